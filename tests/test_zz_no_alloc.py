"""pa_decode_builtin_scratch: decode for callers that cannot allocate device memory.

Such callers (a plugin whose host program owns every device allocation, a
foreign runtime that only passes pointers to tensors it already owns, a
latency-critical loop that must not call cudaMalloc) get the split decode's
scratch from an array the library owns.  These tests call the entry point
through the C ABI and compare it with pa_decode given a caller workspace,
within the attention tolerance, on two calls in a row with different inputs
(so the second call cannot lean on what the first left in the shared array).
"""
import ctypes

import numpy as np
import pytest

import workloads as W
from tests.gpu_helpers import ATOL_MAX, ATOL_MEAN, bf16_dev, i32_dev

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch


def _args(case, tensors, out):
    q, k, v, t, lens = tensors
    return (P(out.data_ptr()), P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(t.data_ptr()),
            case.max_blocks_per_seq, P(lens.data_ptr()), case.batch, case.max_seq_len, case.num_q_heads,
            case.num_kv_heads, case.head_dim, case.block_size, case.num_blocks, float(case.scale),
            case.partition_tokens)


def _tensors(case):
    return (bf16_dev(case.q), bf16_dev(case.k_cache), bf16_dev(case.v_cache), i32_dev(case.block_tables),
            i32_dev(case.seq_lens))


def test_builtin_scratch_matches_caller_workspace_two_calls(torch_cuda):
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    from paged_kv_cache_349_b200._lib import lib
    stream = P(torch.cuda.current_stream().cuda_stream)
    for seed in (21, 22):  # two calls in a row, different inputs and lengths
        case = W.make_case(5, seed=seed, batch=3, max_len=2000 + 300 * (seed - 21), num_blocks=1024,
                           num_copy_pairs=0, partition_tokens=256, fill=W.BF16_ZERO)
        tens = _tensors(case)
        need = pa.pa_decode_workspace_size(case.batch, case.num_q_heads, case.num_kv_heads, case.head_dim,
                                           case.block_size, case.max_seq_len, case.partition_tokens)
        assert 0 < need <= pa.PA_DECODE_BUILTIN_SCRATCH_BYTES
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        want = torch.empty(case.q.shape, dtype=torch.float32, device="cuda")
        got = torch.full(case.q.shape, float("nan"), dtype=torch.float32, device="cuda")
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert lib.pa_decode(*_args(case, tens, want), P(ws.data_ptr()), need, P(flag.data_ptr()), stream) == 0
        before = pa.launch_count()
        assert lib.pa_decode_builtin_scratch(*_args(case, tens, got), P(flag.data_ptr()), stream) == 0
        assert pa.launch_count() - before == 2  # split decode + log-sum-exp reduce
        torch.cuda.synchronize()
        assert int(flag.item()) == 0
        g = got.cpu().numpy().astype(np.float64)
        w = want.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(g))
        err = np.abs(g - w)
        assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (err.max(), err.mean())


def test_builtin_scratch_rejects_oversize_split(torch_cuda):
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    from paged_kv_cache_349_b200._lib import lib
    # 16-token partitions of 32768 tokens for 8 x 64 heads need ~2.2 GB of scratch
    case = W.make_case(1)
    B, Hq, Hkv, d, bs, L = 8, 64, 8, 128, 16, 32768
    need = pa.pa_decode_workspace_size(B, Hq, Hkv, d, bs, L, 16)
    assert need > pa.PA_DECODE_BUILTIN_SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    p = P(dummy.data_ptr())
    before = pa.launch_count()
    st = lib.pa_decode_builtin_scratch(p, p, p, p, p, L // bs, p, B, L, Hq, Hkv, d, bs, 4096, 0.1, 16, None,
                                       P(torch.cuda.current_stream().cuda_stream))
    assert st == pa.PA_ERR_UNSUPPORTED
    assert pa.launch_count() == before
    del case
