"""pa_decode_builtin_scratch: decode for callers that cannot allocate device memory.

Such callers (a plugin whose host program owns every device allocation, a
foreign runtime that only passes pointers to tensors it already owns, a
latency-critical loop that must not call cudaMalloc) get the split decode's
scratch from an array the library owns.  These tests call the entry point
through the C ABI and compare it with pa_decode given a caller workspace.
Both run the same kernels with the same partitioning on the same inputs, so
the outputs must agree bit for bit:
  - two calls in a row with different inputs, synchronised in between;
  - two calls queued back to back on one stream with no synchronisation, so
    the second call's partial states overwrite the shared array right after
    the first call's merge has read them;
  - a call that does not split (no scratch used) and an empty batch.
"""
import ctypes

import numpy as np
import pytest

import workloads as W
from tests.gpu_helpers import bf16_dev, i32_dev

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


def _case(seed, **kw):
    kw.setdefault("partition_tokens", 256)
    return W.make_case(5, seed=seed, batch=3, max_len=2000 + 300 * (seed % 2), num_blocks=1024,
                       num_copy_pairs=0, fill=W.BF16_ZERO, **kw)


def _reference(torch, lib, pa, case, tens, stream):
    """pa_decode with a caller-owned workspace (filled with garbage: it needs no clearing)."""
    need = pa.pa_decode_workspace_size(case.batch, case.num_q_heads, case.num_kv_heads, case.head_dim,
                                       case.block_size, case.max_seq_len, case.partition_tokens)
    ws = torch.randint(0, 256, (max(need, 16),), dtype=torch.uint8, device="cuda")
    want = torch.empty(case.q.shape, dtype=torch.float32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.pa_decode(*_args(case, tens, want), P(ws.data_ptr()), need, P(flag.data_ptr()), stream) == 0
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    return want, need


def test_builtin_scratch_bit_identical_to_caller_workspace_two_calls(torch_cuda):
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    from paged_kv_cache_349_b200._lib import lib
    stream = P(torch.cuda.current_stream().cuda_stream)
    for seed in (21, 22):  # two calls in a row, different inputs and lengths
        case = _case(seed)
        tens = _tensors(case)
        want, need = _reference(torch, lib, pa, case, tens, stream)
        assert 0 < need <= pa.PA_DECODE_BUILTIN_SCRATCH_BYTES
        got = torch.full(case.q.shape, float("nan"), dtype=torch.float32, device="cuda")
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")
        before = pa.launch_count()
        assert lib.pa_decode_builtin_scratch(*_args(case, tens, got), P(flag.data_ptr()), stream) == 0
        assert pa.launch_count() - before == 2  # split decode + log-sum-exp reduce
        torch.cuda.synchronize()
        assert int(flag.item()) == 0
        assert torch.equal(got, want)


def test_builtin_scratch_back_to_back_on_one_stream(torch_cuda):
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    from paged_kv_cache_349_b200._lib import lib
    stream = P(torch.cuda.current_stream().cuda_stream)
    cases = [_case(31), _case(32)]
    tens = [_tensors(c) for c in cases]
    wants = [_reference(torch, lib, pa, c, t, stream)[0] for c, t in zip(cases, tens)]
    gots = [torch.full(c.q.shape, float("nan"), dtype=torch.float32, device="cuda") for c in cases]
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    for c, t, g in zip(cases, tens, gots):  # queued with no synchronisation in between
        assert lib.pa_decode_builtin_scratch(*_args(c, t, g), P(flag.data_ptr()), stream) == 0
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    for g, w in zip(gots, wants):
        assert torch.equal(g, w)


def test_builtin_scratch_single_pass_and_empty_batch(torch_cuda):
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    from paged_kv_cache_349_b200._lib import lib
    stream = P(torch.cuda.current_stream().cuda_stream)
    # max_seq_len within one partition: no split, no scratch, one launch
    case = _case(41, partition_tokens=4096)
    assert pa.pa_decode_partition_tokens(case.batch, case.num_q_heads, case.num_kv_heads, case.head_dim,
                                         case.block_size, case.max_seq_len, case.partition_tokens) == -1
    tens = _tensors(case)
    want, need = _reference(torch, lib, pa, case, tens, stream)
    assert need == 0
    got = torch.full(case.q.shape, float("nan"), dtype=torch.float32, device="cuda")
    before = pa.launch_count()
    assert lib.pa_decode_builtin_scratch(*_args(case, tens, got), None, stream) == 0
    assert pa.launch_count() - before == 1
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    # an empty batch: PA_OK, nothing launched
    before = pa.launch_count()
    args = list(_args(case, tens, got))
    args[7] = 0
    assert lib.pa_decode_builtin_scratch(*args, None, stream) == pa.PA_OK
    assert pa.launch_count() == before


def test_builtin_scratch_rejects_oversize_split(torch_cuda):
    torch = torch_cuda
    import paged_kv_cache_349_b200 as pa
    from paged_kv_cache_349_b200._lib import lib
    # 16-token partitions of 32768 tokens for 8 x 64 heads need ~2.2 GB of scratch
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
