"""pa_decode_append (cache write fused into decode) vs the oracle and vs the unfused step."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import DeviceCase, assert_close, bits_host, run_fused_step, run_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _check(case, pt=None, what=""):
    fused = DeviceCase(case)
    got = run_fused_step(fused, pt)
    want, k_ref, v_ref = oracle.decode_step(case)
    assert np.array_equal(bits_host(fused.k), k_ref), f"{what}: K pool differs"
    assert np.array_equal(bits_host(fused.v), v_ref), f"{what}: V pool differs"
    assert int(fused.flag.item()) == 0
    assert_close(got, want, what)
    unfused = DeviceCase(case)
    ref = run_step(unfused, pt)
    assert np.array_equal(got, ref), f"{what}: fused and unfused outputs differ"


@pytest.mark.parametrize("cfg,kw", [
    (1, {}),
    (2, dict(batch=6, max_len=300, num_blocks=256)),
    (3, dict(batch=8, max_len=260, num_blocks=512)),
    (4, dict(batch=9, max_len=700, num_blocks=256)),
    (5, dict(batch=2, max_len=2048, num_blocks=640, num_copy_pairs=40)),
])
def test_workloads(cfg, kw):
    _check(W.make_case(cfg, **kw), what=f"cfg{cfg}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32, 64])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_ragged_shapes(d, bs, G):
    lens = [0, 1, 2, 15, 16, 17, 31, 32, 33, 48, 49, 257]
    case = W.make_custom_case(lens, num_q_heads=2 * G, num_kv_heads=2, head_dim=d, block_size=bs,
                              seed=100 + d + bs + G)
    for pt in (-1, bs, 2 * bs):
        _check(case, pt, what=f"d{d} bs{bs} G{G} pt{pt}")


def test_full_size_llama2_7b_sampled_rows():
    from tests.gpu_helpers import sample_rows
    case = W.make_case(2)
    dc = DeviceCase(case)
    got = run_fused_step(dc)
    rows = sample_rows(case, 64, seed=9)
    want, k_ref, v_ref = oracle.decode_step(case, rows=rows)
    assert np.array_equal(bits_host(dc.k), k_ref) and np.array_equal(bits_host(dc.v), v_ref)
    assert_close(got[rows[:, 0], rows[:, 1]], want, "cfg2 full fused")


@pytest.mark.parametrize("cfg,kw,chunks,pinned_out,inputs", [
    (2, dict(batch=6, max_len=300, num_blocks=256), 1, True, "pinned"),
    (2, dict(batch=6, max_len=300, num_blocks=256), 8, True, "pinned"),      # one sequence per chunk
    (2, dict(batch=64, max_len=300, num_blocks=2048), 0, True, "pinned"),    # auto: ~2.6 MB over the link
    (2, dict(batch=67, max_len=300, num_blocks=2048), 5, True, "pinned"),    # ragged chunk sizes
    (2, dict(batch=67, max_len=300, num_blocks=2048), 5, False, "pinned"),   # pageable output: staged
    (2, dict(batch=67, max_len=300, num_blocks=2048), 5, True, "pageable"),  # inputs copied, not read
    (4, dict(batch=9, max_len=1500, num_blocks=512), 1, True, "pinned"),
    (4, dict(batch=9, max_len=1500, num_blocks=512), 1, False, "misaligned"),  # 8-byte aligned inputs
    (4, dict(batch=9, max_len=1500, num_blocks=512), 4, True, "pinned"),     # split: a workspace slice per chunk
    (5, dict(batch=2, max_len=2048, num_blocks=640, num_copy_pairs=40), 1, True, "pinned"),
    (5, dict(batch=3, max_len=2048, num_blocks=960, num_copy_pairs=40), 3, True, "pinned"),  # copies first
    (5, dict(batch=3, max_len=2048, num_blocks=960, num_copy_pairs=40), 3, True, "misaligned"),
])
def test_host_step_matches_device_path(cfg, kw, chunks, pinned_out, inputs):
    """pa_decode_step_host (uploads, copies, fused decode, output to the host) == the device-resident
    path, bit for bit, whether or not the step is cut into pipelined chunks, whether the output buffer
    is page-locked (written by the kernels) or pageable (staged and copied back), and whether the
    inputs are read by the upload kernel (page-locked, 16-byte aligned) or copied (pageable, or only
    8-byte aligned)."""
    import torch
    import paged_kv_cache_349_b200 as pa
    case = W.make_case(cfg, **kw)
    k_last, v_last, other = W.split_last_tokens(case)
    assert other.size == 0
    ref = DeviceCase(case)
    want = run_fused_step(ref)
    dc = DeviceCase(case)

    def pinned(a, dtype):
        t = torch.from_numpy(np.ascontiguousarray(a))
        t = t.view(dtype) if dtype is torch.bfloat16 else t.to(dtype)
        if inputs == "pageable":
            return t
        if inputs == "misaligned":      # a contiguous view 8 bytes into a page-locked buffer
            esz = t.element_size()
            buf = torch.empty(t.numel() + 8 // esz, dtype=dtype).pin_memory()
            v = buf[8 // esz:].view(t.shape)
            v.copy_(t)
            assert v.data_ptr() % 16 == 8
            return v
        return t.pin_memory()

    out_h = torch.full(case.q.shape, float("nan"), dtype=torch.float32)
    if pinned_out:
        out_h = out_h.pin_memory()
    pairs = case.copy_pairs.reshape(-1, 2)
    max_pairs = max(1, pairs.shape[0])
    pairs_np = np.zeros((max_pairs, 2), np.int32)
    pairs_np[:pairs.shape[0]] = pairs
    pairs_h = pinned(pairs_np, torch.int32)
    size = pa.pa_decode_step_staging_size(case.batch, case.max_blocks_per_seq, max_pairs, case.num_q_heads,
                                          case.num_kv_heads, case.head_dim, case.block_size, case.max_seq_len,
                                          case.partition_tokens)
    staging = torch.empty(size, dtype=torch.uint8, device="cuda")
    step = pa.DecodeStepHost(out_host=out_h, q_host=pinned(case.q.view(np.int16), torch.bfloat16),
                             k_new_host=pinned(k_last.view(np.int16), torch.bfloat16),
                             v_new_host=pinned(v_last.view(np.int16), torch.bfloat16),
                             tables_host=pinned(case.block_tables, torch.int32),
                             lens_host=pinned(case.seq_lens, torch.int32), pairs_host=pairs_h,
                             k_cache=dc.k, v_cache=dc.v, scale=float(case.scale), max_seq_len_cap=case.max_seq_len,
                             partition_tokens=case.partition_tokens, num_chunks=chunks, staging=staging,
                             err_flag=dc.flag)
    step(case.max_seq_len, pairs.shape[0])
    torch.cuda.synchronize()
    got = out_h.numpy().astype(np.float64)
    assert np.array_equal(got, want)
    assert np.array_equal(bits_host(dc.k), bits_host(ref.k)) and np.array_equal(bits_host(dc.v), bits_host(ref.v))
    assert int(dc.flag.item()) == 0


@pytest.mark.parametrize("chunks", [1, 3])
def test_one_call_host_step_matches_plan(chunks):
    """pa_decode_step_host (everything resolved per call) and a prepared step
    (pa_decode_step_plan_create once, pa_decode_step_plan_run per step) give the same output and
    pools, bit for bit, over two steps; the plan refuses a run past its caps."""
    import ctypes
    import torch
    import paged_kv_cache_349_b200 as pa
    from paged_kv_cache_349_b200._lib import lib
    case = W.make_case(3, batch=12, max_len=300, num_blocks=1024)
    k_last, v_last, other = W.split_last_tokens(case)
    pairs = case.copy_pairs.reshape(-1, 2)
    P = ctypes.c_void_p

    def pinned(a, dtype):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(dtype) if dtype is torch.bfloat16 else t.to(dtype)).pin_memory()

    hq = pinned(case.q.view(np.int16), torch.bfloat16)
    hk, hv = pinned(k_last.view(np.int16), torch.bfloat16), pinned(v_last.view(np.int16), torch.bfloat16)
    ht, hl = pinned(case.block_tables, torch.int32), pinned(case.seq_lens, torch.int32)
    hp = pinned(pairs, torch.int32)
    cap = case.max_seq_len + 8
    size = pa.pa_decode_step_staging_size(case.batch, case.max_blocks_per_seq, pairs.shape[0], case.num_q_heads,
                                          case.num_kv_heads, case.head_dim, case.block_size, cap,
                                          case.partition_tokens)
    results = []
    for use_plan in (False, True):
        dc = DeviceCase(case)
        if other.size:  # the copy-on-write rows other than each sequence's last, written beforehand
            pa.pa_copy_blocks(dc.k, dc.v, dc.pairs, err_flag=dc.flag)
            pa.pa_reshape_and_cache(dc.k_new[torch.from_numpy(other).cuda()].contiguous(),
                                    dc.v_new[torch.from_numpy(other).cuda()].contiguous(), dc.k, dc.v,
                                    dc.slots[torch.from_numpy(other).cuda()].contiguous(), err_flag=dc.flag)
        staging = torch.empty(size, dtype=torch.uint8, device="cuda")
        out_h = torch.full(case.q.shape, float("nan"), dtype=torch.float32).pin_memory()
        stream = P(torch.cuda.current_stream().cuda_stream)
        head = (P(out_h.data_ptr()), P(hq.data_ptr()), P(hk.data_ptr()), P(hv.data_ptr()), P(ht.data_ptr()),
                case.max_blocks_per_seq, P(hl.data_ptr()), P(hp.data_ptr()))
        shape = (case.num_q_heads, case.num_kv_heads, case.head_dim, case.block_size, case.num_blocks,
                 float(case.scale), case.partition_tokens, chunks, P(staging.data_ptr()), size)
        outs = []
        plan = P()
        if use_plan:
            assert lib.pa_decode_step_plan_create(*head, pairs.shape[0], P(dc.k.data_ptr()), P(dc.v.data_ptr()),
                                                  case.batch, cap, *shape, 0, 1.0, 1.0, ctypes.byref(plan)) == 0
            # past the caps: refused, nothing enqueued
            assert lib.pa_decode_step_plan_run(plan, cap + 1, 0, P(dc.flag.data_ptr()), stream) == \
                pa.PA_ERR_INVALID_ARG
            assert lib.pa_decode_step_plan_run(plan, cap, pairs.shape[0] + 1, P(dc.flag.data_ptr()), stream) == \
                pa.PA_ERR_INVALID_ARG
        for step in range(2):  # the second step re-runs on the updated pools (same inputs)
            if use_plan:
                rc = lib.pa_decode_step_plan_run(plan, case.max_seq_len, 0, P(dc.flag.data_ptr()), stream)
            else:
                rc = lib.pa_decode_step_host(*head, 0, pairs.shape[0], P(dc.k.data_ptr()), P(dc.v.data_ptr()),
                                             case.batch, case.max_seq_len, *shape, P(dc.flag.data_ptr()), stream)
            assert rc == 0
            torch.cuda.synchronize()
            outs.append(out_h.numpy().copy())
        if use_plan:
            lib.pa_decode_step_plan_destroy(plan)
        assert int(dc.flag.item()) == 0
        results.append((outs, bits_host(dc.k), bits_host(dc.v)))
    (o1, k1, v1), (o2, k2, v2) = results
    assert all(np.array_equal(a, b) for a, b in zip(o1, o2))
    assert np.array_equal(k1, k2) and np.array_equal(v1, v2)
    want, k_ref, v_ref = oracle.decode_step(case)
    assert np.array_equal(k1, k_ref) and np.array_equal(v1, v_ref)
    assert_close(o1[0].astype(np.float64), want, "host step")

