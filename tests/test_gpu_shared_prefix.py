"""Shared-prefix decode (pa_decode_shared_prefix) vs the fp64 oracle, through the C ABI.

The method is still standard attention per sequence ("PagedAttention & vLLM",
Copy-on-write sharing: the n samples of one prompt keep its KV once); only the
reading order changes, so the oracle is the plain per-sequence decode on each
member's own table.  Pools written by the fused step are compared bit-exact,
outputs within max-abs 1e-2 / mean-abs 1e-3.  Batches are laid out in groups of
``group_size`` consecutive sequences whose first ``prefix_lens[g]`` tokens hold
the same K/V: shared physical blocks, plus a copy for a partly shared block.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import DeviceCase, assert_close, bf16_dev, bits_host, i32_dev, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import paged_kv_cache_349_b200  # noqa: F401


def grouped_case(lens, group_size, prefix, *, Hq, Hkv, d, bs, seed):
    """A custom decode step whose groups share their first tokens with the group's first member.

    Member m of group g shares s = min(prefix[g], L_m - 1, L_first - 1) tokens: whole blocks by
    pointing its table at the first member's blocks, the rest of a partly shared block by copying
    those rows into its own block (what a copy-on-write leaves behind)."""
    case = W.make_custom_case(lens, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d, block_size=bs, seed=seed)
    t, k, v = case.block_tables, case.k_cache, case.v_cache
    B = case.batch
    for g in range(-(-B // group_size)):
        lead = g * group_size
        for m in range(lead + 1, min(lead + group_size, B)):
            s = min(int(prefix[g]), int(lens[m]) - 1, int(lens[lead]) - 1)
            if s <= 0:
                continue
            full, r = divmod(s, bs)
            t[m, :full] = t[lead, :full]
            if r:
                k[t[m, full], :, :r] = k[t[lead, full], :, :r]
                v[t[m, full], :, :r] = v[t[lead, full], :, :r]
    return case


def run_prefix(case, prefix, group_size, pt, fused=True, ws_fill=None):
    """copy pairs -> cache write of rows other than each sequence's last -> shared-prefix decode
    (with the last rows written by the decode launch when ``fused``)."""
    import torch
    import paged_kv_cache_349_b200 as pa
    dc = DeviceCase(case)
    k_last, v_last, other = W.split_last_tokens(case)
    pa.pa_copy_blocks(dc.k, dc.v, dc.pairs, err_flag=dc.flag)
    if fused:
        if other.size:
            pa.pa_reshape_and_cache(bf16_dev(case.k_new[other]), bf16_dev(case.v_new[other]), dc.k, dc.v,
                                    i32_dev(case.slot_mapping[other]), err_flag=dc.flag)
    else:
        pa.pa_reshape_and_cache(dc.k_new, dc.v_new, dc.k, dc.v, dc.slots, err_flag=dc.flag)
    need = pa.pa_decode_shared_prefix_workspace_size(case.batch, group_size, case.num_q_heads, case.num_kv_heads,
                                                     case.head_dim, case.block_size, case.max_seq_len, pt)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    if ws_fill is not None:
        ws.fill_(ws_fill)
    before = pa.launch_count()
    pa.pa_decode_shared_prefix(dc.out, dc.q, dc.k, dc.v, dc.tables, dc.lens, i32_dev(np.asarray(prefix)),
                               group_size=group_size, max_seq_len=case.max_seq_len, scale=float(case.scale),
                               partition_tokens=pt, workspace=ws, err_flag=dc.flag,
                               k_new=bf16_dev(k_last) if fused else None, v_new=bf16_dev(v_last) if fused else None)
    assert pa.launch_count() - before == 2  # decode + log-sum-exp reduce
    torch.cuda.synchronize()
    return dc, dc.out.cpu().numpy().astype(np.float64)


def check(case, prefix, group_size, pt, fused=True, rows=None, what="", flag=0):
    dc, got = run_prefix(case, prefix, group_size, pt, fused)
    want, k_ref, v_ref = oracle.decode_step(case, rows=rows)
    assert np.array_equal(bits_host(dc.k), k_ref), f"{what}: K pool differs"
    assert np.array_equal(bits_host(dc.v), v_ref), f"{what}: V pool differs"
    assert int(dc.flag.item()) == flag, f"{what}: error flag {int(dc.flag.item()):#x}"
    if rows is not None:
        got = got[rows[:, 0], rows[:, 1]]
    assert_close(got, want, what)
    return got


@pytest.mark.parametrize("pt", [-1, 0, 64, 16])
def test_chat_workload_small_every_output(pt):
    """The n=4 chat mix shrunk: groups share min(prefix cap, prompt) tokens, the partly shared
    block copied on write by three members."""
    case = W.make_case(3, batch=12, max_len=400, num_blocks=1024)
    check(case, case.shared_tokens[::4], 4, pt, what=f"chat small pt {pt}")


LENS = [40, 57, 33, 100, 17, 17, 17, 17, 300, 1, 200, 250, 0, 50, 60, 70, 95, 95, 130]
LENS_NO_EMPTY = [40, 57, 33, 100, 17, 17, 17, 17, 300, 21, 200, 250, 90, 50, 60, 70, 95, 95, 130]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32, 64])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_groups_all_shapes(d, bs, G):
    n = 4
    prefix = [35, 16, 200, 30, 94]  # a partly shared block, exactly one tile, a short member, an empty one
    case = grouped_case(LENS, n, prefix, Hq=2 * G, Hkv=2, d=d, bs=bs, seed=d + bs + G)
    for pt in (-1, 2 * bs):
        check(case, prefix, n, pt, what=f"d{d} bs{bs} G{G} pt{pt}")


@pytest.mark.parametrize("n", [1, 2, 3, 8, 19])
def test_group_sizes_and_ragged_last_group(n):
    groups = -(-len(LENS_NO_EMPTY) // n)
    prefix = [10_000] * groups  # everything a group can share
    case = grouped_case(LENS_NO_EMPTY, n, prefix, Hq=8, Hkv=8, d=128, bs=16, seed=n)
    check(case, prefix, n, -1, what=f"n{n}")
    check(case, prefix, n, 32, fused=False, what=f"n{n} unfused split")


def test_no_sharing_and_negative_prefix():
    import paged_kv_cache_349_b200 as pa
    case = grouped_case(LENS, 4, [0] * 5, Hq=4, Hkv=4, d=128, bs=16, seed=3)
    check(case, [0] * 5, 4, -1, what="prefix 0")
    # a negative prefix length reads as 0 and is reported
    check(case, [0, -7, 0, 0, 0], 4, -1, what="prefix -7", flag=pa.PA_FLAG_BAD_LEN)


def test_matches_plain_decode_and_is_placement_invariant():
    """Against pa_decode on the same pools (within tolerance: different partitioning), and bit
    identical under a relocation of every physical block."""
    import torch
    import paged_kv_cache_349_b200 as pa
    case = W.make_case(3, batch=16, max_len=600, num_blocks=1500)
    prefix = case.shared_tokens[::4]
    dc, got = run_prefix(case, prefix, 4, -1)
    plain = torch.empty_like(dc.out)
    pa.pa_decode(plain, dc.q, dc.k, dc.v, dc.tables, dc.lens, max_seq_len=case.max_seq_len,
                 scale=float(case.scale), partition_tokens=-1)
    torch.cuda.synchronize()
    err = np.abs(got - plain.cpu().numpy())
    assert err.max() <= 2e-5, err.max()
    # relocate: every block moves, tables are rewritten, the pools after the step are permuted
    perm = np.random.default_rng(9).permutation(case.num_blocks)
    idx = torch.from_numpy(perm).cuda()
    k2, v2 = torch.empty_like(dc.k), torch.empty_like(dc.v)
    k2[idx] = dc.k
    v2[idx] = dc.v
    t = case.block_tables.copy()
    t[t >= 0] = perm[t[t >= 0]]
    out2 = torch.empty_like(dc.out)
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_size(case.batch, 4, case.num_q_heads,
                                                               case.num_kv_heads, case.head_dim, case.block_size,
                                                               case.max_seq_len, -1),
                     dtype=torch.uint8, device="cuda")
    # the pools already hold the step's new tokens: decode without the fused write, on both placements
    pa.pa_decode_shared_prefix(dc.out, dc.q, dc.k, dc.v, dc.tables, dc.lens, i32_dev(prefix), group_size=4,
                               max_seq_len=case.max_seq_len, scale=float(case.scale), partition_tokens=-1,
                               workspace=ws)
    torch.cuda.synchronize()
    a = dc.out.clone()
    pa.pa_decode_shared_prefix(out2, dc.q, k2, v2, i32_dev(t), dc.lens, i32_dev(prefix), group_size=4,
                               max_seq_len=case.max_seq_len, scale=float(case.scale), partition_tokens=-1,
                               workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, out2)
    assert torch.equal(a, torch.from_numpy(got.astype(np.float32)).cuda())


def test_full_size_chat_workload_sampled_rows():
    """The chat workload at full size, in the launch configuration the benchmark times."""
    case = W.make_case(3)
    rows = sample_rows(case, 96, seed=33)
    check(case, case.shared_tokens[::4], 4, 0, rows=rows, what="chat full")


def _pinned(torch, a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(dtype) if dtype is torch.bfloat16 else t.to(dtype)).pin_memory()


@pytest.mark.parametrize("kind,chunks", [("chat", 1), ("chat", 2), ("chat", 3), ("ragged", 2), ("ragged", 5)])
def test_prepared_host_step_matches_device_path(kind, chunks):
    """A prepared host step in shared-prefix mode (pa_decode_step_plan_set_shared_prefix): inputs
    uploaded from pinned host memory, chunks of whole groups, output stored into pinned host memory --
    bit-identical to pa_decode_shared_prefix on device-resident inputs, pools included."""
    import torch
    import paged_kv_cache_349_b200 as pa
    if kind == "chat":
        case = W.make_case(3, batch=12, max_len=400, num_blocks=1024)
        n, prefix = 4, case.shared_tokens[::4]
    else:  # 19 sequences in groups of 4: the last group has 3
        n, prefix = 4, [35, 16, 200, 30, 94]
        case = grouped_case(LENS_NO_EMPTY, n, prefix, Hq=8, Hkv=2, d=128, bs=16, seed=71)
    ref, want = run_prefix(case, prefix, n, case.partition_tokens)
    dc = DeviceCase(case)
    k_last, v_last, other = W.split_last_tokens(case)
    pa.pa_copy_blocks(dc.k, dc.v, dc.pairs, err_flag=dc.flag)
    if other.size:
        pa.pa_reshape_and_cache(bf16_dev(case.k_new[other]), bf16_dev(case.v_new[other]), dc.k, dc.v,
                                i32_dev(case.slot_mapping[other]), err_flag=dc.flag)
    B = case.batch
    args = (B, n, case.max_blocks_per_seq, 1, case.num_q_heads, case.num_kv_heads, case.head_dim, case.block_size,
            case.max_seq_len, case.partition_tokens)
    size = pa.pa_decode_step_staging_size_shared_prefix(*args)
    plain = pa.pa_decode_step_staging_size(B, *args[2:])
    assert size > plain > 0
    staging = torch.empty(size, dtype=torch.uint8, device="cuda")
    out_h = torch.full(case.q.shape, float("nan"), dtype=torch.float32).pin_memory()
    step = pa.DecodeStepHost(out_host=out_h, q_host=_pinned(torch, case.q.view(np.int16), torch.bfloat16),
                             k_new_host=_pinned(torch, k_last.view(np.int16), torch.bfloat16),
                             v_new_host=_pinned(torch, v_last.view(np.int16), torch.bfloat16),
                             tables_host=_pinned(torch, case.block_tables, torch.int32),
                             lens_host=_pinned(torch, case.seq_lens, torch.int32),
                             pairs_host=_pinned(torch, np.zeros((1, 2), np.int32), torch.int32),
                             k_cache=dc.k, v_cache=dc.v, scale=float(case.scale), max_seq_len_cap=case.max_seq_len,
                             partition_tokens=case.partition_tokens, num_chunks=chunks, staging=staging,
                             err_flag=dc.flag, prefix_lens_host=_pinned(torch, np.asarray(prefix), torch.int32),
                             group_size=n)
    step(case.max_seq_len, 0)
    torch.cuda.synchronize()
    assert int(dc.flag.item()) == 0 and int(ref.flag.item()) == 0
    assert np.array_equal(out_h.numpy().astype(np.float64), want)
    assert np.array_equal(bits_host(dc.k), bits_host(ref.k)) and np.array_equal(bits_host(dc.v), bits_host(ref.v))
    step.close()


def test_prepared_host_step_shared_prefix_argument_errors():
    """set_shared_prefix refuses a bad group size, a missing prefix buffer, a staging buffer sized
    for the plain decode (the plan stays a working plain step) and fp8 pools."""
    import ctypes
    import torch
    import paged_kv_cache_349_b200 as pa
    from paged_kv_cache_349_b200._lib import lib
    case = W.make_case(3, batch=8, max_len=200, num_blocks=512)
    k_last, v_last, other = W.split_last_tokens(case)
    dc = DeviceCase(case)
    B = case.batch
    plain = pa.pa_decode_step_staging_size(B, case.max_blocks_per_seq, 1, case.num_q_heads, case.num_kv_heads,
                                           case.head_dim, case.block_size, case.max_seq_len, case.partition_tokens)
    staging = torch.empty(plain, dtype=torch.uint8, device="cuda")
    out_h = torch.empty(case.q.shape, dtype=torch.float32).pin_memory()
    prefix_h = _pinned(torch, case.shared_tokens[::4], torch.int32)
    step = pa.DecodeStepHost(out_host=out_h, q_host=_pinned(torch, case.q.view(np.int16), torch.bfloat16),
                             k_new_host=_pinned(torch, k_last.view(np.int16), torch.bfloat16),
                             v_new_host=_pinned(torch, v_last.view(np.int16), torch.bfloat16),
                             tables_host=_pinned(torch, case.block_tables, torch.int32),
                             lens_host=_pinned(torch, case.seq_lens, torch.int32),
                             pairs_host=_pinned(torch, np.zeros((1, 2), np.int32), torch.int32),
                             k_cache=dc.k, v_cache=dc.v, scale=float(case.scale), max_seq_len_cap=case.max_seq_len,
                             staging=staging, err_flag=dc.flag)
    P = ctypes.c_void_p
    setp = lib.pa_decode_step_plan_set_shared_prefix
    assert setp(None, P(prefix_h.data_ptr()), 4) == pa.PA_ERR_INVALID_ARG
    assert setp(step._plan, P(prefix_h.data_ptr()), 65) == pa.PA_ERR_INVALID_ARG
    assert setp(step._plan, P(prefix_h.data_ptr()), -1) == pa.PA_ERR_INVALID_ARG
    assert setp(step._plan, None, 4) == pa.PA_ERR_INVALID_ARG
    assert setp(step._plan, P(prefix_h.data_ptr()), 4) == pa.PA_ERR_INVALID_ARG  # staging sized for the plain decode
    assert setp(step._plan, None, 0) == pa.PA_OK  # back to (still) the plain decode
    step(case.max_seq_len, 0)  # runs as the plain step
    torch.cuda.synchronize()
    assert int(dc.flag.item()) == 0
    step.close()
    # fp8 pools: no shared-prefix decode
    k8 = torch.zeros(dc.k.shape, dtype=torch.uint8, device="cuda")
    v8 = torch.zeros(dc.v.shape, dtype=torch.uint8, device="cuda")
    big = torch.empty(plain * 2, dtype=torch.uint8, device="cuda")
    step8 = pa.DecodeStepHost(out_host=out_h, q_host=_pinned(torch, case.q.view(np.int16), torch.bfloat16),
                              k_new_host=_pinned(torch, k_last.view(np.int16), torch.bfloat16),
                              v_new_host=_pinned(torch, v_last.view(np.int16), torch.bfloat16),
                              tables_host=_pinned(torch, case.block_tables, torch.int32),
                              lens_host=_pinned(torch, case.seq_lens, torch.int32),
                              pairs_host=_pinned(torch, np.zeros((1, 2), np.int32), torch.int32),
                              k_cache=k8, v_cache=v8, scale=float(case.scale), max_seq_len_cap=case.max_seq_len,
                              staging=big, err_flag=dc.flag, k_scale=1.0, v_scale=1.0)
    assert setp(step8._plan, P(prefix_h.data_ptr()), 4) == pa.PA_ERR_UNSUPPORTED
    step8.close()


def test_prepared_host_step_full_size_chat_sampled_rows():
    """The chat workload at full size through a prepared host step in shared-prefix mode, in the launch
    configuration the benchmark's end-to-end leg uses (automatic chunking: 8 chunks of whole groups,
    first and last half-size), against the oracle on sampled rows; pools bit-exact."""
    import torch
    import paged_kv_cache_349_b200 as pa
    case = W.make_case(3)
    n, prefix = 4, case.shared_tokens[::4]
    dc = DeviceCase(case)
    k_last, v_last, other = W.split_last_tokens(case)
    pa.pa_copy_blocks(dc.k, dc.v, dc.pairs, err_flag=dc.flag)
    if other.size:
        pa.pa_reshape_and_cache(bf16_dev(case.k_new[other]), bf16_dev(case.v_new[other]), dc.k, dc.v,
                                i32_dev(case.slot_mapping[other]), err_flag=dc.flag)
    B = case.batch
    size = pa.pa_decode_step_staging_size_shared_prefix(B, n, case.max_blocks_per_seq, 1, case.num_q_heads,
                                                        case.num_kv_heads, case.head_dim, case.block_size,
                                                        case.max_seq_len, case.partition_tokens)
    staging = torch.empty(size, dtype=torch.uint8, device="cuda")
    out_h = torch.full(case.q.shape, float("nan"), dtype=torch.float32).pin_memory()
    step = pa.DecodeStepHost(out_host=out_h, q_host=_pinned(torch, case.q.view(np.int16), torch.bfloat16),
                             k_new_host=_pinned(torch, k_last.view(np.int16), torch.bfloat16),
                             v_new_host=_pinned(torch, v_last.view(np.int16), torch.bfloat16),
                             tables_host=_pinned(torch, case.block_tables, torch.int32),
                             lens_host=_pinned(torch, case.seq_lens, torch.int32),
                             pairs_host=_pinned(torch, np.zeros((1, 2), np.int32), torch.int32),
                             k_cache=dc.k, v_cache=dc.v, scale=float(case.scale), max_seq_len_cap=case.max_seq_len,
                             partition_tokens=case.partition_tokens, num_chunks=0, staging=staging,
                             err_flag=dc.flag, prefix_lens_host=_pinned(torch, np.asarray(prefix), torch.int32),
                             group_size=n)
    step(case.max_seq_len, 0)
    torch.cuda.synchronize()
    step.close()
    assert int(dc.flag.item()) == 0
    rows = sample_rows(case, 96, seed=34)
    want, k_ref, v_ref = oracle.decode_step(case, rows=rows)
    assert np.array_equal(bits_host(dc.k), k_ref) and np.array_equal(bits_host(dc.v), v_ref)
    got = out_h.numpy().astype(np.float64)
    assert not np.isnan(got).any()
    assert_close(got[rows[:, 0], rows[:, 1]], want, "chat full, prepared host step")
