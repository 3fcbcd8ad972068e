"""CUDA path vs the fp64 oracle, through the C ABI.

Cache writes and block copies must be bit-exact over the whole pool
(untouched blocks included); attention outputs must lie within max-abs 1e-2
and mean-abs 1e-3 of the oracle.  Small cases compare every output; the five
workloads at full size compare sampled rows the oracle computes one by one,
in the launch configuration the benchmark times.
"""
import numpy as np
import pytest

import oracle
import workloads as W
from tests.gpu_helpers import DeviceCase, assert_close, bits_host, bf16_dev, i32_dev, run_step, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import paged_kv_cache_349_b200  # noqa: F401  (fails loudly if libpa.so is missing)


def _check_step(case, partition_tokens=None, rows=None, what=""):
    dc = DeviceCase(case)
    got = run_step(dc, partition_tokens)
    want, k_ref, v_ref = oracle.decode_step(case, rows=rows)
    assert np.array_equal(bits_host(dc.k), k_ref), f"{what}: K pool differs"
    assert np.array_equal(bits_host(dc.v), v_ref), f"{what}: V pool differs"
    assert int(dc.flag.item()) == 0, f"{what}: error flag {int(dc.flag.item()):#x}"
    if rows is not None:
        got = got[rows[:, 0], rows[:, 1]]
    return assert_close(got, want, what), dc, got


def test_tiny_workload_every_output():
    case = W.make_case(1)
    (mx, mean), dc, got = _check_step(case, what="tiny")
    # seq 0 has one token: the output is that token's value row, exactly
    want, k_ref, v_ref = oracle.decode_step(case)
    for g in range(case.num_q_heads):
        assert np.array_equal(got[0, g], want[0, g]), "single-token row must be exact"


@pytest.mark.parametrize("cfg,kw", [
    (2, dict(batch=6, max_len=300, num_blocks=256)),
    (3, dict(batch=8, max_len=260, num_blocks=512)),
    (4, dict(batch=9, max_len=700, num_blocks=256)),
    (5, dict(batch=2, max_len=2048, num_blocks=640, num_copy_pairs=40)),
])
def test_small_workloads_every_output(cfg, kw):
    case = W.make_case(cfg, **kw)
    _check_step(case, what=f"cfg{cfg} small")


@pytest.mark.parametrize("pt", [-1, 16, 32, 64, 512, 0])
def test_split_and_single_pass_agree_with_oracle(pt):
    case = W.make_case(2, batch=5, max_len=600, num_blocks=256)
    _check_step(case, partition_tokens=pt, what=f"partition {pt}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32, 64])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_ragged_lengths_all_shapes(d, bs, G):
    lens = [1, 2, 15, 16, 17, 31, 32, 33, 47, 48, 49, 95, 257]
    case = W.make_custom_case(lens, num_q_heads=2 * G, num_kv_heads=2, head_dim=d, block_size=bs,
                              seed=d + bs + G)
    for pt in (-1, 2 * bs):
        _check_step(case, partition_tokens=pt, what=f"d{d} bs{bs} G{G} pt{pt}")


def test_empty_sequences_give_zero_rows():
    case = W.make_custom_case([0, 5, 0, 40], num_q_heads=4, num_kv_heads=4, head_dim=128, block_size=16,
                              seed=11)
    for pt in (-1, 16):
        (_, _), dc, got = _check_step(case, partition_tokens=pt, what="empty")
        assert np.all(got[0] == 0) and np.all(got[2] == 0)


def test_physical_permutation_is_bit_identical():
    """Relocating blocks (and rewriting the tables) must not change a single output bit."""
    import torch
    case = W.make_case(4, batch=7, max_len=900, num_blocks=256)
    dc = DeviceCase(case)
    out_a = run_step(dc, -1)
    perm = np.random.default_rng(5).permutation(case.num_blocks)
    k_b = torch.empty_like(dc.k)
    v_b = torch.empty_like(dc.v)
    idx = torch.from_numpy(perm).cuda()
    k_b[idx] = dc.k
    v_b[idx] = dc.v
    t = case.block_tables.copy()
    t[t >= 0] = perm[t[t >= 0]]
    out_b_dev = torch.empty_like(dc.out)
    import paged_kv_cache_349_b200 as pa
    pa.pa_decode(out_b_dev, dc.q, k_b, v_b, i32_dev(t), dc.lens, max_seq_len=case.max_seq_len,
                 scale=float(case.scale), partition_tokens=-1)
    torch.cuda.synchronize()
    assert np.array_equal(out_a, out_b_dev.cpu().numpy().astype(np.float64))


def test_shared_blocks_equal_private_copies_bit_identical():
    import torch
    import paged_kv_cache_349_b200 as pa
    case = W.make_case(3, batch=12, max_len=300, num_blocks=1024)
    dc = DeviceCase(case)
    out_shared = run_step(dc, -1)
    bs = case.block_size
    nblk = [-(-int(L) // bs) for L in case.seq_lens]
    total = sum(nblk)
    k2 = torch.zeros((total,) + tuple(dc.k.shape[1:]), dtype=dc.k.dtype, device="cuda")
    v2 = torch.zeros_like(k2)
    t2 = np.full((case.batch, case.max_blocks_per_seq), -1, np.int32)
    src = np.concatenate([case.block_tables[b, :n] for b, n in enumerate(nblk)])
    k2[:] = dc.k[torch.from_numpy(src.astype(np.int64)).cuda()]
    v2[:] = dc.v[torch.from_numpy(src.astype(np.int64)).cuda()]
    c = 0
    for b, n in enumerate(nblk):
        t2[b, :n] = np.arange(c, c + n)
        c += n
    assert len(set(src.tolist())) < src.size, "case must contain shared blocks"
    out2 = torch.empty_like(dc.out)
    pa.pa_decode(out2, dc.q, k2, v2, i32_dev(t2), dc.lens, max_seq_len=case.max_seq_len,
                 scale=float(case.scale), partition_tokens=-1)
    torch.cuda.synchronize()
    assert np.array_equal(out_shared, out2.cpu().numpy().astype(np.float64))


def test_error_flags_and_skipped_accesses():
    import torch
    import paged_kv_cache_349_b200 as pa
    case = W.make_custom_case([20, 33], num_q_heads=2, num_kv_heads=2, head_dim=128, block_size=16,
                              seed=12)
    dc = DeviceCase(case)
    NB, bs = case.num_blocks, case.block_size
    k0 = dc.k.clone()
    # bad slot: reported, nothing written; -1 silently skipped
    bad = i32_dev(np.array([NB * bs, -1], np.int32))
    pa.pa_reshape_and_cache(dc.k_new[:2].contiguous(), dc.v_new[:2].contiguous(), dc.k, dc.v, bad,
                            err_flag=dc.flag)
    torch.cuda.synchronize()
    assert int(dc.flag.item()) == pa.PA_FLAG_BAD_SLOT
    assert torch.equal(dc.k.view(torch.int16), k0.view(torch.int16))
    # bad copy pair
    dc.flag.zero_()
    pa.pa_copy_blocks(dc.k, dc.v, i32_dev(np.array([[0, NB]], np.int32)), err_flag=dc.flag)
    torch.cuda.synchronize()
    assert int(dc.flag.item()) == pa.PA_FLAG_BAD_PAIR and torch.equal(dc.k.view(torch.int16), k0.view(torch.int16))
    # bad block id inside the used part of a table
    dc.flag.zero_()
    t = case.block_tables.copy()
    t[1, 1] = NB + 5
    pa.pa_decode(dc.out, dc.q, dc.k, dc.v, i32_dev(t), dc.lens, max_seq_len=case.max_seq_len,
                 scale=float(case.scale), partition_tokens=-1, err_flag=dc.flag)
    torch.cuda.synchronize()
    assert int(dc.flag.item()) & pa.PA_FLAG_BAD_BLOCK
    # a sequence longer than max_seq_len (split modes: test_bad_lengths_flagged_in_every_mode)
    dc.flag.zero_()
    pa.pa_decode(dc.out, dc.q, dc.k, dc.v, dc.tables, dc.lens, max_seq_len=20,
                 scale=float(case.scale), partition_tokens=-1, err_flag=dc.flag)
    torch.cuda.synchronize()
    assert int(dc.flag.item()) & pa.PA_FLAG_BAD_LEN


@pytest.mark.parametrize("pt", [-1, 16, 0])
def test_bad_lengths_flagged_in_every_mode(pt):
    """A negative length reads nothing and gives zero rows; a length past max_seq_len is cut to it.
    Both raise PA_FLAG_BAD_LEN, single pass, 16-token partitions and the default split alike."""
    import torch
    import paged_kv_cache_349_b200 as pa
    case = W.make_custom_case([20, 33, 700, 1500], num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                              seed=13)
    dc = DeviceCase(case)
    # the default of this shape splits (4 sequences x 2 kv heads, up to 1500 tokens)
    assert pt != 0 or pa.pa_decode_partition_tokens(4, 8, 2, 128, 16, case.max_seq_len, 0) > 0
    # complete the pools with the step's new tokens, on both sides
    pa.pa_reshape_and_cache(dc.k_new, dc.v_new, dc.k, dc.v, dc.slots, err_flag=dc.flag)
    k_ref, v_ref = case.k_cache.copy(), case.v_cache.copy()
    assert oracle.reshape_and_cache(case.k_new, case.v_new, k_ref, v_ref, case.slot_mapping, 16) == 0
    for lens, max_len in (([-5, 33, 700, 1500], case.max_seq_len), ([20, 33, 700, 1500], 1000)):
        bad = np.array(lens, np.int32)
        ws_bytes = pa.pa_decode_workspace_size(case.batch, 8, 2, 128, 16, max_len, pt)
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
        dc.flag.zero_()
        dc.out.fill_(float("nan"))
        pa.pa_decode(dc.out, dc.q, dc.k, dc.v, dc.tables, i32_dev(bad), max_seq_len=max_len,
                     scale=float(case.scale), partition_tokens=pt, workspace=ws, err_flag=dc.flag)
        torch.cuda.synchronize()
        assert int(dc.flag.item()) == pa.PA_FLAG_BAD_LEN, (lens, max_len, pt)
        got = dc.out.cpu().numpy().astype(np.float64)
        clamped = np.clip(bad, 0, max_len)
        want = oracle.decode(case.q, k_ref, v_ref, case.block_tables, clamped,
                             num_kv_heads=2, block_size=16, scale=case.scale)
        assert_close(got, want, f"lens {lens} max {max_len} pt {pt}")
        if lens[0] < 0:
            assert np.all(got[0] == 0)


def test_split_workspace_needs_no_clearing():
    """Every partial state the reduce reads is written earlier in the same call: a workspace
    full of zeros, of random bytes or of all-ones bytes gives bit-identical outputs, and a call
    queued right behind another on the same workspace (different inputs, no synchronisation)
    does too."""
    import torch
    import paged_kv_cache_349_b200 as pa
    case = W.make_case(5, batch=3, max_len=3000, num_blocks=800, num_copy_pairs=0, partition_tokens=256,
                       fill=W.BF16_ZERO)
    dc = DeviceCase(case)
    need = pa.pa_decode_workspace_size(case.batch, case.num_q_heads, case.num_kv_heads, case.head_dim,
                                       case.block_size, case.max_seq_len, 256)
    outs = []
    for fill in ("zero", "random", "ones"):
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
        if fill == "random":
            ws = torch.randint(0, 256, (need,), dtype=torch.uint8, device="cuda")
        elif fill == "ones":
            ws.fill_(255)
        out = torch.empty_like(dc.out)
        pa.pa_decode(out, dc.q, dc.k, dc.v, dc.tables, dc.lens, max_seq_len=case.max_seq_len,
                     scale=float(case.scale), partition_tokens=256, workspace=ws, err_flag=dc.flag)
        torch.cuda.synchronize()
        outs.append(out)
    assert int(dc.flag.item()) == 0
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    want = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.seq_lens,
                         num_kv_heads=case.num_kv_heads, block_size=16, scale=case.scale)
    assert_close(outs[0].cpu().numpy(), want, "split 256")
    # back to back on one workspace: q, then -q (a different softmax), no sync in between
    ws = torch.randint(0, 256, (need,), dtype=torch.uint8, device="cuda")
    q2 = (-dc.q.float()).to(torch.bfloat16)
    a, b = torch.empty_like(dc.out), torch.empty_like(dc.out)
    for qq, o in ((dc.q, a), (q2, b)):
        pa.pa_decode(o, qq, dc.k, dc.v, dc.tables, dc.lens, max_seq_len=case.max_seq_len,
                     scale=float(case.scale), partition_tokens=256, workspace=ws, err_flag=dc.flag)
    torch.cuda.synchronize()
    b_alone = torch.empty_like(dc.out)
    pa.pa_decode(b_alone, q2, dc.k, dc.v, dc.tables, dc.lens, max_seq_len=case.max_seq_len,
                 scale=float(case.scale), partition_tokens=256, workspace=torch.zeros_like(ws), err_flag=dc.flag)
    torch.cuda.synchronize()
    assert torch.equal(a, outs[0]) and torch.equal(b, b_alone)


def test_split_decode_replays_in_a_cuda_graph():
    """A captured split call (decode + programmatic-dependent reduce) replays correctly."""
    import torch
    import paged_kv_cache_349_b200 as pa
    case = W.make_case(4, batch=6, max_len=2500, num_blocks=700, partition_tokens=512, fill=W.BF16_ZERO)
    dc = DeviceCase(case)
    need = pa.pa_decode_workspace_size(case.batch, case.num_q_heads, case.num_kv_heads, case.head_dim,
                                       case.block_size, case.max_seq_len, 512)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")

    def call():
        pa.pa_decode(dc.out, dc.q, dc.k, dc.v, dc.tables, dc.lens, max_seq_len=case.max_seq_len,
                     scale=float(case.scale), partition_tokens=512, workspace=ws, err_flag=dc.flag)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()  # warm-up outside the capture (kernel attributes, tensor maps)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    eager = dc.out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for _ in range(3):
        dc.out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(dc.out, eager)
    assert int(dc.flag.item()) == 0
    del g


@pytest.mark.parametrize("pt", [-1, 16])
def test_nan_in_an_attended_row_propagates(pt):
    """A NaN in a row the decode attends gives NaN in that sequence's outputs, as in the oracle;
    sequences that do not read the row are unaffected and empty ones stay zero."""
    import torch
    import paged_kv_cache_349_b200 as pa
    case = W.make_custom_case([0, 40, 70], num_q_heads=4, num_kv_heads=2, head_dim=128, block_size=16, seed=17)
    dc = DeviceCase(case)
    pa.pa_reshape_and_cache(dc.k_new, dc.v_new, dc.k, dc.v, dc.slots, err_flag=dc.flag)
    k_ref, v_ref = case.k_cache.copy(), case.v_cache.copy()
    oracle.reshape_and_cache(case.k_new, case.v_new, k_ref, v_ref, case.slot_mapping, 16)
    blk = int(case.block_tables[1, 1])  # token 20 of sequence 1, kv head 0
    k_ref[blk, 0, 4, 7] = 0x7FC0
    dc.k[blk, 0, 4, 7] = float("nan")
    ws = torch.empty(max(pa.pa_decode_workspace_size(3, 4, 2, 128, 16, 70, pt), 16), dtype=torch.uint8,
                     device="cuda")
    pa.pa_decode(dc.out, dc.q, dc.k, dc.v, dc.tables, dc.lens, max_seq_len=70, scale=float(case.scale),
                 partition_tokens=pt, workspace=ws, err_flag=dc.flag)
    torch.cuda.synchronize()
    got = dc.out.cpu().numpy().astype(np.float64)
    want = oracle.decode(case.q, k_ref, v_ref, case.block_tables, case.seq_lens, num_kv_heads=2, block_size=16,
                         scale=case.scale)
    assert np.all(np.isnan(want[1, :2])) and np.all(np.isnan(got[1, :2]))
    assert np.all(got[0] == 0)
    assert_close(got[1, 2:], want[1, 2:], "other kv head")
    assert_close(got[2], want[2], "other sequence")


def test_kernels_are_native_launches():
    import paged_kv_cache_349_b200 as pa
    before = pa.launch_count()
    case = W.make_case(1)
    run_step(DeviceCase(case), -1)
    assert pa.launch_count() - before == 2  # reshape + decode (no copy pairs in the tiny case)


# ---------------------------------------------------------------------------
# Full-size workloads, sampled rows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("cfg,n_rows", [(2, 96), (3, 96), (4, 96), (5, 24)])
def test_full_size_workload_sampled_rows(cfg, n_rows):
    case = W.make_case(cfg)
    rows = sample_rows(case, n_rows, seed=cfg)
    (mx, mean), dc, _ = _check_step(case, rows=rows, what=f"cfg{cfg} full")
