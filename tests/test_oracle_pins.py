"""Pins for the fp64 oracle: what the pages print, closed forms, invariants, brute force.

Each test is chosen so that a plausible slip in the oracle (a dropped scale, a
sign, a swapped index, a transposed operand, a wrong head mapping, an
off-by-one in the sequence length) fails at least one of them.
"""
import math

import numpy as np
import pytest

import oracle
import workloads as W


# ---------------------------------------------------------------------------
# bf16 decoding
# ---------------------------------------------------------------------------

def test_bf16_widening_known_patterns():
    pats = {0x3F80: 1.0, 0xC000: -2.0, 0x3FC0: 1.5, 0x4049: 3.140625, 0x0000: 0.0,
            0x8000: -0.0, 0x0001: 2.0 ** -133, 0x7F7F: (2 - 2 ** -7) * 2.0 ** 127,
            0x3E00: 0.125, 0xBF00: -0.5}
    got = oracle.bf16_to_f64(np.array(list(pats.keys()), dtype=np.uint16))
    assert list(got) == list(pats.values())
    assert math.isinf(oracle.bf16_to_f64(np.array([0x7F80], np.uint16))[0])
    assert math.isnan(oracle.bf16_to_f64(np.array([0x7FC0], np.uint16))[0])


def test_bf16_rounding_of_generator_is_nearest_even():
    # 1 + 2^-8 is exactly half-way between bf16 1.0 and 1+2^-7: ties go to even (1.0).
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.5, 1.0 + 2 ** -9], dtype=np.float32)
    assert list(W.bf16_bits(x)) == [0x3F80, 0x3F82, 0xBFC0, 0x3F80]


# ---------------------------------------------------------------------------
# Page arithmetic, from the golden fixture
# ---------------------------------------------------------------------------

def test_block_count_and_slack(golden):
    for e in golden["block_count_and_slack"]:
        assert oracle.blocks_needed(e["tokens"], e["block_size"]) == e["blocks"], e["cite"]
        if "slack" in e:
            assert oracle.last_block_slack(e["tokens"], e["block_size"]) == e["slack"], e["cite"]


def test_max_slack_is_block_size_minus_one(golden):
    for e in golden["max_slack"]:
        bs = e["block_size"]
        worst = max(oracle.last_block_slack(n, bs) for n in range(1, 10 * bs))
        assert worst == e["max_slack"] == bs - 1


def test_naive_waste(golden):
    for e in golden["naive_waste"]:
        w = 100 * oracle.naive_waste(e["used"], e["reserved"])
        if "percent" in e:
            assert w == e["percent"]
            assert e["reserved"] - e["used"] == e["empty_tokens"]
        else:
            assert math.floor(w) == e["percent_floor"], e["cite"]


def test_capacity_worked_example(golden):
    ex, model = golden["capacity"]
    # 2 (K,V) x 40 layers x 40 heads x 128 x 2 bytes = 819,200 B = 0.78125 MiB, printed as 0.78 MB
    b = oracle.kv_bytes_per_token(model["num_layers"], model["num_kv_heads"], model["head_dim"], model["elem_bytes"])
    assert b == 819200
    assert round(b / 2 ** 20, 2) == model["mb_per_token_printed"]
    naive = oracle.max_concurrent_requests(ex["kv_gb"], ex["mb_per_token"], ex["naive_tokens"])
    paged = oracle.max_concurrent_requests(ex["kv_gb"], ex["mb_per_token"], ex["paged_tokens"])
    assert (naive, paged) == (ex["naive_requests"], ex["paged_requests"])
    assert round(ex["mb_per_token"] * ex["naive_tokens"] / 1024, 2) == ex["naive_gb_per_request"]
    assert round(ex["mb_per_token"] * ex["paged_tokens"] / 1024, 3) == ex["paged_gb_per_request"]
    assert round(paged / naive) == ex["ratio_printed"]


def test_chat_workload_arithmetic(golden):
    e = golden["chat_workload"][0]
    bs = e["block_size"]
    per_req = oracle.blocks_needed(e["avg_prompt"], bs) + oracle.blocks_needed(e["avg_gen"], bs)
    assert per_req == e["blocks_per_request"]
    assert e["users"] * per_req == e["peak_blocks"]
    assert bs * e["mb_per_token"] == e["mb_per_block"]
    assert round(e["peak_blocks"] * e["mb_per_block"] / 1000) == e["kv_gb_printed"]
    shared = oracle.blocks_needed(e["shared_prompt_tokens"], bs)
    assert shared == e["shared_blocks"]
    # The shared prompt is stored once instead of once per user.
    m = oracle.AllocModel(num_blocks=shared * 2, block_size=bs)
    root = m.create()
    for _ in range(e["shared_prompt_tokens"]):
        m.append(root)
    for _ in range(e["users"] - 1):
        m.fork(root)
    assert m.blocks_in_use() == e["shared_blocks"]
    saved_mb = shared * (e["users"] - 1) * e["mb_per_block"]
    assert round(saved_mb / 1000) == e["savings_gb_printed"]


# ---------------------------------------------------------------------------
# Attention core: closed forms on tiny inputs
# ---------------------------------------------------------------------------

def _pool_case(lens, Hq, Hkv, d, bs, NB, seed, fill=W.BF16_QNAN):
    """A small paged case with scattered placement; unaddressed rows poisoned."""
    rng = np.random.default_rng(seed)
    nblk = [-(-L // bs) for L in lens]
    ids = rng.choice(NB, size=sum(nblk), replace=False)
    maxb = max(max(nblk), 1)
    unused = np.setdiff1d(np.arange(NB), ids)
    tables = np.full((len(lens), maxb), unused[0] if unused.size else -1, dtype=np.int32)
    c = 0
    for b, n in enumerate(nblk):
        tables[b, :n] = ids[c:c + n]
        c += n
    k = np.full((NB, Hkv, bs, d), fill, np.uint16)
    v = np.full((NB, Hkv, bs, d), fill, np.uint16)
    for b, L in enumerate(lens):
        for p in range(L):
            blk = tables[b, p // bs]
            k[blk, :, p % bs, :] = W.bf16_normal(rng, (Hkv, d))
            v[blk, :, p % bs, :] = W.bf16_normal(rng, (Hkv, d))
    q = W.bf16_normal(rng, (len(lens), Hq, d))
    return q, k, v, tables, np.array(lens, np.int32)


def test_single_token_returns_its_value_exactly():
    q, k, v, t, lens = _pool_case([1, 1], Hq=2, Hkv=1, d=8, bs=4, NB=6, seed=1)
    out = oracle.decode(q, k, v, t, lens, num_kv_heads=1, block_size=4, scale=0.125)
    for b in range(2):
        v0 = oracle.bf16_to_f64(v[t[b, 0], 0, 0])
        for g in range(2):
            assert np.array_equal(out[b, g], v0)


def test_zero_query_gives_mean_of_values():
    q, k, v, t, lens = _pool_case([7, 16, 9], Hq=2, Hkv=2, d=8, bs=4, NB=16, seed=2)
    q[:] = 0
    out = oracle.decode(q, k, v, t, lens, num_kv_heads=2, block_size=4, scale=0.3)
    for b, L in enumerate(lens):
        for h in range(2):
            rows = np.stack([oracle.bf16_to_f64(v[t[b, p // 4], h, p % 4]) for p in range(L)])
            np.testing.assert_allclose(out[b, h], rows.mean(axis=0), rtol=0, atol=1e-15)


def test_equal_keys_give_mean_of_values():
    q, k, v, t, lens = _pool_case([11], Hq=1, Hkv=1, d=8, bs=4, NB=5, seed=3)
    row = W.bf16_normal(np.random.default_rng(33), (8,))
    for p in range(11):
        k[t[0, p // 4], 0, p % 4] = row
    out = oracle.decode(q, k, v, t, lens, num_kv_heads=1, block_size=4, scale=1.0)
    rows = np.stack([oracle.bf16_to_f64(v[t[0, p // 4], 0, p % 4]) for p in range(11)])
    np.testing.assert_allclose(out[0, 0], rows.mean(axis=0), rtol=0, atol=1e-15)


@pytest.mark.parametrize("G", [1, 2])
def test_dominant_key_selects_its_value_at_every_position(G):
    """One key scores 64 above all others: the output is that position's value.

    Run for every logical position, across block boundaries and into the
    partial last block, with scattered blocks and a distinct winning
    position per kv head -- this pins the table dereference, the row offset
    and the query-head -> kv-head mapping (g -> g // G).
    """
    bs, d, L, Hkv = 4, 8, 11, 2
    Hq = Hkv * G
    q, k, v, t, lens = _pool_case([L], Hq=Hq, Hkv=Hkv, d=d, bs=bs, NB=9, seed=4)
    q[:] = 0
    q[0, :, 0] = 0x4100  # 8.0
    for star in range(L):
        kk = k.copy()
        for p in range(L):
            kk[t[0, p // bs], :, p % bs, :] = 0
        star_of = [(star + 3 * h) % L for h in range(Hkv)]
        for h in range(Hkv):
            p = star_of[h]
            kk[t[0, p // bs], h, p % bs, 0] = 0x4100  # 8.0 -> score 64 at scale 1
        out = oracle.decode(q, kk, v, t, lens, num_kv_heads=Hkv, block_size=bs, scale=1.0)
        for g in range(Hq):
            h = g // G
            p = star_of[h]
            want = oracle.bf16_to_f64(v[t[0, p // bs], h, p % bs])
            np.testing.assert_allclose(out[0, g], want, rtol=0, atol=1e-20)


def test_two_tokens_logistic_closed_form():
    d, scale = 4, 0.125
    q = np.zeros((1, 1, d), np.uint16)
    q[0, 0, 0] = 0x4000  # 2.0
    k = np.zeros((2, 1, 1, d), np.uint16)
    v = np.zeros((2, 1, 1, d), np.uint16)
    k[0, 0, 0, 0] = 0x3F80   # +1 -> score 2*scale
    k[1, 0, 0, 0] = 0xBF80   # -1 -> score -2*scale
    v[0, 0, 0] = [0x3F80, 0x4000, 0x0000, 0xBF80]  # 1, 2, 0, -1
    v[1, 0, 0] = [0x4040, 0x0000, 0x3F00, 0x3F80]  # 3, 0, 0.5, 1
    # block size 1: token p lives in block p
    t = np.array([[0, 1]], np.int32)
    out = oracle.decode(q, k, v, t, np.array([2], np.int32), num_kv_heads=1, block_size=1, scale=scale)
    sig = 1.0 / (1.0 + math.exp(-4 * scale))
    want = sig * np.array([1, 2, 0, -1.0]) + (1 - sig) * np.array([3, 0, 0.5, 1.0])
    np.testing.assert_allclose(out[0, 0], want, rtol=0, atol=1e-15)


def test_three_tokens_known_weights():
    # scores (0, ln 2, ln 3) -> weights 1:2:3
    q = np.array([1.0])
    K = np.array([[0.0], [math.log(2)], [math.log(3)]])
    V = np.array([[6.0], [-3.0], [2.0]])
    out = oracle.attend(q, K, V, scale=1.0)
    assert abs(out[0] - (6 - 6 + 6) / 6.0) < 1e-15


def test_empty_sequence_gives_zero_row():
    q, k, v, t, lens = _pool_case([0, 3], Hq=1, Hkv=1, d=8, bs=4, NB=4, seed=5)
    out = oracle.decode(q, k, v, t, lens, num_kv_heads=1, block_size=4, scale=0.5)
    assert np.all(out[0] == 0)
    assert np.all(np.isfinite(out[1]))


def test_matches_library_softmax_on_random_small_cases():
    from scipy.special import softmax
    rng = np.random.default_rng(6)
    for L in (1, 2, 5, 37):
        q = rng.standard_normal(16)
        K = rng.standard_normal((L, 16))
        V = rng.standard_normal((L, 16))
        want = softmax(0.25 * (K @ q)) @ V
        np.testing.assert_allclose(oracle.attend(q, K, V, 0.25), want, rtol=1e-13, atol=1e-14)


def test_gqa_head_mapping_constant_values():
    """Every value of kv head h equals h+1, so query head g must return g//G + 1."""
    Hq, Hkv, d, bs = 8, 2, 4, 4
    q, k, v, t, lens = _pool_case([9, 5], Hq=Hq, Hkv=Hkv, d=d, bs=bs, NB=8, seed=7)
    for b, L in enumerate(lens):
        for p in range(L):
            for h in range(Hkv):
                v[t[b, p // bs], h, p % bs, :] = W.bf16_bits(np.full(d, h + 1.0, np.float32))
    out = oracle.decode(q, k, v, t, lens, num_kv_heads=Hkv, block_size=bs, scale=0.5)
    for g in range(Hq):
        np.testing.assert_allclose(out[:, g], g // (Hq // Hkv) + 1.0, rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# Layout independence
# ---------------------------------------------------------------------------

def test_paged_equals_contiguous_attention():
    """Scatter a contiguous [L, d] history into blocks with numpy reshapes; decode == attend."""
    rng = np.random.default_rng(8)
    L, d, bs, NB, Hkv = 37, 16, 8, 12, 1
    Kc = W.bf16_normal(rng, (L, d))
    Vc = W.bf16_normal(rng, (L, d))
    q = W.bf16_normal(rng, (1, 1, d))
    n = -(-L // bs)
    ids = rng.choice(NB, size=n, replace=False)
    pad = n * bs - L
    Kb = np.concatenate([Kc, np.full((pad, d), W.BF16_QNAN, np.uint16)]).reshape(n, bs, d)
    Vb = np.concatenate([Vc, np.full((pad, d), W.BF16_QNAN, np.uint16)]).reshape(n, bs, d)
    k = np.full((NB, Hkv, bs, d), W.BF16_QNAN, np.uint16)
    v = np.full((NB, Hkv, bs, d), W.BF16_QNAN, np.uint16)
    k[ids, 0] = Kb
    v[ids, 0] = Vb
    out = oracle.decode(q, k, v, ids.reshape(1, -1).astype(np.int32), np.array([L], np.int32),
                        num_kv_heads=1, block_size=bs, scale=0.25)
    want = oracle.attend(oracle.bf16_to_f64(q[0, 0]), oracle.bf16_to_f64(Kc), oracle.bf16_to_f64(Vc), 0.25)
    assert np.array_equal(out[0, 0], want)


def test_permutation_of_physical_blocks_is_invisible():
    case = W.make_case(2, batch=6, max_len=150, num_blocks=128)
    out_a, k_a, v_a = oracle.decode_step(case)
    assert np.all(np.isfinite(out_a))
    rng = np.random.default_rng(9)
    perm = rng.permutation(case.num_blocks)          # new id of old block i
    k_b = np.empty_like(k_a)
    v_b = np.empty_like(v_a)
    k_b[perm] = k_a
    v_b[perm] = v_a
    tables = case.block_tables.copy()
    valid = tables >= 0
    tables[valid] = perm[tables[valid]]
    out_b = oracle.decode(case.q, k_b, v_b, tables, case.seq_lens, num_kv_heads=case.num_kv_heads,
                          block_size=case.block_size, scale=case.scale)
    assert np.array_equal(out_a, out_b)


def test_shared_prefix_tables_match_unshared_copies():
    case = W.make_case(3, batch=8, max_len=120, num_blocks=256)
    out_shared, k, v = oracle.decode_step(case)
    assert np.all(np.isfinite(out_shared))
    # Give every sequence private copies of all its blocks.
    bs = case.block_size
    tables = case.block_tables.copy()
    k2 = np.full((k.shape[0] + tables.size, *k.shape[1:]), W.BF16_QNAN, np.uint16)
    v2 = np.full_like(k2, W.BF16_QNAN)
    k2[:k.shape[0]] = k
    v2[:v.shape[0]] = v
    nxt = k.shape[0]
    shared_seen = 0
    counts = np.bincount(np.concatenate([tables[b, :-(-int(L) // bs)] for b, L in enumerate(case.seq_lens)]))
    for b, L in enumerate(case.seq_lens):
        for j in range(-(-int(L) // bs)):
            old = tables[b, j]
            shared_seen += counts[old] > 1
            k2[nxt] = k[old]
            v2[nxt] = v[old]
            tables[b, j] = nxt
            nxt += 1
    assert shared_seen > 0, "the chat case must contain shared blocks"
    out_copy = oracle.decode(case.q, k2, v2, tables, case.seq_lens, num_kv_heads=case.num_kv_heads,
                             block_size=bs, scale=case.scale)
    assert np.array_equal(out_shared, out_copy)


def test_poisoned_slack_and_padding_stay_out():
    case = W.make_case(1)
    out, _, _ = oracle.decode_step(case)
    assert np.all(np.isfinite(out))
    assert out.shape == (4, 4, 64)


def test_row_subset_matches_full_decode():
    case = W.make_case(4, batch=5, max_len=100, num_blocks=64)
    full, _, _ = oracle.decode_step(case)
    rows = np.array([[4, 31], [0, 0], [2, 17]], np.int32)
    sub, _, _ = oracle.decode_step(case, rows=rows)
    for r, (b, g) in enumerate(rows):
        assert np.array_equal(sub[r], full[b, g])


# ---------------------------------------------------------------------------
# Cache write and block copy: literal tiny examples
# ---------------------------------------------------------------------------

def test_reshape_and_cache_literal():
    k = np.zeros((3, 2, 2, 2), np.uint16)
    v = np.zeros((3, 2, 2, 2), np.uint16)
    k_new = np.arange(1, 9, dtype=np.uint16).reshape(2, 2, 2)        # [T=2, Hkv=2, d=2]
    v_new = np.arange(11, 19, dtype=np.uint16).reshape(2, 2, 2)
    bad = oracle.reshape_and_cache(k_new, v_new, k, v, np.array([5, -1], np.int32), block_size=2)
    assert bad == 0
    want_k = np.zeros_like(k)
    want_k[2, 0, 1] = [1, 2]       # slot 5 = block 2, row 1; head 0 of token 0
    want_k[2, 1, 1] = [3, 4]       # head 1 of token 0
    want_v = np.zeros_like(v)
    want_v[2, 0, 1] = [11, 12]
    want_v[2, 1, 1] = [13, 14]
    assert np.array_equal(k, want_k) and np.array_equal(v, want_v)
    # slot 6 == NB*bs is out of range: reported, nothing written
    bad = oracle.reshape_and_cache(k_new, v_new, k, v, np.array([6, 0], np.int32), block_size=2)
    assert bad == 1
    want_k[0, 0, 0] = [5, 6]
    want_k[0, 1, 0] = [7, 8]
    assert np.array_equal(k, want_k)


def test_copy_blocks_literal():
    k = np.arange(4 * 1 * 2 * 2, dtype=np.uint16).reshape(4, 1, 2, 2)
    v = k + 100
    k0, v0 = k.copy(), v.copy()
    bad = oracle.copy_blocks(k, v, np.array([[1, 3], [1, 0]], np.int32))
    assert bad == 0
    want = k0.copy()
    want[3] = k0[1]
    want[0] = k0[1]
    assert np.array_equal(k, want)
    assert np.array_equal(v, want + 100)
    assert oracle.copy_blocks(k, v, np.array([[4, 0]], np.int32)) == 1


def test_swap_blocks_literal():
    dev_k = np.arange(3 * 1 * 2 * 2, dtype=np.uint16).reshape(3, 1, 2, 2)
    dev_v = dev_k + 50
    host_k = np.zeros((5, 1, 2, 2), np.uint16)
    host_v = np.zeros_like(host_k)
    assert oracle.swap_blocks(host_k, host_v, dev_k, dev_v, np.array([[2, 4], [0, 1]], np.int32)) == 0
    want = np.zeros_like(host_k)
    want[4] = [[[8, 9], [10, 11]]]
    want[1] = [[[0, 1], [2, 3]]]
    assert np.array_equal(host_k, want) and np.array_equal(host_v[[1, 4]], want[[1, 4]] + 50)
    assert not host_v[[0, 2, 3]].any()
    assert oracle.swap_blocks(host_k, host_v, dev_k, dev_v, np.array([[3, 0], [0, 5]], np.int32)) == 2


# ---------------------------------------------------------------------------
# Allocator model
# ---------------------------------------------------------------------------

def test_model_append_allocates_on_block_boundary(golden):
    m = oracle.AllocModel(num_blocks=8, block_size=16)
    s = m.create()
    slots = [m.append(s)[0] for _ in range(33)]
    assert len(m.tables[s]) == 3 and m.num_free() == 5
    b0, b1, b2 = m.tables[s]
    assert slots[:16] == [b0 * 16 + i for i in range(16)]
    assert slots[16:32] == [b1 * 16 + i for i in range(16)]
    assert slots[32] == b2 * 16
    assert 3 * 16 - 33 == 15


def test_model_fork_and_copy_on_write():
    m = oracle.AllocModel(num_blocks=8, block_size=16)
    p = m.create()
    for _ in range(20):
        m.append(p)
    c = m.fork(p)
    b0, b1 = m.tables[p]
    assert m.ref[b0] == 2 and m.ref[b1] == 2 and m.num_free() == 6
    slot, cow = m.append(c)
    assert cow is not None and cow[0] == b1
    new = cow[1]
    assert slot == new * 16 + 4
    assert m.tables[c] == [b0, new] and m.tables[p] == [b0, b1]
    assert m.ref[b1] == 1 and m.ref[new] == 1 and m.ref[b0] == 2
    # the last owner writes in place
    slot, cow = m.append(p)
    assert cow is None and slot == b1 * 16 + 4


def test_model_n4_sampling_stores_prompt_once():
    m = oracle.AllocModel(num_blocks=64, block_size=16)
    root = m.create()
    for _ in range(500):
        m.append(root)
    members = [root] + [m.fork(root) for _ in range(3)]
    assert m.blocks_in_use() == 32
    cows = [m.append(s)[1] for s in members[1:]] + [m.append(root)[1]]
    assert sum(c is not None for c in cows) == 3 and cows[-1] is None
    assert m.blocks_in_use() == 35


def test_model_free_returns_blocks_and_oom_keeps_state():
    m = oracle.AllocModel(num_blocks=2, block_size=16)
    s = m.create()
    for _ in range(32):
        m.append(s)
    with pytest.raises(oracle.OutOfBlocks):
        m.append(s)
    assert m.ntok[s] == 32 and len(m.tables[s]) == 2
    c = m.fork(s)
    m.free_seq(s)
    assert m.num_free() == 0
    m.free_seq(c)
    assert m.num_free() == 2


def test_model_logical_views_survive_sharing():
    """Random create/append/fork/free; every sequence reads back exactly its own tokens."""
    rng = np.random.default_rng(10)
    bs, NB = 4, 48
    m = oracle.AllocModel(num_blocks=NB, block_size=bs, order=rng.permutation(NB))
    content = {}            # slot -> token value
    expect = {}             # sid -> list of token values
    val = 0
    for step in range(3000):
        live = list(m.tables)
        r = rng.random()
        try:
            if r < 0.05 or not live:
                sid = m.create()
                expect[sid] = []
            elif r < 0.12:
                parent = int(rng.choice(live))
                sid = m.fork(parent)
                expect[sid] = list(expect[parent])
            elif r < 0.2:
                sid = int(rng.choice(live))
                m.free_seq(sid)
                del expect[sid]
            else:
                sid = int(rng.choice(live))
                slot, cow = m.append(sid)
                if cow is not None:
                    for row in range(bs):
                        if cow[0] * bs + row in content:
                            content[cow[1] * bs + row] = content[cow[0] * bs + row]
                val += 1
                content[slot] = val
                expect[sid].append(val)
        except oracle.OutOfBlocks:
            pass
        for sid, toks in expect.items():
            got = [content.get(m.tables[sid][p // bs] * bs + p % bs) for p in range(len(toks))]
            assert got == toks
        used = {b for t in m.tables.values() for b in t}
        assert len(used) + m.num_free() == NB
        for b in range(NB):
            assert m.ref[b] == sum(t.count(b) for t in m.tables.values())


# ---------------------------------------------------------------------------
# fp8 (E4M3) pools
# ---------------------------------------------------------------------------

def test_e4m3_known_codes():
    # worked by hand from the format: sign | exponent (bias 7) | 3-bit mantissa
    table = {1.0: 0x38, 0.5: 0x30, 448.0: 0x7E, -2.0: 0xC0, 2.0 ** -9: 0x01, 2.0 ** -6: 0x08,
             7 * 2.0 ** -9: 0x07, 240.0: 0x77, 30.0: 0x5F, 0.0: 0x00, 1.125: 0x39, -448.0: 0xFE}
    assert list(oracle.e4m3_code(list(table))) == list(table.values())
    assert list(oracle.e4m3_value(list(table.values()))) == list(table)


def test_e4m3_round_trip_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_value(codes)
    assert np.all(np.isfinite(vals))
    assert np.array_equal(oracle.e4m3_code(vals.astype(np.float32)), codes)
    assert np.isnan(oracle.e4m3_value([0x7F, 0xFF])).all()
    pos = vals[(codes < 0x80)]
    assert np.all(np.diff(pos) > 0) and pos.max() == 448.0


def test_e4m3_ties_to_even_and_nearest():
    codes = np.arange(0, 0x7E, dtype=np.uint8)           # adjacent finite positive pairs (c, c+1)
    lo = oracle.e4m3_value(codes)
    hi = oracle.e4m3_value(codes + 1)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)  # midpoints are exact in fp32
    even = np.where(codes % 2 == 0, codes, codes + 1).astype(np.uint8)
    assert np.array_equal(oracle.e4m3_code(mid), even)
    below = np.nextafter(mid, np.float32(0))
    above = np.nextafter(mid, np.float32(1000))
    assert np.array_equal(oracle.e4m3_code(below), codes)
    assert np.array_equal(oracle.e4m3_code(above), (codes + 1).astype(np.uint8))


def test_e4m3_saturates():
    big = np.array([448.5, 463.9, 464.0, 1e6, np.inf], np.float32)
    assert list(oracle.e4m3_code(big)) == [0x7E] * 5
    assert list(oracle.e4m3_code(-big)) == [0xFE] * 5


def test_quantize_uses_fp32_product():
    # inv = fp32(1/0.1) = 10.000000149...; 3 * inv in fp32 = 30.0000004 -> code of 30
    x = W.bf16_bits(np.array([3.0], np.float32))
    assert oracle.inv_scale(0.1) == np.float32(1) / np.float32(0.1)
    assert list(oracle.quantize_e4m3(x, 0.1)) == [0x5F]
    # 1.0625 * 1 is a tie between 1.0 and 1.125 -> even code 0x38
    assert list(oracle.quantize_e4m3(W.bf16_bits(np.array([1.0625], np.float32)), 1.0)) == [0x38]


def test_fp8_decode_equals_bf16_decode_on_dequantised_pool():
    """With a power-of-two scale the dequantised rows are exact bf16 values: both paths agree bitwise."""
    case = W.make_case(2, batch=4, max_len=90, num_blocks=64)
    _, k_pool, v_pool = oracle.decode_step(case)     # pools after the step's cache write
    k_codes = oracle.quantize_e4m3(k_pool, 0.5)
    v_codes = oracle.quantize_e4m3(v_pool, 0.25)
    # rebuild bf16 pools from the codes' values (exact in bf16 after scaling by a power of two)
    k_deq = W.bf16_bits((oracle.e4m3_value(k_codes) * 0.5).astype(np.float32))
    v_deq = W.bf16_bits((oracle.e4m3_value(v_codes) * 0.25).astype(np.float32))
    kw = dict(num_kv_heads=case.num_kv_heads, block_size=case.block_size, scale=case.scale)
    got = oracle.decode_fp8(case.q, k_codes, v_codes, case.block_tables, case.seq_lens, k_scale=0.5,
                            v_scale=0.25, **kw)
    want = oracle.decode(case.q, k_deq, v_deq, case.block_tables, case.seq_lens, **kw)
    finite = np.isfinite(want).all(axis=-1)  # rows never read poisoned slots
    assert finite.all()
    assert np.array_equal(got, want)
    # v_scale is linear in the output
    twice = oracle.decode_fp8(case.q, k_codes, v_codes, case.block_tables, case.seq_lens, k_scale=0.5,
                              v_scale=0.5, **kw)
    assert np.array_equal(twice, 2 * got)


def test_fp8_cache_write_literal():
    k = np.zeros((2, 1, 2, 2), np.uint8)
    v = np.zeros_like(k)
    k_new = W.bf16_bits(np.array([[[1.0, -2.0]]], np.float32))     # [T=1, Hkv=1, d=2]
    v_new = W.bf16_bits(np.array([[[448.0, 0.5]]], np.float32))
    assert oracle.reshape_and_cache_fp8(k_new, v_new, k, v, np.array([3], np.int32), 2, 1.0, 2.0) == 0
    # v: 448 / 2 = 224 = 1.75 * 2^7 -> 0x76; 0.5 / 2 = 0.25 -> 0x28
    assert list(k[1, 0, 1]) == [0x38, 0xC0] and list(v[1, 0, 1]) == [0x76, 0x28]
    assert not k[0].any() and not k[1, 0, 0].any()
