"""The C++ block allocator against the oracle's allocator model and the pages' examples.

The pages let an allocator hand out *any* free block, so the comparison is on
what every correct allocator agrees on: token counts, block counts, which
appends need a copy, refcount multisets, free-pool size, and -- checked by
replaying the token contents through the tables -- that every sequence reads
back exactly its own tokens.
"""
import numpy as np
import pytest

import oracle
import paged_kv_cache_349_b200 as pa
import workloads as W


def test_page_example_33_tokens():
    a = pa.Allocator(8, 16)
    s = a.create()
    slots = [a.append(s)[0] for _ in range(33)]
    table, n = a.block_table(s)
    assert n == 33 and len(table) == 3 and a.num_free() == 5
    assert slots == [int(table[p // 16]) * 16 + p % 16 for p in range(33)]
    assert oracle.last_block_slack(n, 16) == 15
    s2 = a.create()
    for _ in range(32):
        a.append(s2)
    assert len(a.block_table(s2)[0]) == 2


def test_ordered_pool_deals_in_order():
    order = np.random.default_rng(0).permutation(20).astype(np.int32)
    a = pa.Allocator(20, 16, order=order)
    s = a.create()
    for _ in range(40):
        a.append(s)
    assert list(a.block_table(s)[0]) == list(order[:3])


def test_fork_cow_and_in_place_write():
    a = pa.Allocator(8, 16)
    p = a.create()
    for _ in range(20):
        a.append(p)
    c = a.fork(p)
    b0, b1 = a.block_table(p)[0]
    assert a.refcount(b0) == 2 and a.refcount(b1) == 2
    slot, cow = a.append(c)
    assert cow is not None and cow[0] == b1 and slot == cow[1] * 16 + 4
    assert a.refcount(b1) == 1 and a.refcount(cow[1]) == 1
    slot, cow = a.append(p)
    assert cow is None and slot == b1 * 16 + 4


def test_n4_sampling_prompt_stored_once():
    a = pa.Allocator(64, 16)
    root = a.create()
    for _ in range(500):
        a.append(root)
    members = [root] + [a.fork(root) for _ in range(3)]
    assert a.num_free() == 64 - 32
    slots, pairs = a.append_batch(members[1:] + [root])
    assert pairs.shape == (3, 2)
    assert a.num_free() == 64 - 35


def test_oom_leaves_state_unchanged():
    a = pa.Allocator(2, 16)
    s = a.create()
    for _ in range(32):
        a.append(s)
    with pytest.raises(pa.PaError) as e:
        a.append(s)
    assert e.value.status == pa.PA_ERR_OOM
    assert a.block_table(s)[1] == 32
    # batched append is all-or-nothing
    b = pa.Allocator(3, 8)
    x, y = b.create(), b.create()
    for _ in range(8):
        b.append(x)
    for _ in range(7):
        b.append(y)
    before = (b.block_table(x), b.block_table(y), b.num_free())
    b.append(y)                     # y fills its block
    z = b.fork(x)                   # x's block now shared
    free_before = b.num_free()
    with pytest.raises(pa.PaError):
        b.append_batch([x, y, z, y])  # needs 1 (x new) + 1 (y new) + 1 (z new) + ... > free
    assert b.num_free() == free_before
    assert b.block_table(x)[1] == 8 and b.block_table(y)[1] == 8 and b.block_table(z)[1] == 8
    del before


def test_bad_ids():
    a = pa.Allocator(4, 16)
    with pytest.raises(pa.PaError) as e:
        a.append(7)
    assert e.value.status == pa.PA_ERR_BAD_INDEX
    s = a.create()
    a.free(s)
    with pytest.raises(pa.PaError):
        a.free(s)                   # double free
    assert a.refcount(-1) == -1 and a.refcount(4) == -1


def test_export_pads_tables():
    a = pa.Allocator(16, 16)
    s1, s2 = a.create(), a.create()
    for _ in range(17):
        a.append(s1)
    a.append(s2)
    t, lens = a.export([s1, s2], max_blocks=3, pad=-7)
    assert list(lens) == [17, 1]
    assert t[0, 2] == -7 and t[1, 1] == -7 and t[1, 2] == -7
    assert list(t[0, :2]) == list(a.block_table(s1)[0])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_ops_match_model(seed):
    """Random create/append/batch-append/fork/free on the C++ allocator and the model."""
    rng = np.random.default_rng(seed)
    bs, NB = 8, 40
    a = pa.Allocator(NB, bs)
    m = oracle.AllocModel(NB, bs)
    ids = {}                 # product id -> model id
    content = {}             # slot -> token value (product pool contents)
    expect = {}              # product id -> token list
    val = 0

    def write(slot):
        nonlocal val
        val += 1
        content[slot] = val
        return val

    def apply_copy(src, dst):
        for r in range(bs):
            if src * bs + r in content:
                content[dst * bs + r] = content[src * bs + r]

    for step in range(1500):
        live = list(ids)
        r = rng.random()
        if r < 0.06 or not live:
            s = a.create()
            ids[s] = m.create()
            expect[s] = []
        elif r < 0.12:
            p = int(rng.choice(live))
            c = a.fork(p)
            ids[c] = m.fork(ids[p])
            expect[c] = list(expect[p])
        elif r < 0.18:
            s = int(rng.choice(live))
            a.free(s)
            m.free_seq(ids.pop(s))
            del expect[s]
        elif r < 0.3:
            batch = [int(x) for x in rng.choice(live, size=min(len(live), 4), replace=False)]
            free0 = a.num_free()
            try:
                slots, pairs = a.append_batch(batch)
            except pa.PaError as e:
                assert e.status == pa.PA_ERR_OOM and a.num_free() == free0
                with pytest.raises(oracle.OutOfBlocks):
                    snapshot = (list(m.free), list(m.ref), {k: list(v) for k, v in m.tables.items()}, dict(m.ntok))
                    try:
                        for s in batch:
                            m.append(ids[s])
                    finally:
                        m.free, m.ref = snapshot[0], snapshot[1]
                        m.tables, m.ntok = snapshot[2], snapshot[3]
                continue
            mc = [m.append(ids[s])[1] for s in batch]
            assert len(pairs) == sum(c is not None for c in mc)
            for src, dst in pairs:
                apply_copy(src, dst)
            for s, slot in zip(batch, slots):
                expect[s].append(write(int(slot)))
        else:
            s = int(rng.choice(live))
            try:
                slot, cow = a.append(s)
            except pa.PaError as e:
                assert e.status == pa.PA_ERR_OOM
                with pytest.raises(oracle.OutOfBlocks):
                    m.append(ids[s])
                continue
            _, mcow = m.append(ids[s])
            assert (cow is None) == (mcow is None)
            if cow is not None:
                apply_copy(*cow)
            expect[s].append(write(slot))
        # policy-free agreement
        assert a.num_free() == m.num_free()
        for s, ms in ids.items():
            table, n = a.block_table(s)
            assert n == m.ntok[ms] and len(table) == len(m.tables[ms])
            got = [content.get(int(table[p // bs]) * bs + p % bs) for p in range(n)]
            assert got == expect[s]
        prod_refs = sorted(a.refcount(b) for b in range(NB))
        assert prod_refs == sorted(m.ref)


def test_replays_generator_placement():
    """Dealing blocks in the generator's order reproduces its tables exactly."""
    case = W.make_case(2, batch=5, max_len=100, num_blocks=64)
    a = pa.Allocator(case.num_blocks, case.block_size, order=case.free_order)
    sids = [a.create() for _ in range(case.batch)]
    for s, L in zip(sids, case.seq_lens):
        for _ in range(int(L)):
            a.append(s)
    t, lens = a.export(sids, case.max_blocks_per_seq)
    assert np.array_equal(lens, case.seq_lens)
    for b, L in enumerate(case.seq_lens):
        n = -(-int(L) // case.block_size)
        assert np.array_equal(t[b, :n], case.block_tables[b, :n])


def _twin_allocators(seed):
    """Two allocators in the same state: sequences with random lengths, some forked (shared blocks)."""
    rng = np.random.default_rng(seed)
    twins = [pa.Allocator(600, 16), pa.Allocator(600, 16)]
    ids = []
    for a in twins:
        r = np.random.default_rng(seed)
        got = []
        for _ in range(6):
            s = a.create()
            for _ in range(int(r.integers(0, 70))):
                a.append(s)
            got.append(s)
            if r.random() < 0.5:
                got.append(a.fork(s))
        ids.append(np.array(got, np.int32))
    assert np.array_equal(ids[0], ids[1])
    return twins, ids[0], rng


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_alloc_step_equals_append_batch_then_export(seed):
    """pa_alloc_step == pa_seq_append_batch followed by pa_alloc_export, step after step, forks and
    copies on write included."""
    (a, b), ids, _ = _twin_allocators(seed)
    n, max_blocks = ids.size, 12
    tables = np.zeros((n, max_blocks), np.int32)
    lens = np.zeros(n, np.int32)
    pairs = np.zeros((n, 2), np.int32)
    step = a.step_fn(ids, tables, lens, pairs)
    saw_copy = False
    for _ in range(40):
        n_cow, max_len = step()
        _, want_pairs = b.append_batch(ids)
        want_t, want_l = b.export(ids, max_blocks)
        assert np.array_equal(tables, want_t) and np.array_equal(lens, want_l)
        assert n_cow == want_pairs.shape[0] and np.array_equal(pairs[:n_cow], want_pairs)
        assert max_len == int(want_l.max())
        assert a.num_free() == b.num_free()
        saw_copy |= n_cow > 0
    assert saw_copy  # the forks made some appends copy
    a.close(), b.close()


def test_alloc_step_all_or_nothing():
    """A table that would outgrow max_blocks, or a pool that runs dry, leaves the allocator as it was."""
    a = pa.Allocator(5, 16)
    s1, s2 = a.create(), a.create()
    for _ in range(32):
        a.append(s1)                        # 2 full blocks: the next append needs a third
    a.append(s2)
    ids = np.array([s2, s1], np.int32)
    tables = np.zeros((2, 2), np.int32)
    lens = np.zeros(2, np.int32)
    pairs = np.zeros((2, 2), np.int32)
    before = (a.num_free(), a.block_table(s1), a.block_table(s2))
    with pytest.raises(RuntimeError, match="PA_ERR_INVALID_ARG"):
        a.step_fn(ids, tables, lens, pairs)()
    after = (a.num_free(), a.block_table(s1), a.block_table(s2))
    assert before[0] == after[0] and all(np.array_equal(x[0], y[0]) and x[1] == y[1]
                                         for x, y in zip(before[1:], after[1:]))
    # pool of 5: s1 holds 2, s2 holds 1; a fork of s1 then 3 appends each need fresh blocks
    c = a.fork(s1)
    ids = np.array([s1, c, s2], np.int32)
    tables = np.zeros((3, 8), np.int32)
    lens = np.zeros(3, np.int32)
    pairs = np.zeros((3, 2), np.int32)
    step = a.step_fn(ids, tables, lens, pairs)
    step()                                  # s1 -> new block 3, c -> new block 4: pool empty
    free = a.num_free()
    assert free == 0
    snap = [a.block_table(x) for x in (s1, c, s2)]
    for _ in range(14):
        step()                              # s2 fills its block (16 tokens); s1, c write in place
    with pytest.raises(RuntimeError, match="PA_ERR_OOM"):
        step()                              # s1 and c append in place, then s2 needs a block: none left
    assert a.num_free() == 0
    assert [a.block_table(x)[1] for x in (s1, c, s2)] == [snap[0][1] + 14, snap[1][1] + 14, snap[2][1] + 14]
    a.close()


def test_validate_tables_accepts_workloads_and_locates_corruption():
    case = W.make_case(2, batch=6, max_len=300, num_blocks=256)
    t, L, NB, bs = case.block_tables, case.seq_lens, case.num_blocks, case.block_size
    assert pa.validate_tables(t, L, NB, bs) is None
    chat = W.make_case(3, batch=8, max_len=260, num_blocks=512)  # rows share prefix blocks: allowed
    assert pa.validate_tables(chat.block_tables, chat.seq_lens, chat.num_blocks, chat.block_size) is None
    used = (L + bs - 1) // bs
    b = int(np.argmax(used >= 2))
    bad = t.copy()
    bad[b, used[b] - 1] = NB                      # id out of range in the last attended entry
    assert pa.validate_tables(bad, L, NB, bs) == (b, int(used[b]) - 1)
    bad = t.copy()
    bad[b, 1] = bad[b, 0]                         # a block twice in one row
    assert pa.validate_tables(bad, L, NB, bs) == (b, 1)
    bad = t.copy()
    bad[b, 0] = -1                                # padding value where a block is needed
    assert pa.validate_tables(bad, L, NB, bs) == (b, 0)
    long_l = L.copy()
    long_l[4] = t.shape[1] * bs + 1               # longer than its row can hold
    assert pa.validate_tables(t, long_l, NB, bs) == (4, -1)
    pad = t.copy()
    pad[0, used[0]:] = -7                         # entries past the attended ones are never read
    assert pa.validate_tables(pad, L, NB, bs) is None
    assert pa.validate_tables(np.zeros((0, 4), np.int32), np.zeros(0, np.int32), NB, bs) is None


@pytest.mark.parametrize("cfg,kw", [
    (2, dict(batch=6, max_len=300, num_blocks=256)),
    (3, dict(batch=8, max_len=260, num_blocks=512)),
    (5, dict(batch=2, max_len=2048, num_blocks=640, num_copy_pairs=0)),
])
def test_bench_e2e_host_state_matches_workload(cfg, kw):
    """The bench's e2e leg rebuilds the pre-append state with the allocator and runs pa_alloc_step:
    the step's lengths are the workload's, every table it exports is valid, and max_seq_len is the
    longest length.  (Placement may differ from the generator's for a token that opens a block:
    the allocator deals that block at step time.)"""
    import bench
    case = W.make_case(cfg, **kw)
    alloc, sids = bench.replay_allocator(pa, case)
    B, mb = case.batch, case.block_tables.shape[1]
    tables = np.zeros((B, mb), np.int32)
    lens = np.zeros(B, np.int32)
    pairs = np.zeros((B, 2), np.int32)
    n_pairs, max_len = alloc.step_fn(sids, tables, lens, pairs)()
    assert np.array_equal(lens, case.seq_lens)
    assert max_len == int(case.seq_lens.max())
    assert pa.validate_tables(tables, lens, case.num_blocks, case.block_size) is None
    assert n_pairs == 0  # copy-on-write already happened while the state was rebuilt
    alloc.close()


def test_create_rejects_sizes_the_kernels_cannot_address():
    """Slot ids are int32 (block * block_size + row): a pool whose slots overflow int32 is refused,
    and so is a block size the kernels do not support; neither creates an allocator."""
    for nb, bs in ((1 << 27, 16), ((1 << 31) // 16 + 1, 16), (8, 4), (8, 12), (8, 128)):
        with pytest.raises(pa.PaError) as e:
            pa.Allocator(nb, bs)
        assert e.value.status in (pa.PA_ERR_INVALID_ARG, pa.PA_ERR_UNSUPPORTED)
    # the largest pool whose slots still fit int32
    a = pa.Allocator((1 << 31) // 64 - 1, 64)
    s = a.create()
    slot, _ = a.append(s)
    assert 0 <= slot < (1 << 31)
    a.close()
