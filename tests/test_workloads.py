"""Structure of the seeded synthetic workloads (shapes, placement, sharing)."""
import numpy as np
import pytest

import workloads as W


def _used_blocks(case):
    bs = case.block_size
    return [case.block_tables[b, :-(-int(L) // bs)] for b, L in enumerate(case.seq_lens)]


def test_tiny_case_shape():
    c = W.make_case(1)
    assert list(c.seq_lens) == [1, 16, 33, 47]
    assert [len(u) for u in _used_blocks(c)] == [1, 1, 3, 3]
    ids = np.concatenate(_used_blocks(c))
    assert len(set(ids.tolist())) == 8 and ids.min() >= 0 and ids.max() < 32
    assert c.scale == np.float32(0.125)
    assert c.q.shape == (4, 4, 64) and c.k_cache.shape == (32, 2, 16, 64)
    assert c.k_new.shape == (4, 2, 64) and sorted(c.slot_mapping.tolist()) == sorted(
        (c.block_tables[b, (L - 1) // 16] * 16 + (L - 1) % 16) for b, L in enumerate(c.seq_lens))


def test_same_seed_same_case():
    a = W.make_case(2, batch=4, max_len=64, num_blocks=64)
    b = W.make_case(2, batch=4, max_len=64, num_blocks=64)
    assert np.array_equal(a.k_cache, b.k_cache) and np.array_equal(a.block_tables, b.block_tables)
    c = W.make_case(2, batch=4, max_len=64, num_blocks=64, seed=7)
    assert not np.array_equal(a.q, c.q)


@pytest.mark.parametrize("cfg", [2, 4, 5])
def test_private_blocks_are_distinct(cfg):
    c = W.make_case(cfg, batch=6, max_len=300, num_blocks=1024)
    ids = np.concatenate(_used_blocks(c))
    assert len(set(ids.tolist())) == ids.size
    assert ids.min() >= 0 and ids.max() < c.num_blocks


def test_chat_case_sharing_and_cow():
    c = W.make_case(3, batch=16, max_len=200, num_blocks=2048)
    bs = c.block_size
    used = _used_blocks(c)
    for g in range(4):
        S = int(c.shared_tokens[4 * g])
        full = S // bs
        tabs = [used[4 * g + m] for m in range(4)]
        for m in range(1, 4):
            assert np.array_equal(tabs[m][:full], tabs[0][:full])
        if S % bs:
            # members 0..2 hold private copies of the partial block, member 3 the original
            part = [t[full] for t in tabs]
            assert len(set(part)) == 4
            for m in range(3):
                assert [part[3], part[m]] in c.copy_pairs.tolist()
    assert c.copy_pairs.shape[1] == 2
    dsts = c.copy_pairs[:, 1]
    assert len(set(dsts.tolist())) == dsts.size
    assert not set(dsts.tolist()) & set(c.copy_pairs[:, 0].tolist())


def test_long_context_copy_pairs():
    c = W.make_case(5, batch=2, max_len=256, num_blocks=256, num_copy_pairs=10)
    used = set(np.concatenate(_used_blocks(c)).tolist())
    assert c.copy_pairs.shape == (10, 2)
    assert set(c.copy_pairs[:, 0].tolist()) <= used
    assert not set(c.copy_pairs[:, 1].tolist()) & used
    assert c.partition_tokens == 512


def test_gqa_lengths_lognormal_capped():
    L = W.gqa_lengths(np.random.default_rng(1004), 20000)
    assert L.min() >= 1 and L.max() <= 4096
    assert 750 < np.median(L) < 850
    assert 0.03 < np.mean(L == 4096) < 0.07
    c = W.make_case(4, batch=3, max_len=64, num_blocks=64)
    assert c.group_size == 4 and c.block_size == 32


def test_algorithmic_bytes():
    c = W.make_case(1)
    kv = 97 * 2 * 64 * 2 * 2
    assert W.algorithmic_decode_bytes(c) == kv + 4 * 4 * 64 * 2 + 4 * 4 * 64 * 4 + 8 * 4 + 4 * 4


@pytest.mark.parametrize("bs", [8, 32, 64])
def test_workload_2_repaged_keeps_lengths_and_pool_bytes(bs):
    """Re-paging the Llama-2-7B-shaped workload changes only the paging: the same lengths, the same
    pool bytes, every sequence's blocks distinct and in range, padding never read."""
    base = W.make_case(2, fill=W.BF16_ZERO, batch=16, max_len=600, num_blocks=2048)
    case = W.make_case(2, fill=W.BF16_ZERO, batch=16, max_len=600, num_blocks=2048 * 16 // bs, block_size=bs)
    assert case.block_size == bs
    assert np.array_equal(case.seq_lens, base.seq_lens)
    assert case.num_blocks * bs == base.num_blocks * 16
    used = []
    for b, L in enumerate(case.seq_lens):
        n = -(-int(L) // bs)
        row = case.block_tables[b, :n]
        assert np.all((row >= 0) & (row < case.num_blocks))
        used.extend(row.tolist())
    assert len(used) == len(set(used))
    with pytest.raises(ValueError):
        W.make_case(3, block_size=8)
