"""Seeded synthetic inputs for paged decode.

This module only *draws inputs*: lengths, physical block placement, bf16
query/key/value values, the new tokens of a decode step, their slot ids and
block-copy pairs.  It holds none of the attention arithmetic and none of the
allocator logic; both the CUDA path and the fp64 oracle consume what it
produces.  The one piece of addressing it needs to *encode* its inputs is the
slot id of a cached row, ``slot = physical_block * block_size + row``, which
is how a slot is defined in "Walk through paged attention end to end"
(zenaique.com, conceptual ``paged_attention_decode``: ``last_block`` and
``offset``); decoding a slot back into (block, row) is left to each consumer.

Workloads follow the five decode shapes of this library's test plan:

1. tiny: 4 seqs, lengths {1,16,33,47}, 4 q / 2 kv heads, d 64, bs 16, 32 blocks.
2. Llama-2-7B-shaped: 64 seqs, 32/32 heads, d 128, bs 16, lengths U{128..2048},
   16384-block pool, placement by a seeded permutation.
3. Llama-2-13B-shaped chat mix with n=4 sampling: 128 seqs = 32 groups of 4,
   40/40 heads, d 128, bs 16, length = prompt U{100..2000} (per group) +
   generated U{50..500} (per member); the first min(512, prompt) tokens of a
   group live in shared physical blocks; a partially filled shared block is
   copied-on-write by members 0..2 (member 3 keeps it), the copies arriving via
   ``copy_pairs``.
4. Llama-3-8B-shaped GQA: 256 seqs, 32/8 heads, d 128, bs 32, lengths
   lognormal(median 800, sigma 1.0) rounded and clamped to [1, 4096].
5. long context: 8 seqs x 32768 tokens, 64/8 heads, d 128, bs 16, split into
   512-token partitions, plus 1024 copy pairs (used block -> unused block).

Every decode step is "append, then attend" (zenaique.com conceptual code): the
pool handed out (``k_cache``/``v_cache``) holds every token before the last
one; the token at position ``L_b - 1`` of each sequence is delivered in
``k_new``/``v_new`` through ``slot_mapping`` (token order shuffled), and the
step applies ``copy_pairs`` first, then the cache write, then decode.

All values are bf16 bit patterns (``uint16``) rounded to nearest-even from
fp32 N(0,1) draws of ``numpy.random.default_rng(seed)``; default seed is
1000 + config number.  Unaddressed pool rows are filled with ``fill`` (a bf16
quiet NaN for parity runs, 0 for timing).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

BF16_QNAN = np.uint16(0x7FC0)
BF16_ZERO = np.uint16(0)

_CHUNK_ROWS = 1 << 16


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (nearest-even); return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_normal(rng: np.random.Generator, shape) -> np.ndarray:
    """bf16 bit patterns of N(0,1) fp32 draws."""
    return bf16_bits(rng.standard_normal(shape, dtype=np.float32))


@dataclasses.dataclass
class DecodeCase:
    """One decode step's inputs.  Arrays are host numpy; bf16 values are uint16 bits."""

    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: np.float32
    seq_lens: np.ndarray          # int32 [B]  (length after this step's append)
    block_tables: np.ndarray      # int32 [B, max_blocks]; unused entries are padding
    q: np.ndarray                 # uint16 [B, Hq, d]
    k_cache: np.ndarray           # uint16 [NB, Hkv, bs, d]  (state before the step)
    v_cache: np.ndarray           # uint16 [NB, Hkv, bs, d]
    k_new: np.ndarray             # uint16 [T, Hkv, d]
    v_new: np.ndarray             # uint16 [T, Hkv, d]
    slot_mapping: np.ndarray      # int32 [T]
    copy_pairs: np.ndarray        # int32 [n, 2]  (src, dst), applied before the write
    partition_tokens: int         # 0 = library default, -1 = single pass, >0 = split size
    seed: int
    # Placement bookkeeping (for the bench's allocator replay and for tests).
    free_order: Optional[np.ndarray] = None   # int32 [NB] order blocks were dealt in
    groups: Optional[np.ndarray] = None       # int32 [B] sharing group of each seq (cfg3)
    shared_tokens: Optional[np.ndarray] = None  # int32 [B] tokens shared within the group

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if self.seq_lens.size else 0

    @property
    def group_size(self) -> int:
        return self.num_q_heads // self.num_kv_heads


def _slots_of(tables: np.ndarray, b: np.ndarray, pos: np.ndarray, bs: int) -> np.ndarray:
    """Slot ids of logical positions ``pos`` of sequences ``b`` (input encoding only)."""
    return (tables[b, pos // bs].astype(np.int64) * bs + pos % bs).astype(np.int64)


def _fill_rows(pool: np.ndarray, slots: np.ndarray, rng: np.random.Generator, bs: int) -> None:
    """Write fresh N(0,1) bf16 values into every (block, row) named by ``slots``."""
    nb, hkv, _, d = pool.shape
    for start in range(0, slots.size, _CHUNK_ROWS):
        s = slots[start:start + _CHUNK_ROWS]
        vals = bf16_normal(rng, (s.size, hkv, d))
        pool[s // bs, :, s % bs, :] = vals


def _finish(name, rng, seed, *, Hq, Hkv, d, bs, NB, lens, tables, fill,
            skip_rows=None, late_rows=None, copy_pairs=None, partition_tokens=0,
            free_order=None, groups=None, shared_tokens=None,
            scale=None) -> DecodeCase:
    """Fill the pool with the tokens that precede this step and draw the step's inputs.

    ``tables`` must already be padded.  Rows listed in ``skip_rows`` (pairs of
    (seq, position)) are *not* pre-filled (they sit in a copy destination, which
    ``copy_pairs`` fills); those also listed in ``late_rows`` are delivered as new
    tokens of the step, written after the copy.
    """
    B = lens.shape[0]
    lens = lens.astype(np.int32)
    q = bf16_normal(rng, (B, Hq, d))
    k_cache = np.full((NB, Hkv, bs, d), fill, dtype=np.uint16)
    v_cache = np.full((NB, Hkv, bs, d), fill, dtype=np.uint16)

    # Positions already cached: 0 .. L_b-2 of every sequence.
    prev = np.maximum(lens - 1, 0)
    b_idx = np.repeat(np.arange(B), prev)
    p_idx = np.concatenate([np.arange(n) for n in prev]) if B else np.zeros(0, np.int64)
    new_b = [np.nonzero(lens > 0)[0]]
    new_p = [lens[lens > 0] - 1]
    if skip_rows is not None and len(skip_rows):
        # Remove (seq, pos) pairs that land in a copy destination block.
        key_all = b_idx.astype(np.int64) * (1 << 32) + p_idx
        key_skip = skip_rows[:, 0].astype(np.int64) * (1 << 32) + skip_rows[:, 1]
        keep = ~np.isin(key_all, key_skip)
        b_idx, p_idx = b_idx[keep], p_idx[keep]
    if late_rows is not None and len(late_rows):
        new_b.append(late_rows[:, 0])
        new_p.append(late_rows[:, 1])
    slots = np.unique(_slots_of(tables, b_idx, p_idx, bs))
    _fill_rows(k_cache, slots, rng, bs)
    _fill_rows(v_cache, slots, rng, bs)

    nb = np.concatenate(new_b).astype(np.int64)
    npos = np.concatenate(new_p).astype(np.int64)
    T = nb.size
    k_new = bf16_normal(rng, (T, Hkv, d))
    v_new = bf16_normal(rng, (T, Hkv, d))
    order = rng.permutation(T)
    k_new, v_new = k_new[order], v_new[order]
    slot_mapping = _slots_of(tables, nb[order], npos[order], bs).astype(np.int32)

    if copy_pairs is None:
        copy_pairs = np.zeros((0, 2), dtype=np.int32)
    if scale is None:
        scale = np.float32(1.0) / np.sqrt(np.float32(d))
    return DecodeCase(
        name=name, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d, block_size=bs,
        num_blocks=NB, scale=np.float32(scale), seq_lens=lens, block_tables=tables.astype(np.int32),
        q=q, k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
        slot_mapping=slot_mapping, copy_pairs=np.asarray(copy_pairs, dtype=np.int32).reshape(-1, 2),
        partition_tokens=partition_tokens, seed=seed, free_order=free_order,
        groups=groups, shared_tokens=shared_tokens)


def _deal_tables(lens: np.ndarray, order: np.ndarray, bs: int, max_blocks: int,
                 pad: np.ndarray) -> np.ndarray:
    """Give sequence 0 the first ceil(L_0/bs) blocks of ``order``, then sequence 1, ...

    Unused table entries take values from ``pad`` (cycled), e.g. -1 or ids of
    poisoned blocks.
    """
    B = lens.shape[0]
    tables = np.empty((B, max_blocks), dtype=np.int64)
    tables[:] = np.resize(pad, (B, max_blocks)) if pad.size else -1
    cursor = 0
    need = int((-(-lens // bs)).sum())
    if need > order.size:
        raise ValueError(f"pool of {order.size} blocks cannot hold {need} blocks of tables")
    for b in range(B):
        n = -(-int(lens[b]) // bs)
        tables[b, :n] = order[cursor:cursor + n]
        cursor += n
    return tables


def _padding_ids(order: np.ndarray, used: int, rng: np.random.Generator, poison_padding: bool) -> np.ndarray:
    """Padding values for table entries past a sequence's last block.

    With ``poison_padding`` the padding names real but unused (poisoned) blocks,
    so a kernel that reads past the last block pulls NaN into its output instead
    of tripping a bounds check; otherwise the padding is -1.
    """
    unused = order[used:]
    if poison_padding and unused.size:
        return rng.choice(unused, size=min(unused.size, 64), replace=False)
    return np.array([-1], dtype=np.int64)


def make_case(config: int, *, seed: Optional[int] = None, fill=BF16_QNAN,
              batch: Optional[int] = None, max_len: Optional[int] = None,
              num_blocks: Optional[int] = None, poison_padding: bool = True,
              num_copy_pairs: Optional[int] = None,
              partition_tokens: Optional[int] = None,
              block_size: Optional[int] = None) -> DecodeCase:
    """Build decode workload ``config`` (1..5).

    ``batch``/``max_len``/``num_blocks``/``num_copy_pairs`` shrink a workload
    (same recipe, smaller numbers) so the oracle can check every output.
    ``block_size`` (workload 2 only) re-pages the Llama-2-7B-shaped workload
    with another block size: the same lengths and pool bytes (the block count
    scales inversely), the blocks dealt from a fresh permutation.
    """
    if block_size is not None and config != 2:
        raise ValueError("block_size applies to workload 2 only")
    if seed is None:
        seed = 1000 + config
    rng = np.random.default_rng(seed)

    if config == 1:
        Hq, Hkv, d, bs, NB = 4, 2, 64, 16, 32 if num_blocks is None else num_blocks
        lens = np.array([1, 16, 33, 47], dtype=np.int64)
        if batch is not None:
            lens = lens[:batch]
        nblk = -(-lens // bs)
        chosen = rng.choice(NB, size=int(nblk.sum()), replace=False)
        rest = np.setdiff1d(np.arange(NB), chosen)
        order = np.concatenate([chosen, rest])
        max_blocks = int(nblk.max()) if lens.size else 1
        pad = _padding_ids(order, int(nblk.sum()), rng, poison_padding)
        tables = _deal_tables(lens, order, bs, max_blocks, pad)
        return _finish("tiny", rng, seed, Hq=Hq, Hkv=Hkv, d=d, bs=bs, NB=NB, lens=lens,
                       tables=tables, fill=fill, free_order=order.astype(np.int32),
                       scale=np.float32(1.0 / 8.0),
                       partition_tokens=-1 if partition_tokens is None else partition_tokens)

    if config == 2:
        Hq = Hkv = 32
        d = 128
        bs = 16 if block_size is None else block_size
        NB = 16384 * 16 // bs if num_blocks is None else num_blocks
        B = 64 if batch is None else batch
        hi = 2048 if max_len is None else max_len
        lo = min(128, hi)
        lens = rng.integers(lo, hi + 1, size=B)
        order = rng.permutation(NB)
        max_blocks = -(-hi // bs)
        used = int((-(-lens // bs)).sum())
        pad = _padding_ids(order, used, rng, poison_padding)
        tables = _deal_tables(lens, order, bs, max_blocks, pad)
        return _finish("llama2-7b", rng, seed, Hq=Hq, Hkv=Hkv, d=d, bs=bs, NB=NB, lens=lens,
                       tables=tables, fill=fill, free_order=order.astype(np.int32),
                       partition_tokens=0 if partition_tokens is None else partition_tokens)

    if config == 3:
        return _make_chat_case(rng, seed, fill=fill, batch=batch, max_len=max_len,
                               num_blocks=num_blocks, poison_padding=poison_padding,
                               partition_tokens=partition_tokens)

    if config == 4:
        Hq, Hkv, d, bs = 32, 8, 128, 32
        NB = 32768 if num_blocks is None else num_blocks
        B = 256 if batch is None else batch
        cap = 4096 if max_len is None else max_len
        lens = gqa_lengths(rng, B, cap)
        order = rng.permutation(NB)
        max_blocks = -(-cap // bs)
        used = int((-(-lens // bs)).sum())
        pad = _padding_ids(order, used, rng, poison_padding)
        tables = _deal_tables(lens, order, bs, max_blocks, pad)
        return _finish("llama3-8b-gqa", rng, seed, Hq=Hq, Hkv=Hkv, d=d, bs=bs, NB=NB, lens=lens,
                       tables=tables, fill=fill, free_order=order.astype(np.int32),
                       partition_tokens=0 if partition_tokens is None else partition_tokens)

    if config == 5:
        Hq, Hkv, d, bs = 64, 8, 128, 16
        NB = 32768 if num_blocks is None else num_blocks
        B = 8 if batch is None else batch
        L = 32768 if max_len is None else max_len
        lens = np.full(B, L, dtype=np.int64)
        order = rng.permutation(NB)
        max_blocks = -(-L // bs)
        used = int((-(-lens // bs)).sum())
        pad = _padding_ids(order, used, rng, poison_padding)
        tables = _deal_tables(lens, order, bs, max_blocks, pad)
        n_pairs = 1024 if num_copy_pairs is None else num_copy_pairs
        n_pairs = min(n_pairs, used, NB - used)
        src = rng.choice(order[:used], size=n_pairs, replace=False)
        dst = rng.choice(order[used:], size=n_pairs, replace=False)
        pairs = np.stack([src, dst], axis=1)
        return _finish("long-context", rng, seed, Hq=Hq, Hkv=Hkv, d=d, bs=bs, NB=NB, lens=lens,
                       tables=tables, fill=fill, copy_pairs=pairs, free_order=order.astype(np.int32),
                       partition_tokens=512 if partition_tokens is None else partition_tokens)

    raise ValueError(f"unknown workload {config}")


def make_custom_case(lens, *, num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int,
                     num_blocks: Optional[int] = None, seed: int = 0, fill=BF16_QNAN,
                     poison_padding: bool = True, extra_table_cols: int = 0,
                     partition_tokens: int = 0, scale=None) -> DecodeCase:
    """A decode step with the given lengths and shape, blocks placed by a seeded permutation."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int64)
    bs = block_size
    used = int((-(-lens // bs)).sum())
    NB = num_blocks if num_blocks is not None else max(8, 2 * used + 8)
    order = rng.permutation(NB)
    max_blocks = max(1, int((-(-lens // bs)).max()) if lens.size else 1) + extra_table_cols
    pad = _padding_ids(order, used, rng, poison_padding)
    tables = _deal_tables(lens, order, bs, max_blocks, pad)
    return _finish("custom", rng, seed, Hq=num_q_heads, Hkv=num_kv_heads, d=head_dim, bs=bs, NB=NB,
                   lens=lens, tables=tables, fill=fill, free_order=order.astype(np.int32),
                   partition_tokens=partition_tokens, scale=scale)


def gqa_lengths(rng: np.random.Generator, batch: int, cap: int = 4096) -> np.ndarray:
    """Lengths of workload 4: lognormal with median 800 and sigma 1.0, rounded, clamped to [1, cap]."""
    return np.clip(np.rint(rng.lognormal(np.log(800.0), 1.0, size=batch)), 1, cap).astype(np.int64)


def _make_chat_case(rng, seed, *, fill, batch, max_len, num_blocks, poison_padding,
                    partition_tokens) -> DecodeCase:
    """Chat mix with n=4 sampling (workload 3).

    Group g's four members share the physical blocks of the first
    S_g = min(512, prompt_g) tokens.  When S_g is not a multiple of the block
    size the last shared block is partial: members 0..2 each get a private copy
    (a (src, dst) pair, applied by the step's block copy) and member 3 keeps the
    original; the rows of a copy from S_g on are that member's own tokens and
    are delivered as new tokens of the step.
    """
    Hq = Hkv = 40
    d, bs = 128, 16
    NB = 24576 if num_blocks is None else num_blocks
    B = 128 if batch is None else batch
    if B % 4:
        raise ValueError("chat workload batch must be a multiple of 4")
    G4 = B // 4
    plo, phi = 100, 2000
    glo, ghi = 50, 500
    if max_len is not None:  # shrink: keep the 4:1 prompt:generation shape
        phi = max(2, (max_len * 4) // 5)
        plo = min(plo, phi)
        ghi = max(1, max_len - phi)
        glo = min(glo, ghi)
    prompt = rng.integers(plo, phi + 1, size=G4)
    gen = rng.integers(glo, ghi + 1, size=B)
    lens = prompt[np.arange(B) // 4] + gen
    share_cap = 512 if max_len is None else max(1, min(512, phi // 2))
    S = np.minimum(share_cap, prompt)
    order = rng.permutation(NB)
    max_blocks = -(-int(lens.max()) // bs)

    tables = np.full((B, max_blocks), -1, dtype=np.int64)
    cursor = 0
    pairs = []
    skip_rows = []
    late_rows = []
    for g in range(G4):
        n_shared = -(-int(S[g]) // bs)
        shared = order[cursor:cursor + n_shared]
        cursor += n_shared
        partial = int(S[g]) % bs
        for m in range(4):
            b = 4 * g + m
            n = -(-int(lens[b]) // bs)
            tables[b, :n_shared] = shared
            if partial and m < 3:
                dst = order[cursor]
                cursor += 1
                pairs.append((shared[-1], dst))
                tables[b, n_shared - 1] = dst
                # The copy block starts poisoned; rows below S_g arrive via the
                # copy, rows S_g .. end of block are this member's own tokens.
                for p in range((n_shared - 1) * bs, min(n_shared * bs, int(lens[b]) - 1)):
                    skip_rows.append((b, p))
                    if p >= int(S[g]):
                        late_rows.append((b, p))
            tables[b, n_shared:n] = order[cursor:cursor + (n - n_shared)]
            cursor += n - n_shared
    used = cursor
    pad = _padding_ids(order, used, rng, poison_padding)
    padded = np.resize(pad, tables.shape)
    for b in range(B):
        n = -(-int(lens[b]) // bs)
        tables[b, n:] = padded[b, n:]
    groups = (np.arange(B) // 4).astype(np.int32)
    shared_tokens = S[groups].astype(np.int32)
    return _finish("llama2-13b-chat-n4", rng, seed, Hq=Hq, Hkv=Hkv, d=d, bs=bs, NB=NB, lens=lens,
                   tables=tables, fill=fill,
                   skip_rows=np.array(skip_rows, dtype=np.int64).reshape(-1, 2),
                   late_rows=np.array(late_rows, dtype=np.int64).reshape(-1, 2),
                   copy_pairs=np.array(pairs, dtype=np.int64).reshape(-1, 2),
                   free_order=order.astype(np.int32), groups=groups, shared_tokens=shared_tokens,
                   partition_tokens=0 if partition_tokens is None else partition_tokens)


def split_last_tokens(case: DecodeCase):
    """Split a step's new tokens into each sequence's token at position L-1 (ordered by
    sequence, zero rows for empty sequences) and the remaining token indices.

    Returns (k_last [B, Hkv, d], v_last [B, Hkv, d], other: int64 indices into k_new).
    """
    bs = case.block_size
    want = {}
    for b, L in enumerate(case.seq_lens):
        if L > 0:
            want[int(case.block_tables[b, (L - 1) // bs]) * bs + (int(L) - 1) % bs] = b
    B, Hkv, d = case.batch, case.num_kv_heads, case.head_dim
    k_last = np.zeros((B, Hkv, d), np.uint16)
    v_last = np.zeros((B, Hkv, d), np.uint16)
    other = []
    for t, s in enumerate(case.slot_mapping):
        b = want.get(int(s))
        if b is None:
            other.append(t)
        else:
            k_last[b] = case.k_new[t]
            v_last[b] = case.v_new[t]
    return k_last, v_last, np.array(other, dtype=np.int64)


def algorithmic_decode_bytes(case_or_lens, *, num_q_heads=None, num_kv_heads=None,
                             head_dim=None, block_size=None, kv_elem_bytes: int = 2) -> int:
    """Bytes a decode call must move at minimum: K+V rows once, q, fp32 out, table entries, lengths.

    ``kv_elem_bytes`` is 2 for bf16 pools and 1 for fp8 pools."""
    if isinstance(case_or_lens, DecodeCase):
        c = case_or_lens
        lens, Hq, Hkv, d, bs = c.seq_lens, c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size
    else:
        lens, Hq, Hkv, d, bs = case_or_lens, num_q_heads, num_kv_heads, head_dim, block_size
    lens = np.asarray(lens, dtype=np.int64)
    B = lens.size
    kv = int(lens.sum()) * Hkv * d * kv_elem_bytes * 2
    qb = B * Hq * d * 2
    ob = B * Hq * d * 4
    tb = int((-(-lens // bs)).sum()) * 4
    return kv + qb + ob + tb + B * 4
