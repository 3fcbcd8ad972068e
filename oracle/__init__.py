"""fp64 CPU oracle for paged decode -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library (``paged_kv_cache_349_b200``) and neither imports the other.

Contents
--------
* ``oracle.c`` (built to ``liboracle.so`` with gcc, IEEE double, OpenMP over
  independent output rows): gather through the block table, textbook softmax
  attention, decode, cache write, block copy.  See that file's header for the
  definitions and the passages they follow.
* Page arithmetic (pure Python): block counts and last-block slack, naive
  reservation waste, the naive-vs-paged capacity example, KV bytes per token.
* ``AllocModel``: a list-of-lists model of the refcounted block allocator with
  on-demand append, fork and copy-on-write.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against values the pages print, closed forms, invariants or brute force.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from typing import List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i32, i64 = ctypes.c_int, ctypes.c_int64
            lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_f64.restype = ctypes.c_double
            lib.oracle_num_threads.restype = i32
            lib.oracle_set_num_threads.argtypes = [i32]
            lib.oracle_gather.argtypes = [P, i64, i32, i32, i32, P, i32, i32, i32, P]
            lib.oracle_gather.restype = i32
            lib.oracle_attend.argtypes = [P, P, P, i32, i32, ctypes.c_double, P]
            lib.oracle_attend.restype = None
            lib.oracle_decode_rows.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64,
                                               ctypes.c_float, P, i32, P]
            lib.oracle_decode_rows.restype = i32
            lib.oracle_decode.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64,
                                          ctypes.c_float, P]
            lib.oracle_decode.restype = i32
            lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32]
            lib.oracle_reshape_and_cache.restype = i32
            lib.oracle_copy_blocks.argtypes = [P, P, P, i32, i64, i32, i32, i32]
            lib.oracle_copy_blocks.restype = i32
            lib.oracle_swap_blocks.argtypes = [P, P, i64, P, P, i64, P, i32, i32, i32, i32]
            lib.oracle_swap_blocks.restype = i32
            lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_decode.restype = ctypes.c_double
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_quantize_e4m3.argtypes = [P, P, i64, ctypes.c_float]
            lib.oracle_quantize_e4m3.restype = None
            lib.oracle_reshape_and_cache_fp8.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32,
                                                         ctypes.c_float, ctypes.c_float]
            lib.oracle_reshape_and_cache_fp8.restype = i32
            lib.oracle_decode_rows_fp8.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64,
                                                   ctypes.c_float, ctypes.c_float, ctypes.c_float, P, i32, P]
            lib.oracle_decode_rows_fp8.restype = i32
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------------------
# Numeric kernels (C, fp64)
# ---------------------------------------------------------------------------

def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def bf16_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64 (element by element, in C)."""
    lib = _load()
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    out = np.array([lib.oracle_bf16_to_f64(int(b)) for b in flat], dtype=np.float64)
    return out.reshape(np.shape(bits))


def gather(pool: np.ndarray, table: np.ndarray, seq_len: int, h: int, block_size: int) -> np.ndarray:
    """K (or V) rows of kv head ``h`` for logical positions 0..seq_len-1, float64 [L, d]."""
    pool = _c(pool, np.uint16)
    table = _c(table, np.int32)
    nb, hkv, bs, d = pool.shape
    assert bs == block_size
    out = np.zeros((max(seq_len, 0), d), dtype=np.float64)
    st = _load().oracle_gather(_ptr(pool), nb, hkv, bs, d, _ptr(table), table.size, seq_len, h, _ptr(out))
    if st:
        raise IndexError(f"oracle_gather: status {st}")
    return out


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """Softmax attention of one float64 query over float64 K [L, d], V [L, d]."""
    q = _c(q, np.float64)
    K = _c(K, np.float64).reshape(-1, q.size)
    V = _c(V, np.float64).reshape(-1, q.size)
    out = np.zeros(q.size, dtype=np.float64)
    _load().oracle_attend(_ptr(q), _ptr(K), _ptr(V), K.shape[0], q.size, float(scale), _ptr(out))
    return out


def decode(q, k_pool, v_pool, block_tables, seq_lens, *, num_kv_heads: int, block_size: int,
           scale, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """Paged decode in fp64.

    q: uint16 [B, Hq, d]; pools: uint16 [NB, Hkv, bs, d]; tables int32 [B, max_blocks];
    seq_lens int32 [B].  Returns float64 [B, Hq, d], or [n, d] for ``rows`` (int32 [n, 2]
    of (b, g)).
    """
    q = _c(q, np.uint16)
    k_pool = _c(k_pool, np.uint16)
    v_pool = _c(v_pool, np.uint16)
    tables = _c(block_tables, np.int32)
    lens = _c(seq_lens, np.int32)
    B, Hq, d = q.shape
    nb = k_pool.shape[0]
    assert k_pool.shape == v_pool.shape and k_pool.shape[1] == num_kv_heads
    assert k_pool.shape[2] == block_size and k_pool.shape[3] == d
    lib = _load()
    if rows is None:
        out = np.zeros((B, Hq, d), dtype=np.float64)
        st = lib.oracle_decode(_ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(tables), tables.shape[1],
                               _ptr(lens), B, Hq, num_kv_heads, d, block_size, nb,
                               ctypes.c_float(float(scale)), _ptr(out))
    else:
        rows = _c(rows, np.int32).reshape(-1, 2)
        out = np.zeros((rows.shape[0], d), dtype=np.float64)
        st = lib.oracle_decode_rows(_ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(tables), tables.shape[1],
                                    _ptr(lens), B, Hq, num_kv_heads, d, block_size, nb,
                                    ctypes.c_float(float(scale)), _ptr(rows), rows.shape[0], _ptr(out))
    if st:
        raise IndexError(f"oracle_decode: status {st}")
    return out


def reshape_and_cache(k_new, v_new, k_pool: np.ndarray, v_pool: np.ndarray, slot_mapping,
                      block_size: int) -> int:
    """In-place cache write; returns the number of out-of-range slots (skipped)."""
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    assert k_pool.dtype == np.uint16 and v_pool.dtype == np.uint16
    k_new = _c(k_new, np.uint16)
    v_new = _c(v_new, np.uint16)
    slots = _c(slot_mapping, np.int32)
    nb, hkv, bs, d = k_pool.shape
    assert bs == block_size
    return int(_load().oracle_reshape_and_cache(_ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool),
                                                _ptr(slots), slots.size, nb, hkv, bs, d))


def copy_blocks(k_pool: np.ndarray, v_pool: np.ndarray, pairs) -> int:
    """In-place block copy of (src, dst) pairs; returns the number of invalid pairs."""
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    pairs = _c(pairs, np.int32).reshape(-1, 2)
    nb, hkv, bs, d = k_pool.shape
    return int(_load().oracle_copy_blocks(_ptr(k_pool), _ptr(v_pool), _ptr(pairs), pairs.shape[0],
                                          nb, hkv, bs, d))


def swap_blocks(dst_k: np.ndarray, dst_v: np.ndarray, src_k, src_v, pairs) -> int:
    """In-place copy of (src, dst) block pairs from the source pools into the destination pools."""
    assert dst_k.flags.c_contiguous and dst_v.flags.c_contiguous
    src_k = _c(src_k, np.uint16)
    src_v = _c(src_v, np.uint16)
    pairs = _c(pairs, np.int32).reshape(-1, 2)
    nbd, hkv, bs, d = dst_k.shape
    assert src_k.shape[1:] == dst_k.shape[1:]
    return int(_load().oracle_swap_blocks(_ptr(dst_k), _ptr(dst_v), nbd, _ptr(src_k), _ptr(src_v),
                                          src_k.shape[0], _ptr(pairs), pairs.shape[0], hkv, bs, d))


# ---------------------------------------------------------------------------
# fp8 (E4M3) pools
# ---------------------------------------------------------------------------

def e4m3_value(codes) -> np.ndarray:
    """Value of each E4M3 code (float64; NaN for the NaN codes)."""
    lib = _load()
    flat = np.asarray(codes, dtype=np.uint8).ravel()
    return np.array([lib.oracle_e4m3_decode(int(c)) for c in flat], np.float64).reshape(np.shape(codes))


def e4m3_code(x) -> np.ndarray:
    """Nearest E4M3 code of each fp32 value (ties to even, saturating at 448)."""
    lib = _load()
    flat = np.asarray(x, dtype=np.float32).ravel()
    return np.array([lib.oracle_e4m3_encode(float(v)) for v in flat], np.uint8).reshape(np.shape(x))


def inv_scale(scale) -> np.float32:
    """The fp32 reciprocal both sides quantize with: 1 / scale rounded to fp32."""
    return np.float32(1.0) / np.float32(scale)


def quantize_e4m3(bf16_bits, scale) -> np.ndarray:
    """Codes E4M3(bf16 * (1/scale)) with the product in fp32."""
    src = _c(bf16_bits, np.uint16)
    dst = np.empty(src.shape, np.uint8)
    _load().oracle_quantize_e4m3(_ptr(src), _ptr(dst), src.size, ctypes.c_float(float(inv_scale(scale))))
    return dst


def reshape_and_cache_fp8(k_new, v_new, k_pool: np.ndarray, v_pool: np.ndarray, slot_mapping, block_size: int,
                          k_scale, v_scale) -> int:
    assert k_pool.dtype == np.uint8 and v_pool.dtype == np.uint8
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    k_new = _c(k_new, np.uint16)
    v_new = _c(v_new, np.uint16)
    slots = _c(slot_mapping, np.int32)
    nb, hkv, bs, d = k_pool.shape
    assert bs == block_size
    return int(_load().oracle_reshape_and_cache_fp8(
        _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool), _ptr(slots), slots.size, nb, hkv, bs, d,
        ctypes.c_float(float(inv_scale(k_scale))), ctypes.c_float(float(inv_scale(v_scale)))))


def decode_fp8(q, k_pool, v_pool, block_tables, seq_lens, *, num_kv_heads: int, block_size: int, scale,
               k_scale, v_scale, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """Paged decode in fp64 over fp8 pools (rows dequantised as E4M3 value * scale)."""
    q = _c(q, np.uint16)
    k_pool = _c(k_pool, np.uint8)
    v_pool = _c(v_pool, np.uint8)
    tables = _c(block_tables, np.int32)
    lens = _c(seq_lens, np.int32)
    B, Hq, d = q.shape
    if rows is None:
        rows = np.array([(b, g) for b in range(B) for g in range(Hq)], np.int32).reshape(-1, 2)
        full = True
    else:
        rows = _c(rows, np.int32).reshape(-1, 2)
        full = False
    out = np.zeros((rows.shape[0], d), np.float64)
    st = _load().oracle_decode_rows_fp8(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(tables), tables.shape[1], _ptr(lens), B, Hq, num_kv_heads, d,
        block_size, k_pool.shape[0], ctypes.c_float(float(scale)), ctypes.c_float(float(k_scale)),
        ctypes.c_float(float(v_scale)), _ptr(rows), rows.shape[0], _ptr(out))
    if st:
        raise IndexError(f"oracle_decode_fp8: status {st}")
    return out.reshape(B, Hq, d) if full else out


def decode_step(case, rows: Optional[np.ndarray] = None):
    """Apply one decode step of a ``workloads.DecodeCase`` on host copies of its pools.

    Order: block copies, then the cache write, then decode (append, then attend).
    Returns (out, k_pool_after, v_pool_after).
    """
    k_pool = case.k_cache.copy()
    v_pool = case.v_cache.copy()
    bad = copy_blocks(k_pool, v_pool, case.copy_pairs)
    bad += reshape_and_cache(case.k_new, case.v_new, k_pool, v_pool, case.slot_mapping, case.block_size)
    if bad:
        raise IndexError(f"{bad} invalid slots/pairs in the case")
    out = decode(case.q, k_pool, v_pool, case.block_tables, case.seq_lens,
                 num_kv_heads=case.num_kv_heads, block_size=case.block_size, scale=case.scale,
                 rows=rows)
    return out, k_pool, v_pool


# ---------------------------------------------------------------------------
# Page arithmetic
# ---------------------------------------------------------------------------

def blocks_needed(num_tokens: int, block_size: int) -> int:
    """Blocks a sequence of ``num_tokens`` occupies: ceil(n / bs)
    ("PagedAttention Explained", Grow allocation with the sequence)."""
    return -(-num_tokens // block_size)


def last_block_slack(num_tokens: int, block_size: int) -> int:
    """Unused token positions in the last block: blocks*bs - n (at most bs-1)."""
    return blocks_needed(num_tokens, block_size) * block_size - num_tokens


def naive_waste(used_tokens: int, reserved_tokens: int) -> float:
    """Fraction of a contiguous max-length reservation left empty
    ("PagedAttention & vLLM", The problem: contiguous pre-allocation)."""
    return (reserved_tokens - used_tokens) / reserved_tokens


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, elem_bytes: int = 2) -> int:
    """K and V bytes one token occupies across all layers."""
    return 2 * num_layers * num_kv_heads * head_dim * elem_bytes


def max_concurrent_requests(kv_gb: float, mb_per_token: float, tokens_per_request: int) -> int:
    """Requests that fit in ``kv_gb`` of KV memory at ``tokens_per_request`` each.

    Follows the arithmetic of "PagedAttention & vLLM", Worked example: naive
    vs paged: per-request GB = MB/token x tokens / 1024, then the quotient is
    rounded to the nearest request.
    """
    per_request_gb = mb_per_token * tokens_per_request / 1024.0
    return int(math.floor(kv_gb / per_request_gb + 0.5))


# ---------------------------------------------------------------------------
# Allocator model
# ---------------------------------------------------------------------------

class OutOfBlocks(Exception):
    pass


class AllocModel:
    """List-of-lists model of a refcounted block allocator.

    * append: the token at position n goes to block n // bs, row n % bs; a new
      block is taken from the pool when n % bs == 0 ("Walk through paged
      attention end to end", append step; "What is PagedAttention",
      ``append_token``).  Writing into a block whose refcount is above one
      first copies it to a fresh block (copy-on-write, "PagedAttention &
      vLLM", Copy-on-write sharing); the old block loses one reference.
    * fork: the child references every block of the parent, the partially
      filled last one included, and each refcount grows by one.
    * free: refcounts drop; blocks reaching zero return to the pool.

    Blocks are taken from the front of ``free`` (initially ``order``); the
    pages allow any free block, so tests compare only policy-free facts.
    """

    def __init__(self, num_blocks: int, block_size: int, order: Optional[Sequence[int]] = None):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free: List[int] = list(range(num_blocks)) if order is None else [int(b) for b in order]
        self.ref: List[int] = [0] * num_blocks
        self.tables: dict = {}
        self.ntok: dict = {}
        self._next = 0

    def _take(self) -> int:
        if not self.free:
            raise OutOfBlocks()
        b = self.free.pop(0)
        self.ref[b] = 1
        return b

    def create(self) -> int:
        sid = self._next
        self._next += 1
        self.tables[sid] = []
        self.ntok[sid] = 0
        return sid

    def append(self, sid: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        """Append one token; return (slot, cow) with cow = (src, dst) or None."""
        n = self.ntok[sid]
        j, row = n // self.block_size, n % self.block_size
        table = self.tables[sid]
        cow = None
        if row == 0:
            table.append(self._take())
        else:
            old = table[j]
            if self.ref[old] > 1:
                new = self._take()
                self.ref[old] -= 1
                table[j] = new
                cow = (old, new)
        self.ntok[sid] = n + 1
        return table[j] * self.block_size + row, cow

    def fork(self, parent: int) -> int:
        child = self.create()
        self.tables[child] = list(self.tables[parent])
        self.ntok[child] = self.ntok[parent]
        for b in self.tables[child]:
            self.ref[b] += 1
        return child

    def free_seq(self, sid: int) -> None:
        for b in self.tables.pop(sid):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del self.ntok[sid]

    def num_free(self) -> int:
        return len(self.free)

    def blocks_in_use(self) -> int:
        return sum(1 for r in self.ref if r > 0)
