"""B200-native paged KV-cache decode: Python binding of ``libpa.so``.

Argument marshalling only: every function below turns torch tensors (or
host numpy arrays for the allocator) into the plain pointers and sizes of
the C ABI declared in ``include/pa.h`` and raises ``PaError`` on a non-zero
status.  All device work runs in the library's CUDA kernels.

Device ops on bf16 pools (names as in the C ABI):
    pa_reshape_and_cache, pa_copy_blocks, pa_swap_blocks, pa_decode,
    pa_decode_append, pa_decode_shared_prefix, pa_decode_builtin_scratch,
    pa_decode_workspace_size, pa_decode_shared_prefix_workspace_size,
    pa_decode_partition_tokens
Device ops on fp8 (E4M3) pools:
    pa_quantize_fp8, pa_reshape_and_cache_fp8, pa_copy_blocks_fp8,
    pa_swap_blocks_fp8, pa_decode_fp8 (with k_new/v_new: the fused write)
A whole decode step from pinned host buffers:
    pa_decode_step_staging_size[_shared_prefix], DecodeStepHost (pa_decode_step_plan_*; the
    one-call form is pa_decode_step_host[_fp8] in the C ABI)
Host allocator:
    Allocator (pa_alloc_* / pa_seq_* / pa_block_refcount; step_fn = pa_alloc_step)
    validate_tables (pa_validate_tables: host-side check of decode tables)
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence, Tuple

import numpy as np

from ._lib import lib

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_CUDA = 3
PA_ERR_BAD_INDEX = 4
PA_ERR_TIMEOUT = 5
PA_ERR_OOM = 6
PA_ERR_STATE = 7

PA_FLAG_BAD_SLOT = 0x1
PA_FLAG_BAD_BLOCK = 0x2
PA_FLAG_BAD_PAIR = 0x4
PA_FLAG_BAD_LEN = 0x8
PA_FLAG_TIMEOUT = 0x10


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.pa_status_string(status).decode()} ({status})")


def _check(status: int, where: str) -> None:
    if status != PA_OK:
        raise PaError(status, where)


def status_string(status: int) -> str:
    return lib.pa_status_string(status).decode()


def version() -> int:
    return lib.pa_version()


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(lib.pa_launch_count())


# ---------------------------------------------------------------------------
# Device ops (torch tensors in, pointers out)
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _dev(t, dtype, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _opt_flag(err_flag):
    if err_flag is None:
        return None
    return _dev(err_flag, _torch().int32, "err_flag")


def _stream(stream):
    torch = _torch()
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def pa_reshape_and_cache(k_new, v_new, k_cache, v_cache, slot_mapping, err_flag=None, stream=None) -> None:
    """Write k_new/v_new [T, Hkv, d] into the pools [NB, Hkv, bs, d] at slot_mapping [T]."""
    torch = _torch()
    T, Hkv, d = k_new.shape
    NB, Hkv2, bs, d2 = k_cache.shape
    if (Hkv2, d2) != (Hkv, d) or v_new.shape != k_new.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if slot_mapping.numel() != T:
        raise ValueError("slot_mapping must have one entry per token")
    _check(lib.pa_reshape_and_cache(
        _dev(k_new, torch.bfloat16, "k_new"), _dev(v_new, torch.bfloat16, "v_new"),
        _dev(k_cache, torch.bfloat16, "k_cache"), _dev(v_cache, torch.bfloat16, "v_cache"),
        _dev(slot_mapping, torch.int32, "slot_mapping"), T, NB, Hkv, bs, d,
        _opt_flag(err_flag), _stream(stream)), "pa_reshape_and_cache")


def pa_copy_blocks(k_cache, v_cache, pairs, err_flag=None, stream=None) -> None:
    """Copy whole blocks src -> dst in both pools; pairs is int32 [n, 2] on the device."""
    torch = _torch()
    NB, Hkv, bs, d = k_cache.shape
    n = pairs.shape[0] if pairs.dim() == 2 else pairs.numel() // 2
    if n and (pairs.numel() != 2 * n):
        raise ValueError("pairs must be [n, 2]")
    _check(lib.pa_copy_blocks(
        _dev(k_cache, torch.bfloat16, "k_cache"), _dev(v_cache, torch.bfloat16, "v_cache"),
        _dev(pairs, torch.int32, "pairs") if n else None, n, NB, Hkv, bs, d,
        _opt_flag(err_flag), _stream(stream)), "pa_copy_blocks")


def _dev_or_pinned(t, dtype, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not (t.is_cuda or t.is_pinned()):
        raise TypeError(f"{name} must be a CUDA tensor or a pinned host tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, pairs, err_flag=None, stream=None) -> None:
    """Copy blocks between two pools [NB, Hkv, bs, d]; either side may be pinned host memory.

    pairs: int32 [n, 2] (src block, dst block), a CUDA tensor or a pinned host tensor.
    """
    torch = _torch()
    if dst_k.shape[1:] != src_k.shape[1:] or dst_v.shape != dst_k.shape or src_v.shape != src_k.shape:
        raise ValueError("pools must share [Hkv, bs, d]")
    NBd, Hkv, bs, d = dst_k.shape
    n = pairs.shape[0] if pairs.dim() == 2 else pairs.numel() // 2
    _check(lib.pa_swap_blocks(
        _dev_or_pinned(dst_k, torch.bfloat16, "dst_k"), _dev_or_pinned(dst_v, torch.bfloat16, "dst_v"), NBd,
        _dev_or_pinned(src_k, torch.bfloat16, "src_k"), _dev_or_pinned(src_v, torch.bfloat16, "src_v"),
        src_k.shape[0], _dev_or_pinned(pairs, torch.int32, "pairs") if n else None, n, Hkv, bs, d,
        _opt_flag(err_flag), _stream(stream)), "pa_swap_blocks")


def pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len,
                             partition_tokens=0) -> int:
    return int(lib.pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, block_size,
                                            max_seq_len, partition_tokens))


def pa_decode_partition_tokens(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len,
                               partition_tokens=0) -> int:
    return int(lib.pa_decode_partition_tokens(batch, num_q_heads, num_kv_heads, head_dim, block_size,
                                              max_seq_len, partition_tokens))


def pa_decode(out, q, k_cache, v_cache, block_tables, seq_lens, *, max_seq_len: int, scale: float,
              partition_tokens: int = 0, workspace=None, err_flag=None, stream=None) -> None:
    """Paged decode: out fp32 [B, Hq, d] <- attention of q bf16 [B, Hq, d] over the pools.

    block_tables int32 [B, max_blocks], seq_lens int32 [B] (device tensors);
    ``workspace`` is a uint8 CUDA tensor of at least ``pa_decode_workspace_size`` bytes.
    """
    torch = _torch()
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    if d2 != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.numel() != B:
        raise ValueError("block_tables must be [B, max_blocks] and seq_lens [B]")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, workspace.dtype, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.pa_decode(
        _dev(out, torch.float32, "out"), _dev(q, torch.bfloat16, "q"),
        _dev(k_cache, torch.bfloat16, "k_cache"), _dev(v_cache, torch.bfloat16, "v_cache"),
        _dev(block_tables, torch.int32, "block_tables"), block_tables.shape[1],
        _dev(seq_lens, torch.int32, "seq_lens"), B, int(max_seq_len), Hq, Hkv, d, bs, NB,
        float(scale), int(partition_tokens), ws_ptr, ws_bytes, _opt_flag(err_flag),
        _stream(stream)), "pa_decode")


def pa_decode_append(out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens, *, max_seq_len: int,
                     scale: float, partition_tokens: int = 0, workspace=None, err_flag=None, stream=None) -> None:
    """Fused decode step: write each sequence's new token (k_new/v_new bf16 [B, Hkv, d], at
    position seq_lens[b]-1) into the pools and decode, in one launch."""
    torch = _torch()
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    if d2 != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if tuple(k_new.shape) != (B, Hkv, d) or v_new.shape != k_new.shape:
        raise ValueError("k_new/v_new must be [B, Hkv, d]")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.numel() != B:
        raise ValueError("block_tables must be [B, max_blocks] and seq_lens [B]")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, workspace.dtype, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_append(
        _dev(out, torch.float32, "out"), _dev(q, torch.bfloat16, "q"),
        _dev(k_new, torch.bfloat16, "k_new"), _dev(v_new, torch.bfloat16, "v_new"),
        _dev(k_cache, torch.bfloat16, "k_cache"), _dev(v_cache, torch.bfloat16, "v_cache"),
        _dev(block_tables, torch.int32, "block_tables"), block_tables.shape[1],
        _dev(seq_lens, torch.int32, "seq_lens"), B, int(max_seq_len), Hq, Hkv, d, bs, NB,
        float(scale), int(partition_tokens), ws_ptr, ws_bytes, _opt_flag(err_flag),
        _stream(stream)), "pa_decode_append")


def pa_decode_shared_prefix_workspace_size(batch, group_size, num_q_heads, num_kv_heads, head_dim, block_size,
                                           max_seq_len, partition_tokens=0) -> int:
    return int(lib.pa_decode_shared_prefix_workspace_size(batch, group_size, num_q_heads, num_kv_heads, head_dim,
                                                          block_size, max_seq_len, partition_tokens))


def pa_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, seq_lens, prefix_lens, *, group_size: int,
                            max_seq_len: int, scale: float, partition_tokens: int = 0, workspace=None,
                            err_flag=None, stream=None, k_new=None, v_new=None) -> None:
    """Decode of a batch laid out in groups of ``group_size`` sequences whose first
    ``prefix_lens[g]`` tokens (int32 device tensor, one entry per group) hold the same
    K/V: the shared tiles are read once per group and kv head.  With k_new/v_new
    (bf16 [B, Hkv, d]) each sequence's new token is written first, as pa_decode_append."""
    torch = _torch()
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    if d2 != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.numel() != B:
        raise ValueError("block_tables must be [B, max_blocks] and seq_lens [B]")
    if group_size < 1 or prefix_lens.numel() != -(-B // group_size):
        raise ValueError("prefix_lens must hold one entry per group of group_size sequences")
    if (k_new is None) != (v_new is None):
        raise ValueError("pass both k_new and v_new, or neither")
    new = (None, None)
    if k_new is not None:
        if tuple(k_new.shape) != (B, Hkv, d) or v_new.shape != k_new.shape:
            raise ValueError("k_new/v_new must be [B, Hkv, d]")
        new = (_dev(k_new, torch.bfloat16, "k_new"), _dev(v_new, torch.bfloat16, "v_new"))
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, workspace.dtype, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_shared_prefix(
        _dev(out, torch.float32, "out"), _dev(q, torch.bfloat16, "q"), *new,
        _dev(k_cache, torch.bfloat16, "k_cache"), _dev(v_cache, torch.bfloat16, "v_cache"),
        _dev(block_tables, torch.int32, "block_tables"), block_tables.shape[1],
        _dev(seq_lens, torch.int32, "seq_lens"), _dev(prefix_lens, torch.int32, "prefix_lens"), int(group_size),
        B, int(max_seq_len), Hq, Hkv, d, bs, NB, float(scale), int(partition_tokens), ws_ptr, ws_bytes,
        _opt_flag(err_flag), _stream(stream)), "pa_decode_shared_prefix")


def pa_decode_step_staging_size(batch, max_blocks_per_seq, max_copy_pairs, num_q_heads, num_kv_heads, head_dim,
                                block_size, max_seq_len, partition_tokens=0) -> int:
    return int(lib.pa_decode_step_staging_size(batch, max_blocks_per_seq, max_copy_pairs, num_q_heads,
                                               num_kv_heads, head_dim, block_size, max_seq_len, partition_tokens))


def pa_decode_step_staging_size_shared_prefix(batch, group_size, max_blocks_per_seq, max_copy_pairs, num_q_heads,
                                              num_kv_heads, head_dim, block_size, max_seq_len,
                                              partition_tokens=0) -> int:
    return int(lib.pa_decode_step_staging_size_shared_prefix(batch, group_size, max_blocks_per_seq, max_copy_pairs,
                                                             num_q_heads, num_kv_heads, head_dim, block_size,
                                                             max_seq_len, partition_tokens))


class DecodeStepHost:
    """Repeated decode steps from fixed pinned host buffers: a prepared step
    (``pa_decode_step_plan_create``) over bf16 pools, or uint8 E4M3 pools given
    ``k_scale`` and ``v_scale``; each call is one ``pa_decode_step_plan_run``.

    Host arrays are torch CPU tensors (pinned); pools and staging are CUDA
    tensors, all kept alive by this object.  ``max_seq_len_cap`` bounds the
    ``max_seq_len`` of every call (staging must be sized with it).
    ``num_chunks``: 0 lets the library pick how many chunks of sequences to
    pipeline, 1 disables pipelining, 2..8 forces that many.  With
    ``prefix_lens_host`` (int32, one entry per group) and ``group_size`` the
    step decodes with ``pa_decode_shared_prefix``
    (``pa_decode_step_plan_set_shared_prefix``; staging sized by
    ``pa_decode_step_staging_size_shared_prefix``).  ``close()`` (or garbage
    collection) releases the plan.
    """

    def __init__(self, *, out_host, q_host, k_new_host, v_new_host, tables_host, lens_host, pairs_host,
                 k_cache, v_cache, scale: float, max_seq_len_cap: int, partition_tokens: int = 0,
                 num_chunks: int = 0, staging=None, err_flag=None, stream=None, k_scale: Optional[float] = None,
                 v_scale: Optional[float] = None, prefix_lens_host=None, group_size: int = 0):
        torch = _torch()
        B, Hq, d = q_host.shape
        NB, Hkv, bs, d2 = k_cache.shape
        if d2 != d or tuple(out_host.shape) != (B, Hq, d) or tuple(k_new_host.shape) != (B, Hkv, d):
            raise ValueError("shape mismatch")
        for t, dt, name in ((out_host, torch.float32, "out_host"), (q_host, torch.bfloat16, "q_host"),
                            (k_new_host, torch.bfloat16, "k_new_host"), (v_new_host, torch.bfloat16, "v_new_host"),
                            (tables_host, torch.int32, "tables_host"), (lens_host, torch.int32, "lens_host"),
                            (pairs_host, torch.int32, "pairs_host")):
            if t.is_cuda or t.dtype != dt or not t.is_contiguous():
                raise TypeError(f"{name} must be a contiguous host {dt} tensor")
        self.fp8 = k_cache.dtype == torch.uint8
        if self.fp8 != (k_scale is not None and v_scale is not None):
            raise ValueError("uint8 (E4M3) pools need k_scale and v_scale; bf16 pools take neither")
        pool_dt = torch.uint8 if self.fp8 else torch.bfloat16
        self.max_blocks = int(tables_host.shape[1])
        self.max_pairs = int(pairs_host.shape[0])
        self._keep = (out_host, q_host, k_new_host, v_new_host, tables_host, lens_host, pairs_host, k_cache, v_cache,
                      staging, err_flag)
        self._plan = ctypes.c_void_p()
        _check(lib.pa_decode_step_plan_create(
            ctypes.c_void_p(out_host.data_ptr()), ctypes.c_void_p(q_host.data_ptr()),
            ctypes.c_void_p(k_new_host.data_ptr()), ctypes.c_void_p(v_new_host.data_ptr()),
            ctypes.c_void_p(tables_host.data_ptr()), self.max_blocks, ctypes.c_void_p(lens_host.data_ptr()),
            ctypes.c_void_p(pairs_host.data_ptr()), self.max_pairs, _dev(k_cache, pool_dt, "k_cache"),
            _dev(v_cache, pool_dt, "v_cache"), B, int(max_seq_len_cap), Hq, Hkv, d, bs, NB, float(scale),
            int(partition_tokens), int(num_chunks), ctypes.c_void_p(staging.data_ptr()),
            staging.numel() * staging.element_size(), int(self.fp8), float(k_scale or 1.0), float(v_scale or 1.0),
            ctypes.byref(self._plan)), "pa_decode_step_plan_create")
        if group_size:
            if prefix_lens_host is None or prefix_lens_host.is_cuda or prefix_lens_host.dtype != torch.int32 \
                    or not prefix_lens_host.is_contiguous() or prefix_lens_host.numel() < -(-B // group_size):
                self.close()
                raise TypeError("prefix_lens_host must be a contiguous host int32 tensor, one entry per group")
            self._keep = self._keep + (prefix_lens_host,)
            rc = lib.pa_decode_step_plan_set_shared_prefix(self._plan, ctypes.c_void_p(prefix_lens_host.data_ptr()),
                                                          int(group_size))
            if rc != 0:
                self.close()
            _check(rc, "pa_decode_step_plan_set_shared_prefix")
        self._flag = _opt_flag(err_flag)
        self._stream = _stream(stream)
        self._run = lib.pa_decode_step_plan_run

    def __call__(self, max_seq_len: int, num_pairs: int = 0) -> None:
        _check(self._run(self._plan, max_seq_len, num_pairs, self._flag, self._stream), "pa_decode_step_plan_run")

    def close(self) -> None:
        if self._plan:
            lib.pa_decode_step_plan_destroy(self._plan)
            self._plan = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---------------------------------------------------------------------------
# fp8 (E4M3) pools: uint8 tensors of codes, one scale per pool
# ---------------------------------------------------------------------------

def pa_quantize_fp8(src, dst, scale: float, stream=None) -> None:
    """dst (uint8 codes) = E4M3(bf16 src * (1/scale)), element by element."""
    torch = _torch()
    if src.numel() != dst.numel():
        raise ValueError("size mismatch")
    _check(lib.pa_quantize_fp8(_dev(src, torch.bfloat16, "src"), _dev(dst, torch.uint8, "dst"), src.numel(),
                               float(scale), _stream(stream)), "pa_quantize_fp8")


def pa_reshape_and_cache_fp8(k_new, v_new, k_cache, v_cache, slot_mapping, *, k_scale: float, v_scale: float,
                             err_flag=None, stream=None) -> None:
    torch = _torch()
    T, Hkv, d = k_new.shape
    NB, Hkv2, bs, d2 = k_cache.shape
    if (Hkv2, d2) != (Hkv, d) or v_new.shape != k_new.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    _check(lib.pa_reshape_and_cache_fp8(
        _dev(k_new, torch.bfloat16, "k_new"), _dev(v_new, torch.bfloat16, "v_new"),
        _dev(k_cache, torch.uint8, "k_cache"), _dev(v_cache, torch.uint8, "v_cache"),
        _dev(slot_mapping, torch.int32, "slot_mapping"), T, NB, Hkv, bs, d, float(k_scale), float(v_scale),
        _opt_flag(err_flag), _stream(stream)), "pa_reshape_and_cache_fp8")


def pa_copy_blocks_fp8(k_cache, v_cache, pairs, err_flag=None, stream=None) -> None:
    torch = _torch()
    NB, Hkv, bs, d = k_cache.shape
    n = pairs.shape[0] if pairs.dim() == 2 else pairs.numel() // 2
    _check(lib.pa_copy_blocks_fp8(
        _dev(k_cache, torch.uint8, "k_cache"), _dev(v_cache, torch.uint8, "v_cache"),
        _dev(pairs, torch.int32, "pairs") if n else None, n, NB, Hkv, bs, d, _opt_flag(err_flag),
        _stream(stream)), "pa_copy_blocks_fp8")


def pa_swap_blocks_fp8(dst_k, dst_v, src_k, src_v, pairs, err_flag=None, stream=None) -> None:
    torch = _torch()
    if dst_k.shape[1:] != src_k.shape[1:] or dst_v.shape != dst_k.shape or src_v.shape != src_k.shape:
        raise ValueError("pools must share [Hkv, bs, d]")
    NBd, Hkv, bs, d = dst_k.shape
    n = pairs.shape[0] if pairs.dim() == 2 else pairs.numel() // 2
    _check(lib.pa_swap_blocks_fp8(
        _dev_or_pinned(dst_k, torch.uint8, "dst_k"), _dev_or_pinned(dst_v, torch.uint8, "dst_v"), NBd,
        _dev_or_pinned(src_k, torch.uint8, "src_k"), _dev_or_pinned(src_v, torch.uint8, "src_v"), src_k.shape[0],
        _dev_or_pinned(pairs, torch.int32, "pairs") if n else None, n, Hkv, bs, d, _opt_flag(err_flag),
        _stream(stream)), "pa_swap_blocks_fp8")


def pa_decode_fp8(out, q, k_cache, v_cache, block_tables, seq_lens, *, max_seq_len: int, scale: float,
                  k_scale: float, v_scale: float, partition_tokens: int = 0, workspace=None, err_flag=None,
                  stream=None, k_new=None, v_new=None) -> None:
    """pa_decode over uint8 E4M3 pools; with k_new/v_new, pa_decode_append_fp8 (fused write)."""
    torch = _torch()
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    if d2 != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, workspace.dtype, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    head = (_dev(out, torch.float32, "out"), _dev(q, torch.bfloat16, "q"))
    pools = (_dev(k_cache, torch.uint8, "k_cache"), _dev(v_cache, torch.uint8, "v_cache"))
    tail = (_dev(block_tables, torch.int32, "block_tables"), block_tables.shape[1],
            _dev(seq_lens, torch.int32, "seq_lens"), B, int(max_seq_len), Hq, Hkv, d, bs, NB, float(scale),
            float(k_scale), float(v_scale), int(partition_tokens), ws_ptr, ws_bytes, _opt_flag(err_flag),
            _stream(stream))
    if k_new is None:
        _check(lib.pa_decode_fp8(*head, *pools, *tail), "pa_decode_fp8")
    else:
        if tuple(k_new.shape) != (B, Hkv, d) or v_new.shape != k_new.shape:
            raise ValueError("k_new/v_new must be [B, Hkv, d]")
        new = (_dev(k_new, torch.bfloat16, "k_new"), _dev(v_new, torch.bfloat16, "v_new"))
        _check(lib.pa_decode_append_fp8(*head, *new, *pools, *tail), "pa_decode_append_fp8")


PA_DECODE_BUILTIN_SCRATCH_BYTES = 32 << 20


def pa_decode_builtin_scratch(out, q, k_cache, v_cache, block_tables, seq_lens, *, max_seq_len: int,
                              scale: float, partition_tokens: int = 0, err_flag=None, stream=None) -> None:
    """pa_decode for callers that cannot allocate a workspace: split states go to a
    library-owned device array of PA_DECODE_BUILTIN_SCRATCH_BYTES (shared by all calls;
    calls that overlap on the GPU race on it)."""
    torch = _torch()
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    if d2 != d or out.shape != q.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.numel() != B:
        raise ValueError("block_tables must be [B, max_blocks] and seq_lens [B]")
    _check(lib.pa_decode_builtin_scratch(
        _dev(out, torch.float32, "out"), _dev(q, torch.bfloat16, "q"),
        _dev(k_cache, torch.bfloat16, "k_cache"), _dev(v_cache, torch.bfloat16, "v_cache"),
        _dev(block_tables, torch.int32, "block_tables"), block_tables.shape[1],
        _dev(seq_lens, torch.int32, "seq_lens"), B, int(max_seq_len), Hq, Hkv, d, bs, NB,
        float(scale), int(partition_tokens), _opt_flag(err_flag), _stream(stream)),
        "pa_decode_builtin_scratch")


# ---------------------------------------------------------------------------
# Host allocator
# ---------------------------------------------------------------------------

def _np_ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def validate_tables(tables: np.ndarray, seq_lens: np.ndarray, num_blocks: int, block_size: int):
    """Host-side check of decode tables (``pa_validate_tables``).

    Returns None when every attended entry is a block id in range, unrepeated within its row,
    and every length fits its row; otherwise (bad_seq, bad_entry) of the first offence
    (bad_entry -1: the length itself).
    """
    t = np.ascontiguousarray(tables, dtype=np.int32)
    lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    if t.ndim != 2 or lens.shape != (t.shape[0],):
        raise ValueError("tables [B, max_blocks] and seq_lens [B] expected")
    bs_, be = ctypes.c_int(), ctypes.c_int()
    st = lib.pa_validate_tables(_np_ptr(t), t.shape[0], t.shape[1], _np_ptr(lens), int(num_blocks), int(block_size),
                                ctypes.byref(bs_), ctypes.byref(be))
    if st == PA_OK:
        return None
    if st == PA_ERR_BAD_INDEX:
        return bs_.value, be.value
    _check(st, "pa_validate_tables")


class Allocator:
    """Refcounted block allocator with fork and copy-on-write (host memory only)."""

    def __init__(self, num_blocks: int, block_size: int, order: Optional[Sequence[int]] = None):
        h = ctypes.c_void_p()
        if order is None:
            _check(lib.pa_alloc_create(num_blocks, block_size, ctypes.byref(h)), "pa_alloc_create")
        else:
            o = np.ascontiguousarray(order, dtype=np.int32)
            if o.size != num_blocks:
                raise ValueError("order must list every block once")
            _check(lib.pa_alloc_create_ordered(num_blocks, block_size, _np_ptr(o), ctypes.byref(h)),
                   "pa_alloc_create_ordered")
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self) -> None:
        if self._h:
            lib.pa_alloc_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def create(self) -> int:
        sid = ctypes.c_int()
        _check(lib.pa_seq_create(self._h, ctypes.byref(sid)), "pa_seq_create")
        return sid.value

    def append(self, seq_id: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        slot, src, dst = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib.pa_seq_append(self._h, seq_id, ctypes.byref(slot), ctypes.byref(src), ctypes.byref(dst)),
               "pa_seq_append")
        return slot.value, ((src.value, dst.value) if src.value >= 0 else None)

    def append_batch(self, seq_ids) -> Tuple[np.ndarray, np.ndarray]:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
        slots = np.empty(ids.size, dtype=np.int32)
        pairs = np.empty((max(ids.size, 1), 2), dtype=np.int32)
        n = ctypes.c_int()
        _check(lib.pa_seq_append_batch(self._h, _np_ptr(ids), ids.size, _np_ptr(slots), _np_ptr(pairs),
                                       ctypes.byref(n)), "pa_seq_append_batch")
        return slots, pairs[:n.value].copy()

    def fork(self, parent: int) -> int:
        c = ctypes.c_int()
        _check(lib.pa_seq_fork(self._h, parent, ctypes.byref(c)), "pa_seq_fork")
        return c.value

    def free(self, seq_id: int) -> None:
        _check(lib.pa_seq_free(self._h, seq_id), "pa_seq_free")

    def block_table(self, seq_id: int) -> Tuple[np.ndarray, int]:
        nb, nt = ctypes.c_int(), ctypes.c_int()
        st = lib.pa_seq_block_table(self._h, seq_id, None, 0, ctypes.byref(nb), ctypes.byref(nt))
        if st not in (PA_OK, PA_ERR_INVALID_ARG):
            _check(st, "pa_seq_block_table")
        out = np.empty(max(nb.value, 1), dtype=np.int32)
        _check(lib.pa_seq_block_table(self._h, seq_id, _np_ptr(out), out.size, ctypes.byref(nb),
                                      ctypes.byref(nt)), "pa_seq_block_table")
        return out[:nb.value].copy(), nt.value

    def export(self, seq_ids, max_blocks: int, pad: int = -1, tables: Optional[np.ndarray] = None,
               lens: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
        """Padded int32 tables [n, max_blocks] and lengths [n]; written into ``tables`` /
        ``lens`` when given (e.g. numpy views of pinned buffers)."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
        if tables is None:
            tables = np.empty((ids.size, max_blocks), dtype=np.int32)
        if lens is None:
            lens = np.empty(ids.size, dtype=np.int32)
        if (tables.dtype != np.int32 or not tables.flags.c_contiguous or tables.shape != (ids.size, max_blocks)
                or lens.dtype != np.int32 or not lens.flags.c_contiguous or lens.shape != (ids.size,)):
            raise ValueError("tables/lens must be contiguous int32 [n, max_blocks] / [n]")
        _check(lib.pa_alloc_export(self._h, _np_ptr(ids), ids.size, _np_ptr(tables), max_blocks, pad,
                                   _np_ptr(lens)), "pa_alloc_export")
        return tables, lens

    def step_fn(self, seq_ids, tables: np.ndarray, lens: np.ndarray, pairs: np.ndarray, pad: int = -1):
        """A callable for the host side of repeated decode steps on fixed buffers (``pa_alloc_step``).

        Each call appends one token to every sequence of ``seq_ids``, writes their padded tables into
        ``tables`` (int32 [n, max_blocks]) and lengths into ``lens`` (int32 [n]), and the copy-on-write
        pairs into ``pairs`` (int32 [>= n, 2]); it returns ``(num_pairs, max_seq_len)``.  The arrays
        may be numpy views of pinned buffers; their pointers are taken once, here.
        """
        ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
        n = ids.size
        for a, shape, name in ((tables, None, "tables"), (lens, (n,), "lens"), (pairs, None, "pairs")):
            if a.dtype != np.int32 or not a.flags.c_contiguous:
                raise ValueError(f"{name} must be a contiguous int32 array")
        if tables.ndim != 2 or tables.shape[0] != n or lens.shape != (n,) or pairs.ndim != 2 or \
                pairs.shape[1] != 2 or pairs.shape[0] < n:
            raise ValueError("tables [n, max_blocks], lens [n], pairs [>= n, 2] expected")
        n_cow, max_len = ctypes.c_int(), ctypes.c_int()
        args = (self._h, _np_ptr(ids), n, _np_ptr(tables), int(tables.shape[1]), int(pad), _np_ptr(lens),
                _np_ptr(pairs), ctypes.byref(n_cow), ctypes.byref(max_len))
        fn = lib.pa_alloc_step

        def step():
            _check(fn(*args), "pa_alloc_step")
            return n_cow.value, max_len.value

        step.ids = ids  # keeps the id array alive with the callable
        return step

    def num_free(self) -> int:
        return int(lib.pa_alloc_num_free(self._h))

    def refcount(self, block: int) -> int:
        return int(lib.pa_block_refcount(self._h, block))
