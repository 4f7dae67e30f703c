"""Python binding of libpagedattn.so (the C ABI in include/pagedattn.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or fails, these
functions raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_OK = 0
PA_ERR_INVALID_ARG = -1
PA_ERR_UNSUPPORTED = -2
PA_ERR_WORKSPACE = -3
PA_ERR_CUDA = -4
PA_ERR_SCRATCH_LIMIT = -5
PA_ERR_OUT_OF_BLOCKS = -6
NOALLOC_SCRATCH_BYTES = 32 << 20

PA_DTYPE_F32 = 0
PA_DTYPE_BF16 = 1

PA_DEVERR_SLOT_OOB = 1
PA_DEVERR_BLOCK_OOB = 2
PA_DEVERR_SEQ_LEN = 4
PA_DEVERR_TIMEOUT = 8
PA_DEVERR_PREFIX = 16
PA_DEVERR_Q_RANGE = 32

# every symbol the header declares, with (restype, argtypes)
_P, _I32, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_DECODE_ARGS = [_P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _F, _I32, _P, _SZ, _P, _I32, _P]
SIGNATURES = {
    "pa_cache_write": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _P, _P, _I32, _I32, _I32, _P]),
    "pa_cache_write_fp8": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _P, _P, _I32, _I32, _P, _P, _P]),
    "pa_decode_fp8": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I32,
                                     _F, _I32, _P, _SZ, _P, _P]),
    "pa_decode_fp8_partitions": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32,
                                                _I32, _I32, _F, _I32, _P, _SZ, _P, _P]),
    "pa_decode_fp8_reduce": (ctypes.c_int, [_P, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _P, _SZ, _P, _P]),
    "pa_decode_partition_blocks": (_I32, [_I32, _I32, _I32, _I32, _I32]),
    "pa_decode_workspace_size": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32, _I32]),
    "pa_decode": (ctypes.c_int, _DECODE_ARGS),
    "pa_decode_partitions": (ctypes.c_int, _DECODE_ARGS),
    "pa_decode_reduce": (ctypes.c_int, [_P, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _P, _SZ, _P, _I32, _P]),
    "pa_decode_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _F,
                                         _I32, _P, _I32, _P]),
    "pa_decode_shared_prefix": (ctypes.c_int, [_P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I32,
                                               _I32, _F, _I32, _P, _SZ, _P, _I32, _P]),
    "pa_decode_shared_prefix_workspace_size": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32]),
    "pa_decode_shared_prefix_groups": (ctypes.c_int, [_P, _P, _P, _P, _I32, _P, _I32, _P, _P, _I32, _I32, _I32,
                                                      _I32, _I32, _I32, _I32, _I32, _F, _I32, _P, _SZ, _P, _I32,
                                                      _P]),
    "pa_decode_shared_prefix_groups_workspace_size": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32]),
    "pa_decode_multi": (ctypes.c_int, [_P, _P, _I32, _I32, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32,
                                       _I32, _I32, _F, _I32, _P, _SZ, _P, _I32, _P]),
    "pa_decode_multi_workspace_size": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32]),
    "pa_copy_blocks": (ctypes.c_int, [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P]),
    "pa_bm_create": (_P, [_I32, _I32, _I32]),
    "pa_bm_destroy": (None, [_P]),
    "pa_bm_add_sequence": (ctypes.c_int, [_P, _I32]),
    "pa_bm_fork": (ctypes.c_int, [_P, _I32, _I32]),
    "pa_bm_append": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _P, _P]),
    "pa_bm_free_sequence": (ctypes.c_int, [_P, _I32]),
    "pa_bm_num_free": (_I32, [_P]),
    "pa_bm_refcount": (_I32, [_P, _I32]),
    "pa_bm_export_tables": (ctypes.c_int, [_P, _P, _I32, _P, _I32, _P]),
    "pa_get_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _I32, _P]),
    "pa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}

_lib = None


class PagedAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = lib().pa_status_string(status).decode()
        super().__init__(f"{fn} returned {status}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m paged_kv_cache_432_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _check(fn: str, rc: int):
    if rc != PA_OK:
        raise PagedAttnError(fn, rc)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return PA_DTYPE_F32
    if dt == torch.bfloat16:
        return PA_DTYPE_BF16
    raise TypeError(f"unsupported dtype {dt}")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def cache_write(k, v, slot_mapping, k_cache, v_cache, stream=None) -> None:
    """pa_cache_write: k, v [T, Hkv, D]; caches [NB, Hkv, 16, D]; slots int64 [T]."""
    T, H, D = k.shape
    NB, H2, B, D2 = k_cache.shape
    rc = lib().pa_cache_write(_ptr(k), _ptr(v), _ptr(slot_mapping), T, H, D, _ptr(k_cache),
                              _ptr(v_cache), NB, B, dtype_code(k.dtype), _stream(stream))
    _check("pa_cache_write", rc)


def cache_write_fp8(k, v, slot_mapping, k_cache, v_cache, k_inv_scale, v_inv_scale, stream=None) -> None:
    """pa_cache_write_fp8: k, v bf16 [T, Hkv, D]; caches uint8 (E4M3 codes)
    [NB, Hkv, 16, D]; inverse scales fp32 [Hkv]; slots int64 [T]."""
    T, H, D = k.shape
    NB, H2, B, D2 = k_cache.shape
    rc = lib().pa_cache_write_fp8(_ptr(k), _ptr(v), _ptr(slot_mapping), T, H, D, _ptr(k_cache), _ptr(v_cache),
                                  NB, B, _ptr(k_inv_scale), _ptr(v_inv_scale), _stream(stream))
    _check("pa_cache_write_fp8", rc)


def decode_fp8(q, k_cache, v_cache, k_scale, v_scale, block_tables, seq_lens, scale, out=None, max_seq_len=0,
               partition_blocks=0, workspace=None, stream=None) -> torch.Tensor:
    """pa_decode_fp8: q bf16 [N, Hq, D]; caches uint8 E4M3 [NB, Hkv, 16, D];
    scales fp32 [Hkv].  Returns out (bf16 [N, Hq, D])."""
    N, Hq, D = q.shape
    NB, Hkv, B, _ = k_cache.shape
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(N, Hq, Hkv, D, max_seq_len if max_seq_len > 0 else block_tables.shape[1] * 16,
                                    partition_blocks, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().pa_decode_fp8(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
                             _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), max_seq_len, N, Hq, Hkv, D,
                             NB, B, float(scale), partition_blocks, _ptr(workspace), ws_bytes, _ptr(out),
                             _stream(stream))
    _check("pa_decode_fp8", rc)
    return out


def decode_fp8_partitions(q, k_cache, v_cache, k_scale, v_scale, block_tables, seq_lens, scale, out, max_seq_len,
                          partition_blocks, workspace, stream=None) -> None:
    """pa_decode_fp8_partitions: the E4M3 block-table walk alone (final rows + partials)."""
    N, Hq, D = q.shape
    NB, Hkv, B, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().pa_decode_fp8_partitions(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
                                        _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), max_seq_len, N,
                                        Hq, Hkv, D, NB, B, float(scale), partition_blocks, _ptr(workspace),
                                        ws_bytes, _ptr(out), _stream(stream))
    _check("pa_decode_fp8_partitions", rc)


def decode_fp8_reduce(seq_lens, out, num_kv_heads, max_blocks_per_seq, max_seq_len, partition_blocks,
                      workspace, stream=None) -> None:
    """pa_decode_fp8_reduce: the log-sum-exp merge of an E4M3 partition step."""
    N, Hq, D = out.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().pa_decode_fp8_reduce(_ptr(seq_lens), max_seq_len, N, Hq, num_kv_heads, D, max_blocks_per_seq, 16,
                                    partition_blocks, _ptr(workspace), ws_bytes, _ptr(out), _stream(stream))
    _check("pa_decode_fp8_reduce", rc)


def partition_blocks(num_seqs, num_kv_heads, max_seq_len, partition_blocks=0, block_size=16) -> int:
    r = lib().pa_decode_partition_blocks(num_seqs, num_kv_heads, max_seq_len, block_size, partition_blocks)
    if r < 0:
        raise PagedAttnError("pa_decode_partition_blocks", r)
    return r


def workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len, partition_blocks=0,
                   block_size=16) -> int:
    return int(lib().pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                              max_seq_len, block_size, partition_blocks))


def alloc_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len, partition_blocks=0,
                    device=None) -> Optional[torch.Tensor]:
    n = workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len, partition_blocks)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


def _decode_call(name, q, k_cache, v_cache, block_tables, seq_lens, scale, out, max_seq_len,
                 partition_blocks, workspace, stream):
    N, Hq, D = q.shape
    NB, Hkv, B, _ = k_cache.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = getattr(lib(), name)(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1],
        _ptr(seq_lens), max_seq_len, N, Hq, Hkv, D, NB, B, float(scale), partition_blocks,
        _ptr(workspace), ws_bytes, _ptr(out), dtype_code(q.dtype), _stream(stream))
    _check(name, rc)


def decode(q, k_cache, v_cache, block_tables, seq_lens, scale, out=None, max_seq_len=0,
           partition_blocks=0, workspace=None, stream=None) -> torch.Tensor:
    """pa_decode: out [N, Hq, D] = paged decode attention.  Allocates `out` and the
    workspace with PyTorch when they are not given."""
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(q.shape[0], q.shape[1], k_cache.shape[1], q.shape[2],
                                    max_seq_len if max_seq_len > 0 else block_tables.shape[1] * 16,
                                    partition_blocks, device=q.device)
    _decode_call("pa_decode", q, k_cache, v_cache, block_tables, seq_lens, scale, out, max_seq_len,
                 partition_blocks, workspace, stream)
    return out


def shared_prefix_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len, shared_blocks,
                                 partition_blocks=0, block_size=16) -> int:
    return int(lib().pa_decode_shared_prefix_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                            max_seq_len, shared_blocks, block_size,
                                                            partition_blocks))


def decode_shared_prefix(q, k_cache, v_cache, block_tables, seq_lens, scale, shared_blocks, out=None,
                         max_seq_len=0, partition_blocks=0, workspace=None, stream=None) -> torch.Tensor:
    """pa_decode_shared_prefix: the decode when the first `shared_blocks` blocks of
    every table are one shared prefix (read once per kv head for all sequences)."""
    N, Hq, D = q.shape
    NB, Hkv, B, _ = k_cache.shape
    msl = max_seq_len if max_seq_len > 0 else block_tables.shape[1] * 16
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        n = shared_prefix_workspace_size(N, Hq, Hkv, D, msl, shared_blocks, partition_blocks)
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device) if n else None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().pa_decode_shared_prefix(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens),
        max_seq_len, shared_blocks, N, Hq, Hkv, D, NB, B, float(scale), partition_blocks, _ptr(workspace),
        ws_bytes, _ptr(out), dtype_code(q.dtype), _stream(stream))
    _check("pa_decode_shared_prefix", rc)
    return out


def shared_prefix_groups_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len,
                                        max_shared_blocks, num_groups, partition_blocks=0, block_size=16) -> int:
    return int(lib().pa_decode_shared_prefix_groups_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                                   max_seq_len, max_shared_blocks, num_groups,
                                                                   block_size, partition_blocks))


def decode_shared_prefix_groups(q, k_cache, v_cache, block_tables, seq_lens, scale, group_start,
                                group_shared_blocks, max_shared_blocks, out=None, max_seq_len=0, partition_blocks=0,
                                workspace=None, stream=None) -> torch.Tensor:
    """pa_decode_shared_prefix_groups: group i = sequences group_start[i] ..
    group_start[i+1]-1 (int32 device tensors), sharing their first
    group_shared_blocks[i] blocks; max_shared_blocks bounds those counts."""
    N, Hq, D = q.shape
    NB, Hkv, B, _ = k_cache.shape
    G = group_start.numel() - 1
    msl = max_seq_len if max_seq_len > 0 else block_tables.shape[1] * 16
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        n = shared_prefix_groups_workspace_size(N, Hq, Hkv, D, msl, max_shared_blocks, G, partition_blocks)
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device) if n else None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().pa_decode_shared_prefix_groups(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens),
        max_seq_len, _ptr(group_start), _ptr(group_shared_blocks), G, max_shared_blocks, N, Hq, Hkv, D, NB, B,
        float(scale), partition_blocks, _ptr(workspace), ws_bytes, _ptr(out), dtype_code(q.dtype), _stream(stream))
    _check("pa_decode_shared_prefix_groups", rc)
    return out


def decode_partitions(q, k_cache, v_cache, block_tables, seq_lens, scale, out, max_seq_len,
                      partition_blocks, workspace, stream=None) -> None:
    """pa_decode_partitions: the block-table walk alone (final rows + partials)."""
    _decode_call("pa_decode_partitions", q, k_cache, v_cache, block_tables, seq_lens, scale, out,
                 max_seq_len, partition_blocks, workspace, stream)


def decode_reduce(seq_lens, out, num_kv_heads, max_blocks_per_seq, max_seq_len, partition_blocks,
                  workspace, stream=None) -> None:
    """pa_decode_reduce: the log-sum-exp merge alone."""
    N, Hq, D = out.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().pa_decode_reduce(_ptr(seq_lens), max_seq_len, N, Hq, num_kv_heads, D,
                                max_blocks_per_seq, 16, partition_blocks, _ptr(workspace), ws_bytes,
                                _ptr(out), dtype_code(out.dtype), _stream(stream))
    _check("pa_decode_reduce", rc)


def decode_noalloc(q, k_cache, v_cache, block_tables, seq_lens, scale, out, max_seq_len=0,
                   partition_blocks=0, stream=None) -> torch.Tensor:
    """pa_decode_noalloc: the decode without any device allocation (its split-K
    partials live in the library's fixed 32 MiB buffer); `out` is required."""
    N, Hq, D = q.shape
    NB, Hkv, B, _ = k_cache.shape
    rc = lib().pa_decode_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1],
        _ptr(seq_lens), max_seq_len, N, Hq, Hkv, D, NB, B, float(scale), partition_blocks,
        _ptr(out), dtype_code(q.dtype), _stream(stream))
    _check("pa_decode_noalloc", rc)
    return out


def multi_workspace_size(num_seqs, num_q_rows, num_q_heads, num_kv_heads, head_dim, max_seq_len,
                         partition_blocks=0, block_size=16) -> int:
    return int(lib().pa_decode_multi_workspace_size(num_seqs, num_q_rows, num_q_heads, num_kv_heads, head_dim,
                                                    max_seq_len, block_size, partition_blocks))


def decode_multi(q, q_start, k_cache, v_cache, block_tables, seq_lens, scale, max_q_len, out=None, max_seq_len=0,
                 partition_blocks=0, workspace=None, stream=None) -> torch.Tensor:
    """pa_decode_multi: q [rows, Hq, D] packs each sequence's new query tokens
    (rows q_start[s] .. q_start[s+1]-1); causal among them.  Returns out [rows, Hq, D]."""
    T, Hq, D = q.shape
    NB, Hkv, B, _ = k_cache.shape
    N = seq_lens.numel()
    msl = max_seq_len if max_seq_len > 0 else block_tables.shape[1] * 16
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        n = multi_workspace_size(N, T, Hq, Hkv, D, msl, partition_blocks)
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device) if n else None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().pa_decode_multi(_ptr(q), _ptr(q_start), T, max_q_len, _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                               block_tables.shape[1], _ptr(seq_lens), max_seq_len, N, Hq, Hkv, D, NB, B,
                               float(scale), partition_blocks, _ptr(workspace), ws_bytes, _ptr(out),
                               dtype_code(q.dtype), _stream(stream))
    _check("pa_decode_multi", rc)
    return out


def copy_blocks(k_cache, v_cache, src, dst, stream=None) -> None:
    """pa_copy_blocks: block dst[i] of both pools <- block src[i] (int32 device tensors)."""
    NB, Hkv, B, D = k_cache.shape
    rc = lib().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(src), _ptr(dst), int(src.numel()), Hkv, D,
                              NB, B, dtype_code(k_cache.dtype), _stream(stream))
    _check("pa_copy_blocks", rc)


class BlockManager:
    """The library's host-side block manager (pa_bm_*): free list, reference
    counts, per-sequence tables; copy-on-write of shared partial blocks."""

    def __init__(self, num_blocks: int, block_size: int = 16, max_blocks_per_seq: int = 1 << 20):
        self.h = lib().pa_bm_create(num_blocks, block_size, max_blocks_per_seq)
        if not self.h:
            raise PagedAttnError("pa_bm_create", PA_ERR_INVALID_ARG)

    def __del__(self):
        if getattr(self, "h", None):
            lib().pa_bm_destroy(self.h)
            self.h = None

    def add(self, seq: int):
        _check("pa_bm_add_sequence", lib().pa_bm_add_sequence(self.h, seq))

    def fork(self, parent: int, child: int):
        _check("pa_bm_fork", lib().pa_bm_fork(self.h, parent, child))

    def append(self, seq: int, n: int):
        """-> (slots: list[int], copies: list[(src, dst)])"""
        slots = (ctypes.c_int64 * max(n, 1))()
        src, dst, nc = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        rc = lib().pa_bm_append(self.h, seq, n, slots, ctypes.byref(src), ctypes.byref(dst), ctypes.byref(nc))
        _check("pa_bm_append", rc)
        return list(slots[:n]), ([(src.value, dst.value)] if nc.value else [])

    def release(self, seq: int):
        _check("pa_bm_free_sequence", lib().pa_bm_free_sequence(self.h, seq))

    def num_free(self) -> int:
        return int(lib().pa_bm_num_free(self.h))

    def refcount(self, block: int) -> int:
        return int(lib().pa_bm_refcount(self.h, block))

    def tables(self, seq_ids, width: int):
        """-> (int32 tables [n][width] padded with -1, int32 lens [n]) as CPU tensors."""
        ids = (ctypes.c_int32 * max(len(seq_ids), 1))(*seq_ids)
        tab = torch.empty((len(seq_ids), width), dtype=torch.int32)
        lens = torch.empty(len(seq_ids), dtype=torch.int32)
        rc = lib().pa_bm_export_tables(self.h, ids, len(seq_ids), tab.data_ptr(), width, lens.data_ptr())
        _check("pa_bm_export_tables", rc)
        return tab, lens


def device_error(clear: bool = True, stream=None) -> int:
    """Sticky device error bits (PA_DEVERR_*) of the current device."""
    bits = ctypes.c_uint32(0)
    rc = lib().pa_get_device_error(ctypes.byref(bits), 1 if clear else 0, _stream(stream))
    _check("pa_get_device_error", rc)
    return int(bits.value)


def workspace_views(workspace: torch.Tensor, num_seqs, num_q_heads, head_dim, max_parts, num_kv_heads=None):
    """(m, l, acc, parts) views of a workspace, following the layout the header
    documents: float [rows][P], [rows][P], [rows][P][D] and int32 [N*Hkv], each
    on a 256-byte boundary (parts is None when num_kv_heads is not given)."""
    rows = num_seqs * num_q_heads
    a256 = lambda x: (x + 255) // 256 * 256
    ml = a256(rows * max_parts * 4)
    off_parts = 2 * ml + a256(rows * max_parts * head_dim * 4)
    f = workspace.view(torch.uint8)
    m = f[:rows * max_parts * 4].view(torch.float32).view(num_seqs, num_q_heads, max_parts)
    l = f[ml:ml + rows * max_parts * 4].view(torch.float32).view(num_seqs, num_q_heads, max_parts)
    acc = f[2 * ml:2 * ml + rows * max_parts * head_dim * 4].view(torch.float32).view(
        num_seqs, num_q_heads, max_parts, head_dim)
    parts = None
    if num_kv_heads is not None:
        parts = f[off_parts:off_parts + num_seqs * num_kv_heads * 4].view(torch.int32).view(
            num_seqs, num_kv_heads)
    return m, l, acc, parts
