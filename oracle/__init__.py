"""CPU oracle for the paged KV-cache decode path (fp64, single-threaded).

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The CUDA
library never calls it and shares no code with it; the only code both sides
use is the seeded input generator, which holds none of the method's arithmetic.

``oracle.c`` holds the arithmetic (plain loops, fp64, built with gcc without
fast-math); this module only marshals numpy arrays into it, plus the block
accounting of the pages' worked example, which is plain integer arithmetic.

Sources: "Was ändert PagedAttention an der KV-Speicherzuweisung für LLMs?"
(slavadubrov.com), introduction and §"Ungenutzten Platz in Blöcken berechnen";
"PagedAttention et vLLM" (aiunderstanding.org), §"Plongée profonde".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, IEEE semantics kept)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I32, I64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_cache_write.restype = I64
        lib.oracle_cache_write.argtypes = [P, P, P, I64, I32, I32, I32, P, P, I64, I32]
        lib.oracle_paged_decode.restype = ctypes.c_int
        lib.oracle_paged_decode.argtypes = [P, P, P, P, I32, P, I32, I32, I32, I32, I32, I64,
                                            I32, D, P, P, I32, P]
        lib.oracle_decode_partials.restype = ctypes.c_int
        lib.oracle_decode_partials.argtypes = [P, P, P, P, I32, P, I32, I32, I32, I32, I32, I64,
                                               I32, D, I32, I32, P, P, P, P]
        lib.oracle_paged_decode_multi.restype = ctypes.c_int
        lib.oracle_paged_decode_multi.argtypes = [P, P, P, P, I32, P, P, I32, I32, I32, I32, I32, I64,
                                                  I32, D, P]
        lib.oracle_e4m3_decode.restype = D
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_cache_write_fp8.restype = I64
        lib.oracle_cache_write_fp8.argtypes = [P, P, P, I64, I32, I32, P, P, I64, I32, P, P]
        lib.oracle_paged_decode_fp8.restype = ctypes.c_int
        lib.oracle_paged_decode_fp8.argtypes = [P, P, P, P, I32, P, I32, I32, I32, I32, I32, I64, P, P, D, P]
        lib.oracle_copy_blocks.restype = I64
        lib.oracle_copy_blocks.argtypes = [P, P, P, P, I64, I64, I64]
        lib.oracle_lse_merge.restype = None
        lib.oracle_lse_merge.argtypes = [P, P, P, P, I32, I32, I32, I32, P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:  # raw bf16 bits
        return BF16
    raise TypeError(f"oracle takes float32 or bf16 bits (uint16), got {a.dtype}")


# ---------------------------------------------------------------- block accounting
def blocks_needed(seq_len: int, block_size: int = 16) -> int:
    """Blocks a sequence occupies: ceil(L / B)."""
    return -(-seq_len // block_size)


def allocated_slots(seq_len: int, block_size: int = 16) -> int:
    return blocks_needed(seq_len, block_size) * block_size


def unused_slots(seq_len: int, block_size: int = 16) -> int:
    """Slots left empty; all of them are in the last block."""
    return allocated_slots(seq_len, block_size) - seq_len


def slot_utilisation(lens, block_size: int = 16) -> float:
    """Occupied token positions / allocated token positions over a batch."""
    alloc = sum(allocated_slots(L, block_size) for L in lens)
    return (sum(lens) / alloc) if alloc else 1.0


# ---------------------------------------------------------------- cache write
def cache_write(k, v, slot_mapping, k_cache, v_cache, inplace=False):
    """Scatter new tokens into copies of the caches (or into the given C-contiguous
    caches when inplace=True); returns (k_cache, v_cache, n_bad).

    k, v: [T, Hkv, D]; caches [NB, Hkv, B, D]; slot_mapping int64 [T].
    """
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    if inplace:
        assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
        kc, vc = k_cache, v_cache
    else:
        kc = np.array(k_cache, copy=True, order="C")
        vc = np.array(v_cache, copy=True, order="C")
    dt = _dtype_code(k)
    assert kc.dtype == k.dtype == v.dtype == vc.dtype
    T, H, D = k.shape
    NB, H2, B, D2 = kc.shape
    assert (H, D) == (H2, D2)
    bad = _load().oracle_cache_write(_ptr(k), _ptr(v), _ptr(sm), T, H, D, dt, _ptr(kc), _ptr(vc), NB, B)
    return kc, vc, int(bad)


def e4m3_decode(code: int) -> float:
    """Value of an FP8 E4M3 code (NaN for S.1111.111)."""
    return _load().oracle_e4m3_decode(int(code) & 0xFF)


def e4m3_encode(y: float) -> int:
    """Nearest E4M3 code of a float32 value (ties to even, saturating at 448)."""
    return int(_load().oracle_e4m3_encode(float(np.float32(y))))


def cache_write_fp8(k, v, slot_mapping, k_cache, v_cache, k_inv_scale, v_inv_scale):
    """Quantising scatter into E4M3 caches (uint8 [NB, Hkv, B, D]); k, v bf16 bits.
    Returns (k_cache, v_cache, n_bad) as copies."""
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    kc = np.array(k_cache, dtype=np.uint8, copy=True, order="C")
    vc = np.array(v_cache, dtype=np.uint8, copy=True, order="C")
    ks = np.ascontiguousarray(k_inv_scale, dtype=np.float32)
    vs = np.ascontiguousarray(v_inv_scale, dtype=np.float32)
    T, H, D = k.shape
    NB, _, B, _ = kc.shape
    bad = _load().oracle_cache_write_fp8(_ptr(k), _ptr(v), _ptr(sm), T, H, D, _ptr(kc), _ptr(vc), NB, B,
                                         _ptr(ks), _ptr(vs))
    return kc, vc, int(bad)


def paged_decode_fp8(q, k_cache, v_cache, block_tables, seq_lens, k_scale, v_scale, scale):
    """fp64 decode over E4M3 caches (value = decode(code) * scale of the kv head);
    q as bf16 bits.  Returns [N, Hq, D]."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    kc = np.ascontiguousarray(k_cache, dtype=np.uint8)
    vc = np.ascontiguousarray(v_cache, dtype=np.uint8)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    ks = np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = np.ascontiguousarray(v_scale, dtype=np.float32)
    N, Hq, D = q.shape
    NB, Hkv, B, _ = kc.shape
    out = np.zeros((N, Hq, D), dtype=np.float64)
    rc = _load().oracle_paged_decode_fp8(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), bt.shape[1], _ptr(sl), N, Hq, Hkv,
                                         D, B, NB, _ptr(ks), _ptr(vs), float(scale), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_paged_decode_fp8 failed ({rc})")
    return out


def copy_blocks(k_cache, v_cache, src, dst):
    """Copies of the pools where block dst[i] = block src[i] (both pools, all
    heads); returns (k_cache, v_cache, n_bad)."""
    kc = np.array(k_cache, copy=True, order="C")
    vc = np.array(v_cache, copy=True, order="C")
    src = np.ascontiguousarray(src, dtype=np.int32)
    dst = np.ascontiguousarray(dst, dtype=np.int32)
    assert src.shape == dst.shape
    NB = kc.shape[0]
    bb = kc[0].nbytes
    bad = _load().oracle_copy_blocks(_ptr(kc), _ptr(vc), _ptr(src), _ptr(dst), len(src), NB, bb)
    return kc, vc, int(bad)


# ---------------------------------------------------------------- decode
def _decode_args(q, k_cache, v_cache, block_tables, seq_lens):
    q = np.ascontiguousarray(q)
    kc = np.ascontiguousarray(k_cache)
    vc = np.ascontiguousarray(v_cache)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    assert q.dtype == kc.dtype == vc.dtype
    return q, kc, vc, bt, sl


def paged_decode(q, k_cache, v_cache, block_tables, seq_lens, scale, rows=None):
    """fp64 decode attention through block tables.

    q [N, Hq, D]; caches [NB, Hkv, B, D]; block_tables int32 [N, max_blocks];
    seq_lens int32 [N]; scale: the float32 value the kernel receives.
    rows: optional list of (seq, q_head) pairs -> returns [len(rows), D];
    otherwise returns [N, Hq, D].
    """
    q, kc, vc, bt, sl = _decode_args(q, k_cache, v_cache, block_tables, seq_lens)
    N, Hq, D = q.shape
    NB, Hkv, B, _ = kc.shape
    if rows is None:
        out = np.zeros((N, Hq, D), dtype=np.float64)
        sel_s = sel_h = None
        nsel = 0
    else:
        rows = np.asarray(rows, dtype=np.int32).reshape(-1, 2)
        sel_s = np.ascontiguousarray(rows[:, 0])
        sel_h = np.ascontiguousarray(rows[:, 1])
        nsel = len(rows)
        out = np.zeros((nsel, D), dtype=np.float64)
    rc = _load().oracle_paged_decode(
        _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), bt.shape[1], _ptr(sl), N, Hq, Hkv, D, B, NB,
        _dtype_code(q), float(scale),
        _ptr(sel_s) if sel_s is not None else None,
        _ptr(sel_h) if sel_h is not None else None, nsel, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_paged_decode failed ({rc})")
    return out


def paged_decode_multi(q, k_cache, v_cache, block_tables, seq_lens, q_start, scale):
    """fp64 attention of several new query tokens per sequence (causal among
    them).  q [rows, Hq, D] packs each sequence's query tokens (rows
    q_start[s] .. q_start[s+1]-1), which are the sequence's last positions.
    Returns [rows, Hq, D]."""
    q, kc, vc, bt, sl = _decode_args(q, k_cache, v_cache, block_tables, seq_lens)
    qs = np.ascontiguousarray(q_start, dtype=np.int32)
    T, Hq, D = q.shape
    NB, Hkv, B, _ = kc.shape
    N = len(sl)
    assert len(qs) == N + 1 and qs[-1] == T
    out = np.zeros((T, Hq, D), dtype=np.float64)
    rc = _load().oracle_paged_decode_multi(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), bt.shape[1], _ptr(sl),
                                           _ptr(qs), N, Hq, Hkv, D, B, NB, _dtype_code(q), float(scale),
                                           _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_paged_decode_multi failed ({rc})")
    return out


def decode_partials(q, k_cache, v_cache, block_tables, seq_lens, scale, partition_tokens):
    """Per-partition (m, l, acc) of the split-K form; returns (m, l, acc, nparts)."""
    q, kc, vc, bt, sl = _decode_args(q, k_cache, v_cache, block_tables, seq_lens)
    N, Hq, D = q.shape
    NB, Hkv, B, _ = kc.shape
    max_parts = max(1, max((int(L) + partition_tokens - 1) // partition_tokens for L in sl) if N else 1)
    m = np.zeros((N, Hq, max_parts), dtype=np.float64)
    l = np.zeros((N, Hq, max_parts), dtype=np.float64)
    acc = np.zeros((N, Hq, max_parts, D), dtype=np.float64)
    nparts = np.zeros(N, dtype=np.int32)
    rc = _load().oracle_decode_partials(
        _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), bt.shape[1], _ptr(sl), N, Hq, Hkv, D, B, NB,
        _dtype_code(q), float(scale), partition_tokens, max_parts, _ptr(m), _ptr(l), _ptr(acc),
        _ptr(nparts))
    if rc != 0:
        raise ValueError(f"oracle_decode_partials failed ({rc})")
    return m, l, acc, nparts


def lse_merge(m, l, acc, nparts):
    """Log-sum-exp merge of decode_partials' output -> [N, Hq, D]."""
    m = np.ascontiguousarray(m, dtype=np.float64)
    l = np.ascontiguousarray(l, dtype=np.float64)
    acc = np.ascontiguousarray(acc, dtype=np.float64)
    nparts = np.ascontiguousarray(nparts, dtype=np.int32)
    N, Hq, P, D = acc.shape
    out = np.zeros((N, Hq, D), dtype=np.float64)
    _load().oracle_lse_merge(_ptr(m), _ptr(l), _ptr(acc), _ptr(nparts), N, Hq, D, P, _ptr(out))
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bit patterns (test helper for comparisons)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
