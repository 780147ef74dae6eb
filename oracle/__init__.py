"""Python face of the double-precision CPU oracle (``rope_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` are the only callers.  Nothing here touches the CUDA library, and the
CUDA library never imports this package.

Arrays are numpy arrays holding the raw element bits: ``uint16`` for bf16 / f16 data,
``float32`` for f32 data.  Outputs (``q_out``, ``output``, the cache storage) are written in
place, exactly like the documented destination-passing-style operations.  Every function
returns the data-dependent error bits (``ERR_*``) it met; 0 means every token was written.

Parity status of the functions (what pins each one is stated in the test-suite):
  rope_split_store_paged_ragged, fused_qk_rmsnorm_rope_paged (multiply_before_cast=1),
  fused_dual_qk_rmsnorm_rope_paged, qk_rope_bshd_continuous, kv_cache_radd, and bands whose
  K is updated in place (k_col < 0; pinned against the store mode on a cache that holds the
  input's K): pinned.
  multiply_before_cast=0: parity unpinned (the pages name the flag without defining it; the
  reading implemented rounds the normalised value to the element type before the gamma
  multiply; what is checked is that the oracle implements that reading: at position 0 it
  equals single half-precision roundings done by Python's own float packing, and it reduces
  to the plain op at unit gamma).
  The choice of rotated columns under partial RoPE is a reading of an open point; it is
  pinned only against the reading it implements.
  FP8 (E4M3) caches: the element codec is pinned against torch's float8_e4m3fn; the format
  around it (one float32 scale per K / V plane, code = e4m3(value / scale), saturating) is
  parity unpinned: the pages name a scale type and a quantisation granularity only.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

DTYPES = {"bf16": 0, "f16": 1, "f32": 2, "fp8": 3}  # fp8: OCP E4M3 (cache elements only)
ERR_ROW_OFFSETS = 0x1
ERR_POSITION = 0x2
ERR_PAGE_INDEX = 0x4
ERR_PAGE_ID = 0x8
ERR_BATCH = 0x10
ERR_ARGS = 0x80000000

_c_void_p = ctypes.c_void_p
_i32, _i64, _u32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32


class _Paged(ctypes.Structure):
    _fields_ = [("k", _c_void_p), ("v", _c_void_p), ("dtype", _i32),
                ("n_kv_heads", _i32), ("head_dim", _i32), ("page_size", _i32),
                ("num_pages", _i32), ("num_layers", _i32),
                ("page_stride", _i64), ("layer_stride", _i64), ("slot_stride", _i64),
                ("head_stride", _i64), ("page_table", _c_void_p), ("page_table_stride", _i64),
                ("max_pages_per_seq", _i32), ("cache_lengths", _c_void_p), ("n_seqs", _i32),
                ("k_scale", _c_void_p), ("v_scale", _c_void_p)]


class _Cont(ctypes.Structure):
    _fields_ = [("k", _c_void_p), ("v", _c_void_p), ("dtype", _i32),
                ("n_kv_heads", _i32), ("head_dim", _i32), ("num_slots", _i32),
                ("num_layers", _i32), ("max_seq_len", _i32),
                ("slot_stride", _i64), ("layer_stride", _i64), ("pos_stride", _i64),
                ("head_stride", _i64), ("lookup_table", _c_void_p),
                ("cache_lengths", _c_void_p), ("n_seqs", _i32)]


class _Rope(ctypes.Structure):
    _fields_ = [("table", _c_void_p), ("dtype", _i32), ("max_seq_len", _i32),
                ("rope_dim", _i32), ("interleaved", _i32), ("rope_col_offset", _i32)]


class _Band(ctypes.Structure):
    _fields_ = [("input", _c_void_p), ("input_row_stride", _i64), ("q_col", _i64),
                ("k_col", _i64), ("v_col", _i64), ("n_q_heads", _i32),
                ("cache", ctypes.POINTER(_Paged)), ("q_gamma", _c_void_p),
                ("k_gamma", _c_void_p), ("epsilon", ctypes.c_double), ("q_out", _c_void_p),
                ("q_out_row_stride", _i64), ("written", _c_void_p), ("q_out_dtype", _i32)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        P = ctypes.POINTER
        lib.orc_rope_split_store_paged_ragged.argtypes = [
            _i32, _c_void_p, _i64, _i32, _i32, _c_void_p, _i32, P(_Rope), P(_Paged), _u32,
            _c_void_p, _i64, _i32, _c_void_p]
        lib.orc_fused_qk_rmsnorm_rope_paged.argtypes = [
            _i32, P(_Band), _c_void_p, _i32, _i32, P(_Rope), ctypes.c_double, _i32, _u32]
        lib.orc_fused_dual_qk_rmsnorm_rope_paged.argtypes = [
            _i32, P(_Band), P(_Band), _c_void_p, _i32, _i32, P(_Rope), ctypes.c_double, _i32,
            _u32]
        lib.orc_qk_rope_bshd_continuous.argtypes = [
            _i32, _c_void_p, _i32, _i32, _i32, _i32, P(_Cont), P(_Rope), _u32, _c_void_p,
            _c_void_p, _c_void_p]
        lib.orc_kv_cache_radd.argtypes = [
            _i32, _c_void_p, _i64, _i32, P(_Paged), _c_void_p, _i32, _u32, _u32, _c_void_p]
        lib.orc_matmul_fused_partial_rmsnorm.argtypes = [
            _i32, _c_void_p, _c_void_p, _i64, _i32, _i32, _c_void_p, ctypes.c_double,
            ctypes.c_double, _c_void_p, _i32, _c_void_p]
        for f in ("orc_rope_split_store_paged_ragged", "orc_fused_qk_rmsnorm_rope_paged",
                  "orc_fused_dual_qk_rmsnorm_rope_paged", "orc_qk_rope_bshd_continuous",
                  "orc_kv_cache_radd", "orc_matmul_fused_partial_rmsnorm"):
            getattr(lib, f).restype = _u32
        lib.orc_decode.argtypes = [_i32, _c_void_p, _i64]
        lib.orc_decode.restype = ctypes.c_double
        lib.orc_encode.argtypes = [_i32, _c_void_p, _i64, ctypes.c_double]
        lib.orc_encode.restype = None
        _lib = lib
    return _lib


# ----------------------------------------------------------------------------- inputs --

@dataclass
class PagedCache:
    """A paged K/V cache held in one flat host array ``storage``.

    K element (page, layer, slot, head, d) is ``storage[k_offset + page*page_stride +
    layer*layer_stride + slot*slot_stride + head*head_stride + d]``; V likewise from
    ``v_offset`` (None for a K-only cache)."""
    storage: np.ndarray
    k_offset: int
    v_offset: Optional[int]
    dtype: str
    n_kv_heads: int
    head_dim: int
    page_size: int
    num_pages: int
    num_layers: int
    page_stride: int
    layer_stride: int
    slot_stride: int
    head_stride: int
    page_table: np.ndarray      # uint32 [n_seqs, width]
    max_pages_per_seq: int
    cache_lengths: np.ndarray   # uint32 [n_seqs]
    k_scale: Optional[np.ndarray] = None  # float32 [1] each, for an fp8 cache
    v_scale: Optional[np.ndarray] = None


@dataclass
class ContCache:
    """A continuous-batching K/V cache: K element (slot, layer, pos, head, d) at
    ``storage[k_offset + slot*slot_stride + layer*layer_stride + pos*pos_stride +
    head*head_stride + d]``."""
    storage: np.ndarray
    k_offset: int
    v_offset: Optional[int]
    dtype: str
    n_kv_heads: int
    head_dim: int
    num_slots: int
    num_layers: int
    max_seq_len: int
    slot_stride: int
    layer_stride: int
    pos_stride: int
    head_stride: int
    lookup_table: np.ndarray    # uint32 [n_seqs]
    cache_lengths: np.ndarray   # uint32 [n_seqs]


@dataclass
class Rope:
    """freqs_cis [max_seq_len, rope_dim] (cos, sin interleaved) and the layout flags."""
    table: np.ndarray           # float32, or uint16 bits for bf16 / f16
    dtype: str
    interleaved: bool
    rope_col_offset: int = -1   # -1: the last rope_dim columns of a head are rotated


@dataclass
class Band:
    """One band of the per-head RMSNorm + RoPE op: where its Q / K / V heads sit in the
    token-major input, its cache, its gammas, epsilon and Q output."""
    input: np.ndarray           # 2-D [tokens, columns]
    q_col: int
    k_col: int
    v_col: int                  # -1: K-only cache (or V not stored)
    # k_col -1: K heads read from the token's cache slot and updated there (in place)
    n_q_heads: int
    cache: PagedCache
    q_gamma: np.ndarray
    k_gamma: np.ndarray
    epsilon: float
    q_out: np.ndarray           # 2-D [tokens, n_q_heads*head_dim]
    written: Optional[np.ndarray] = None


def _ptr(a: Optional[np.ndarray], offset_elems: int = 0) -> Optional[int]:
    if a is None:
        return None
    return a.ctypes.data + offset_elems * a.itemsize


def _row_stride(a: np.ndarray) -> int:
    assert a.ndim == 2 and a.strides[1] == a.itemsize, "rows must be contiguous"
    return a.strides[0] // a.itemsize


def _as_u32(a: np.ndarray) -> np.ndarray:
    assert a.dtype == np.uint32 and a.flags.c_contiguous
    return a


def _paged(c: PagedCache) -> _Paged:
    pt = _as_u32(c.page_table)
    return _Paged(_ptr(c.storage, c.k_offset),
                  None if c.v_offset is None else _ptr(c.storage, c.v_offset),
                  DTYPES[c.dtype], c.n_kv_heads, c.head_dim, c.page_size, c.num_pages,
                  c.num_layers, c.page_stride, c.layer_stride, c.slot_stride, c.head_stride,
                  _ptr(pt), pt.shape[1], c.max_pages_per_seq, _ptr(_as_u32(c.cache_lengths)),
                  pt.shape[0], _ptr(c.k_scale), _ptr(c.v_scale))


def _rope(r: Rope) -> _Rope:
    t = r.table
    assert t.ndim == 2 and t.flags.c_contiguous
    return _Rope(_ptr(t), DTYPES[r.dtype], t.shape[0], t.shape[1], int(bool(r.interleaved)),
                 r.rope_col_offset)


def _band(b: Band, keep: list) -> _Band:
    pc = _paged(b.cache)
    keep.append(pc)
    return _Band(_ptr(b.input), _row_stride(b.input), b.q_col, b.k_col, b.v_col, b.n_q_heads,
                 ctypes.pointer(pc), _ptr(b.q_gamma), _ptr(b.k_gamma), float(b.epsilon),
                 _ptr(b.q_out), _row_stride(b.q_out), _ptr(b.written), -1)


# ------------------------------------------------------------------------ operations --

def rope_split_store_paged_ragged(qkv, n_q_heads, input_row_offsets, rope: Rope,
                                  cache: PagedCache, layer_idx, q_out, written=None,
                                  dtype="bf16", q_out_dtype=None) -> int:
    offs = _as_u32(input_row_offsets)
    pc, rp = _paged(cache), _rope(rope)
    return _load().orc_rope_split_store_paged_ragged(
        DTYPES[dtype], _ptr(qkv), _row_stride(qkv), qkv.shape[0], n_q_heads, _ptr(offs),
        offs.shape[0] - 1, ctypes.byref(rp), ctypes.byref(pc), layer_idx, _ptr(q_out),
        _row_stride(q_out), DTYPES[q_out_dtype] if q_out_dtype else -1, _ptr(written))


def fused_qk_rmsnorm_rope_paged(band: Band, input_row_offsets, rope: Rope, weight_offset=0.0,
                                multiply_before_cast=True, layer_idx=0, dtype="bf16") -> int:
    offs = _as_u32(input_row_offsets)
    keep: list = []
    bd, rp = _band(band, keep), _rope(rope)
    return _load().orc_fused_qk_rmsnorm_rope_paged(
        DTYPES[dtype], ctypes.byref(bd), _ptr(offs), offs.shape[0] - 1, band.input.shape[0],
        ctypes.byref(rp), float(weight_offset), int(bool(multiply_before_cast)), layer_idx)


def fused_dual_qk_rmsnorm_rope_paged(main: Band, index: Band, input_row_offsets, rope: Rope,
                                     weight_offset=0.0, multiply_before_cast=True, layer_idx=0,
                                     dtype="bf16") -> int:
    offs = _as_u32(input_row_offsets)
    keep: list = []
    bm, bi, rp = _band(main, keep), _band(index, keep), _rope(rope)
    return _load().orc_fused_dual_qk_rmsnorm_rope_paged(
        DTYPES[dtype], ctypes.byref(bm), ctypes.byref(bi), _ptr(offs), offs.shape[0] - 1,
        main.input.shape[0], ctypes.byref(rp), float(weight_offset),
        int(bool(multiply_before_cast)), layer_idx)


def qk_rope_bshd_continuous(q_proj, cache: ContCache, rope: Rope, layer_idx, valid_lengths,
                            output, written=None, dtype="bf16") -> int:
    assert q_proj.ndim == 4 and q_proj.flags.c_contiguous and output.flags.c_contiguous
    B, S, H, D = q_proj.shape
    lt, cl = _as_u32(cache.lookup_table), _as_u32(cache.cache_lengths)
    cc = _Cont(_ptr(cache.storage, cache.k_offset),
               None if cache.v_offset is None else _ptr(cache.storage, cache.v_offset),
               DTYPES[cache.dtype], cache.n_kv_heads, cache.head_dim, cache.num_slots,
               cache.num_layers, cache.max_seq_len, cache.slot_stride, cache.layer_stride,
               cache.pos_stride, cache.head_stride, _ptr(lt), _ptr(cl), lt.shape[0])
    rp = _rope(rope)
    return _load().orc_qk_rope_bshd_continuous(
        DTYPES[dtype], _ptr(q_proj), B, S, H, D, ctypes.byref(cc), ctypes.byref(rp), layer_idx,
        _ptr(_as_u32(valid_lengths)), _ptr(output), _ptr(written))


def kv_cache_radd(a, cache: PagedCache, input_row_offsets, batch_offset, layer_idx,
                  written=None, dtype="bf16") -> int:
    offs = _as_u32(input_row_offsets)
    pc = _paged(cache)
    return _load().orc_kv_cache_radd(
        DTYPES[dtype], _ptr(a), _row_stride(a), a.shape[0], ctypes.byref(pc), _ptr(offs),
        offs.shape[0] - 1, batch_offset, layer_idx, _ptr(written))


# -------------------------------------------------------------------- element codecs --

def decode(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Element bits -> float64 values, through the oracle's own codec."""
    src = np.ascontiguousarray(bits)
    out = np.empty(src.size, dtype=np.float64)
    lib, code, p = _load(), DTYPES[dtype], _ptr(src)
    for i in range(src.size):
        out[i] = lib.orc_decode(code, p, i)
    return out.reshape(bits.shape)


def encode(values, dtype: str) -> np.ndarray:
    """float64 values -> element bits, rounded once to nearest-even by the oracle's codec."""
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.size, dtype={"f32": np.float32, "fp8": np.uint8}.get(dtype, np.uint16))
    lib, code, p = _load(), DTYPES[dtype], _ptr(out)
    flat = v.reshape(-1)
    for i in range(flat.size):
        lib.orc_encode(code, p, i, float(flat[i]))
    return out.reshape(v.shape)


def matmul_fused_partial_rmsnorm(x, weight, gamma, epsilon, weight_offset, normed_output,
                                 unnormed_output, dtype="bf16") -> int:
    """MatmulFusedPartialRMSNorm (one input row): x [k], weight [n, k] (rows may be padded),
    gamma [n_normed]; normed_output [n_normed] and unnormed_output [n - n_normed] are written
    in place."""
    n, k = weight.shape
    nn = normed_output.shape[0]
    assert unnormed_output.shape[0] == n - nn and x.shape[0] == k
    return _load().orc_matmul_fused_partial_rmsnorm(
        DTYPES[dtype], _ptr(x), _ptr(weight), _row_stride(weight), n, k, _ptr(gamma),
        float(epsilon), float(weight_offset), _ptr(normed_output), nn, _ptr(unnormed_output))
