"""Python binding of ``librope_store.so`` (include/rope_store.h): argument marshalling only.

Every function takes torch CUDA tensors (for memory) and an optional torch CUDA stream,
builds the C descriptors from their data pointers and calls the C entry point of the same
name.  All arithmetic runs in the library's sm_100a kernels; there is no fallback, and a
missing library raises at import time.

Descriptors
-----------
Freqs(table, interleaved, rope_col_offset=-1)
    freqs_cis [max_seq_len, rope_dim] (f32 / bf16 / f16): (cos, sin) of pair i at columns
    2i, 2i+1.  rope_col_offset: first rotated column of a head (-1 = head_dim - rope_dim).
PagedCache(k, v, page_table, cache_lengths, n_kv_heads, head_dim, page_size, num_pages,
           num_layers, page_stride, layer_stride, slot_stride, head_stride)
    k / v: tensors whose data pointers are the K / V plane bases (v may be None for a K-only
    cache); strides in elements; page_table int32/uint32 [n_seqs, width]; cache_lengths
    [n_seqs].
ContCache(k, v, lookup_table, cache_lengths, n_kv_heads, head_dim, num_slots, num_layers,
          max_seq_len, slot_stride, layer_stride, pos_stride, head_stride)
NormBand(input, q_col, k_col, v_col, n_q_heads, cache, q_gamma, k_gamma, epsilon, q_out)

Scheduling workspace and launch overlap
---------------------------------------
The staged entry points take ``sched``: None (a static token schedule) or a device tensor of
at least SCHED_WORDS int32 words that is zero before its first use (``sched_workspace()``);
every call leaves it zero.  Concurrent calls on different streams need separate
workspaces.  ``set_launch_overlap(mode)`` picks how launches overlap the previous kernel of
the stream (OVERLAP_OFF, OVERLAP_PDL = default, OVERLAP_PDL_EARLY_METADATA).
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_PKG, "librope_store.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "rope_store.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA = 0, 1, 2, 3
DEVERR_ROW_OFFSETS, DEVERR_POSITION, DEVERR_PAGE_INDEX = 0x1, 0x2, 0x4
DEVERR_PAGE_ID, DEVERR_BATCH, DEVERR_TIMEOUT = 0x8, 0x10, 0x20
SCHED_WORDS = 2
OVERLAP_OFF, OVERLAP_PDL, OVERLAP_PDL_EARLY_METADATA = 0, 1, 2

_DTYPE_CODE = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2,
               torch.float8_e4m3fn: 3}

if not os.path.exists(LIBRARY_PATH):
    raise ImportError(f"{LIBRARY_PATH} is missing: build it with "
                      f"`python rope_paged_kv_b200/build.py` (nvcc, sm_100a)")
_lib = ctypes.CDLL(LIBRARY_PATH)

_vp, _i32, _i64, _u32, _f32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                               ctypes.c_uint32, ctypes.c_float)


class c_freqs(ctypes.Structure):
    _fields_ = [("data", _vp), ("dtype", _i32), ("max_seq_len", _i32), ("rope_dim", _i32),
                ("interleaved", _i32), ("rope_col_offset", _i32)]


class c_paged_cache(ctypes.Structure):
    _fields_ = [("k", _vp), ("v", _vp), ("dtype", _i32), ("n_kv_heads", _i32),
                ("head_dim", _i32), ("page_size", _i32), ("num_pages", _i32),
                ("num_layers", _i32), ("page_stride", _i64), ("layer_stride", _i64),
                ("slot_stride", _i64), ("head_stride", _i64), ("page_table", _vp),
                ("page_table_stride", _i64), ("max_pages_per_seq", _i32),
                ("cache_lengths", _vp), ("n_seqs", _i32), ("k_scale", _vp), ("v_scale", _vp)]


class c_cont_cache(ctypes.Structure):
    _fields_ = [("k", _vp), ("v", _vp), ("dtype", _i32), ("n_kv_heads", _i32),
                ("head_dim", _i32), ("num_slots", _i32), ("num_layers", _i32),
                ("max_seq_len", _i32), ("slot_stride", _i64), ("layer_stride", _i64),
                ("pos_stride", _i64), ("head_stride", _i64), ("lookup_table", _vp),
                ("cache_lengths", _vp), ("n_seqs", _i32)]


class c_norm_band(ctypes.Structure):
    _fields_ = [("input", _vp), ("input_row_stride", _i64), ("q_col", _i64), ("k_col", _i64),
                ("v_col", _i64), ("n_q_heads", _i32), ("cache", ctypes.POINTER(c_paged_cache)),
                ("q_gamma", _vp), ("k_gamma", _vp), ("epsilon", _f32), ("q_out", _vp),
                ("q_out_row_stride", _i64)]


_P = ctypes.POINTER
_lib.rope_split_store_paged_ragged.argtypes = [
    _vp, _i64, _i32, _i32, _i32, _vp, _i32, _P(c_freqs), _P(c_paged_cache), _u32, _vp, _i64,
    _i32, _vp, _vp, _vp]
_lib.fused_qk_rmsnorm_rope_paged.argtypes = [
    _vp, _i64, _i32, _i32, _i32, _vp, _i32, _P(c_freqs), _P(c_paged_cache), _vp, _vp, _f32,
    _f32, _i32, _u32, _vp, _i64, _vp, _vp, _vp]
_lib.fused_dual_qk_rmsnorm_rope_paged.argtypes = [
    _P(c_norm_band), _P(c_norm_band), _i32, _vp, _i32, _i32, _P(c_freqs), _f32, _i32, _u32,
    _vp, _vp, _vp]
_lib.qk_rope_bshd_continuous.argtypes = [
    _vp, _i32, _i32, _i32, _i32, _P(c_cont_cache), _P(c_freqs), _u32, _vp, _vp, _vp, _vp]
_lib.kv_cache_radd.argtypes = [
    _vp, _i64, _i32, _P(c_paged_cache), _vp, _i32, _u32, _u32, _vp, _vp, _vp]
_lib.rope_split_store_paged_ragged_noalloc.argtypes = [
    _vp, _i64, _i32, _i32, _i32, _vp, _i32, _P(c_freqs), _P(c_paged_cache), _u32, _vp, _i64,
    _i32, _vp, _vp]
_lib.matmul_fused_partial_rmsnorm.argtypes = [
    _vp, _vp, _i64, _i32, _i32, _i32, _vp, _f32, _f32, _vp, _i32, _vp, _i32, _vp, _vp, _i64,
    _vp]
_lib.rope_set_launch_overlap.argtypes = [_i32]
_lib.rope_get_launch_overlap.argtypes = []
_lib.rope_get_launch_overlap.restype = _i32
_lib.rope_set_stall_test.argtypes = [_u32]
_lib.rope_get_stall_test.argtypes = []
_lib.rope_get_stall_test.restype = _u32
for _f in ("rope_split_store_paged_ragged", "fused_qk_rmsnorm_rope_paged",
           "fused_dual_qk_rmsnorm_rope_paged", "qk_rope_bshd_continuous", "kv_cache_radd",
           "rope_set_launch_overlap", "rope_split_store_paged_ragged_noalloc",
           "rope_set_stall_test",
           "matmul_fused_partial_rmsnorm"):
    getattr(_lib, _f).restype = ctypes.c_int
_lib.rope_status_string.argtypes = [ctypes.c_int]
_lib.rope_status_string.restype = ctypes.c_char_p


def header_functions() -> list:
    """Names of the functions include/rope_store.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return re.findall(r"^(?:rope_status_t|int32_t|const char \*)\s*\n?\s*\**(\w+)\(", text,
                      re.M)


class RopeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.rope_status_string(status).decode()} "
                         f"(status {status})")


def _check(status: int, where: str) -> None:
    if status != OK:
        raise RopeError(status, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _sched(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if (t.dtype not in (torch.int32, torch.uint32) or not t.is_contiguous()
            or t.numel() < SCHED_WORDS or not t.is_cuda):
        raise ValueError(f"sched must be a contiguous CUDA int32 tensor of >= {SCHED_WORDS} words")
    return t.data_ptr()


def sched_workspace(device=None) -> torch.Tensor:
    """A zeroed scheduling workspace for the staged entry points."""
    return torch.zeros(SCHED_WORDS, dtype=torch.int32,
                       device=device if device is not None else torch.cuda.current_device())


def set_launch_overlap(mode: int) -> None:
    """How launches overlap the previous kernel of their stream (process-wide)."""
    _check(_lib.rope_set_launch_overlap(int(mode)), "rope_set_launch_overlap")


def get_launch_overlap() -> int:
    return int(_lib.rope_get_launch_overlap())


def set_stall_test(timeout_us: int) -> None:
    """A diagnostic of the timeout path (process-wide): with timeout_us > 0 the staged
    kernels of the launches that follow start with a wait that nothing completes, bounded by
    timeout_us; when it runs out they take the path of a wait that runs out.  0: off."""
    _check(_lib.rope_set_stall_test(int(timeout_us)), "rope_set_stall_test")


def get_stall_test() -> int:
    return int(_lib.rope_get_stall_test())


def _row_stride(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with contiguous rows")
    return t.stride(0)


def _code(t: torch.Tensor) -> int:
    """rope_dtype_t of a tensor's element type."""
    try:
        return _DTYPE_CODE[t.dtype]
    except KeyError:
        raise ValueError(f"unsupported element type {t.dtype}") from None


def _idx(t: torch.Tensor) -> torch.Tensor:
    if t.dtype not in (torch.int32, torch.uint32) or not t.is_contiguous():
        raise ValueError("index arrays must be contiguous int32/uint32")
    return t


@dataclass
class Freqs:
    table: torch.Tensor
    interleaved: bool
    rope_col_offset: int = -1

    def c(self) -> c_freqs:
        t = self.table
        if t.dim() != 2 or not t.is_contiguous():
            raise ValueError("freqs_cis must be a contiguous [max_seq_len, rope_dim] tensor")
        return c_freqs(t.data_ptr(), _code(t), t.shape[0], t.shape[1],
                       int(bool(self.interleaved)), self.rope_col_offset)


@dataclass
class PagedCache:
    k: torch.Tensor
    v: Optional[torch.Tensor]
    page_table: torch.Tensor
    cache_lengths: torch.Tensor
    n_kv_heads: int
    head_dim: int
    page_size: int
    num_pages: int
    num_layers: int
    page_stride: int
    layer_stride: int
    slot_stride: int
    head_stride: int
    max_pages_per_seq: Optional[int] = None
    k_scale: Optional[torch.Tensor] = None  # float32 [1] each, for an fp8 (E4M3) cache
    v_scale: Optional[torch.Tensor] = None

    def c(self) -> c_paged_cache:
        pt = _idx(self.page_table)
        width = pt.shape[1] if self.max_pages_per_seq is None else self.max_pages_per_seq
        return c_paged_cache(self.k.data_ptr(), _ptr(self.v), _code(self.k),
                             self.n_kv_heads, self.head_dim, self.page_size, self.num_pages,
                             self.num_layers, self.page_stride, self.layer_stride,
                             self.slot_stride, self.head_stride, pt.data_ptr(), pt.stride(0),
                             width, _idx(self.cache_lengths).data_ptr(), pt.shape[0],
                             _ptr(self.k_scale), _ptr(self.v_scale))


@dataclass
class ContCache:
    k: torch.Tensor
    v: Optional[torch.Tensor]
    lookup_table: torch.Tensor
    cache_lengths: torch.Tensor
    n_kv_heads: int
    head_dim: int
    num_slots: int
    num_layers: int
    max_seq_len: int
    slot_stride: int
    layer_stride: int
    pos_stride: int
    head_stride: int

    def c(self) -> c_cont_cache:
        lt = _idx(self.lookup_table)
        return c_cont_cache(self.k.data_ptr(), _ptr(self.v), _code(self.k),
                            self.n_kv_heads, self.head_dim, self.num_slots, self.num_layers,
                            self.max_seq_len, self.slot_stride, self.layer_stride,
                            self.pos_stride, self.head_stride, lt.data_ptr(),
                            _idx(self.cache_lengths).data_ptr(), lt.shape[0])


@dataclass
class NormBand:
    input: torch.Tensor
    q_col: int
    k_col: int
    v_col: int
    n_q_heads: int
    cache: PagedCache
    q_gamma: torch.Tensor
    k_gamma: torch.Tensor
    epsilon: float
    q_out: torch.Tensor

    def c(self, keep: list) -> c_norm_band:
        pc = self.cache.c()
        keep.append(pc)
        return c_norm_band(self.input.data_ptr(), _row_stride(self.input), self.q_col,
                           self.k_col, self.v_col, self.n_q_heads, ctypes.pointer(pc),
                           self.q_gamma.data_ptr(), self.k_gamma.data_ptr(), self.epsilon,
                           self.q_out.data_ptr(), _row_stride(self.q_out))


# ------------------------------------------------------------------------ entry points --

def rope_split_store_paged_ragged(qkv, n_q_heads, input_row_offsets, freqs: Freqs,
                                  kv: PagedCache, layer_idx, q_out, err_word=None,
                                  stream=None, sched=None) -> None:
    """Rotate Q and K of a flat ragged QKV batch, write Q to q_out (in q_out's element type)
    and store K and V into the paged cache `kv` (rope_split_store_paged_ragged page:
    signature, Parameters, Args).  qkv [T, (Hq + 2 Hk) D]; input_row_offsets [batch + 1]."""
    offs = _idx(input_row_offsets)
    f, c = freqs.c(), kv.c()
    _check(_lib.rope_split_store_paged_ragged(
        qkv.data_ptr(), _row_stride(qkv), _code(qkv), qkv.shape[0], n_q_heads,
        offs.data_ptr(),
        offs.shape[0] - 1, ctypes.byref(f), ctypes.byref(c), layer_idx, q_out.data_ptr(),
        _row_stride(q_out), _code(q_out), _ptr(err_word), _sched(sched),
        _stream(stream)), "rope_split_store_paged_ragged")


def rope_split_store_paged_ragged_noalloc(qkv, n_q_heads, input_row_offsets, freqs: Freqs,
                                          kv: PagedCache, layer_idx, q_out, err_word=None,
                                          stream=None) -> None:
    """rope_split_store_paged_ragged for callers that cannot allocate device memory: the
    scheduling workspace is the library's own per-device array (calls on different streams
    must not overlap)."""
    offs = _idx(input_row_offsets)
    f, c = freqs.c(), kv.c()
    _check(_lib.rope_split_store_paged_ragged_noalloc(
        qkv.data_ptr(), _row_stride(qkv), _code(qkv), qkv.shape[0], n_q_heads,
        offs.data_ptr(),
        offs.shape[0] - 1, ctypes.byref(f), ctypes.byref(c), layer_idx, q_out.data_ptr(),
        _row_stride(q_out), _code(q_out), _ptr(err_word), _stream(stream)),
        "rope_split_store_paged_ragged_noalloc")


def fused_qk_rmsnorm_rope_paged(qkv, n_q_heads, input_row_offsets, freqs: Freqs,
                                kv: PagedCache, q_gamma, k_gamma, epsilon, weight_offset,
                                layer_idx, q_out, multiply_before_cast=True, err_word=None,
                                stream=None, sched=None) -> None:
    """Per-head RMSNorm, then RoPE, of Q and K, with the paged store of
    rope_split_store_paged_ragged: the single-band op that the
    fused_dual_qk_rms_norm_rope_ragged_paged page fuses twice (its first paragraph)."""
    offs = _idx(input_row_offsets)
    f, c = freqs.c(), kv.c()
    _check(_lib.fused_qk_rmsnorm_rope_paged(
        qkv.data_ptr(), _row_stride(qkv), _code(qkv), qkv.shape[0], n_q_heads,
        offs.data_ptr(),
        offs.shape[0] - 1, ctypes.byref(f), ctypes.byref(c), q_gamma.data_ptr(),
        k_gamma.data_ptr(), epsilon, weight_offset, int(bool(multiply_before_cast)), layer_idx,
        q_out.data_ptr(), _row_stride(q_out), _ptr(err_word), _sched(sched), _stream(stream)),
        "fused_qk_rmsnorm_rope_paged")


def fused_dual_qk_rmsnorm_rope_paged(main_band: NormBand, index_band: Optional[NormBand],
                                     input_row_offsets, total_tokens, freqs: Freqs,
                                     weight_offset, layer_idx, multiply_before_cast=True,
                                     err_word=None, stream=None, sched=None) -> None:
    """The main band and the index band in one launch (fused_dual_qk_rms_norm_rope_ragged_paged
    page: signature and both paragraphs); index_band None launches the main band alone.  A
    band with k_col < 0 reads its K heads from the token's cache slot and writes them back
    there (the key cache updated in place)."""
    offs = _idx(input_row_offsets)
    keep: list = []
    m, f = main_band.c(keep), freqs.c()
    i = None if index_band is None else ctypes.byref(index_band.c(keep))
    _check(_lib.fused_dual_qk_rmsnorm_rope_paged(
        ctypes.byref(m), i, _code(main_band.input), offs.data_ptr(),
        offs.shape[0] - 1, total_tokens,
        ctypes.byref(f), weight_offset, int(bool(multiply_before_cast)), layer_idx,
        _ptr(err_word), _sched(sched), _stream(stream)), "fused_dual_qk_rmsnorm_rope_paged")


def qk_rope_bshd_continuous(q_proj, kv: ContCache, freqs: Freqs, layer_idx, valid_lengths,
                            output, err_word=None, stream=None) -> None:
    """Continuous-batching decode RoPE: Q of q_proj [B, S, H, D] rotated into output, K
    rotated in place in its cache slot, for s < valid_lengths[b]
    (generic_fused_qk_rope_bshd_continuous_batch page: signature, description, Args)."""
    if q_proj.dim() != 4 or not q_proj.is_contiguous() or not output.is_contiguous():
        raise ValueError("q_proj / output must be contiguous [batch, seq_len, heads, head_dim]")
    B, S, H, D = q_proj.shape
    c, f = kv.c(), freqs.c()
    _check(_lib.qk_rope_bshd_continuous(
        q_proj.data_ptr(), B, S, H, D, ctypes.byref(c), ctypes.byref(f), layer_idx,
        _idx(valid_lengths).data_ptr(), output.data_ptr(), _ptr(err_word), _stream(stream)),
        "qk_rope_bshd_continuous")


def kv_cache_radd(a, kv: PagedCache, input_row_offsets, batch_offset, layer_idx,
                  err_word=None, stream=None, sched=None) -> None:
    """Add a [T, 2 Hk D] into the K (first half of the columns) and V rows of the paged
    cache at each token's position (generic_kv_cache_radd_dispatch page: description,
    Args)."""
    offs = _idx(input_row_offsets)
    c = kv.c()
    _check(_lib.kv_cache_radd(
        a.data_ptr(), _row_stride(a), a.shape[0], ctypes.byref(c), offs.data_ptr(),
        offs.shape[0] - 1, batch_offset, layer_idx, _ptr(err_word), _sched(sched),
        _stream(stream)), "kv_cache_radd")


def gemv_workspace_bytes(n_normed: int) -> int:
    return 16 + 4 * int(n_normed)


def gemv_workspace(n_normed: int, device=None) -> torch.Tensor:
    """A zeroed workspace for matmul_fused_partial_rmsnorm (16-byte aligned)."""
    return torch.zeros(gemv_workspace_bytes(n_normed) // 4, dtype=torch.int32,
                       device=device if device is not None else torch.cuda.current_device())


def matmul_fused_partial_rmsnorm(input, weight, gamma, epsilon, weight_offset, normed_output,
                                 unnormed_output, workspace=None, stream=None,
                                 err_word=None) -> None:
    """y = input @ weight.T (input [k], weight [n, k]); normed_output [n_normed] gets the RMS
    normalised first entries times gamma, unnormed_output [n - n_normed] the rest
    (MatmulFusedPartialRMSNorm page: description, execute, Args)."""
    n, k = weight.shape
    nn = normed_output.shape[0]
    if unnormed_output.shape[0] != n - nn or input.shape[-1] != k:
        raise ValueError("output sizes must split n; input must have k entries")
    dtype = _code(weight)
    for name, t in (("input", input), ("gamma", gamma), ("normed_output", normed_output),
                    ("unnormed_output", unnormed_output)):
        if t is not None and t.numel() and t.dtype != weight.dtype:
            raise ValueError(f"{name} must have the weight's element type {weight.dtype}")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.matmul_fused_partial_rmsnorm(
        input.data_ptr(), weight.data_ptr(), _row_stride(weight), n, k, 1,
        gamma.data_ptr() if nn else None, epsilon, weight_offset,
        normed_output.data_ptr() if nn else None, nn,
        unnormed_output.data_ptr() if n > nn else None, dtype, _ptr(err_word), _ptr(workspace),
        ws_bytes, _stream(stream)), "matmul_fused_partial_rmsnorm")


def raw_library() -> ctypes.CDLL:
    """The loaded C library, for callers that pass raw pointers themselves."""
    return _lib
