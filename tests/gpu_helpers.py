"""Run workloads through the C ABI on the GPU (via the rope_paged_kv_b200 binding)."""
from __future__ import annotations

import torch

import rope_paged_kv_b200 as rs
import workloads as W

DEV = "cuda:0"


def to_dev(t: torch.Tensor) -> torch.Tensor:
    return t.to(DEV, non_blocking=False).contiguous() if t.is_contiguous() else t.to(DEV)


def freqs(r: W.RopeSpec) -> rs.Freqs:
    return rs.Freqs(to_dev(r.table), r.interleaved, r.rope_col_offset)


def paged(kv: W.PagedKV, storage: torch.Tensor) -> rs.PagedCache:
    v = None if kv.v_offset is None else storage[kv.v_offset:]
    return rs.PagedCache(storage[kv.k_offset:], v, to_dev(kv.page_table),
                         to_dev(kv.cache_lengths), kv.n_kv_heads, kv.head_dim, kv.page_size,
                         kv.num_pages, kv.num_layers, kv.page_stride, kv.layer_stride,
                         kv.slot_stride, kv.head_stride,
                         k_scale=None if kv.k_scale is None else to_dev(kv.k_scale),
                         v_scale=None if kv.v_scale is None else to_dev(kv.v_scale))


def cont(kv: W.ContKV, storage: torch.Tensor) -> rs.ContCache:
    v = None if kv.v_offset is None else storage[kv.v_offset:]
    return rs.ContCache(storage[kv.k_offset:], v, to_dev(kv.lookup_table),
                        to_dev(kv.cache_lengths), kv.n_kv_heads, kv.head_dim, kv.num_slots,
                        kv.num_layers, kv.max_seq_len, kv.slot_stride, kv.layer_stride,
                        kv.pos_stride, kv.head_stride)


def padded_rows(t: torch.Tensor) -> torch.Tensor:
    """A device copy that keeps a host tensor's row stride (for padded-row inputs)."""
    if t.is_contiguous():
        return to_dev(t)
    base = torch.empty(t.shape[0], t.stride(0), dtype=t.dtype, device=DEV)
    base[:, :t.shape[1]] = t.to(DEV)
    return base[:, :t.shape[1]]


def err_word() -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=DEV)


# The staged entry points run with a scheduling workspace (the claimed-tail token schedule)
# unless a test switches this off to get the static schedule.
USE_SCHED = True


def sched_of(s) -> torch.Tensor | None:
    if not USE_SCHED:
        return None
    if getattr(s, "sched", None) is None:
        s.sched = rs.sched_workspace(DEV)
    return s.sched


class Staged:
    """A workload's tensors on the device, with the binding's descriptors."""


def stage_ragged(w: W.RaggedStore) -> Staged:
    s = Staged()
    s.qkv = padded_rows(w.qkv)
    s.offs = to_dev(w.offsets)
    s.storage = to_dev(w.cache.storage)
    s.kv = paged(w.cache, s.storage)
    s.freqs = freqs(w.rope)
    s.q_out = to_dev(w.q_out)
    s.err = err_word()
    if w.q_gamma is not None:
        s.q_gamma, s.k_gamma = to_dev(w.q_gamma), to_dev(w.k_gamma)
    return s


def launch_ragged(w: W.RaggedStore, s: Staged, stream=None, multiply_before_cast=True) -> None:
    if w.q_gamma is None:
        rs.rope_split_store_paged_ragged(s.qkv, w.n_q_heads, s.offs, s.freqs, s.kv,
                                         w.layer_idx, s.q_out, s.err, stream, sched_of(s))
    else:
        rs.fused_qk_rmsnorm_rope_paged(s.qkv, w.n_q_heads, s.offs, s.freqs, s.kv, s.q_gamma,
                                       s.k_gamma, w.epsilon, w.weight_offset, w.layer_idx,
                                       s.q_out, multiply_before_cast, s.err, stream,
                                       sched_of(s))


def run_ragged(w: W.RaggedStore, multiply_before_cast=True):
    s = stage_ragged(w)
    launch_ragged(w, s, multiply_before_cast=multiply_before_cast)
    torch.cuda.synchronize()
    return s


def stage_dual(w: W.DualBand) -> Staged:
    """The dual-band workload staged; a workload without an index band stages the main
    band alone (s.index is None)."""
    s = Staged()
    s.input = to_dev(w.input)
    s.offs = to_dev(w.offsets)
    s.main_storage = to_dev(w.main_cache.storage)
    s.q_main_out = to_dev(w.q_main_out)
    g = [None if x is None else to_dev(x) for x in w.gammas]
    s.main = rs.NormBand(s.input, *w.main_cols, w.main_q_heads,
                         paged(w.main_cache, s.main_storage), g[0], g[1], w.main_eps,
                         s.q_main_out)
    s.index = None
    if w.index_cache is not None:
        s.index_storage = to_dev(w.index_cache.storage)
        s.q_index_out = to_dev(w.q_index_out)
        s.index = rs.NormBand(s.input, *w.index_cols, w.index_q_heads,
                              paged(w.index_cache, s.index_storage), g[2], g[3], w.index_eps,
                              s.q_index_out)
    s.freqs = freqs(w.rope)
    s.err = err_word()
    return s


def launch_dual(w: W.DualBand, s: Staged, stream=None, multiply_before_cast=True) -> None:
    rs.fused_dual_qk_rmsnorm_rope_paged(s.main, s.index, s.offs, w.total_tokens, s.freqs,
                                        w.weight_offset, w.layer_idx, multiply_before_cast,
                                        s.err, stream, sched_of(s))


def run_dual(w: W.DualBand, multiply_before_cast=True):
    s = stage_dual(w)
    launch_dual(w, s, multiply_before_cast=multiply_before_cast)
    torch.cuda.synchronize()
    return s


def stage_bshd(w: W.BshdDecode) -> Staged:
    s = Staged()
    s.q = to_dev(w.q_proj)
    s.storage = to_dev(w.cache.storage)
    s.kv = cont(w.cache, s.storage)
    s.freqs = freqs(w.rope)
    s.valid = to_dev(w.valid_lengths)
    s.out = to_dev(w.output)
    s.err = err_word()
    return s


def launch_bshd(w: W.BshdDecode, s: Staged, stream=None) -> None:
    rs.qk_rope_bshd_continuous(s.q, s.kv, s.freqs, w.layer_idx, s.valid, s.out, s.err, stream)


def run_bshd(w: W.BshdDecode):
    s = stage_bshd(w)
    launch_bshd(w, s)
    torch.cuda.synchronize()
    return s


def stage_radd(w: W.Radd) -> Staged:
    s = Staged()
    s.a = to_dev(w.a)
    s.offs = to_dev(w.offsets)
    s.storage = to_dev(w.cache.storage)
    s.kv = paged(w.cache, s.storage)
    s.err = err_word()
    return s


def launch_radd(w: W.Radd, s: Staged, stream=None) -> None:
    rs.kv_cache_radd(s.a, s.kv, s.offs, w.batch_offset, w.layer_idx, s.err, stream,
                     sched_of(s))


def run_radd(w: W.Radd):
    s = stage_radd(w)
    launch_radd(w, s)
    torch.cuda.synchronize()
    return s


def compare_cont_cache(w: W.BshdDecode, s: Staged, pristine: torch.Tensor, oracle_storage,
                       written, fp_cols):
    """Continuous cache: rows the oracle did not write are unchanged (checked on the device
    against a pristine copy); written K rows match the oracle (rotated columns within
    tolerance, the rest bit for bit)."""
    import numpy as np
    import helpers as H
    kv = w.cache
    rows_per_slot_plane = kv.num_layers * kv.max_seq_len
    n_rows = kv.num_slots * kv.planes * rows_per_slot_plane
    got = s.storage.view(n_rows, kv.n_kv_heads * kv.head_dim)
    ref = pristine.view(n_rows, kv.n_kv_heads * kv.head_dim)
    changed = (got.view(torch.int16) != ref.view(torch.int16)).any(dim=1).cpu().numpy()
    # row index of (slot, plane 0, layer, pos)
    wr = written.reshape(kv.num_slots, kv.max_seq_len).astype(bool)
    allowed = np.zeros((kv.num_slots, kv.planes, kv.num_layers, kv.max_seq_len), dtype=bool)
    allowed[:, 0, w.layer_idx, :] = wr
    allowed = allowed.reshape(-1)
    assert not (changed & ~allowed).any(), "rows outside the written set changed"
    idx = np.flatnonzero(allowed)
    if idx.size == 0:
        return 1.0
    got_rows = H.bits(got[torch.from_numpy(idx).to(got.device)])
    want_rows = oracle_storage.reshape(n_rows, -1)[idx]
    g = got_rows.reshape(-1, kv.n_kv_heads, kv.head_dim)
    o = want_rows.reshape(-1, kv.n_kv_heads, kv.head_dim)
    H.assert_bits_equal(g[..., ~fp_cols], o[..., ~fp_cols], "K pass-through columns")
    return H.assert_close_bf16(g[..., fp_cols], o[..., fp_cols], "K rotated columns",
                               dtype=kv.dtype)
