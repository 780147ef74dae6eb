"""Run the oracle on the seeded workloads (test infrastructure only).

Converts a workload's host tensors to the oracle's numpy arrays (raw element bits) and
calls the oracle operation it stands for.  Callers: the test-suite, the smoke check and
the benchmark's CPU-baseline leg.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def bits(t: torch.Tensor) -> np.ndarray:
    """A host copy of a tensor's raw element bits (uint16 for 16-bit types, uint8 for fp8)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy().copy()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    if t.dtype == torch.float32:
        return t.numpy().copy()
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32).copy()
    raise TypeError(t.dtype)


def oracle_rope(r: "W.RopeSpec") -> oracle.Rope:
    return oracle.Rope(bits(r.table), r.dtype, r.interleaved, r.rope_col_offset)


def oracle_paged(kv: "W.PagedKV", storage: np.ndarray) -> oracle.PagedCache:
    return oracle.PagedCache(storage, kv.k_offset, kv.v_offset, kv.dtype, kv.n_kv_heads,
                             kv.head_dim, kv.page_size, kv.num_pages, kv.num_layers,
                             kv.page_stride, kv.layer_stride, kv.slot_stride, kv.head_stride,
                             bits(kv.page_table), kv.max_pages_per_seq, bits(kv.cache_lengths),
                             None if kv.k_scale is None else bits(kv.k_scale),
                             None if kv.v_scale is None else bits(kv.v_scale))


def oracle_cont(kv: "W.ContKV", storage: np.ndarray) -> oracle.ContCache:
    return oracle.ContCache(storage, kv.k_offset, kv.v_offset, kv.dtype, kv.n_kv_heads,
                            kv.head_dim, kv.num_slots, kv.num_layers, kv.max_seq_len,
                            kv.slot_stride, kv.layer_stride, kv.pos_stride, kv.head_stride,
                            bits(kv.lookup_table), bits(kv.cache_lengths))


class OracleResult(dict):
    """Named host arrays the oracle produced (element bits) plus its error bits."""

    def __getattr__(self, k):
        return self[k]


def oracle_ragged_store(w: "W.RaggedStore", dtype: str = "bf16",
                        multiply_before_cast: bool = True) -> OracleResult:
    """The oracle on a ragged store workload: no-norm op when the workload has no gammas,
    else the single-band norm op."""
    store = bits(w.cache.storage)
    q_out = bits(w.q_out)
    qkv = bits(w.qkv)
    written = np.zeros(w.cache.num_pages * w.cache.page_size, dtype=np.uint8)
    cache = oracle_paged(w.cache, store)
    rope = oracle_rope(w.rope)
    if w.q_gamma is None:
        q_dtype = {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}[
            w.q_out.dtype]
        err = oracle.rope_split_store_paged_ragged(qkv, w.n_q_heads, bits(w.offsets), rope,
                                                   cache, w.layer_idx, q_out, written, dtype,
                                                   q_dtype)
    else:
        D = w.cache.head_dim
        Hq, Hk = w.n_q_heads, w.cache.n_kv_heads
        band = oracle.Band(qkv, 0, Hq * D, (Hq + Hk) * D, Hq, cache, bits(w.q_gamma),
                           bits(w.k_gamma), w.epsilon, q_out, written)
        err = oracle.fused_qk_rmsnorm_rope_paged(band, bits(w.offsets), rope, w.weight_offset,
                                                 multiply_before_cast, w.layer_idx, dtype)
    return OracleResult(q_out=q_out, storage=store, written=written, err=err)


def oracle_dual(w: "W.DualBand", dtype: str = "bf16",
                multiply_before_cast: bool = True) -> OracleResult:
    """The two-band op, or the single-band op when the workload has no index band."""
    inp = bits(w.input)
    ms = bits(w.main_cache.storage)
    qm = bits(w.q_main_out)
    wm = np.zeros(w.main_cache.num_pages * w.main_cache.page_size, dtype=np.uint8)
    g = [None if x is None else bits(x) for x in w.gammas]
    main = oracle.Band(inp, *w.main_cols, w.main_q_heads, oracle_paged(w.main_cache, ms), g[0],
                       g[1], w.main_eps, qm, wm)
    if w.index_cache is None:
        err = oracle.fused_qk_rmsnorm_rope_paged(main, bits(w.offsets), oracle_rope(w.rope),
                                                 w.weight_offset, multiply_before_cast,
                                                 w.layer_idx, dtype)
        return OracleResult(q_main_out=qm, main_storage=ms, main_written=wm, err=err)
    ist = bits(w.index_cache.storage)
    qi = bits(w.q_index_out)
    wi = np.zeros(w.index_cache.num_pages * w.index_cache.page_size, dtype=np.uint8)
    index = oracle.Band(inp, *w.index_cols, w.index_q_heads, oracle_paged(w.index_cache, ist),
                        g[2], g[3], w.index_eps, qi, wi)
    err = oracle.fused_dual_qk_rmsnorm_rope_paged(main, index, bits(w.offsets),
                                                  oracle_rope(w.rope), w.weight_offset,
                                                  multiply_before_cast, w.layer_idx, dtype)
    return OracleResult(q_main_out=qm, q_index_out=qi, main_storage=ms, index_storage=ist,
                        main_written=wm, index_written=wi, err=err)


def oracle_bshd(w: "W.BshdDecode", dtype: str = "bf16") -> OracleResult:
    store = bits(w.cache.storage)
    out = bits(w.output)
    written = np.zeros(w.cache.num_slots * w.cache.max_seq_len, dtype=np.uint8)
    err = oracle.qk_rope_bshd_continuous(bits(w.q_proj), oracle_cont(w.cache, store),
                                         oracle_rope(w.rope), w.layer_idx,
                                         bits(w.valid_lengths), out, written, dtype)
    return OracleResult(output=out, storage=store, written=written, err=err)


def oracle_radd(w: "W.Radd", dtype: str = "bf16") -> OracleResult:
    store = bits(w.cache.storage)
    written = np.zeros(w.cache.num_pages * w.cache.page_size, dtype=np.uint8)
    err = oracle.kv_cache_radd(bits(w.a), oracle_paged(w.cache, store), bits(w.offsets),
                               w.batch_offset, w.layer_idx, written, dtype)
    return OracleResult(storage=store, written=written, err=err)


def oracle_gemv(w: "W.GemvNorm", dtype: str = "bf16") -> OracleResult:
    normed, unnormed = bits(w.normed_output), bits(w.unnormed_output)
    err = oracle.matmul_fused_partial_rmsnorm(bits(w.x), bits(w.weight), bits(w.gamma),
                                              w.epsilon, w.weight_offset, normed, unnormed,
                                              dtype)
    return OracleResult(normed=normed, unnormed=unnormed, err=err)
