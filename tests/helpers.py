"""Test-side glue: run the CPU oracle on a workload and compare device results with it.

The conversions here only move bits between torch tensors and numpy arrays and describe
memory layouts; none of the operations' arithmetic lives here.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as W


def bits(t: torch.Tensor) -> np.ndarray:
    """A host copy of a tensor's raw element bits (uint16 for 16-bit types)."""
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    if t.dtype == torch.float32:
        return t.numpy().copy()
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32).copy()
    raise TypeError(t.dtype)


def values(b: np.ndarray, dtype: str) -> np.ndarray:
    """Element bits -> float64 (bit reinterpretation through numpy / torch, not the oracle)."""
    if dtype == "f32":
        return b.astype(np.float64)
    if dtype == "f16":
        return b.view(np.float16).astype(np.float64)
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).double().numpy()


def oracle_rope(r: W.RopeSpec) -> oracle.Rope:
    return oracle.Rope(bits(r.table), r.dtype, r.interleaved, r.rope_col_offset)


def oracle_paged(kv: W.PagedKV, storage: np.ndarray) -> oracle.PagedCache:
    return oracle.PagedCache(storage, kv.k_offset, kv.v_offset, kv.dtype, kv.n_kv_heads,
                             kv.head_dim, kv.page_size, kv.num_pages, kv.num_layers,
                             kv.page_stride, kv.layer_stride, kv.slot_stride, kv.head_stride,
                             bits(kv.page_table), kv.max_pages_per_seq, bits(kv.cache_lengths))


def oracle_cont(kv: W.ContKV, storage: np.ndarray) -> oracle.ContCache:
    return oracle.ContCache(storage, kv.k_offset, kv.v_offset, kv.dtype, kv.n_kv_heads,
                            kv.head_dim, kv.num_slots, kv.num_layers, kv.max_seq_len,
                            kv.slot_stride, kv.layer_stride, kv.pos_stride, kv.head_stride,
                            bits(kv.lookup_table), bits(kv.cache_lengths))


class OracleResult(dict):
    """Named host arrays the oracle produced (element bits) plus its error bits."""

    def __getattr__(self, k):
        return self[k]


def oracle_ragged_store(w: W.RaggedStore, dtype: str = "bf16",
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
        err = oracle.rope_split_store_paged_ragged(qkv, w.n_q_heads, bits(w.offsets), rope,
                                                   cache, w.layer_idx, q_out, written, dtype)
    else:
        D = w.cache.head_dim
        Hq, Hk = w.n_q_heads, w.cache.n_kv_heads
        band = oracle.Band(qkv, 0, Hq * D, (Hq + Hk) * D, Hq, cache, bits(w.q_gamma),
                           bits(w.k_gamma), w.epsilon, q_out, written)
        err = oracle.fused_qk_rmsnorm_rope_paged(band, bits(w.offsets), rope, w.weight_offset,
                                                 multiply_before_cast, w.layer_idx, dtype)
    return OracleResult(q_out=q_out, storage=store, written=written, err=err)


def oracle_dual(w: W.DualBand, dtype: str = "bf16") -> OracleResult:
    inp = bits(w.input)
    ms, ist = bits(w.main_cache.storage), bits(w.index_cache.storage)
    qm, qi = bits(w.q_main_out), bits(w.q_index_out)
    wm = np.zeros(w.main_cache.num_pages * w.main_cache.page_size, dtype=np.uint8)
    wi = np.zeros(w.index_cache.num_pages * w.index_cache.page_size, dtype=np.uint8)
    g = [bits(x) for x in w.gammas]
    main = oracle.Band(inp, *w.main_cols, w.main_q_heads, oracle_paged(w.main_cache, ms), g[0],
                       g[1], w.main_eps, qm, wm)
    index = oracle.Band(inp, *w.index_cols, w.index_q_heads, oracle_paged(w.index_cache, ist),
                        g[2], g[3], w.index_eps, qi, wi)
    err = oracle.fused_dual_qk_rmsnorm_rope_paged(main, index, bits(w.offsets),
                                                  oracle_rope(w.rope), w.weight_offset, True,
                                                  w.layer_idx, dtype)
    return OracleResult(q_main_out=qm, q_index_out=qi, main_storage=ms, index_storage=ist,
                        main_written=wm, index_written=wi, err=err)


def oracle_bshd(w: W.BshdDecode, dtype: str = "bf16") -> OracleResult:
    store = bits(w.cache.storage)
    out = bits(w.output)
    written = np.zeros(w.cache.num_slots * w.cache.max_seq_len, dtype=np.uint8)
    err = oracle.qk_rope_bshd_continuous(bits(w.q_proj), oracle_cont(w.cache, store),
                                         oracle_rope(w.rope), w.layer_idx,
                                         bits(w.valid_lengths), out, written, dtype)
    return OracleResult(output=out, storage=store, written=written, err=err)


def oracle_radd(w: W.Radd, dtype: str = "bf16") -> OracleResult:
    store = bits(w.cache.storage)
    written = np.zeros(w.cache.num_pages * w.cache.page_size, dtype=np.uint8)
    err = oracle.kv_cache_radd(bits(w.a), oracle_paged(w.cache, store), bits(w.offsets),
                               w.batch_offset, w.layer_idx, written, dtype)
    return OracleResult(storage=store, written=written, err=err)


# ----------------------------------------------------------------------- comparisons --

def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bfloat16 numbers at |v| (2^(e-7) for |v| in [2^e, 2^(e+1)), subnormal
    spacing 2^-133 below 2^-126)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.exp2(e - 7)


def assert_close_bf16(got_bits: np.ndarray, want_bits: np.ndarray, what: str,
                      abs_tol: float = 1e-3, dtype: str = "bf16"):
    """|got - want| <= max(1 ulp of want, abs_tol) elementwise (want = oracle, already
    rounded once); returns the fraction of bit-identical elements."""
    g, w = values(got_bits, dtype), values(want_bits, dtype)
    if dtype == "bf16":
        ulp = bf16_ulp(w)
    elif dtype == "f16":
        a = np.maximum(np.abs(w), 2.0 ** -14)
        ulp = np.exp2(np.floor(np.log2(a)) - 10)
    else:
        ulp = np.spacing(np.abs(w).astype(np.float32)).astype(np.float64)
    tol = np.maximum(ulp, abs_tol)
    bad = ~(np.abs(g - w) <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:8]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside max(1 ulp, {abs_tol}); "
            f"first at {idx.tolist()}: got {g[bad][:8].tolist()} want {w[bad][:8].tolist()}")
    return float((got_bits == want_bits).mean()) if got_bits.size else 1.0


def assert_bits_equal(got: np.ndarray, want: np.ndarray, what: str):
    if not np.array_equal(got, want):
        diff = np.argwhere(got != want)
        raise AssertionError(f"{what}: {len(diff)} elements differ; first at "
                             f"{diff[:8].tolist()}")


def paged_rows_mask(kv: W.PagedKV, written: np.ndarray, layer_idx: int) -> np.ndarray:
    """Boolean [num_pages, planes, layers, page_size] mask of the (page, slot) rows of
    `layer_idx` that the oracle marked as written."""
    m = np.zeros((kv.num_pages, kv.planes, kv.num_layers, kv.page_size), dtype=bool)
    m[:, :, layer_idx, :] = written.reshape(kv.num_pages, 1, kv.page_size).astype(bool)
    return m


def compare_paged_cache(kv: W.PagedKV, got_storage: np.ndarray, want_storage: np.ndarray,
                        written: np.ndarray, layer_idx: int, fp_cols_k: np.ndarray,
                        what: str, v_exact: bool = True):
    """Rows the oracle did not write: bit-identical (untouched).  Written K rows: columns in
    fp_cols_k within tolerance, other columns bit-identical.  Written V rows: bit-identical
    (or within tolerance when v_exact is False, for radd the tolerance is still exact)."""
    shp = (kv.num_pages, kv.planes, kv.num_layers, kv.page_size, kv.n_kv_heads, kv.head_dim)
    g = got_storage.reshape(shp)
    w = want_storage.reshape(shp)
    rows = paged_rows_mask(kv, written, layer_idx)
    untouched = ~rows
    assert_bits_equal(g[untouched], w[untouched], f"{what}: untouched cache rows")
    kr = rows.copy()
    kr[:, 1:] = False
    gk, wk = g[kr], w[kr]            # [n, Hk, D]
    exact_cols = ~fp_cols_k
    assert_bits_equal(gk[..., exact_cols], wk[..., exact_cols], f"{what}: K pass-through cols")
    frac = assert_close_bf16(gk[..., fp_cols_k], wk[..., fp_cols_k], f"{what}: K roped cols",
                             dtype=kv.dtype)
    if kv.planes == 2:
        vr = rows.copy()
        vr[:, 0] = False
        if v_exact:
            assert_bits_equal(g[vr], w[vr], f"{what}: V rows")
        else:
            assert_close_bf16(g[vr], w[vr], f"{what}: V rows", dtype=kv.dtype)
    return frac


def rope_cols(head_dim: int, rope_dim: int, offset: int = -1) -> np.ndarray:
    o = head_dim - rope_dim if offset < 0 else offset
    m = np.zeros(head_dim, dtype=bool)
    m[o:o + rope_dim] = True
    return m


# --------------------------------------------------------- hand-worked single tokens --

def golden_problem(case: dict, norm: bool, dtype: str = "bf16") -> W.RaggedStore:
    """One token, one Q head and one KV head, at position 1 (cache_length 1) of a two-row
    freqs_cis whose row 0 is the identity and row 1 is the case's row.  Q and K both carry
    the case's x; V carries 1, 2, 3, ...; the expected Q / K row is the case's `expect`."""
    D, R = case["head_dim"], case["rope_dim"]
    td = W.TORCH_DTYPES[dtype]
    x = torch.tensor(case["x"], dtype=torch.float64)
    v = torch.arange(1, D + 1, dtype=torch.float64)
    qkv = torch.cat([x, x, v]).to(td).view(1, 3 * D)
    table = torch.zeros(2, R, dtype=torch.float32)
    table[0, 0::2] = 1.0
    table[1] = torch.tensor(case["freqs_row"], dtype=torch.float32)
    gen = W.generator(7)
    P = 2
    storage = W.random_bits(gen, 1 * 2 * 1 * P * 1 * D, dtype)
    cache = W.PagedKV(storage, 2, 1, 1, P, 1, D, torch.zeros(1, 1, dtype=torch.int32),
                      torch.ones(1, dtype=torch.int32), dtype)
    rope = W.RopeSpec(table, "f32", bool(case["interleaved"]))
    q_out = W.random_bits(gen, D, dtype).view(1, D)
    g = None
    if norm:
        g = torch.tensor(case["gamma"], dtype=torch.float64).to(td)
    return W.RaggedStore(qkv, torch.tensor([0, 1], dtype=torch.int32), 1, cache, rope, 0,
                         q_out, [1], g, None if g is None else g.clone(),
                         case.get("eps", 1e-6), case.get("weight_offset", 0.0),
                         case["name"])
