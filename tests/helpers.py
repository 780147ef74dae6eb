"""Test-side glue: run the CPU oracle on a workload and compare device results with it.

The conversions here only move bits between torch tensors and numpy arrays and describe
memory layouts; none of the operations' arithmetic lives here.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as W


from oracle.runners import (bits, oracle_rope, oracle_paged, oracle_cont,  # noqa: F401
                            OracleResult, oracle_ragged_store, oracle_dual, oracle_bshd,
                            oracle_radd, oracle_gemv)


def values(b: np.ndarray, dtype: str) -> np.ndarray:
    """Element bits -> float64 (bit reinterpretation through numpy / torch, not the oracle)."""
    if dtype == "f32":
        return b.astype(np.float64)
    if dtype == "f16":
        return b.view(np.float16).astype(np.float64)
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).double().numpy()


# ----------------------------------------------------------------------- comparisons --

def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bfloat16 numbers at |v| (2^(e-7) for |v| in [2^e, 2^(e+1)), subnormal
    spacing 2^-133 below 2^-126)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.exp2(e - 7)


def ulp_of(v: np.ndarray, dtype: str) -> np.ndarray:
    """Spacing of the element type's numbers at |v|."""
    if dtype == "bf16":
        return bf16_ulp(v)
    if dtype == "f16":
        a = np.maximum(np.abs(v), 2.0 ** -14)
        return np.exp2(np.floor(np.log2(a)) - 10)
    return np.spacing(np.abs(v).astype(np.float32)).astype(np.float64)


def assert_close_bf16(got_bits: np.ndarray, want_bits: np.ndarray, what: str,
                      abs_tol: float = 1e-3, dtype: str = "bf16", extra=None):
    """|got - want| <= max(1 ulp of want, abs_tol) (+ extra, elementwise, where a reading
    adds an intermediate rounding) elementwise (want = oracle, already rounded once);
    returns the fraction of bit-identical elements."""
    g, w = values(got_bits, dtype), values(want_bits, dtype)
    ulp = ulp_of(w, dtype)
    tol = np.maximum(ulp, abs_tol)
    if extra is not None:
        tol = tol + extra
    same = _as_bits(np.ascontiguousarray(got_bits)) == _as_bits(np.ascontiguousarray(want_bits))
    with np.errstate(invalid="ignore"):  # equal infinities / NaN bits compare as bits
        bad = ~(same | (np.abs(g - w) <= tol))
    if bad.any():
        idx = np.argwhere(bad)[:8]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside max(1 ulp, {abs_tol}); "
            f"first at {idx.tolist()}: got {g[bad][:8].tolist()} want {w[bad][:8].tolist()}")
    return float((_as_bits(np.ascontiguousarray(got_bits)) ==
                  _as_bits(np.ascontiguousarray(want_bits))).mean()) if got_bits.size else 1.0


def _as_bits(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint32) if a.dtype == np.float32 else a


def assert_bits_equal(got: np.ndarray, want: np.ndarray, what: str):
    got, want = _as_bits(np.ascontiguousarray(got)), _as_bits(np.ascontiguousarray(want))
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
                        what: str, v_exact: bool = True, k_extra=None):
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
    ek = None if k_extra is None else k_extra.reshape(shp)[kr][..., fp_cols_k]
    frac = assert_close_bf16(gk[..., fp_cols_k], wk[..., fp_cols_k], f"{what}: K roped cols",
                             dtype=kv.dtype, extra=ek)
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


def tile_golden(case: dict, head_dim: int = 64) -> dict:
    """The same worked example on a wider head: the pass-through columns and the rotated
    columns are each repeated until the head is `head_dim` wide, keeping every rotation
    pair's partner and (cos, sin) entry, so the expected row is the same repetition of the
    expected values.  With no pass-through columns the mean square is unchanged too."""
    D0, R0 = case["head_dim"], case["rope_dim"]
    o0 = D0 - R0
    R = head_dim if o0 == 0 else head_dim // 2
    o = head_dim - R
    rep_r = R // R0
    assert rep_r * R0 == R and (o0 == 0 or (o // o0) * o0 == o)

    def tile_row(x):
        x = list(x)
        head = (x[:o0] * (o // o0)) if o0 else []
        rot = x[o0:]
        if case["interleaved"]:
            tail = rot * rep_r
        else:
            h = R0 // 2
            tail = rot[:h] * rep_r + rot[h:] * rep_r
        return head + tail

    c = dict(case)
    c["head_dim"], c["rope_dim"] = head_dim, R
    c["x"] = tile_row(case["x"])
    c["expect"] = tile_row(case["expect"])
    c["freqs_row"] = list(case["freqs_row"]) * rep_r
    if "gamma" in case:
        assert o0 == 0
        c["gamma"] = tile_row(case["gamma"])
    return c


# ------------------------------------------- the multiply-after-cast reading's tolerance --

def rope_pairs(head_dim: int, rope: W.RopeSpec) -> np.ndarray:
    """partner[d] = the column rotated together with column d (d itself if unrotated)."""
    R = rope.rope_dim
    o = head_dim - R if rope.rope_col_offset < 0 else rope.rope_col_offset
    partner = np.arange(head_dim)
    for i in range(R // 2):
        a, b = (o + 2 * i, o + 2 * i + 1) if rope.interleaved else (o + i, o + i + R // 2)
        partner[a], partner[b] = b, a
    return partner


def multiply_after_cast_slack(x: np.ndarray, gamma: np.ndarray, weight_offset: float,
                              eps: float, dtype: str, rope: W.RopeSpec) -> np.ndarray:
    """Extra tolerance of multiply_before_cast = 0, elementwise for head rows x [..., D]
    (float64 values) of the input.  That reading rounds the normalised value n = x * r to the
    element type before the gamma multiply: both sides round n, the kernel from a float32 n
    (rsqrtf, float32 products), the oracle from the exact one, so where n lies within a few
    float32 ulps of a rounding midpoint they may keep neighbouring values of the element
    type.  Such a flip moves the gamma-scaled value by ulp(n) * |gamma + weight_offset|, and
    the rotation mixes it into both columns of the pair (|cos|, |sin| <= 1)."""
    D = x.shape[-1]
    r = 1.0 / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)
    n = x * r
    u = ulp_of(n * (1.0 + 2.0 ** -7), dtype) * np.abs(gamma + weight_offset)
    partner = rope_pairs(D, rope)
    rotated = partner != np.arange(D)
    return np.where(rotated, u + u[..., partner], u)


def scatter_slots(kv: W.PagedKV, per_token: np.ndarray, cache_lengths, lengths,
                  layer_idx: int) -> np.ndarray:
    """Per-token K-row values [T, Hk, D] placed at the cache rows the tokens map to (K plane
    of layer_idx), zeros elsewhere: storage-shaped."""
    out = np.zeros((kv.num_pages, kv.planes, kv.num_layers, kv.page_size, kv.n_kv_heads,
                    kv.head_dim))
    for i, (page, slot) in enumerate(W.token_slots(kv, list(cache_lengths), list(lengths))):
        out[page, 0, layer_idx, slot] = per_token[i]
    return out


# ------------------------------------------------- weight_offset as an element-type scalar --

def exact_norm_rows(seed: int, n_rows: int, head_dim: int) -> torch.Tensor:
    """[n_rows, head_dim] float64 rows of +-1 and +-3 with exactly 3 * head_dim / 8 threes
    per row (seeded places and signs).  Every row's mean square is exactly 4, so with
    epsilon 0 its normalised value x * rsqrt(mean(x^2)) is exactly x / 2, in {+-0.5, +-1.5}:
    exact in every element type."""
    gen = W.generator(seed)
    rows = torch.ones(n_rows, head_dim, dtype=torch.float64)
    for r in range(n_rows):
        rows[r, torch.randperm(head_dim, generator=gen)[:3 * head_dim // 8]] = 3.0
    sign = torch.randint(0, 2, (n_rows, head_dim), generator=gen).double() * 2 - 1
    return rows * sign


def bf16_weight_offset_case(rows: torch.Tensor, weight_offset: float):
    """For exact_norm_rows `rows`, gamma 0 and epsilon 0 at position 0 (identity rotation):
    the outputs (rows / 2) * bf16(weight_offset), which are bfloat16 numbers for the offsets
    the tests use, and the outputs an unrounded weight_offset would give.  Returns (want,
    unrounded) as bfloat16 tensors; raises if `want` is not exact."""
    wo_b = torch.tensor(weight_offset, dtype=torch.float64).to(torch.bfloat16).double()
    want = rows / 2 * wo_b
    want_b = want.to(torch.bfloat16)
    assert torch.equal(want_b.double(), want), "the expected outputs must be bf16 numbers"
    unrounded = (rows / 2 * weight_offset).to(torch.bfloat16)
    return want_b, unrounded
