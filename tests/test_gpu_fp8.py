"""FP8 (E4M3) paged caches, CUDA path vs the oracle.

An FP8 cache element holds the E4M3 code of value / scale, one float32 scale per plane.
V rows are copied: the kernel rounds value / scale exactly once (its float32 estimate is
checked against the midpoint between the two candidate codes with an exact fused
multiply-add), as the oracle rounds the quotient, so V codes must match bit for bit at any
scale, including scales where a float32 quotient rounded again would not.  K rows are
rotated (and normalised): the kernel rounds a float32 y * (1 / scale), the oracle the exact
y / scale, so where that value lies within float32 error of a midpoint between two codes the
two sides may keep neighbouring codes.  The tolerance derived from that: every K code equal
to the oracle's or one E4M3 step away, and at most one in a thousand not equal.  Every byte
outside the written rows is untouched.  Q outputs as in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import workloads as W
import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gpu_helpers
    return gpu_helpers


def e4m3_values(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


def compare_fp8_cache(kv, got, want, written, layer, what):
    shp = (kv.num_pages, kv.planes, kv.num_layers, kv.page_size, kv.n_kv_heads, kv.head_dim)
    g, w = got.reshape(shp), want.reshape(shp)
    rows = H.paged_rows_mask(kv, written, layer)
    H.assert_bits_equal(g[~rows], w[~rows], f"{what}: untouched bytes")
    kr = rows.copy()
    kr[:, 1:] = False
    gk, wk = g[kr], w[kr]
    same = gk == wk
    gv, wv = e4m3_values(gk), e4m3_values(wk)
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(wv), 2.0 ** -6))) - 3)
    near = np.abs(gv - wv) <= step * (1 + 1e-9)
    assert bool(np.all(same | near)), f"{what}: K codes more than one step from the oracle"
    assert same.mean() >= 0.999, f"{what}: {1 - same.mean():.2e} of K codes differ"
    if kv.planes == 2:
        vr = rows.copy()
        vr[:, 0] = False
        H.assert_bits_equal(g[vr], w[vr], f"{what}: V codes")


def check_store(G, w, s, r):
    assert int(s.err.item()) == r.err == 0
    T, Hq, D = w.total_tokens, w.n_q_heads, w.cache.head_dim
    qd = {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}[w.q_out.dtype]
    H.assert_close_bf16(H.bits(s.q_out).reshape(T, Hq, D), r.q_out.reshape(T, Hq, D), "q_out",
                        dtype=qd)
    compare_fp8_cache(w.cache, H.bits(s.storage), r.storage, r.written, w.layer_idx, "cache")


@pytest.mark.parametrize("interleaved", [True, False])
@pytest.mark.parametrize("dtype,head_dim", [("bf16", 128), ("f32", 64), ("f16", 256)])
def test_store_into_fp8_cache(G, interleaved, dtype, head_dim):
    w = W.ragged_store(50, lengths=[700, 3, 301], cache_lengths=[0, 11, 90], n_q_heads=8,
                       n_kv_heads=2, head_dim=head_dim, page_size=32, rope_dim=head_dim,
                       theta=5e5, interleaved=interleaved, max_seq_len=1024, dtype=dtype,
                       cache_dtype="fp8", kv_scales=(0.5, 0.0625))
    check_store(G, w, G.run_ragged(w), H.oracle_ragged_store(w, dtype))


def test_norm_store_into_fp8_cache(G):
    w = W.ragged_store(51, lengths=[500, 1, 257], cache_lengths=[3, 0, 77], n_q_heads=16,
                       n_kv_heads=4, head_dim=128, page_size=64, rope_dim=64, theta=1e4,
                       interleaved=False, max_seq_len=1024, x_std=2.0, norm=True,
                       cache_dtype="fp8", kv_scales=(0.25, 0.125))
    check_store(G, w, G.run_ragged(w), H.oracle_ragged_store(w, "bf16"))


@pytest.mark.parametrize("main_fp8,index_fp8", [(True, False), (False, True), (True, True)])
def test_dual_band_with_fp8_caches(G, main_fp8, index_fp8):
    w = W.dual_band(52, lengths=[400, 1, 90], cache_lengths=[0, 40, 7], main_q_heads=8,
                    main_kv_heads=2, index_q_heads=2, index_kv_heads=1, head_dim=128,
                    main_page_size=64, index_page_size=32, rope_dim=64, theta=1e4,
                    interleaved=True, max_seq_len=1024,
                    main_cache_dtype="fp8" if main_fp8 else None,
                    index_cache_dtype="fp8" if index_fp8 else None, kv_scales=(0.5, 0.25))
    s = G.run_dual(w)
    r = H.oracle_dual(w)
    assert int(s.err.item()) == r.err == 0
    D = 128
    for which, nq, is8 in (("main", w.main_q_heads, main_fp8),
                           ("index", w.index_q_heads, index_fp8)):
        kv = getattr(w, f"{which}_cache")
        q = H.bits(getattr(s, f"q_{which}_out")).reshape(w.total_tokens, nq, D)
        H.assert_close_bf16(q, r[f"q_{which}_out"].reshape(q.shape), f"q_{which}_out")
        got = H.bits(getattr(s, f"{which}_storage"))
        if is8:
            compare_fp8_cache(kv, got, r[f"{which}_storage"], r[f"{which}_written"],
                              w.layer_idx, f"{which} cache")
        else:
            H.compare_paged_cache(kv, got, r[f"{which}_storage"], r[f"{which}_written"],
                                  w.layer_idx, np.ones(D, bool), f"{which} cache")


def test_fp8_cache_with_the_claimed_schedule_and_every_overlap_mode(G):
    import rope_paged_kv_b200 as rs
    w = W.ragged_store(53, lengths=[1500, 37, 2900, 1, 1700], cache_lengths=[0, 5, 100, 0, 64],
                       n_q_heads=8, n_kv_heads=2, head_dim=128, page_size=64, rope_dim=128,
                       theta=5e5, interleaved=False, max_seq_len=4096, cache_dtype="fp8",
                       kv_scales=(1.0, 0.5))
    r = H.oracle_ragged_store(w, "bf16")
    before = rs.get_launch_overlap()
    try:
        for mode in (0, 1, 2):
            rs.set_launch_overlap(mode)
            check_store(G, w, G.run_ragged(w), r)
    finally:
        rs.set_launch_overlap(before)


@pytest.mark.parametrize("q_out_dtype", ["f32", "f16"])
def test_fp8_cache_with_q_out_in_another_type(G, q_out_dtype):
    # both extended outputs at once: Q rounded into its own type, K and V as E4M3 codes
    w = W.ragged_store(54, lengths=[300, 2, 129], cache_lengths=[1, 0, 64], n_q_heads=16,
                       n_kv_heads=4, head_dim=128, page_size=64, rope_dim=128, theta=1e4,
                       interleaved=True, max_seq_len=512, q_out_dtype=q_out_dtype,
                       cache_dtype="fp8", kv_scales=(0.125, 2.0))
    check_store(G, w, G.run_ragged(w), H.oracle_ragged_store(w, "bf16"))


# ------------------------------------------------------- FP8 V codes at general scales --
# The kernel encodes V as the E4M3 code of value / scale rounded once, exactly like the
# oracle, at any scale: these cases put every finite bf16 (f16) bit pattern in the V columns,
# at scales where a float32 quotient rounded again would be off by one code on some inputs
# (0.7 and 1.3 on 32 bf16 inputs each, 1.7 and 0.1 on 2).  f32 inputs get values next to
# the midpoints between codes.

def _all_patterns(dtype, n):
    """n values: every finite bit pattern of the 16-bit type (non-finite ones become 0),
    repeated to length n."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(W.TORCH_DTYPES[dtype])
    t = torch.where(torch.isfinite(t.float()), t, torch.zeros_like(t))
    return t.repeat((n + 65535) // 65536)[:n]


def _near_midpoints(scale, n, gen):
    """f32 values v with v / scale within a few float32 ulps of a midpoint between two E4M3
    codes, or exactly on one."""
    codes = torch.arange(0, 0x7E, dtype=torch.uint8)
    vals = codes.view(torch.float8_e4m3fn).double()
    mids = (vals[:-1] + vals[1:]) / 2
    m = mids[torch.randint(0, mids.numel(), (n,), generator=gen)]
    m = m * (torch.randint(0, 2, (n,), generator=gen).double() * 2 - 1)
    v = (m * float(np.float32(scale))).float()
    nudge = torch.randint(-3, 4, (n,), generator=gen, dtype=torch.int32)
    return (v.view(torch.int32) + nudge).view(torch.float32)


@pytest.mark.parametrize("scale", [0.7, 1.3, 1.7, 0.1, 0.3])
@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_fp8_v_codes_exact_at_any_scale(G, dtype, scale):
    T, Hk, D = 300, 2, 128
    w = W.ragged_store(55, lengths=[200, 100], cache_lengths=[0, 37], n_q_heads=4,
                       n_kv_heads=Hk, head_dim=D, page_size=64, rope_dim=D, theta=1e4,
                       interleaved=False, max_seq_len=512, dtype=dtype, cache_dtype="fp8",
                       kv_scales=(scale, scale))
    vcols = slice((4 + Hk) * D, (4 + 2 * Hk) * D)
    if dtype == "f32":
        v = _near_midpoints(scale, T * Hk * D, W.generator(56))
    else:
        v = _all_patterns(dtype, T * Hk * D)
    w.qkv[:, vcols] = v.view(T, Hk * D)
    check_store(G, w, G.run_ragged(w), H.oracle_ragged_store(w, dtype))


def test_fp8_general_scales_norm_and_dual_band(G):
    w = W.dual_band(57, lengths=[300, 2, 41], cache_lengths=[0, 9, 70], main_q_heads=8,
                    main_kv_heads=2, index_q_heads=2, index_kv_heads=1, head_dim=128,
                    main_page_size=64, index_page_size=32, rope_dim=64, theta=1e4,
                    interleaved=True, max_seq_len=1024, main_cache_dtype="fp8",
                    index_cache_dtype="fp8", kv_scales=(0.37, 0.7))
    s = G.run_dual(w)
    r = H.oracle_dual(w)
    assert int(s.err.item()) == r.err == 0
    for which in ("main", "index"):
        compare_fp8_cache(getattr(w, f"{which}_cache"), H.bits(getattr(s, f"{which}_storage")),
                          r[f"{which}_storage"], r[f"{which}_written"], w.layer_idx,
                          f"{which} cache")
