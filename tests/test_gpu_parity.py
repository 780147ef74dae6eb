"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bit-exact: page/slot placement, V copies, columns neither normed nor rotated, every cache
byte the operation must not touch, the radd sums, the device error bits.  Rotated / normed
values: |gpu - oracle| <= max(1 ulp of the oracle value in the element type, 1e-3).
Sizes: the five named workloads at full size (with the claimed-tail token schedule the
benchmark uses, under the default launch-overlap mode and the benchmark's own; the
test_gpu_schedule.py cases show every mode bit-identical) plus small cases that span several
tiles and ragged tails, and the edge cases.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gpu_helpers
    return gpu_helpers


def _head_rows(x, col, heads, D):
    return x[:, col:col + heads * D].reshape(x.shape[0], heads, D)


def _slot_rows(kv, storage_bits, cache_lengths, lengths, layer_idx):
    """The K rows a band updated in place held before the call, in token order."""
    v = H.values(storage_bits, kv.dtype).reshape(kv.num_pages, kv.planes, kv.num_layers,
                                                 kv.page_size, kv.n_kv_heads, kv.head_dim)
    return np.stack([v[p, 0, layer_idx, sl] for p, sl in
                     W.token_slots(kv, list(cache_lengths), list(lengths))])


def check_ragged(G, w, s, exact_norm_cols=False, multiply_before_cast=True, r=None):
    if r is None:
        r = H.oracle_ragged_store(w, w.cache.dtype, multiply_before_cast)
    assert int(s.err.item()) == r.err
    D, T, Hq, Hk = w.cache.head_dim, w.total_tokens, w.n_q_heads, w.cache.n_kv_heads
    norm = w.q_gamma is not None
    fpc = np.ones(D, bool) if norm else H.rope_cols(D, w.rope.rope_dim, w.rope.rope_col_offset)
    eq = ek = None
    if not multiply_before_cast:  # the reading's intermediate rounding (helpers.py)
        dt = w.cache.dtype
        x = H.values(H.bits(w.qkv), dt).reshape(T, -1)
        gq, gk = H.values(H.bits(w.q_gamma), dt), H.values(H.bits(w.k_gamma), dt)
        eq = H.multiply_after_cast_slack(_head_rows(x, 0, Hq, D), gq, w.weight_offset,
                                         w.epsilon, dt, w.rope)[..., fpc]
        ek = H.scatter_slots(w.cache, H.multiply_after_cast_slack(
            _head_rows(x, Hq * D, Hk, D), gk, w.weight_offset, w.epsilon, dt, w.rope),
            w.cache.cache_lengths.tolist(), w.lengths, w.layer_idx)
    q = H.bits(s.q_out).reshape(T, Hq, D)
    qo = r.q_out.reshape(T, Hq, D)
    qd = {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}[w.q_out.dtype]
    H.assert_bits_equal(q[..., ~fpc], qo[..., ~fpc], "q_out pass-through columns")
    H.assert_close_bf16(q[..., fpc], qo[..., fpc], "q_out", dtype=qd, extra=eq)
    H.compare_paged_cache(w.cache, H.bits(s.storage), r.storage, r.written, w.layer_idx, fpc,
                          "cache", k_extra=ek)
    return r


# ------------------------------------------------------------- the named workloads --

def test_tiny_ragged(G):
    w = W.tiny_ragged()
    s = G.run_ragged(w)
    r = check_ragged(G, w, s)
    assert r.err == 0 and int(r.written.sum()) == 8


# The full-size cases run under the default launch-overlap mode and under the one the
# benchmark times (descriptor arrays read before the wait for the preceding kernels), each
# compared with the oracle.
FULL_SIZE_MODES = (1, 2)


def _under_modes(run):
    """run() under every mode of FULL_SIZE_MODES, the process-wide mode restored after."""
    import rope_paged_kv_b200 as rs
    before = rs.get_launch_overlap()
    try:
        for mode in FULL_SIZE_MODES:
            rs.set_launch_overlap(mode)
            run()
    finally:
        rs.set_launch_overlap(before)


def test_llama3_8b_prefill_full_size(G):
    w = W.llama3_8b_prefill()
    r = H.oracle_ragged_store(w, w.cache.dtype)
    _under_modes(lambda: check_ragged(G, w, G.run_ragged(w), r=r))


def test_per_head_norm_full_size(G):
    w = W.per_head_norm()
    r = H.oracle_ragged_store(w, w.cache.dtype)
    _under_modes(lambda: check_ragged(G, w, G.run_ragged(w), r=r))


def _check_dual(G, w, s, multiply_before_cast=True, r=None):
    if r is None:
        r = H.oracle_dual(w, multiply_before_cast=multiply_before_cast)
    assert int(s.err.item()) == r.err
    D = w.main_cache.head_dim
    allc = np.ones(D, bool)
    bands = (("main", w.main_q_heads), ("index", w.index_q_heads))
    x = H.values(H.bits(w.input), w.main_cache.dtype)
    for k, (which, nq) in enumerate(bands if w.index_cache is not None else bands[:1]):
        kv = getattr(w, f"{which}_cache")
        eq = ek = None
        if not multiply_before_cast:  # the reading's intermediate rounding (helpers.py)
            cols = getattr(w, f"{which}_cols")
            dt, eps = kv.dtype, getattr(w, f"{which}_eps")
            gq, gk = (H.values(H.bits(g), dt) for g in w.gammas[2 * k:2 * k + 2])
            eq = H.multiply_after_cast_slack(_head_rows(x, cols[0], nq, D), gq,
                                             w.weight_offset, eps, dt, w.rope)
            xk = (_head_rows(x, cols[1], kv.n_kv_heads, D) if cols[1] >= 0 else
                  _slot_rows(kv, H.bits(kv.storage), kv.cache_lengths.tolist(), w.lengths,
                             w.layer_idx))
            ek = H.scatter_slots(kv, H.multiply_after_cast_slack(xk, gk, w.weight_offset, eps,
                                                                 dt, w.rope),
                                 kv.cache_lengths.tolist(), w.lengths, w.layer_idx)
        q = H.bits(getattr(s, f"q_{which}_out")).reshape(w.total_tokens, nq, D)
        H.assert_close_bf16(q, r[f"q_{which}_out"].reshape(q.shape), f"q_{which}_out",
                            extra=eq)
        H.compare_paged_cache(kv, H.bits(getattr(s, f"{which}_storage")),
                              r[f"{which}_storage"], r[f"{which}_written"], w.layer_idx, allc,
                              f"{which} cache", k_extra=ek)
    return r


def test_dual_band_full_size(G):
    w = W.dual_band_minimax()
    r = H.oracle_dual(w)
    _under_modes(lambda: _check_dual(G, w, G.run_dual(w), r=r))


def _check_radd(G, w, s, r=None):
    if r is None:
        r = H.oracle_radd(w, w.cache.dtype)
    assert int(s.err.item()) == r.err
    H.assert_bits_equal(H.bits(s.storage), r.storage, "cache after radd")
    return r


def test_radd_full_size(G):
    w = W.radd_minimax()
    r = H.oracle_radd(w, w.cache.dtype)
    _under_modes(lambda: _check_radd(G, w, G.run_radd(w), r=r))


def _check_bshd(G, w, s, pristine, r=None):
    if r is None:
        r = H.oracle_bshd(w, w.cache.dtype)
    assert int(s.err.item()) == r.err
    D = w.cache.head_dim
    fpc = H.rope_cols(D, w.rope.rope_dim, w.rope.rope_col_offset)
    out = H.bits(s.out)
    H.assert_bits_equal(out[..., ~fpc], r.output[..., ~fpc], "output pass-through columns")
    H.assert_close_bf16(out[..., fpc], r.output[..., fpc], "output", dtype=w.cache.dtype)
    # tokens past valid_lengths: copied bit for bit
    for b in range(w.q_proj.shape[0]):
        vl = int(w.valid_lengths[b])
        if vl < w.q_proj.shape[1]:
            H.assert_bits_equal(out[b, vl:], H.bits(w.q_proj)[b, vl:], "copied tokens")
    G.compare_cont_cache(w, s, pristine, r.storage, r.written, fpc)
    return r


def test_decode_bshd_full_size(G):
    w = W.decode_bshd()
    r = H.oracle_bshd(w, w.cache.dtype)

    def run():
        s = G.stage_bshd(w)
        pristine = s.storage.clone()
        G.launch_bshd(w, s)
        torch.cuda.synchronize()
        _check_bshd(G, w, s, pristine, r=r)
    _under_modes(run)


# ------------------------------------------------------------------------ edge cases --

RAGGED_EDGES = {
    "zero-length seqs, page crossings, half-split partial 32/64": dict(
        lengths=[37, 0, 1, 64, 0, 18], cache_lengths=[5, 9, 0, 120, 3, 15], n_q_heads=4,
        n_kv_heads=2, head_dim=64, page_size=16, rope_dim=32, theta=1e4, interleaved=False,
        max_seq_len=256, width=16),
    "interleaved partial 64/128, rows past many tiles": dict(
        lengths=[300, 257, 1, 500], cache_lengths=[0, 1000, 77, 3], n_q_heads=8, n_kv_heads=2,
        head_dim=128, page_size=32, rope_dim=64, theta=5e5, interleaved=True,
        max_seq_len=2048),
    "head_dim 256, GQA 16/4": dict(
        lengths=[33, 70], cache_lengths=[1, 250], n_q_heads=16, n_kv_heads=4, head_dim=256,
        page_size=64, rope_dim=256, theta=1e6, interleaved=False, max_seq_len=512),
    "f16 elements, head_dim 64": dict(
        lengths=[17, 40, 3], cache_lengths=[0, 31, 2], n_q_heads=6, n_kv_heads=3, head_dim=64,
        page_size=16, rope_dim=64, theta=1e4, interleaved=True, max_seq_len=128, dtype="f16"),
    "f32 elements, head_dim 128, half-split": dict(
        lengths=[21, 9], cache_lengths=[4, 60], n_q_heads=4, n_kv_heads=1, head_dim=128,
        page_size=16, rope_dim=128, theta=1e4, interleaved=False, max_seq_len=128,
        dtype="f32"),
    "bf16 freqs table": dict(
        lengths=[50, 13], cache_lengths=[7, 0], n_q_heads=4, n_kv_heads=2, head_dim=128,
        page_size=16, rope_dim=128, theta=5e5, interleaved=True, max_seq_len=128,
        freq_dtype="bf16"),
    "f16 freqs table, half-split": dict(
        lengths=[50, 13], cache_lengths=[7, 0], n_q_heads=4, n_kv_heads=2, head_dim=128,
        page_size=16, rope_dim=128, theta=5e5, interleaved=False, max_seq_len=128,
        freq_dtype="f16"),
    "padded input rows": dict(
        lengths=[19, 23], cache_lengths=[3, 0], n_q_heads=4, n_kv_heads=2, head_dim=64,
        page_size=16, rope_dim=64, theta=1e4, interleaved=False, max_seq_len=64, row_pad=24),
    "rotation on the leading columns": dict(
        lengths=[10, 30], cache_lengths=[0, 5], n_q_heads=2, n_kv_heads=2, head_dim=128,
        page_size=16, rope_dim=64, theta=1e4, interleaved=True, max_seq_len=64,
        rope_col_offset=0),
    "no rotation (rope_dim 0)": dict(
        lengths=[10, 30], cache_lengths=[0, 5], n_q_heads=2, n_kv_heads=2, head_dim=64,
        page_size=16, rope_dim=0, theta=1e4, interleaved=True, max_seq_len=64),
    "many sequences (offsets beyond the shared-memory stage)": dict(
        lengths=[(i * 7) % 4 for i in range(1500)], cache_lengths=[(i * 13) % 50 for i in range(1500)],
        n_q_heads=2, n_kv_heads=1, head_dim=64, page_size=16, rope_dim=64, theta=1e4,
        interleaved=False, max_seq_len=64),
    "layer 0 of 3": dict(
        lengths=[12, 5], cache_lengths=[3, 4], n_q_heads=2, n_kv_heads=2, head_dim=64,
        page_size=8, rope_dim=64, theta=1e4, interleaved=True, max_seq_len=64, num_layers=3,
        layer_idx=0),
}


@pytest.mark.parametrize("name", list(RAGGED_EDGES))
@pytest.mark.parametrize("norm", [False, True], ids=["store", "norm"])
def test_ragged_edge_cases(G, name, norm):
    kw = dict(RAGGED_EDGES[name])
    if norm:
        kw.update(norm=True, epsilon=1e-5, weight_offset=0.0, x_std=2.0)
    w = W.ragged_store(1000 + len(name), **kw, name=name)
    check_ragged(G, w, G.run_ragged(w))


@pytest.mark.parametrize("n_q,n_kv,mbc", [(32, 8, True), (40, 8, False), (60, 6, True),
                                          (64, 8, True)])
def test_norm_rows_a_thread(G, n_q, n_kv, mbc):
    """The norm's row steps take a thread's rows three at a time, then a tail of one or two.
    In the six-warp shape (24 row groups) Q + K rows of 40 give threads two and one rows, 48
    two, 66 three and two, 72 three: every step size, with either order of cast and gamma."""
    w = W.ragged_store(1300 + n_q + n_kv, lengths=[70, 1, 33], cache_lengths=[0, 11, 90],
                       n_q_heads=n_q, n_kv_heads=n_kv, head_dim=128, page_size=32, rope_dim=128,
                       theta=1e4, interleaved=False, max_seq_len=256, norm=True, epsilon=1e-6,
                       x_std=2.0, weight_offset=0.25)
    check_ragged(G, w, G.run_ragged(w, multiply_before_cast=mbc), multiply_before_cast=mbc)


def test_norm_weight_offset_one(G):
    w = W.ragged_store(1201, lengths=[40, 25], cache_lengths=[0, 9], n_q_heads=8, n_kv_heads=2,
                       head_dim=128, page_size=16, rope_dim=128, theta=1e4, interleaved=False,
                       max_seq_len=128, norm=True, epsilon=1e-6, weight_offset=1.0)
    w.q_gamma.mul_(0.0).add_(torch.randn(128, generator=W.generator(3)).to(torch.bfloat16) * 0.1)
    check_ragged(G, w, G.run_ragged(w))


def _golden_cases():
    here = os.path.join(os.path.dirname(__file__), "golden")
    out = []
    for fname, norm in (("rope_worked_examples.json", False),
                        ("rmsnorm_worked_examples.json", True)):
        for c in json.load(open(os.path.join(here, fname)))["cases"]:
            out.append(pytest.param(c, norm, id=c["name"]))
    return out


@pytest.mark.parametrize("case,norm", _golden_cases())
def test_worked_examples_on_gpu(G, case, norm):
    # the hand-worked rows, tiled across a head_dim-64 head (same pairs, same mean square)
    c = H.tile_golden(case, 64)
    w = H.golden_problem(c, norm)
    s = G.run_ragged(w)
    assert int(s.err.item()) == 0
    want = np.asarray(c["expect"], dtype=np.float64)
    q = H.values(H.bits(s.q_out).reshape(-1), "bf16")
    kv6 = H.bits(s.storage).reshape(1, 2, 1, 2, 1, 64)
    k = H.values(kv6[0, 0, 0, 1, 0], "bf16")
    v = H.values(kv6[0, 1, 0, 1, 0], "bf16")
    tol = np.maximum(H.bf16_ulp(want), 1e-3)
    assert np.all(np.abs(q - want) <= tol) and np.all(np.abs(k - want) <= tol)
    assert v.tolist() == list(range(1, 65))


DUAL_EDGES = {
    "small, zero-length seqs, eps per band, weight_offset 1": dict(
        lengths=[7, 0, 12, 33], cache_lengths=[3, 0, 60, 0], main_q_heads=4, main_kv_heads=2,
        index_q_heads=2, index_kv_heads=1, head_dim=64, main_page_size=16, index_page_size=8,
        rope_dim=32, theta=1e4, interleaved=True, max_seq_len=256, main_eps=1e-6,
        index_eps=1e-3, weight_offset=1.0),
    "half-split, head_dim 128, 300 tokens": dict(
        lengths=[100, 150, 50], cache_lengths=[10, 0, 500], main_q_heads=16, main_kv_heads=4,
        index_q_heads=4, index_kv_heads=1, head_dim=128, main_page_size=64, index_page_size=32,
        rope_dim=64, theta=1e4, interleaved=False, max_seq_len=1024),
}


@pytest.mark.parametrize("name", list(DUAL_EDGES))
def test_dual_band_edge_cases(G, name):
    w = W.dual_band(1300 + len(name), **DUAL_EDGES[name])
    _check_dual(G, w, G.run_dual(w))


@pytest.mark.parametrize("batch_offset", [0, 3])
@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_radd_edge_cases(G, batch_offset, dtype):
    w = W.radd(1400 + batch_offset, lengths=[5, 0, 12, 40], cache_lengths=[3, 8, 30, 100],
               n_kv_heads=2, head_dim=64 if dtype != "f32" else 128, page_size=16,
               batch_offset=batch_offset, max_seq_len=256, dtype=dtype)
    _check_radd(G, w, G.run_radd(w))


BSHD_EDGES = {
    "S 4 with valid_lengths < S, two layers": dict(
        B=3, S=4, n_q_heads=4, n_kv_heads=2, head_dim=128, cache_lengths=[0, 7, 20],
        valid_lengths=[4, 2, 0], max_seq_len=64, rope_dim=128, theta=1e4, interleaved=True,
        freq_dtype="f32", num_slots=5, num_layers=2, layer_idx=1, planes=2),
    "half-split, f16, partial 32/64": dict(
        B=5, S=3, n_q_heads=8, n_kv_heads=1, head_dim=64, cache_lengths=[0, 1, 2, 30, 60],
        valid_lengths=[3, 3, 1, 2, 3], max_seq_len=64, rope_dim=32, theta=1e4,
        interleaved=False, freq_dtype="f16", dtype="f16"),
    "head_dim 256, bf16 table": dict(
        B=2, S=2, n_q_heads=8, n_kv_heads=2, head_dim=256, cache_lengths=[10, 99],
        valid_lengths=[2, 1], max_seq_len=128, rope_dim=256, theta=5e5, interleaved=True,
        freq_dtype="bf16"),
}


@pytest.mark.parametrize("name", list(BSHD_EDGES))
def test_bshd_edge_cases(G, name):
    w = W.bshd_decode(1500 + len(name), **BSHD_EDGES[name])
    s = G.stage_bshd(w)
    pristine = s.storage.clone()
    G.launch_bshd(w, s)
    torch.cuda.synchronize()
    _check_bshd(G, w, s, pristine)


# -------------------------------------------------------------------- device errors --

def test_device_errors_skip_tokens(G):
    # positions past the 16-row freqs table, then a page id past num_pages
    w = W.ragged_store(1601, lengths=[3, 4], cache_lengths=[0, 14], n_q_heads=2, n_kv_heads=1,
                       head_dim=64, page_size=8, rope_dim=64, theta=1e4, interleaved=True,
                       max_seq_len=16, width=2)
    r = check_ragged(G, w, G.run_ragged(w))
    assert r.err == oracle.ERR_POSITION
    w.cache.page_table[1, 1] = w.cache.num_pages + 5
    r = check_ragged(G, w, G.run_ragged(w))
    assert r.err & oracle.ERR_PAGE_ID
    # page index past the table width
    w2 = W.ragged_store(1602, lengths=[10], cache_lengths=[12], n_q_heads=1, n_kv_heads=1,
                        head_dim=64, page_size=8, rope_dim=64, theta=1e4, interleaved=True,
                        max_seq_len=64, width=2)
    r = check_ragged(G, w2, G.run_ragged(w2))
    assert r.err == oracle.ERR_PAGE_INDEX


@pytest.mark.parametrize("bad", ["first", "decreasing", "last"])
def test_bad_offsets_write_nothing(G, bad):
    w = W.ragged_store(1603, lengths=[5, 6, 7], cache_lengths=[0, 0, 0], n_q_heads=2,
                       n_kv_heads=1, head_dim=64, page_size=8, rope_dim=64, theta=1e4,
                       interleaved=True, max_seq_len=64)
    if bad == "first":
        w.offsets[0] = 1
    elif bad == "decreasing":
        w.offsets[1] = 12
    else:
        w.offsets[3] = 17
    s = G.run_ragged(w)
    r = check_ragged(G, w, s)
    assert r.err == oracle.ERR_ROW_OFFSETS and int(r.written.sum()) == 0


def test_radd_and_bshd_errors(G):
    w = W.radd(1604, lengths=[2, 3], cache_lengths=[0, 0], n_kv_heads=1, head_dim=64,
               page_size=8, batch_offset=1, max_seq_len=64)
    w.batch_offset = 2
    r = _check_radd(G, w, G.run_radd(w))
    assert r.err == oracle.ERR_BATCH
    wb = W.bshd_decode(1605, B=3, S=2, n_q_heads=2, n_kv_heads=1, head_dim=64,
                       cache_lengths=[0, 63, 5], valid_lengths=[2, 2, 2], max_seq_len=64,
                       rope_dim=64, theta=1e4, interleaved=True, freq_dtype="f32", num_slots=4)
    wb.cache.lookup_table[2] = 9          # slot past num_slots
    s = G.stage_bshd(wb)
    pristine = s.storage.clone()
    G.launch_bshd(wb, s)
    torch.cuda.synchronize()
    r = _check_bshd(G, wb, s, pristine)
    assert r.err == (oracle.ERR_POSITION | oracle.ERR_BATCH)


def test_empty_batch_launches_nothing(G):
    import rope_paged_kv_b200 as rs
    w = W.ragged_store(1606, lengths=[0, 0], cache_lengths=[0, 0], n_q_heads=2, n_kv_heads=1,
                       head_dim=64, page_size=8, rope_dim=64, theta=1e4, interleaved=True,
                       max_seq_len=64)
    s = G.stage_ragged(w)
    before = s.storage.clone()
    G.launch_ragged(w, s)
    torch.cuda.synchronize()
    assert torch.equal(before.view(torch.int16), s.storage.view(torch.int16))
    assert int(s.err.item()) == 0
