"""Band options beyond the store of the named workloads, CUDA path vs the oracle.

K updated in place (a band whose K heads are read from the token's cache slot and written
back there, V untouched), the single-band launch (no index band), and
multiply_before_cast = 0 (the normalised value rounded to the element type before the
gamma multiply).  Tolerances as in test_gpu_parity.py.
"""
import pytest
import torch

import workloads as W
from test_gpu_parity import _check_dual, check_ragged

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gpu_helpers
    return gpu_helpers


def band_case(seed, **kw):
    base = dict(lengths=[300, 1, 57, 640], cache_lengths=[0, 9, 200, 33], main_q_heads=8,
                main_kv_heads=2, index_q_heads=2, index_kv_heads=1, head_dim=128,
                main_page_size=64, index_page_size=32, rope_dim=64, theta=1e4,
                interleaved=True, max_seq_len=1024)
    base.update(kw)
    return W.dual_band(seed, **base)


@pytest.mark.parametrize("single", [False, True])
@pytest.mark.parametrize("interleaved", [True, False])
def test_k_in_place(G, single, interleaved):
    w = band_case(41, k_in_place=True, single=single, interleaved=interleaved)
    _check_dual(G, w, G.run_dual(w))


def test_single_band_store(G):
    w = band_case(42, single=True)
    _check_dual(G, w, G.run_dual(w))


def test_k_in_place_full_size(G):
    # the dual-band workload with both key caches updated in place (the literal reading)
    w = W.dual_band_minimax_in_place()
    _check_dual(G, w, G.run_dual(w))


@pytest.mark.parametrize("head_dim,dtype", [(128, "bf16"), (64, "f16"), (128, "f32")])
def test_multiply_after_cast_ragged(G, head_dim, dtype):
    w = W.ragged_store(43, lengths=[129, 3, 700], cache_lengths=[0, 17, 64], n_q_heads=8,
                       n_kv_heads=2, head_dim=head_dim, page_size=32, rope_dim=head_dim // 2,
                       theta=1e4, interleaved=False, max_seq_len=1024, x_std=2.0, norm=True,
                       weight_offset=1.0, dtype=dtype)
    s = G.run_ragged(w, multiply_before_cast=False)
    check_ragged(G, w, s, multiply_before_cast=False)


def test_multiply_after_cast_dual_in_place(G):
    w = band_case(44, k_in_place=True, x_std=2.0)
    _check_dual(G, w, G.run_dual(w, multiply_before_cast=False), multiply_before_cast=False)


@pytest.mark.parametrize("dtype,q_dtype,head_dim", [
    ("bf16", "f32", 128), ("bf16", "f16", 128), ("f16", "bf16", 64), ("f32", "bf16", 64),
    ("f32", "f16", 128), ("bf16", "bf16", 128)])
@pytest.mark.parametrize("interleaved", [True, False])
def test_q_out_element_type(G, dtype, q_dtype, head_dim, interleaved):
    # rope_split_store_paged_ragged's q_out_dtype: Q rounded once into its own type;
    # partial rope so that unrotated columns are converted too
    w = W.ragged_store(45, lengths=[300, 2, 257], cache_lengths=[0, 5, 64], n_q_heads=8,
                       n_kv_heads=2, head_dim=head_dim, page_size=32, rope_dim=head_dim // 2,
                       theta=1e4, interleaved=interleaved, max_seq_len=1024, dtype=dtype,
                       q_out_dtype=q_dtype)
    check_ragged(G, w, G.run_ragged(w))


def test_q_out_element_type_many_heads(G):
    # more head rows than the light shape's usual share: the call still takes the shape
    # built with the conversion
    w = W.ragged_store(46, lengths=[130, 70], cache_lengths=[0, 9], n_q_heads=64,
                       n_kv_heads=8, head_dim=128, page_size=64, rope_dim=128, theta=5e5,
                       interleaved=False, max_seq_len=512, q_out_dtype="f32")
    check_ragged(G, w, G.run_ragged(w))


# ---------------------------------------------- weight_offset, a scalar of the element type --
# fused_dual_qk_rms_norm_rope_ragged_paged, signature: weight_offset is a Scalar[dtype].  On
# rows whose normalised value is exactly x / 2 (gamma 0, epsilon 0, position 0), every
# output is (x / 2) * bf16(0.3) exactly, one bf16 step away from what an unrounded 0.3 gives
# on a third of the elements: a tolerance of one step would not see the difference, so the
# outputs are compared bit for bit with the oracle (pinned on this case) and the closed form.

@pytest.mark.parametrize("multiply_before_cast", [True, False])
def test_weight_offset_is_an_element_type_scalar_single_band(G, multiply_before_cast):
    import helpers as H
    from test_oracle_pins import weight_offset_problem
    w, want_q, _ = weight_offset_problem(72, head_dim=128, n_tokens=300)
    s = G.run_ragged(w, multiply_before_cast=multiply_before_cast)
    r = H.oracle_ragged_store(w, "bf16", multiply_before_cast)
    assert int(s.err.item()) == r.err == 0
    H.assert_bits_equal(H.bits(s.q_out).reshape(want_q.shape), H.bits(want_q), "q_out")
    H.assert_bits_equal(H.bits(s.q_out), r.q_out, "q_out vs the oracle")
    H.assert_bits_equal(H.bits(s.storage), r.storage, "cache vs the oracle")


@pytest.mark.parametrize("multiply_before_cast", [True, False])
def test_weight_offset_is_an_element_type_scalar_dual_band(G, multiply_before_cast):
    import helpers as H
    n, D = 200, 128
    w = W.dual_band(73, lengths=[1] * n, cache_lengths=[0] * n, main_q_heads=4,
                    main_kv_heads=2, index_q_heads=2, index_kv_heads=1, head_dim=D,
                    main_page_size=16, index_page_size=8, rope_dim=64, theta=1e4,
                    interleaved=True, max_seq_len=16, main_eps=0.0, index_eps=0.0,
                    weight_offset=0.3)
    for g in w.gammas:
        g.zero_()
    want = {}
    # Q and K head blocks of each band: main [Q 4 | K 2] from column 0, index [Q 2 | K 1]
    # from column 8 * D (after the main V heads)
    for which, lo, nq, hi in (("main", 0, 4, 6), ("index", 8, 2, 11)):
        rows = H.exact_norm_rows(73 + lo, n * (hi - lo), D)
        w.input[:, lo * D:hi * D] = rows.view(n, -1).to(torch.bfloat16)
        want[which] = H.bf16_weight_offset_case(rows, w.weight_offset)[0].view(n, hi - lo, D)
    s = G.run_dual(w, multiply_before_cast=multiply_before_cast)
    r = H.oracle_dual(w, multiply_before_cast=multiply_before_cast)
    assert int(s.err.item()) == r.err == 0
    for which, nq in (("main", 4), ("index", 2)):
        q = H.bits(getattr(s, f"q_{which}_out"))
        H.assert_bits_equal(q.reshape(n, nq, D), H.bits(want[which][:, :nq]), f"q_{which}_out")
        H.assert_bits_equal(q, r[f"q_{which}_out"], f"q_{which}_out vs the oracle")
        H.assert_bits_equal(H.bits(getattr(s, f"{which}_storage")), r[f"{which}_storage"],
                            f"{which} cache vs the oracle")
