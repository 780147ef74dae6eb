"""Pins of the CPU oracle against what the kernel pages and the mathematics fix.

Each test checks the oracle against something other than itself: hand-worked values
(tests/golden, each citing its page), closed forms, invariants of the rotation and of the
normalisation, and special cases that reduce to a library routine (numpy complex products,
rotation matrices, torch / numpy float rounding).  A dropped term, a wrong sign, a wrong
pair index, a wrong position or a transposed operand fails at least one of them.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import helpers as H

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------- element codecs --

def test_bf16_codec_known_bits():
    b = np.array([0x3F80, 0xC000, 0x0001, 0x7F80, 0x0080, 0x3F81], dtype=np.uint16)
    want = [1.0, -2.0, 2.0 ** -133, np.inf, 2.0 ** -126, 1.0 + 2.0 ** -7]
    assert oracle.decode(b, "bf16").tolist() == want
    # ties go to the even neighbour; just above a tie goes up
    v = [1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -30, -(1 + 2 ** -8), 2.0 ** -134,
         3 * 2.0 ** -134, (2 - 2 ** -8) * 2.0 ** 127]
    want = [0x3F80, 0x3F82, 0x3F81, 0xBF80, 0x0000, 0x0002, 0x7F80]
    assert oracle.encode(v, "bf16").tolist() == want


def test_bf16_encode_matches_torch_rne_on_float32_values():
    # for values that are float32 numbers, rounding to bf16 is torch's float32 -> bf16 (RNE)
    g = torch.Generator().manual_seed(3)
    x = torch.randn(20000, generator=g) * torch.exp2(torch.randint(-40, 40, (20000,),
                                                                    generator=g).float())
    want = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.encode(x.double().numpy(), "bf16")
    assert np.array_equal(got, want)


def test_f16_codec_matches_numpy():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(20000) * np.exp2(rng.integers(-26, 14, 20000))
    x[:4] = [65519.99, 65520.0, -70000.0, 2.0 ** -25]   # last finite, first overflow, tie
    got = oracle.encode(x, "f16")
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)  # numpy: correctly rounded, ties to even
    assert np.array_equal(got, want)
    back = oracle.decode(want, "f16")
    assert np.array_equal(back, want.view(np.float16).astype(np.float64))


# ------------------------------------------------------------------- worked examples --

def _run_golden(case, norm, dtype="bf16"):
    w = H.golden_problem(case, norm, dtype)
    r = H.oracle_ragged_store(w, dtype)
    assert r.err == 0
    D = case["head_dim"]
    q = H.values(r.q_out.reshape(-1), dtype)
    kv6 = r.storage.reshape(1, 2, 1, 2, 1, D)  # [page, plane, layer, slot, head, d]
    k = H.values(kv6[0, 0, 0, 1, 0], dtype)
    v = H.values(kv6[0, 1, 0, 1, 0], dtype)
    return q, k, v, r


@pytest.mark.parametrize("case", _golden("rope_worked_examples.json")["cases"],
                         ids=lambda c: c["name"])
def test_rope_worked_examples(case):
    q, k, v, _ = _run_golden(case, norm=False)
    assert q.tolist() == case["expect"]
    assert k.tolist() == case["expect"]
    assert v.tolist() == list(range(1, case["head_dim"] + 1))


@pytest.mark.parametrize("case", _golden("rmsnorm_worked_examples.json")["cases"],
                         ids=lambda c: c["name"])
def test_rmsnorm_worked_examples(case):
    q, k, v, _ = _run_golden(case, norm=True)
    assert q.tolist() == case["expect"]
    assert k.tolist() == case["expect"]
    assert v.tolist() == list(range(1, case["head_dim"] + 1))


@pytest.mark.parametrize("fname,norm", [("rope_worked_examples.json", False),
                                         ("rmsnorm_worked_examples.json", True)])
def test_worked_examples_tiled_to_head_dim_64(fname, norm):
    for case in _golden(fname)["cases"]:
        c = H.tile_golden(case, 64)
        q, k, v, _ = _run_golden(c, norm)
        assert q.tolist() == c["expect"], case["name"]
        assert k.tolist() == c["expect"], case["name"]


def _placement_problem(g, D=8, Hq=1, Hk=1, seed=11):
    gen = W.generator(seed)
    T = sum(g["lengths"])
    P, npg = g["page_size"], g["num_pages"]
    qkv = W.normal(gen, (T, (Hq + 2 * Hk) * D))
    table = torch.tensor(np.array(g["page_table"], dtype=np.uint32).view(np.int32))
    storage = W.random_bits(gen, npg * 2 * 2 * P * Hk * D)
    cache = W.PagedKV(storage, 2, npg, 2, P, Hk, D, table.contiguous(),
                      torch.tensor(g["cache_lengths"], dtype=torch.int32))
    rope = W.RopeSpec(W.freqs_cis(64, D, 1e4), "f32", True)
    q_out = W.random_bits(gen, T * Hq * D).view(T, Hq * D)
    return W.RaggedStore(qkv, W.row_offsets(g["lengths"]), Hq, cache, rope, 1, q_out,
                         g["lengths"])


def test_placement_worked_example():
    g = _golden("placement_worked_example.json")
    w = _placement_problem(g)
    r = H.oracle_ragged_store(w)
    assert r.err == 0
    P = g["page_size"]
    want = {p * P + s for p, s in g["expect_page_slot"]}
    assert set(np.flatnonzero(r.written).tolist()) == want
    kv6 = w.cache.view6(torch.from_numpy(r.storage.view(np.int16)).view(torch.bfloat16))
    qkv = w.qkv
    D = w.cache.head_dim
    for row, (p, s) in enumerate(g["expect_page_slot"]):
        # V of token `row` sits at (page, slot) of layer 1, bit for bit
        assert torch.equal(kv6[p, 1, 1, s, 0].view(torch.int16),
                           qkv[row, 2 * D:3 * D].view(torch.int16))


# ------------------------------------------------------------ rotation: library forms --

def _f32_problem(interleaved, rope_dim=64, head_dim=64, rope_col_offset=-1, seed=21,
                 lengths=(5, 9, 1), cache_lengths=(0, 17, 40), theta=1e4):
    return W.ragged_store(seed, lengths=list(lengths), cache_lengths=list(cache_lengths),
                          n_q_heads=3, n_kv_heads=2, head_dim=head_dim, page_size=8,
                          rope_dim=rope_dim, theta=theta, interleaved=interleaved,
                          max_seq_len=64, rope_col_offset=rope_col_offset, dtype="f32")


def _positions(w):
    pos = []
    for b, n in enumerate(w.lengths):
        pos += [int(w.cache.cache_lengths[b]) + t for t in range(n)]
    return np.array(pos)


def _q_heads(w, arr):
    T = w.total_tokens
    return arr.reshape(T, w.n_q_heads, w.cache.head_dim).astype(np.float64)


def test_interleaved_rope_is_complex_product():
    w = _f32_problem(True)
    r = H.oracle_ragged_store(w, "f32")
    assert r.err == 0
    D, R = 64, 64
    x = _q_heads(w, w.qkv[:, :w.n_q_heads * D].numpy())
    F = w.rope.table.double().numpy()[_positions(w)]          # [T, R]
    z = x[..., 0::2] + 1j * x[..., 1::2]
    cis = (F[:, 0::2] + 1j * F[:, 1::2])[:, None, :]
    want = z * cis
    got = _q_heads(w, r.q_out)
    np.testing.assert_allclose(got[..., 0::2], want.real, rtol=0, atol=1e-6 * np.abs(x).max())
    np.testing.assert_allclose(got[..., 1::2], want.imag, rtol=0, atol=1e-6 * np.abs(x).max())


def test_half_split_rope_is_rotation_matrix_product():
    w = _f32_problem(False, rope_dim=32, head_dim=64)
    r = H.oracle_ragged_store(w, "f32")
    assert r.err == 0
    D, R = 64, 32
    o = D - R
    x = _q_heads(w, w.qkv[:, :w.n_q_heads * D].numpy())
    F = w.rope.table.double().numpy()[_positions(w)]
    T = x.shape[0]
    M = np.zeros((T, D, D))
    M[:, np.arange(o), np.arange(o)] = 1.0
    for i in range(R // 2):
        a, b = o + i, o + i + R // 2
        c, s = F[:, 2 * i], F[:, 2 * i + 1]
        M[:, a, a], M[:, a, b], M[:, b, a], M[:, b, b] = c, -s, s, c
    want = np.einsum("tij,thj->thi", M, x)
    got = _q_heads(w, r.q_out)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-6 * np.abs(x).max())
    # unrotated columns pass through bit for bit
    assert np.array_equal(got[..., :o], x[..., :o])


@pytest.mark.parametrize("interleaved", [True, False])
def test_position_zero_is_identity(interleaved):
    w = W.ragged_store(31, lengths=[4, 3], cache_lengths=[0, 0], n_q_heads=4, n_kv_heads=2,
                       head_dim=64, page_size=16, rope_dim=64, theta=1e4,
                       interleaved=interleaved, max_seq_len=16)
    r = H.oracle_ragged_store(w)
    q_in = H.bits(w.qkv)[:, :4 * 64]
    # token 0 of each sequence sits at position 0: freqs_cis row 0 is (1, 0)
    for row in (0, 4):
        assert np.array_equal(r.q_out[row], q_in[row])
    # other positions do rotate
    assert not np.array_equal(r.q_out[1], q_in[1])


@pytest.mark.parametrize("interleaved", [True, False])
def test_rotation_preserves_pair_norms(interleaved):
    w = _f32_problem(interleaved)
    r = H.oracle_ragged_store(w, "f32")
    D = 64
    x = _q_heads(w, w.qkv[:, :w.n_q_heads * D].numpy())
    y = _q_heads(w, r.q_out)
    F = w.rope.table.double().numpy()[_positions(w)]
    if interleaved:
        nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
        ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    else:
        nx = x[..., :32] ** 2 + x[..., 32:] ** 2
        ny = y[..., :32] ** 2 + y[..., 32:] ** 2
    scale = (F[:, 0::2] ** 2 + F[:, 1::2] ** 2)[:, None, :]   # = 1 up to the f32 table
    np.testing.assert_allclose(ny, scale * nx, rtol=1e-6, atol=1e-9)


@pytest.mark.parametrize("interleaved", [True, False])
def test_inverse_rotation_round_trips(interleaved):
    w = _f32_problem(interleaved)
    r = H.oracle_ragged_store(w, "f32")
    # rotate the output back with the conjugate table (cos, -sin)
    w2 = _f32_problem(interleaved)
    w2.qkv[:, :w.n_q_heads * 64] = torch.from_numpy(r.q_out)
    w2.rope.table[:, 1::2] *= -1
    r2 = H.oracle_ragged_store(w2, "f32")
    x = w.qkv[:, :w.n_q_heads * 64].double().numpy()
    np.testing.assert_allclose(r2.q_out.astype(np.float64), x, rtol=0,
                               atol=4e-7 * np.abs(x).max())


def test_relative_position_property():
    # <R(p) q, R(p') k> depends only on p - p' (closed-form table, f32 elements)
    def roped_first_token(cache_len):
        w = W.ragged_store(41, lengths=[1], cache_lengths=[cache_len], n_q_heads=1,
                           n_kv_heads=1, head_dim=64, page_size=8, rope_dim=64, theta=1e4,
                           interleaved=True, max_seq_len=64, dtype="f32")
        r = H.oracle_ragged_store(w, "f32")
        return r.q_out[0].astype(np.float64)

    dots = []
    for p, pk, delta in [(3, 10, 0), (3, 10, 20), (3, 10, 45)]:
        q = roped_first_token(p + delta)
        k = roped_first_token(pk + delta)
        dots.append(q @ k)
    np.testing.assert_allclose(dots, dots[0], rtol=2e-5)
    # and it does depend on the gap
    assert abs(roped_first_token(3) @ roped_first_token(30) - dots[0]) > 1e-3


def test_half_split_equals_permuted_interleaved():
    w_h = _f32_problem(False, rope_dim=64, head_dim=64)
    w_i = _f32_problem(True, rope_dim=64, head_dim=64)
    perm = np.empty(64, dtype=np.int64)          # interleaved column j <- half-split column
    perm[0::2], perm[1::2] = np.arange(32), np.arange(32, 64)
    Hq = w_h.n_q_heads
    x = w_h.qkv[:, :Hq * 64].view(-1, Hq, 64)
    w_i.qkv[:, :Hq * 64] = x[..., perm].reshape(-1, Hq * 64)
    r_h = H.oracle_ragged_store(w_h, "f32")
    r_i = H.oracle_ragged_store(w_i, "f32")
    inv = np.argsort(perm)
    got = r_i.q_out.reshape(-1, Hq, 64)[..., inv]
    assert np.array_equal(got, r_h.q_out.reshape(-1, Hq, 64))


@pytest.mark.parametrize("interleaved", [True, False])
def test_partial_rope_is_full_rope_of_the_tail(interleaved):
    w_p = _f32_problem(interleaved, rope_dim=32, head_dim=64)
    r_p = H.oracle_ragged_store(w_p, "f32")
    Hq = w_p.n_q_heads
    x = w_p.qkv[:, :Hq * 64].view(-1, Hq, 64)
    # the same rotation on head_dim-32 heads holding only the last 32 columns
    w_f = _f32_problem(interleaved, rope_dim=32, head_dim=32)
    assert w_f.total_tokens == w_p.total_tokens
    w_f.qkv[:, :Hq * 32] = x[..., 32:].reshape(-1, Hq * 32)
    w_f.rope.table.copy_(w_p.rope.table)
    r_f = H.oracle_ragged_store(w_f, "f32")
    got = r_p.q_out.reshape(-1, Hq, 64)
    assert np.array_equal(got[..., :32], x[..., :32].numpy())
    assert np.array_equal(got[..., 32:], r_f.q_out.reshape(-1, Hq, 32))


@pytest.mark.parametrize("interleaved", [True, False])
@pytest.mark.parametrize("offset", [0, 16])
def test_partial_rope_at_another_column_offset(interleaved, offset):
    """The other reading of partial RoPE (rope_col_offset names the first rotated column):
    columns [offset, offset + 32) of each head are rotated exactly as a 32-wide head would
    be, every other column passes through bit for bit."""
    w_p = _f32_problem(interleaved, rope_dim=32, head_dim=64)
    w_p.rope.rope_col_offset = offset
    r_p = H.oracle_ragged_store(w_p, "f32")
    assert r_p.err == 0
    Hq = w_p.n_q_heads
    x = w_p.qkv[:, :Hq * 64].view(-1, Hq, 64)
    w_f = _f32_problem(interleaved, rope_dim=32, head_dim=32)
    w_f.qkv[:, :Hq * 32] = x[..., offset:offset + 32].reshape(-1, Hq * 32)
    w_f.rope.table.copy_(w_p.rope.table)
    r_f = H.oracle_ragged_store(w_f, "f32")
    got = r_p.q_out.reshape(-1, Hq, 64)
    keep = np.ones(64, bool)
    keep[offset:offset + 32] = False
    assert np.array_equal(got[..., keep], x[..., keep].numpy())
    assert np.array_equal(got[..., offset:offset + 32], r_f.q_out.reshape(-1, Hq, 32))


# ----------------------------------------------------------------------- RMSNorm pins --

def _norm_problem(gamma_const=None, eps=0.5, wo=0.0, seed=51, interleaved=True):
    w = W.ragged_store(seed, lengths=[6, 2], cache_lengths=[0, 9], n_q_heads=2, n_kv_heads=1,
                       head_dim=64, page_size=8, rope_dim=64, theta=1e4,
                       interleaved=interleaved, max_seq_len=32, norm=True, epsilon=eps,
                       weight_offset=wo, dtype="f32", x_std=3.0)
    if gamma_const is not None:
        w.q_gamma.fill_(gamma_const)
        w.k_gamma.fill_(gamma_const)
    return w


def test_rmsnorm_rms_closed_form():
    # rows at position 0 are not rotated: rms(y) = |g| sqrt(ms / (ms + eps))
    eps, g = 0.5, 1.75
    w = _norm_problem(gamma_const=g, eps=eps)
    r = H.oracle_ragged_store(w, "f32")
    x = w.qkv[0, :2 * 64].double().view(2, 64).numpy()
    y = r.q_out[0].astype(np.float64).reshape(2, 64)
    ms = (x ** 2).mean(axis=1)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(axis=1)), g * np.sqrt(ms / (ms + eps)),
                               rtol=1e-6)
    # RoPE preserves the row's RMS at every position
    for row in range(w.total_tokens):
        x = w.qkv[row, :2 * 64].double().view(2, 64).numpy()
        y = r.q_out[row].astype(np.float64).reshape(2, 64)
        ms = (x ** 2).mean(axis=1)
        np.testing.assert_allclose(np.sqrt((y ** 2).mean(axis=1)),
                                   g * np.sqrt(ms / (ms + eps)), rtol=1e-6)


def test_rmsnorm_weight_offset_one_gamma_zero_is_plain_rmsnorm():
    w = _norm_problem(gamma_const=0.0, eps=1e-6, wo=1.0)
    r = H.oracle_ragged_store(w, "f32")
    x = w.qkv[0, :2 * 64].double().view(2, 64).numpy()
    y = r.q_out[0].astype(np.float64).reshape(2, 64)
    want = x / np.sqrt((x ** 2).mean(axis=1, keepdims=True) + float(np.float32(1e-6)))
    np.testing.assert_allclose(y, want, rtol=1e-6)


def weight_offset_problem(seed, head_dim=64, n_tokens=6):
    """A bf16 norm store whose every token sits at position 0 (one-token sequences, cache
    length 0) and whose Q and K head rows are exact_norm_rows, with gamma 0, epsilon 0 and
    weight_offset 0.3.  Returns the workload and the expected Q and K rows (bf16)."""
    w = W.ragged_store(seed, lengths=[1] * n_tokens, cache_lengths=[0] * n_tokens,
                       n_q_heads=2, n_kv_heads=1, head_dim=head_dim, page_size=8,
                       rope_dim=head_dim, theta=1e4, interleaved=False, max_seq_len=8,
                       norm=True, epsilon=0.0, weight_offset=0.3)
    Hq, Hk, D = 2, 1, head_dim
    rows = H.exact_norm_rows(seed, n_tokens * (Hq + Hk), D)
    w.qkv[:, :(Hq + Hk) * D] = rows.view(n_tokens, (Hq + Hk) * D).to(torch.bfloat16)
    w.q_gamma.zero_()
    w.k_gamma.zero_()
    want, unrounded = H.bf16_weight_offset_case(rows, w.weight_offset)
    assert not torch.equal(want, unrounded)  # the case tells the two readings apart
    want = want.view(n_tokens, Hq + Hk, D)
    return w, want[:, :Hq], want[:, Hq:]


@pytest.mark.parametrize("multiply_before_cast", [True, False])
def test_rmsnorm_weight_offset_is_a_scalar_of_the_element_type(multiply_before_cast):
    # fused_dual_qk_rms_norm_rope_ragged_paged, signature: weight_offset is a Scalar[dtype],
    # so 0.3 acts as bf16(0.3) = 154 * 2^-9.  gamma = 0 and epsilon = 0 on rows whose
    # normalised value is exactly x / 2 in {+-0.5, +-1.5}, at the identity rotation: every
    # output is (x / 2) * bf16(0.3), a bf16 number (1.5 * 154 * 2^-9 = 231 * 2^-9), where
    # the unrounded 1.5 * 0.3 = 0.45 rounds to 230 * 2^-9.  Both orders of the gamma
    # multiply give it, since x / 2 is exact in bf16.
    w, want_q, want_k = weight_offset_problem(71)
    assert w.total_tokens == 6
    r = H.oracle_ragged_store(w, "bf16", multiply_before_cast)
    assert r.err == 0
    Hq, D = w.n_q_heads, w.cache.head_dim
    H.assert_bits_equal(r.q_out.reshape(-1, Hq, D), H.bits(want_q), "Q rows")
    kv = w.cache
    view = torch.from_numpy(r.storage.view(np.int16)).view(torch.bfloat16)
    view = kv.view6(view)
    for row, (page, slot) in enumerate(W.token_slots(kv, [0] * w.total_tokens,
                                                     [1] * w.total_tokens)):
        H.assert_bits_equal(H.bits(view[page, 0, w.layer_idx, slot]), H.bits(want_k[row]),
                            f"K row of token {row}")


@pytest.mark.parametrize("interleaved", [True, False])
def test_rmsnorm_comes_before_rope(interleaved):
    # undoing the rotation of the output gives x * rsqrt(ms + eps) * gamma_d, column by
    # column, for a gamma that differs per column
    w = _norm_problem(eps=0.25, seed=61, interleaved=interleaved)
    r = H.oracle_ragged_store(w, "f32")
    w2 = W.ragged_store(61, lengths=[6, 2], cache_lengths=[0, 9], n_q_heads=2, n_kv_heads=1,
                        head_dim=64, page_size=8, rope_dim=64, theta=1e4,
                        interleaved=interleaved, max_seq_len=32, dtype="f32")
    w2.qkv[:, :2 * 64] = torch.from_numpy(r.q_out)
    w2.rope.table[:, 1::2] *= -1
    r2 = H.oracle_ragged_store(w2, "f32")
    x = w.qkv[:, :2 * 64].double().view(-1, 2, 64).numpy()
    gam = w.q_gamma.double().numpy()
    want = x / np.sqrt((x ** 2).mean(axis=2, keepdims=True) + 0.25) * gam
    np.testing.assert_allclose(r2.q_out.astype(np.float64).reshape(-1, 2, 64), want, rtol=0,
                               atol=2e-6 * np.abs(want).max())


# ------------------------------------------------------------- placement and untouched --

@pytest.mark.parametrize("cfg", ["tiny", "mid"])
def test_cache_reader_sees_every_token_once(cfg):
    if cfg == "tiny":
        w = W.tiny_ragged()
    else:
        w = W.ragged_store(71, lengths=[37, 1, 0, 64, 18], cache_lengths=[5, 0, 3, 120, 15],
                           n_q_heads=4, n_kv_heads=2, head_dim=64, page_size=16, rope_dim=64,
                           theta=1e4, interleaved=False, max_seq_len=256, width=16)
    r = H.oracle_ragged_store(w)
    assert r.err == 0
    kv = w.cache
    D, Hk = kv.head_dim, kv.n_kv_heads
    v_cols = slice((w.n_q_heads + Hk) * D, (w.n_q_heads + 2 * Hk) * D)
    qkv = H.bits(w.qkv)
    store = r.storage.reshape(kv.num_pages, 2, kv.num_layers, kv.page_size, Hk, D)
    pt = H.bits(kv.page_table)
    seen = 0
    offs = H.bits(w.offsets)
    for b in range(len(w.lengths)):
        for t in range(w.lengths[b]):
            pos = int(kv.cache_lengths[b]) + t
            page = pt[b, pos // kv.page_size]
            got_v = store[page, 1, w.layer_idx, pos % kv.page_size].reshape(-1)
            assert np.array_equal(got_v, qkv[offs[b] + t, v_cols])
            seen += 1
    assert seen == w.total_tokens == int(r.written.sum())
    # every row the op did not write, in every layer and plane, is untouched
    pristine = H.bits(kv.storage).reshape(store.shape)
    mask = H.paged_rows_mask(kv, r.written, w.layer_idx)
    assert np.array_equal(store[~mask], pristine[~mask])
    other = [l for l in range(kv.num_layers) if l != w.layer_idx]
    assert np.array_equal(store[:, :, other], pristine[:, :, other])


# ------------------------------------------------------------------------ BSHD decode --

def _within_half_ulp(y, z):
    # a value rounded once to nearest lies within half a bf16 spacing of the exact value
    return bool(np.all(np.abs(y - z) <= 0.5 * H.bf16_ulp(z) * (1 + 1e-9) + 1e-30))


def test_bshd_valid_lengths_and_in_place_k():
    w = W.bshd_decode(81, B=3, S=4, n_q_heads=2, n_kv_heads=2, head_dim=64,
                      cache_lengths=[0, 7, 20], valid_lengths=[4, 2, 0], max_seq_len=32,
                      rope_dim=64, theta=1e4, interleaved=True, freq_dtype="f32", num_slots=5,
                      num_layers=2, layer_idx=1, planes=2)
    r = H.oracle_bshd(w)
    assert r.err == 0
    q = H.bits(w.q_proj)
    out = r.output
    # beyond valid_lengths: copied unchanged
    assert np.array_equal(out[1, 2:], q[1, 2:])
    assert np.array_equal(out[2], q[2])
    # inside: the complex product with the row of position cache_len + s
    F = w.rope.table.double().numpy()
    for b, s in [(0, 0), (0, 3), (1, 1)]:
        pos = int(w.cache.cache_lengths[b]) + s
        x = H.values(q[b, s], "bf16")
        z = (x[..., 0::2] + 1j * x[..., 1::2]) * (F[pos, 0::2] + 1j * F[pos, 1::2])
        y = H.values(out[b, s], "bf16")
        assert _within_half_ulp(y[..., 0::2], z.real) and _within_half_ulp(y[..., 1::2], z.imag)
    # K rotated in place at (slot, layer 1, pos); everything else untouched
    kv = w.cache
    shp = (kv.num_slots, 2, kv.num_layers, kv.max_seq_len, kv.n_kv_heads, 64)
    before, after = H.bits(kv.storage).reshape(shp), r.storage.reshape(shp)
    touched = np.zeros(shp[:4], dtype=bool)
    for b in range(3):
        for s in range(int(w.valid_lengths[b])):
            slot, pos = int(kv.lookup_table[b]), int(kv.cache_lengths[b]) + s
            touched[slot, 0, 1, pos] = True
            x = H.values(before[slot, 0, 1, pos], "bf16")
            z = (x[..., 0::2] + 1j * x[..., 1::2]) * (F[pos, 0::2] + 1j * F[pos, 1::2])
            y = H.values(after[slot, 0, 1, pos], "bf16")
            assert _within_half_ulp(y[..., 0::2], z.real)
            assert _within_half_ulp(y[..., 1::2], z.imag)
    assert touched.sum() == int(r.written.sum()) == 6
    assert np.array_equal(after[~touched], before[~touched])


def test_bshd_matches_ragged_store_on_the_same_rows():
    # the Q rotation of the two ops agrees when positions and tables agree
    w = W.bshd_decode(82, B=2, S=3, n_q_heads=2, n_kv_heads=1, head_dim=64,
                      cache_lengths=[4, 9], valid_lengths=[3, 3], max_seq_len=16, rope_dim=64,
                      theta=1e4, interleaved=False, freq_dtype="f32")
    r = H.oracle_bshd(w)
    rs = W.ragged_store(83, lengths=[3, 3], cache_lengths=[4, 9], n_q_heads=2, n_kv_heads=1,
                        head_dim=64, page_size=8, rope_dim=64, theta=1e4, interleaved=False,
                        max_seq_len=16)
    rs.qkv[:, :128] = w.q_proj.reshape(6, 128)
    rr = H.oracle_ragged_store(rs)
    assert np.array_equal(rr.q_out, r.output.reshape(6, 128))


# ------------------------------------------------------------------------------ radd --

@pytest.mark.parametrize("batch_offset", [0, 2])
def test_radd_is_the_rounded_sum(batch_offset):
    w = W.radd(91, lengths=[5, 0, 12], cache_lengths=[3, 8, 30], n_kv_heads=2, head_dim=64,
               page_size=16, batch_offset=batch_offset, max_seq_len=128)
    r = H.oracle_radd(w)
    assert r.err == 0
    kv = w.cache
    before = kv.view6().clone()
    after = kv.view6(torch.from_numpy(r.storage.view(np.int16)).view(torch.bfloat16))
    pt = kv.page_table
    offs = w.offsets.tolist()
    hidden = 2 * 64
    mask = torch.zeros(kv.num_pages, 2, kv.num_layers, kv.page_size, dtype=torch.bool)
    for b, n in enumerate(w.lengths):
        seq = b + batch_offset
        for t in range(n):
            pos = int(kv.cache_lengths[seq]) + t
            page, slot = int(pt[seq, pos // 16]), pos % 16
            a = w.a[offs[b] + t]
            for plane, half in ((0, a[:hidden]), (1, a[hidden:])):
                # float32 sum of two bf16 numbers, rounded to bf16 by torch (RNE)
                want = (before[page, plane, 1, slot].float() + half.view(2, 64).float()).to(
                    torch.bfloat16)
                assert torch.equal(after[page, plane, 1, slot].view(torch.int16),
                                   want.view(torch.int16))
            mask[page, :, 1, slot] = True
    assert torch.equal(after[~mask].view(torch.int16), before[~mask].view(torch.int16))


# ---------------------------------------------------------------------------- errors --

def test_out_of_range_rows_are_skipped_with_their_bits():
    w = W.ragged_store(101, lengths=[3, 4], cache_lengths=[0, 14], n_q_heads=2, n_kv_heads=1,
                       head_dim=64, page_size=8, rope_dim=64, theta=1e4, interleaved=True,
                       max_seq_len=16, width=2)
    r = H.oracle_ragged_store(w)
    # seq 1 positions 14..17: 16 and 17 are past the 16-row table
    assert r.err == oracle.ERR_POSITION
    q0 = H.bits(w.q_out)
    assert np.array_equal(r.q_out[5:], q0[5:]) and not np.array_equal(r.q_out[3], q0[3])
    assert int(r.written.sum()) == 5
    # a page-table entry past num_pages
    w.cache.page_table[1, 1] = w.cache.num_pages
    r = H.oracle_ragged_store(W.RaggedStore(**{**w.__dict__}))
    assert r.err & oracle.ERR_PAGE_ID
    # offsets that do not partition [0, T): nothing is written
    w.offsets[1] = 9
    r = H.oracle_ragged_store(w)
    assert r.err == oracle.ERR_ROW_OFFSETS
    assert int(r.written.sum()) == 0 and np.array_equal(r.q_out, q0)


def test_page_index_beyond_table_width():
    w = W.ragged_store(102, lengths=[10], cache_lengths=[12], n_q_heads=1, n_kv_heads=1,
                       head_dim=64, page_size=8, rope_dim=64, theta=1e4, interleaved=True,
                       max_seq_len=64, width=2)
    r = H.oracle_ragged_store(w)
    assert r.err == oracle.ERR_PAGE_INDEX     # positions 16..21 are past 2 pages of 8
    assert int(r.written.sum()) == 16 - 12


def test_radd_batch_offset_past_the_cache():
    w = W.radd(103, lengths=[2, 3], cache_lengths=[0, 0], n_kv_heads=1, head_dim=64,
               page_size=8, batch_offset=1, max_seq_len=64)
    w.batch_offset = 2          # sequence 1 + 2 = 3 is past the 3 sequences of the cache
    r = H.oracle_radd(w)
    assert r.err == oracle.ERR_BATCH and int(r.written.sum()) == 2


# -------------------------------------------------------------------------- dual band --

def test_dual_band_is_two_single_band_ops():
    w = W.dual_band(111, lengths=[7, 0, 12], cache_lengths=[3, 0, 60], main_q_heads=4,
                    main_kv_heads=2, index_q_heads=2, index_kv_heads=1, head_dim=64,
                    main_page_size=16, index_page_size=8, rope_dim=32, theta=1e4,
                    interleaved=True, max_seq_len=128, main_eps=1e-6, index_eps=1e-5,
                    weight_offset=1.0)
    r = H.oracle_dual(w)
    assert r.err == 0
    for which in ("main", "index"):
        cache = getattr(w, f"{which}_cache")
        cols = getattr(w, f"{which}_cols")
        g = w.gammas[:2] if which == "main" else w.gammas[2:]
        nq = getattr(w, f"{which}_q_heads")
        single = W.RaggedStore(w.input, w.offsets, nq, cache, w.rope, w.layer_idx,
                               getattr(w, f"q_{which}_out"), w.lengths, g[0], g[1],
                               getattr(w, f"{which}_eps"), w.weight_offset)
        store = H.bits(cache.storage)
        q_out = H.bits(single.q_out)
        written = np.zeros(cache.num_pages * cache.page_size, dtype=np.uint8)
        band = oracle.Band(H.bits(w.input), *cols, nq, H.oracle_paged(cache, store),
                           H.bits(g[0]), H.bits(g[1]), single.epsilon, q_out, written)
        e = oracle.fused_qk_rmsnorm_rope_paged(band, H.bits(w.offsets), H.oracle_rope(w.rope),
                                               w.weight_offset, True, w.layer_idx)
        assert e == 0
        assert np.array_equal(q_out, r[f"q_{which}_out"])
        assert np.array_equal(store, r[f"{which}_storage"])
        assert np.array_equal(written, r[f"{which}_written"])


def test_dual_band_geometry_mismatch_is_an_argument_error():
    w = W.dual_band(112, lengths=[3], cache_lengths=[0], main_q_heads=2, main_kv_heads=1,
                    index_q_heads=1, index_kv_heads=1, head_dim=64, main_page_size=8,
                    index_page_size=8, rope_dim=64, theta=1e4, interleaved=True,
                    max_seq_len=16)
    w.index_cache.head_dim = 32
    assert H.oracle_dual(w).err == oracle.ERR_ARGS
    w.index_cache.head_dim = 64
    w.index_cache.dtype = "f16"  # neither the input's type nor FP8 codes
    assert H.oracle_dual(w).err == oracle.ERR_ARGS


# ------------------------------------------------------------------- K updated in place --

@pytest.mark.parametrize("single", [False, True])
def test_k_in_place_on_a_cache_holding_the_inputs_k_is_the_store(single):
    """fused_dual_qk_rms_norm_rope_ragged_paged (first paragraph): the key caches are
    updated in place.  When the cache slots already hold the input's K and V rows (as the
    projection would have stored them), normalising and rotating K where it lies must give
    exactly what the store mode gives from the input: same Q outputs, same caches, every
    other byte untouched."""
    import copy
    w = W.dual_band(113, lengths=[7, 12, 1], cache_lengths=[3, 40, 0], main_q_heads=4,
                    main_kv_heads=2, index_q_heads=2, index_kv_heads=1, head_dim=64,
                    main_page_size=16, index_page_size=8, rope_dim=32, theta=1e4,
                    interleaved=False, max_seq_len=128, weight_offset=1.0, single=single)
    store = H.oracle_dual(w)
    assert store.err == 0
    wi = copy.deepcopy(w)
    D = w.main_cache.head_dim
    for kv, cols in ((wi.main_cache, w.main_cols), (wi.index_cache, w.index_cols)):
        if kv is None:
            continue
        Hk = kv.n_kv_heads
        v6 = kv.view6()
        for row, (page, slot) in enumerate(W.token_slots(kv, w.cache_lengths_of(kv),
                                                          w.lengths)):
            v6[page, 0, w.layer_idx, slot] = w.input[row, cols[1]:cols[1] + Hk * D].view(Hk, D)
            if cols[2] >= 0:
                v6[page, 1, w.layer_idx, slot] = \
                    w.input[row, cols[2]:cols[2] + Hk * D].view(Hk, D)
    wi.main_cols = (w.main_cols[0], -1, -1)
    wi.index_cols = (w.index_cols[0], -1, -1)
    inplace = H.oracle_dual(wi)
    assert inplace.err == 0
    for key in store:
        if key != "err":
            assert np.array_equal(inplace[key], store[key]), key


def test_multiply_after_cast_with_unit_gamma_is_multiply_before_cast():
    """multiply_before_cast has no definition on the pages (parity unpinned); the reading
    taken (normalised value rounded to the element type, then scaled by gamma) must still
    reduce to the plain op when gamma + weight_offset == 1 at position 0, where both orders
    round the same normalised value once."""
    w = W.ragged_store(114, lengths=[5], cache_lengths=[0], n_q_heads=2, n_kv_heads=1,
                       head_dim=64, page_size=8, rope_dim=64, theta=1e4, interleaved=True,
                       max_seq_len=8, norm=True, weight_offset=1.0, x_std=3.0)
    w.q_gamma.zero_()
    w.k_gamma.zero_()
    w.cache.cache_lengths.zero_()
    a = H.oracle_ragged_store(w, "bf16", True)
    b = H.oracle_ragged_store(w, "bf16", False)
    # row 0 sits at position 0: identity rotation; later rows rotate a rounded value
    Hq, D = w.n_q_heads, w.cache.head_dim
    assert np.array_equal(a.q_out.reshape(5, Hq * D)[0], b.q_out.reshape(5, Hq * D)[0])


def _half(v):
    """v rounded once to IEEE half (Python's own float packing: nearest, ties to even)."""
    import struct
    return np.array([struct.unpack("<e", struct.pack("<e", float(x)))[0] for x in v])


def test_multiply_after_cast_rounds_the_normalised_value_before_gamma():
    """The reading of multiply_before_cast = 0 (parity unpinned: the pages name the flag
    only), checked against single roundings done by Python's half-precision packing at
    position 0, where the rotation is the identity: flag 1 gives half(n * g) and flag 0
    gives half(half(n) * g), with n = x / sqrt(mean(x^2) + eps) in double and
    g = gamma + weight_offset (both in the element type).  Some elements must differ, so the
    two orders are told apart."""
    w = W.ragged_store(115, lengths=[3], cache_lengths=[0], n_q_heads=4, n_kv_heads=1,
                       head_dim=64, page_size=8, rope_dim=64, theta=1e4, interleaved=False,
                       max_seq_len=8, norm=True, weight_offset=0.5, x_std=3.0, dtype="f16")
    a = H.oracle_ragged_store(w, "f16", True)
    b = H.oracle_ragged_store(w, "f16", False)
    assert a.err == b.err == 0
    Hq, D = w.n_q_heads, w.cache.head_dim
    x = w.qkv[0, :Hq * D].double().numpy().reshape(Hq, D)
    n = x / np.sqrt((x * x).mean(axis=1, keepdims=True) + w.epsilon)
    g = w.q_gamma.double().numpy() + _half([w.weight_offset])[0]
    before = _half((n * g).reshape(-1))
    after = _half((_half(n.reshape(-1)).reshape(Hq, D) * g).reshape(-1))
    got_a = H.values(a.q_out.reshape(3, Hq * D)[0], "f16")
    got_b = H.values(b.q_out.reshape(3, Hq * D)[0], "f16")
    assert np.array_equal(got_a, before)
    assert np.array_equal(got_b, after)
    assert np.any(before != after)


# ------------------------------------------------ GEMV + partial RMSNorm (P5) ----------

def _gemv(n, k, n_normed, dtype="f32", seed=120, **kw):
    return W.gemv_norm(seed, n=n, k=k, n_normed=n_normed, dtype=dtype, **kw)


def _vals(a, dtype):
    return H.values(a, dtype)


def test_gemv_pass_through_is_the_rounded_matmul():
    # MatmulFusedPartialRMSNorm: the columns after n_normed are y = x W^T unchanged; numpy's
    # float64 matmul of the decoded inputs is the exact product up to its summation order
    w = _gemv(37, 300, 5, dtype="bf16", row_pad=8)
    r = H.oracle_gemv(w, "bf16")
    assert r.err == 0
    x = w.x.double().numpy()
    y = w.weight.double().numpy() @ x
    assert _within_half_ulp(_vals(r.unnormed, "bf16"), y[5:])


def test_gemv_normed_rms_closed_form():
    # with gamma = g constant: rms(normed) = |g| sqrt(ms / (ms + eps)) over the normed part
    eps, g = 0.25, 1.5
    w = _gemv(24, 96, 16, epsilon=eps)
    w.gamma.fill_(g)
    r = H.oracle_gemv(w, "f32")
    y = w.weight.double().numpy() @ w.x.double().numpy()
    ms = (y[:16] ** 2).mean()
    got = r.normed.astype(np.float64)
    np.testing.assert_allclose(np.sqrt((got ** 2).mean()), g * np.sqrt(ms / (ms + eps)),
                               rtol=1e-6)
    # the direction of the normed part is y's
    np.testing.assert_allclose(got / np.linalg.norm(got), y[:16] / np.linalg.norm(y[:16]),
                               rtol=1e-5, atol=1e-7)


def test_gemv_scale_invariance_and_gamma():
    # eps = 0: scaling x by 2 (exact) leaves the normed part unchanged bit for bit and doubles
    # the pass-through part; gamma scales the normed part elementwise
    w = _gemv(20, 64, 12, dtype="bf16", epsilon=0.0)
    a = H.oracle_gemv(w, "bf16")
    w2 = W.GemvNorm(w.x * 2, w.weight, w.gamma, 0.0, 0.0, w.normed_output,
                    w.unnormed_output)
    b = H.oracle_gemv(w2, "bf16")
    assert np.array_equal(a.normed, b.normed)
    np.testing.assert_array_equal(_vals(b.unnormed, "bf16"), 2 * _vals(a.unnormed, "bf16"))
    w3 = W.GemvNorm(w.x, w.weight, w.gamma * 4, 0.0, 0.0, w.normed_output, w.unnormed_output)
    c = H.oracle_gemv(w3, "bf16")
    np.testing.assert_array_equal(_vals(c.normed, "bf16"), 4 * _vals(a.normed, "bf16"))


def test_gemv_weight_offset_is_not_consumed_and_partitions_agree():
    w = _gemv(30, 128, 10, dtype="bf16")
    a = H.oracle_gemv(w, "bf16")
    w.weight_offset = 3.0
    b = H.oracle_gemv(w, "bf16")
    assert np.array_equal(a.normed, b.normed) and np.array_equal(a.unnormed, b.unnormed)
    # no normed columns: every column passes through; the 20 trailing ones are a's
    w0 = W.GemvNorm(w.x, w.weight, w.gamma[:0], w.epsilon, 0.0, w.normed_output[:0],
                    W.random_bits(W.generator(1), 30, "bf16"))
    z = H.oracle_gemv(w0, "bf16")
    assert np.array_equal(z.unnormed[10:], a.unnormed)


# ------------------------------------------------------- Q output in another element type --

def test_q_out_f32_at_position_zero_is_the_input_widened():
    # rope_split_store_paged_ragged, Parameters: q_out_dtype.  At position 0 the rotation is
    # the identity, so a float32 q_out holds the bf16 input exactly
    w = W.ragged_store(130, lengths=[1, 1, 1], cache_lengths=[0, 0, 0], n_q_heads=4,
                       n_kv_heads=2, head_dim=64, page_size=8, rope_dim=64, theta=1e4,
                       interleaved=True, max_seq_len=16, q_out_dtype="f32")
    r = H.oracle_ragged_store(w, "bf16")
    assert r.err == 0
    want = w.qkv[:, :4 * 64].float().numpy()
    np.testing.assert_array_equal(r.q_out.view(np.float32), want)


@pytest.mark.parametrize("q_dtype", ["f32", "f16"])
def test_q_out_in_another_type_is_the_same_value_rounded_once(q_dtype):
    # the same rotated value rounded once into each type: the bf16 output lies within half a
    # bf16 spacing of the wider one, and the f32 output is the complex product of the pages'
    # interleaved layout, rounded once
    kw = dict(lengths=[5, 9], cache_lengths=[3, 40], n_q_heads=2, n_kv_heads=1, head_dim=64,
              page_size=16, rope_dim=64, theta=1e4, interleaved=True, max_seq_len=64)
    a = H.oracle_ragged_store(W.ragged_store(131, **kw), "bf16")
    wq = W.ragged_store(131, q_out_dtype=q_dtype, **kw)
    b = H.oracle_ragged_store(wq, "bf16")
    assert a.err == b.err == 0
    qa = H.values(a.q_out, "bf16")
    qb = H.values(b.q_out, q_dtype)
    assert bool(np.all(np.abs(qa - qb) <= 0.5 * H.bf16_ulp(qa) + 0.5 * H.ulp_of(qb, q_dtype)))
    assert np.array_equal(a.storage, b.storage)
    if q_dtype == "f32":
        T = wq.total_tokens
        x = wq.qkv[:, :2 * 64].double().numpy().reshape(T, 2, 32, 2)
        z = x[..., 0] + 1j * x[..., 1]
        pos = np.concatenate([np.arange(3, 8), np.arange(40, 49)])
        f = wq.rope.table.double().numpy()[pos].reshape(T, 1, 32, 2)
        y = z * (f[..., 0] + 1j * f[..., 1])
        got = qb.reshape(T, 2, 32, 2)
        sp = np.spacing(np.abs(np.stack([y.real, y.imag], -1)).astype(np.float32))
        assert bool(np.all(np.abs(got - np.stack([y.real, y.imag], -1)) <= 0.5 * sp * (1 + 1e-9)))


# ------------------------------------------------------------------ FP8 (E4M3) caches --

def _e4m3_roundtrip(vals):
    """The oracle's codec on float64 values, through a one-column fp8 'cache' of the ragged
    store's V plane would be indirect; the codec is exported instead."""
    buf = np.zeros(len(vals), dtype=np.uint8)
    lib = oracle._load()
    for i, v in enumerate(vals):
        lib.orc_encode(3, buf.ctypes.data, i, float(v))
    back = np.array([lib.orc_decode(3, buf.ctypes.data, i) for i in range(len(vals))])
    return buf, back


def test_e4m3_codec_matches_torch():
    # every code decodes as torch's float8_e4m3fn does; float32 values inside the finite
    # range encode as torch rounds them (nearest, ties to even); beyond 448 the reading
    # saturates (torch's plain cast does not, so those are checked against 448 directly)
    codes = np.arange(256, dtype=np.uint8)
    lib = oracle._load()
    dec = np.array([lib.orc_decode(3, codes.ctypes.data, i) for i in range(256)])
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().double().numpy()
    assert np.array_equal(np.isnan(dec), np.isnan(ref))
    assert np.array_equal(dec[~np.isnan(dec)], ref[~np.isnan(ref)])
    g = torch.Generator().manual_seed(7)
    x = (torch.randn(4000, generator=g) * torch.exp2(torch.randint(-12, 9, (4000,),
                                                                   generator=g).float()))
    x = x[x.abs() < 448].float()
    # exact midpoints between neighbouring codes, where ties to even decides
    mids = torch.tensor([(a + b) / 2 for a, b in zip(ref[1:120:7], ref[2:121:7])],
                        dtype=torch.float32)
    x = torch.cat([x, mids, -mids])
    got, _ = _e4m3_roundtrip(x.double().numpy())
    want = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want)
    sat, back = _e4m3_roundtrip([448.0, 460.0, 1e6, float("inf"), -1e6])
    assert np.array_equal(back, [448.0, 448.0, 448.0, 448.0, -448.0])


def test_fp8_store_holds_the_scaled_value_rounded_once():
    # an FP8 cache stores e4m3(value / scale) per plane (the reading of the pages' scale_dtype_
    # and quantization_granularity_: one float32 scale per K / V plane).  V is copied, so its
    # code is torch's cast of the input divided by an exact power-of-two scale; K is rotated,
    # so its dequantised value lies within half an e4m3 spacing (plus half a bf16 one) of the
    # bf16 store's K
    kw = dict(lengths=[6, 11], cache_lengths=[2, 30], n_q_heads=2, n_kv_heads=2, head_dim=64,
              page_size=16, rope_dim=64, theta=1e4, interleaved=False, max_seq_len=64)
    sk, sv = 0.5, 0.0625
    w8 = W.ragged_store(140, cache_dtype="fp8", kv_scales=(sk, sv), **kw)
    wb = W.ragged_store(140, **kw)
    r8, rb = H.oracle_ragged_store(w8), H.oracle_ragged_store(wb)
    assert r8.err == rb.err == 0
    assert np.array_equal(r8.q_out, rb.q_out) and np.array_equal(r8.written, rb.written)
    kv8, kvb = w8.cache, wb.cache
    shp = (kv8.num_pages, 2, kv8.num_layers, kv8.page_size, 2, 64)
    rows = H.paged_rows_mask(kv8, r8.written, w8.layer_idx)
    c8, cb = r8.storage.reshape(shp), rb.storage.reshape(shp)
    # V plane, written rows: code == torch cast of (input V / sv)
    T = w8.total_tokens
    v_in = w8.qkv[:, 4 * 64:6 * 64].float().reshape(T, 2, 64)
    slots = W.token_slots(kv8, [2, 30], [6, 11])
    for t, (pg, sl) in enumerate(slots):
        want = (v_in[t] / sv).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(c8[pg, 1, w8.layer_idx, sl], want)
    # K plane, written rows: dequantised value close to the bf16 store's
    kq = torch.from_numpy(c8[:, 0][rows[:, 0]].copy()).view(torch.float8_e4m3fn).double()
    kq = kq.numpy() * sk
    kbf = H.values(cb[:, 0][rows[:, 0]], "bf16")
    e4_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(kbf) / sk, 2.0 ** -6))) - 3) * sk
    assert bool(np.all(np.abs(kq - kbf) <= 0.5 * e4_ulp + 0.5 * H.bf16_ulp(kbf) + 1e-12))
    # bytes outside the written rows are untouched
    before = H.bits(kv8.storage).reshape(shp)
    assert np.array_equal(c8[~rows], before[~rows])
