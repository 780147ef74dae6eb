"""matmul_fused_partial_rmsnorm on the GPU vs the oracle, through the C ABI binding.

Outputs within max(1 ulp of the element type at the oracle value, 1e-3): y is accumulated in
float32 over k products (relative error ~ sqrt(k) * 2^-24, far below a bf16 ulp), then
normalised and rounded once.  The workspace must be back at zero after every call.
"""
import numpy as np
import pytest
import torch

import workloads as W
import helpers as H

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def rs():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import rope_paged_kv_b200 as rs
    return rs


def run(rs, w, ws=None):
    d = {f: getattr(w, f).to(DEV) for f in ("x", "gamma", "normed_output", "unnormed_output")}
    if w.weight.is_contiguous():
        weight = w.weight.to(DEV)
    else:  # keep the padded row stride
        base = torch.empty(w.weight.shape[0], w.weight.stride(0), dtype=w.weight.dtype,
                           device=DEV)
        base[:, :w.k] = w.weight.to(DEV)
        weight = base[:, :w.k]
    ws = rs.gemv_workspace(w.n_normed, DEV) if ws is None else ws
    rs.matmul_fused_partial_rmsnorm(d["x"], weight, d["gamma"], w.epsilon, w.weight_offset,
                                    d["normed_output"], d["unnormed_output"], ws)
    torch.cuda.synchronize()
    return d, ws


def check(rs, w, dtype="bf16"):
    d, ws = run(rs, w)
    r = H.oracle_gemv(w, dtype)
    assert r.err == 0
    H.assert_close_bf16(H.bits(d["normed_output"]), r.normed, "normed", dtype=dtype)
    H.assert_close_bf16(H.bits(d["unnormed_output"]), r.unnormed, "unnormed", dtype=dtype)
    assert int(ws[0].item()) == 0, "workspace count not returned to zero"
    return d


def test_mla_kv_a_proj_full_size(rs):
    check(rs, W.mla_kv_a_proj())


@pytest.mark.parametrize("n,k,n_normed", [
    (1, 8, 1), (1, 8, 0), (3, 64, 2), (64, 64, 64), (64, 64, 0), (577, 7168, 512),
    (2000, 256, 1500), (150, 1032, 100)])
def test_shapes(rs, n, k, n_normed):
    check(rs, W.gemv_norm(60 + n, n=n, k=k, n_normed=n_normed))


@pytest.mark.parametrize("dtype,k", [("f16", 520), ("f32", 300)])
def test_other_element_types(rs, dtype, k):
    check(rs, W.gemv_norm(70, n=200, k=k, n_normed=150, dtype=dtype), dtype)


def test_padded_rows_and_weight_offset_ignored(rs):
    w = W.gemv_norm(71, n=96, k=512, n_normed=64, row_pad=24, weight_offset=5.0)
    check(rs, w)


def test_two_calls_in_a_row_share_a_workspace(rs):
    w1, w2 = W.gemv_norm(72, n=576, k=1024, n_normed=512), W.gemv_norm(73, n=576, k=1024,
                                                                        n_normed=512)
    ws = rs.gemv_workspace(512, DEV)
    outs = []
    for w in (w1, w2):  # queued without a sync in between
        d = {f: getattr(w, f).to(DEV) for f in ("x", "gamma", "normed_output",
                                                "unnormed_output")}
        rs.matmul_fused_partial_rmsnorm(d["x"], w.weight.to(DEV), d["gamma"], w.epsilon, 0.0,
                                        d["normed_output"], d["unnormed_output"], ws)
        outs.append(d)
    torch.cuda.synchronize()
    assert int(ws[0].item()) == 0
    for w, d in zip((w1, w2), outs):
        r = H.oracle_gemv(w)
        H.assert_close_bf16(H.bits(d["normed_output"]), r.normed, "normed")
        H.assert_close_bf16(H.bits(d["unnormed_output"]), r.unnormed, "unnormed")


def test_chained_calls_under_early_overlap(rs):
    """Launch-overlap mode 2 (programmatic dependent launch): the second call's x is the
    first call's output, queued without a sync in between, so a read of x before the wait
    for the preceding kernel would see the sentinel bits."""
    import dataclasses
    w1 = W.gemv_norm(74, n=1024, k=512, n_normed=0)
    w2 = W.gemv_norm(75, n=576, k=1024, n_normed=512)
    d1 = {f: getattr(w1, f).to(DEV) for f in ("x", "weight", "gamma", "normed_output",
                                              "unnormed_output")}
    d2 = {f: getattr(w2, f).to(DEV) for f in ("weight", "gamma", "normed_output",
                                              "unnormed_output")}
    ws1, ws2 = rs.gemv_workspace(0, DEV), rs.gemv_workspace(512, DEV)
    before = rs.get_launch_overlap()
    rs.set_launch_overlap(2)
    try:
        for _ in range(3):  # the later rounds run behind the earlier ones' kernels
            rs.matmul_fused_partial_rmsnorm(d1["x"], d1["weight"], d1["gamma"], w1.epsilon, 0.0,
                                            d1["normed_output"], d1["unnormed_output"], ws1)
            rs.matmul_fused_partial_rmsnorm(d1["unnormed_output"], d2["weight"], d2["gamma"],
                                            w2.epsilon, 0.0, d2["normed_output"],
                                            d2["unnormed_output"], ws2)
        torch.cuda.synchronize()
    finally:
        rs.set_launch_overlap(before)
    r1 = H.oracle_gemv(w1)
    H.assert_close_bf16(H.bits(d1["unnormed_output"]), r1.unnormed, "first call")
    y1 = d1["unnormed_output"].cpu()
    r2 = H.oracle_gemv(dataclasses.replace(w2, x=y1))
    H.assert_close_bf16(H.bits(d2["normed_output"]), r2.normed, "normed")
    H.assert_close_bf16(H.bits(d2["unnormed_output"]), r2.unnormed, "unnormed")
    assert int(ws2[0].item()) == 0


def test_argument_errors(rs):
    lib = rs.raw_library()
    x = torch.zeros(64, dtype=torch.bfloat16, device=DEV)
    wt = torch.zeros(8, 64, dtype=torch.bfloat16, device=DEV)
    out = torch.zeros(8, dtype=torch.bfloat16, device=DEV)
    ws = rs.gemv_workspace(8, DEV)
    call = lib.matmul_fused_partial_rmsnorm
    ok = (x.data_ptr(), wt.data_ptr(), 64, 8, 64, 1, out.data_ptr(), 1e-6, 0.0, out.data_ptr(),
          8, None, 0, None, ws.data_ptr(), ws.numel() * 4, None)
    assert call(*ok) == rs.OK
    bad = list(ok); bad[5] = 0                # weight stored [k, n]
    assert call(*bad) == rs.ERR_UNSUPPORTED
    bad = list(ok); bad[10] = 9               # n_normed > n
    assert call(*bad) == rs.ERR_INVALID_ARG
    bad = list(ok); bad[15] = 16              # workspace too small
    assert call(*bad) == rs.ERR_INVALID_ARG
    bad = list(ok); bad[4] = 60; bad[2] = 64  # k * 2 bytes not a multiple of 16
    assert call(*bad) == rs.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(ws[0].item()) == 0
