"""The bounded waits: a wait that runs out ends the call with ROPE_DEVERR_TIMEOUT set
instead of hanging, and the context stays usable.

rope_set_stall_test(100) makes every staged kernel start with a wait on a barrier that no
thread ever arrives at (a flag that nothing sets), bounded by 100 us: it runs out, and the
kernel takes the path any wait that runs out takes.  The waits that let a CTA's in-flight
copies land before it exits keep their full limit, so every CTA leaves with its copies done.
Each case checks the timeout bit, that the scheduling workspace (or the GEMV's count) is
back at zero, and then runs the same call with the test off and compares it with the oracle.
No kernel traps or is stopped from outside: the failure is a wait that gives up.
"""
import pytest
import torch

import workloads as W
import helpers as H
from test_gpu_parity import _check_dual, _check_radd, check_ragged

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gpu_helpers
    return gpu_helpers


def _ragged(norm, fp8=False):
    return W.ragged_store(81, lengths=[900, 3, 1100], cache_lengths=[0, 5, 64], n_q_heads=16,
                          n_kv_heads=4, head_dim=128, page_size=64, rope_dim=128, theta=1e4,
                          interleaved=False, max_seq_len=2048, norm=norm,
                          cache_dtype="fp8" if fp8 else None, kv_scales=(0.5, 0.25))


def _short_waits(run):
    """run() with the stall test on (a 100 us wait nothing completes); returns what run()
    returns."""
    import rope_paged_kv_b200 as rs
    assert rs.get_stall_test() == 0
    rs.set_stall_test(100)
    try:
        out = run()
        torch.cuda.synchronize()  # the call returns: nothing hangs
    finally:
        rs.set_stall_test(0)
    return out


@pytest.mark.parametrize("case", ["store", "norm", "fp8"])
def test_timeout_of_the_ragged_stores(G, case):
    import rope_paged_kv_b200 as rs
    w = _ragged(norm=case == "norm", fp8=case == "fp8")
    s = _short_waits(lambda: G.run_ragged(w))
    assert int(s.err.item()) & rs.DEVERR_TIMEOUT
    assert not s.sched.any().item()
    if case != "fp8":
        check_ragged(G, w, G.run_ragged(w))
    else:
        s2 = G.run_ragged(w)
        assert int(s2.err.item()) == 0


def test_timeout_of_the_dual_band(G):
    import rope_paged_kv_b200 as rs
    w = W.dual_band(82, lengths=[700, 1, 400], cache_lengths=[0, 40, 7], main_q_heads=8,
                    main_kv_heads=2, index_q_heads=2, index_kv_heads=1, head_dim=128,
                    main_page_size=64, index_page_size=32, rope_dim=64, theta=1e4,
                    interleaved=True, max_seq_len=1024)
    s = _short_waits(lambda: G.run_dual(w))
    assert int(s.err.item()) & rs.DEVERR_TIMEOUT
    assert not s.sched.any().item()
    _check_dual(G, w, G.run_dual(w))


def test_timeout_of_radd(G):
    import rope_paged_kv_b200 as rs
    w = W.radd(83, lengths=[800, 0, 1200], cache_lengths=[3, 8, 30], n_kv_heads=4,
               head_dim=128, page_size=64, batch_offset=0, max_seq_len=4096)
    s = _short_waits(lambda: G.run_radd(w))
    assert int(s.err.item()) & rs.DEVERR_TIMEOUT
    assert not s.sched.any().item()
    _check_radd(G, w, G.run_radd(w))


def test_timeout_of_the_gemv(G):
    import rope_paged_kv_b200 as rs
    w = W.gemv_norm(84, n=576, k=7168, n_normed=512)
    dev = G.DEV
    ws = rs.gemv_workspace(w.n_normed, dev)
    err = G.err_word()
    x, wt, g = (G.to_dev(t) for t in (w.x, w.weight, w.gamma))
    no, uo = G.to_dev(w.normed_output), G.to_dev(w.unnormed_output)
    _short_waits(lambda: rs.matmul_fused_partial_rmsnorm(x, wt, g, w.epsilon, w.weight_offset,
                                                         no, uo, ws, err_word=err))
    assert int(err.item()) & rs.DEVERR_TIMEOUT
    assert int(ws[0].item()) == 0
    err.zero_()
    rs.matmul_fused_partial_rmsnorm(x, wt, g, w.epsilon, w.weight_offset, no, uo, ws,
                                    err_word=err)
    torch.cuda.synchronize()
    r = H.oracle_gemv(w)
    assert int(err.item()) == r.err == 0
    H.assert_close_bf16(H.bits(no), r.normed, "normed")
    H.assert_close_bf16(H.bits(uo), r.unnormed, "unnormed")
