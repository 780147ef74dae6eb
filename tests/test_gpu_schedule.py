"""The token schedule and the launch-overlap mode change no result.

Every staged entry point gives bit-identical outputs with and without a scheduling
workspace and in every overlap mode (each output element is computed by the same code
whichever CTA takes its token), and the workspace is back to zero after every call.  Calls
queued back to back on one stream, where a launch may start while its predecessor
finishes, still see each other's writes: a store followed by two radd calls on the rows it
wrote equals the same calls run one at a time.  The baseline of these comparisons (plain
launch, static schedule) is checked against the oracle in test_gpu_parity.py; here one
small case per entry point is checked against the oracle as well.
"""
import numpy as np
import pytest
import torch

import workloads as W
import helpers as H

pytestmark = pytest.mark.gpu

MODES = (0, 1, 2)  # off, programmatic dependent launch, the same with early descriptor reads


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gpu_helpers
    return gpu_helpers


@pytest.fixture
def rs():
    import rope_paged_kv_b200 as rs
    before = rs.get_launch_overlap()
    yield rs
    rs.set_launch_overlap(before)


# about 6k tokens: at the light shape's 444 CTAs (and the heavy shape's 296) each CTA has a
# static share of several tokens and the rest is claimed, and a 1-token sequence sits
# between long ones
LENGTHS = [1500, 37, 2900, 1, 1700]
CACHE_LENGTHS = [0, 5, 100, 0, 64]


def ragged(norm):
    return W.ragged_store(11, lengths=LENGTHS, cache_lengths=CACHE_LENGTHS, n_q_heads=8,
                          n_kv_heads=2, head_dim=128, page_size=64, rope_dim=128, theta=5e5,
                          interleaved=False, max_seq_len=4096, norm=norm)


def dual():
    return W.dual_band(12, lengths=LENGTHS, cache_lengths=CACHE_LENGTHS, main_q_heads=8,
                       main_kv_heads=2, index_q_heads=2, index_kv_heads=1, head_dim=128,
                       main_page_size=64, index_page_size=32, rope_dim=64, theta=1e4,
                       interleaved=True, max_seq_len=4096)


def radd():
    return W.radd(13, lengths=LENGTHS, cache_lengths=CACHE_LENGTHS, n_kv_heads=2,
                  head_dim=128, page_size=64, batch_offset=1, max_seq_len=4096)


def run(G, kind, w, use_sched):
    """Stage w, run its entry point once, return the output tensors (on the host) and the
    workspace (None without one)."""
    G.USE_SCHED = use_sched
    try:
        if kind in ("store", "norm"):
            s = G.run_ragged(w)
            outs = [s.q_out, s.storage]
        elif kind == "dual":
            s = G.run_dual(w)
            outs = [s.q_main_out, s.q_index_out, s.main_storage, s.index_storage]
        else:
            s = G.run_radd(w)
            outs = [s.storage]
    finally:
        G.USE_SCHED = True
    assert int(s.err.item()) == 0
    return [H.bits(o) for o in outs], getattr(s, "sched", None) if use_sched else None


CASES = {"store": lambda: ragged(False), "norm": lambda: ragged(True), "dual": dual,
         "radd": radd}


@pytest.mark.parametrize("kind", list(CASES))
def test_schedule_and_overlap_do_not_change_results(G, rs, kind):
    w = CASES[kind]()
    rs.set_launch_overlap(0)
    want, _ = run(G, kind, w, use_sched=False)
    for mode in MODES:
        rs.set_launch_overlap(mode)
        for use_sched in (False, True):
            got, sched = run(G, kind, w, use_sched)
            for g, x in zip(got, want):
                H.assert_bits_equal(g, x, f"{kind} mode {mode} sched {use_sched}")
            if sched is not None:
                assert not sched.any().item(), "workspace not returned to zero"


def test_claimed_schedule_matches_the_oracle(G, rs):
    # the claimed tail against the oracle directly (the store; radd is exact)
    rs.set_launch_overlap(2)
    w = ragged(False)
    s = G.run_ragged(w)
    r = H.oracle_ragged_store(w, w.cache.dtype)
    assert int(s.err.item()) == r.err == 0
    H.assert_close_bf16(H.bits(s.q_out), r.q_out, "q_out")
    H.compare_paged_cache(w.cache, H.bits(s.storage), r.storage, r.written, w.layer_idx,
                          H.rope_cols(128, 128), "cache")
    w = radd()
    s = G.run_radd(w)
    r = H.oracle_radd(w, w.cache.dtype)
    H.assert_bits_equal(H.bits(s.storage), r.storage, "radd cache")


@pytest.mark.parametrize("mode", MODES)
def test_back_to_back_calls_see_each_others_writes(G, rs, mode):
    """store -> radd(a1) -> radd(a2) on the rows the store writes, queued without a sync and
    sharing one workspace, equals the three calls run one at a time."""
    w = ragged(False)
    T, Hk, D = w.total_tokens, w.cache.n_kv_heads, w.cache.head_dim
    gen = torch.Generator().manual_seed(5)
    a = [torch.randn(T, 2 * Hk * D, generator=gen).to(torch.bfloat16).to(G.DEV)
         for _ in range(2)]

    def chain(sync_between):
        s = G.stage_ragged(w)
        sched = rs.sched_workspace(G.DEV)
        rs.rope_split_store_paged_ragged(s.qkv, w.n_q_heads, s.offs, s.freqs, s.kv,
                                         w.layer_idx, s.q_out, s.err, sched=sched)
        for x in a:
            if sync_between:
                torch.cuda.synchronize()
            rs.kv_cache_radd(x, s.kv, s.offs, 0, w.layer_idx, s.err, sched=sched)
        torch.cuda.synchronize()
        assert int(s.err.item()) == 0
        assert not sched.any().item()
        return H.bits(s.q_out), H.bits(s.storage)

    rs.set_launch_overlap(0)
    want = chain(True)
    rs.set_launch_overlap(mode)
    for _ in range(3):
        got = chain(False)
        H.assert_bits_equal(got[0], want[0], "q_out")
        H.assert_bits_equal(got[1], want[1], "cache after store + 2 x radd")


@pytest.mark.parametrize("mode", MODES)
def test_many_queued_calls_share_a_workspace(G, rs, mode):
    """60 calls over two staged copies, queued without a sync on one workspace."""
    rs.set_launch_overlap(0)
    w = ragged(True)
    G.USE_SCHED = False
    try:
        want = G.run_ragged(w)
    finally:
        G.USE_SCHED = True
    rs.set_launch_overlap(mode)
    copies = [G.stage_ragged(w) for _ in range(2)]
    sched = rs.sched_workspace(G.DEV)
    for c in copies:
        c.sched = sched
    for i in range(60):
        G.launch_ragged(w, copies[i % 2])
    torch.cuda.synchronize()
    assert not sched.any().item()
    for c in copies:
        assert int(c.err.item()) == 0
        H.assert_bits_equal(H.bits(c.q_out), H.bits(want.q_out), "q_out")
        H.assert_bits_equal(H.bits(c.storage), H.bits(want.storage), "cache")


@pytest.mark.parametrize("mode", MODES)
def test_invalid_offsets_leave_the_workspace_zero(G, rs, mode):
    rs.set_launch_overlap(mode)
    w = ragged(False)
    s = G.stage_ragged(w)
    pristine_q, pristine_cache = H.bits(s.q_out), H.bits(s.storage)
    bad = s.offs.clone()
    bad[-1] += 1  # the offsets no longer end at total_tokens
    sched = rs.sched_workspace(G.DEV)
    rs.rope_split_store_paged_ragged(s.qkv, w.n_q_heads, bad, s.freqs, s.kv, w.layer_idx,
                                     s.q_out, s.err, sched=sched)
    torch.cuda.synchronize()
    assert int(s.err.item()) == 0x1
    assert not sched.any().item()
    H.assert_bits_equal(H.bits(s.q_out), pristine_q, "q_out untouched")
    H.assert_bits_equal(H.bits(s.storage), pristine_cache, "cache untouched")
    # the same workspace then serves a valid call
    s.err.zero_()
    s.sched = sched
    G.launch_ragged(w, s)
    torch.cuda.synchronize()
    r = H.oracle_ragged_store(w, w.cache.dtype)
    assert int(s.err.item()) == 0
    H.assert_close_bf16(H.bits(s.q_out), r.q_out, "q_out")
    assert not sched.any().item()


def test_decode_overlap_modes_agree(G, rs):
    w = W.bshd_decode(14, B=64, S=2, n_q_heads=8, n_kv_heads=2, head_dim=128,
                      cache_lengths=list(range(0, 640, 10)), valid_lengths=[2, 1] * 32,
                      max_seq_len=1024, rope_dim=128, theta=5e5, interleaved=True)
    rs.set_launch_overlap(0)
    s = G.run_bshd(w)
    want = (H.bits(s.out), H.bits(s.storage))
    for mode in MODES:
        rs.set_launch_overlap(mode)
        s = G.run_bshd(w)
        assert int(s.err.item()) == 0
        H.assert_bits_equal(H.bits(s.out), want[0], f"bshd output mode {mode}")
        H.assert_bits_equal(H.bits(s.storage), want[1], f"bshd cache mode {mode}")
