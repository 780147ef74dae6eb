"""rope_split_store_paged_ragged_noalloc: the store for callers that cannot allocate.

Some callers cannot allocate device memory (an engine that owns the whole device pool, a
latency-critical path that must not call cudaMalloc / cudaFree), so this entry point keeps
its scheduling workspace in the library's own per-device array.  Called twice in a row
through the C ABI, it must give what rope_split_store_paged_ragged gives with a caller-owned
workspace, within the parity tolerance (rotated values) and bit for bit (everything else),
and match the oracle the same way.  It must allocate nothing: the device's free memory is
the same before and after a run of calls.  A call that is rejected, or that has no tokens,
queues nothing, and the next call is still right.  This file is collected last, and it
passes alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
import helpers as H

pytestmark = pytest.mark.gpu


def _workload(seed):
    # ~6k tokens over five sequences: each CTA takes a static share and claims the rest
    return W.ragged_store(seed, lengths=[1500, 37, 2900, 1, 1700],
                          cache_lengths=[0, 5, 100, 0, 64], n_q_heads=8, n_kv_heads=2,
                          head_dim=128, page_size=64, rope_dim=128, theta=5e5,
                          interleaved=False, max_seq_len=4096)


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gpu_helpers
    return gpu_helpers


def _noalloc(lib, w, s, stream, total_tokens=None, kv=None):
    f = s.freqs.c()
    c = s.kv.c() if kv is None else kv
    return lib.rope_split_store_paged_ragged_noalloc(
        s.qkv.data_ptr(), s.qkv.stride(0), -1,
        w.total_tokens if total_tokens is None else total_tokens, w.n_q_heads,
        s.offs.data_ptr(), s.offs.shape[0] - 1, ctypes.byref(f),
        None if c is False else ctypes.byref(c), w.layer_idx, s.q_out.data_ptr(),
        s.q_out.stride(0), -1, s.err.data_ptr(), stream.cuda_stream)


def _check(w, got, want):
    """The no-alloc result against the workspace call's and against the oracle."""
    T, Hq, D = w.total_tokens, w.n_q_heads, w.cache.head_dim
    assert int(got.err.item()) == 0
    H.assert_close_bf16(H.bits(got.q_out).reshape(T, Hq, D),
                        H.bits(want.q_out).reshape(T, Hq, D), "q_out vs the workspace call")
    r = H.oracle_ragged_store(w, w.cache.dtype)
    assert r.err == 0
    H.assert_close_bf16(H.bits(got.q_out).reshape(T, Hq, D), r.q_out.reshape(T, Hq, D),
                        "q_out vs the oracle")
    rope = H.rope_cols(D, w.rope.rope_dim)
    H.compare_paged_cache(w.cache, H.bits(got.storage), H.bits(want.storage), r.written,
                          w.layer_idx, rope, "cache vs the workspace call")
    H.compare_paged_cache(w.cache, H.bits(got.storage), r.storage, r.written, w.layer_idx, rope,
                          "cache vs the oracle")


def test_noalloc_store_matches_the_store_with_a_workspace_and_the_oracle(G):
    import rope_paged_kv_b200 as rs
    lib = rs.raw_library()
    stream = torch.cuda.current_stream()
    for seed in (21, 22):  # two calls in a row, on different inputs
        w = _workload(seed)
        want = G.stage_ragged(w)
        want.sched = rs.sched_workspace(G.DEV)
        G.launch_ragged(w, want)
        got = G.stage_ragged(w)
        assert _noalloc(lib, w, got, stream) == rs.OK
        torch.cuda.synchronize()
        assert not want.sched.any().item()
        _check(w, got, want)


def test_noalloc_store_allocates_nothing_and_rejected_calls_queue_nothing(G):
    import rope_paged_kv_b200 as rs
    lib = rs.raw_library()
    stream = torch.cuda.current_stream()
    w = _workload(23)
    want = G.stage_ragged(w)
    want.sched = rs.sched_workspace(G.DEV)
    G.launch_ragged(w, want)
    staged = [G.stage_ragged(w) for _ in range(4)]
    assert _noalloc(lib, w, staged[0], stream) == rs.OK  # the first call does the set-up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for s in staged[1:]:
        assert _noalloc(lib, w, s, stream) == rs.OK
    # no tokens: returns at once; a rejected call (no cache descriptor) returns its status
    assert _noalloc(lib, w, staged[1], stream, total_tokens=0) == rs.OK
    assert _noalloc(lib, w, staged[1], stream, kv=False) == rs.ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0, "device memory was allocated"
    # every call after the rejected one is still right
    last = G.stage_ragged(w)
    assert _noalloc(lib, w, last, stream) == rs.OK
    torch.cuda.synchronize()
    for s in staged + [last]:
        assert np.array_equal(H.bits(s.q_out), H.bits(staged[0].q_out))
        assert np.array_equal(H.bits(s.storage), H.bits(staged[0].storage))
    _check(w, last, want)
