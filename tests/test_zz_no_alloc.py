"""rope_split_store_paged_ragged_noalloc: the store for callers that cannot allocate.

Some callers cannot allocate device memory (an engine that owns the whole device pool, a
latency-critical path that must not call cudaMalloc / cudaFree), so this entry point keeps
its scheduling workspace in the library's own per-device array.  Called twice in a row
through the C ABI, it must give what rope_split_store_paged_ragged gives with a caller-owned
workspace, within the parity tolerance (rotated values) and bit for bit (everything else).
This file is collected last, and it passes alone in a fresh process as well.
"""
import ctypes

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


def test_noalloc_store_matches_the_store_with_a_workspace():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import gpu_helpers as G
    import rope_paged_kv_b200 as rs

    lib = rs.raw_library()
    stream = torch.cuda.current_stream()
    for seed in (21, 22):  # two calls in a row, on different inputs
        w = _workload(seed)
        want = G.stage_ragged(w)
        want.sched = rs.sched_workspace(G.DEV)
        G.launch_ragged(w, want)
        got = G.stage_ragged(w)
        f, c = got.freqs.c(), got.kv.c()
        st = lib.rope_split_store_paged_ragged_noalloc(
            got.qkv.data_ptr(), got.qkv.stride(0), -1, w.total_tokens, w.n_q_heads,
            got.offs.data_ptr(), got.offs.shape[0] - 1, ctypes.byref(f), ctypes.byref(c),
            w.layer_idx, got.q_out.data_ptr(), got.q_out.stride(0), -1, got.err.data_ptr(),
            stream.cuda_stream)
        assert st == rs.OK
        torch.cuda.synchronize()
        assert int(got.err.item()) == int(want.err.item()) == 0
        assert not want.sched.any().item()
        T, Hq, D = w.total_tokens, w.n_q_heads, w.cache.head_dim
        H.assert_close_bf16(H.bits(got.q_out).reshape(T, Hq, D),
                            H.bits(want.q_out).reshape(T, Hq, D), "q_out")
        written = H.oracle_ragged_store(w, w.cache.dtype).written
        H.compare_paged_cache(w.cache, H.bits(got.storage), H.bits(want.storage), written,
                              w.layer_idx, H.rope_cols(D, w.rope.rope_dim), "cache")
