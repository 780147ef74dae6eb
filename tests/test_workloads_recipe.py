"""The named synthetic workloads have the shapes, sizes, value distributions and structure
their recipe states (the Llama-3-8B prefill, decode, per-head norm, dual-band MiniMax, radd
and latent-attention GEMV shapes): token counts and length bounds, page tables that give
every sequence its own pages, freqs_cis tables of the stated theta, and the moments of the
random inputs.  These are the inputs both the oracle and the kernels are run on."""
import math

import numpy as np
import pytest
import torch

import workloads as W

SENTINEL = -1  # unused page-table entries (0xFFFFFFFF read as uint32)


def _check_page_table(kv, lengths, cache_lengths):
    pt = kv.page_table
    used = []
    for b, (n, c) in enumerate(zip(lengths, cache_lengths)):
        need = max(1, math.ceil((c + n) / kv.page_size))
        row = pt[b].tolist()
        assert all(0 <= p < kv.num_pages for p in row[:need]), "a needed entry is unmapped"
        assert all(p == SENTINEL for p in row[need:]), "entries past the need are not unused"
        used += row[:need]
    assert len(used) == len(set(used)), "two sequences share a page"


def _check_freqs(table, theta, rope_dim, positions=(0, 1, 17, 1000, 8191)):
    i = np.arange(rope_dim // 2)
    inv = theta ** (-2.0 * i / rope_dim)
    t = table.double().numpy()
    for p in positions:
        if p >= t.shape[0]:
            continue
        want = np.stack([np.cos(p * inv), np.sin(p * inv)], -1).reshape(-1)
        got = t[p]
        tol = 2.0 ** -8 if table.dtype == torch.bfloat16 else 2.0 ** -23
        assert np.all(np.abs(got - want) <= tol * np.maximum(1.0, np.abs(want)) + 1e-30), p


def _moments(t, mean, std, rel=0.02):
    x = t.float()
    assert abs(x.mean().item() - mean) < rel * max(std, 1.0)
    assert abs(x.std().item() - std) < rel * std


def test_tiny_ragged():
    w = W.tiny_ragged()
    assert w.lengths == [3, 5] and w.cache.cache_lengths.tolist() == [0, 7]
    assert (w.n_q_heads, w.cache.n_kv_heads, w.cache.head_dim) == (4, 2, 64)
    assert w.cache.page_size == 16 and w.cache.num_pages == 8
    assert sorted(w.cache.page_table.reshape(-1).tolist()) == list(range(8))
    assert w.rope.interleaved and tuple(w.rope.table.shape) == (64, 64)
    _check_freqs(w.rope.table, 1e4, 64)


@pytest.mark.parametrize("fp8", [False, True])
def test_llama3_8b_prefill(fp8):
    w = W.llama3_8b_prefill_fp8_cache() if fp8 else W.llama3_8b_prefill()
    assert len(w.lengths) == 8 and all(256 <= n <= 2048 for n in w.lengths)
    assert w.total_tokens == sum(w.lengths) == 10433
    assert w.cache.cache_lengths.tolist() == [0] * 8
    assert (w.n_q_heads, w.cache.n_kv_heads, w.cache.head_dim, w.cache.page_size) == (
        32, 8, 128, 128)
    assert tuple(w.qkv.shape) == (10433, (32 + 16) * 128) and w.qkv.dtype == torch.bfloat16
    _moments(w.qkv, 0.0, 1.0)
    assert not w.rope.interleaved and tuple(w.rope.table.shape) == (8192, 128)
    assert w.rope.table.dtype == torch.float32
    _check_freqs(w.rope.table, 5e5, 128)
    _check_page_table(w.cache, w.lengths, [0] * 8)
    if fp8:
        assert w.cache.storage.dtype == torch.float8_e4m3fn
        assert (w.cache.k_scale.item(), w.cache.v_scale.item()) == (0.5, 0.25)
    else:
        assert w.cache.storage.dtype == torch.bfloat16


def test_decode_bshd():
    w = W.decode_bshd()
    assert tuple(w.q_proj.shape) == (256, 1, 32, 128) and w.q_proj.dtype == torch.bfloat16
    _moments(w.q_proj, 0.0, 1.0)
    cl = w.cache.cache_lengths.tolist()
    assert len(cl) == 256 and all(1 <= c <= 8191 for c in cl)
    assert w.valid_lengths.tolist() == [1] * 256
    assert (w.cache.num_slots, w.cache.max_seq_len, w.cache.n_kv_heads) == (256, 8192, 8)
    assert sorted(w.cache.lookup_table.tolist()) == list(range(256))
    assert w.rope.interleaved and w.rope.table.dtype == torch.bfloat16
    _check_freqs(w.rope.table, 5e5, 128)


def test_per_head_norm():
    w = W.per_head_norm()
    assert len(w.lengths) == 32 and sum(w.lengths) == w.total_tokens == 16384
    assert all(1 <= n <= 4096 for n in w.lengths)
    cl = w.cache.cache_lengths.tolist()
    assert all(0 <= c <= 4096 for c in cl)
    assert (w.n_q_heads, w.cache.n_kv_heads, w.cache.head_dim) == (64, 8, 128)
    _moments(w.qkv, 0.0, 2.0)
    _moments(w.q_gamma, 1.0, 0.1, rel=0.3)
    _moments(w.k_gamma, 1.0, 0.1, rel=0.3)
    assert w.epsilon == 1e-6 and w.weight_offset == 0.0
    _check_freqs(w.rope.table, 1e4, 128)
    _check_page_table(w.cache, w.lengths, cl)


@pytest.mark.parametrize("in_place", [False, True])
def test_dual_band_minimax(in_place):
    w = W.dual_band_minimax_in_place() if in_place else W.dual_band_minimax()
    assert len(w.lengths) == 64 and sum(w.lengths) == w.total_tokens == 32768
    assert all(1 <= n <= 4096 for n in w.lengths)
    assert w.input.shape[1] == 11392  # Q main 64 | K main 8 | V main 8 | Q index 8 | K index 1
    assert (w.main_q_heads, w.main_cache.n_kv_heads, w.index_q_heads,
            w.index_cache.n_kv_heads) == (64, 8, 8, 1)
    assert (w.main_cache.page_size, w.index_cache.page_size) == (128, 64)
    assert w.main_cache.planes == 2 and w.index_cache.planes == 1
    assert w.rope.rope_dim == 64 and w.rope.interleaved
    if in_place:
        assert w.main_cols[1] < 0 and w.index_cols[1] < 0 and w.main_cols[2] < 0
    else:
        assert w.main_cols == (0, 64 * 128, 72 * 128) and w.index_cols == (80 * 128,
                                                                          88 * 128, -1)
    cl = w.main_cache.cache_lengths.tolist()
    _check_page_table(w.main_cache, w.lengths, cl)
    _check_page_table(w.index_cache, w.lengths, w.index_cache.cache_lengths.tolist())


def test_radd_minimax():
    w = W.radd_minimax()
    assert tuple(w.a.shape) == (32768, 2048) and w.a.dtype == torch.bfloat16
    assert sum(w.lengths) == 32768 and w.batch_offset == 0
    _moments(w.a, 0.0, 1.0)
    assert (w.cache.n_kv_heads, w.cache.head_dim, w.cache.page_size) == (8, 128, 128)


def test_mla_kv_a_proj():
    w = W.mla_kv_a_proj()
    assert (w.n, w.k, w.n_normed) == (576, 7168, 512)
    y = w.weight.double() @ w.x.double()
    assert 0.9 < y.std().item() < 1.1  # W ~ N(0, 1/k) keeps y ~ N(0, 1)
    _moments(w.gamma, 1.0, 0.1, rel=0.3)
