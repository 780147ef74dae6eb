"""The Python binding only marshals arguments: with the C library replaced by a recorder,
every wrapper must hand the library exactly the pointers, sizes, strides, element-type
codes and descriptor fields that include/rope_store.h defines.  CPU tensors only; the real
library is never entered here."""
import ctypes

import pytest
import torch

import workloads as W


class Recorder:
    """Stands in for the loaded library: records each call and returns ROPE_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


@pytest.fixture
def rs(monkeypatch):
    from conftest import build_library
    build_library()
    import rope_paged_kv_b200
    rec = Recorder()
    monkeypatch.setattr(rope_paged_kv_b200, "_lib", rec)
    rope_paged_kv_b200.recorder = rec
    return rope_paged_kv_b200


def _obj(byref_arg):
    return byref_arg._obj


def _paged(rs, kv, storage):
    v = None if kv.v_offset is None else storage[kv.v_offset:]
    return rs.PagedCache(storage[kv.k_offset:], v, kv.page_table, kv.cache_lengths,
                         kv.n_kv_heads, kv.head_dim, kv.page_size, kv.num_pages,
                         kv.num_layers, kv.page_stride, kv.layer_stride, kv.slot_stride,
                         kv.head_stride, k_scale=kv.k_scale, v_scale=kv.v_scale)


def _check_cache(c, kv, storage, code):
    assert c.k == storage[kv.k_offset:].data_ptr()
    assert c.v == (None if kv.v_offset is None else storage[kv.v_offset:].data_ptr())
    assert c.dtype == code
    assert (c.n_kv_heads, c.head_dim, c.page_size, c.num_pages, c.num_layers) == (
        kv.n_kv_heads, kv.head_dim, kv.page_size, kv.num_pages, kv.num_layers)
    assert (c.page_stride, c.layer_stride, c.slot_stride, c.head_stride) == (
        kv.page_stride, kv.layer_stride, kv.slot_stride, kv.head_stride)
    assert c.page_table == kv.page_table.data_ptr()
    assert c.page_table_stride == kv.page_table.stride(0)
    assert c.max_pages_per_seq == kv.page_table.shape[1]
    assert c.cache_lengths == kv.cache_lengths.data_ptr()
    assert c.n_seqs == kv.page_table.shape[0]


@pytest.mark.parametrize("q_out_dtype,cache_dtype", [(None, None), ("f32", None),
                                                      (None, "fp8")])
def test_ragged_store_arguments(rs, q_out_dtype, cache_dtype):
    w = W.ragged_store(1, lengths=[5, 3], cache_lengths=[0, 7], n_q_heads=4, n_kv_heads=2,
                       head_dim=64, page_size=16, rope_dim=64, theta=1e4, interleaved=True,
                       max_seq_len=64, row_pad=8, q_out_dtype=q_out_dtype,
                       cache_dtype=cache_dtype, kv_scales=(0.5, 0.25))
    storage = w.cache.storage
    err = torch.zeros(1, dtype=torch.int32)
    rs.rope_split_store_paged_ragged(w.qkv, 4, w.offsets, rs.Freqs(w.rope.table, True),
                                     _paged(rs, w.cache, storage), 1, w.q_out, err, stream=0)
    (name, a), = rs.recorder.calls
    assert name == "rope_split_store_paged_ragged"
    assert a[0] == w.qkv.data_ptr() and a[1] == w.qkv.stride(0) == (4 + 4) * 64 + 8
    assert a[2] == 0 and a[3] == 8 and a[4] == 4      # bf16 input, T, n_q_heads
    assert a[5] == w.offsets.data_ptr() and a[6] == 2  # offsets, batch
    f = _obj(a[7])
    assert (f.data, f.dtype, f.max_seq_len, f.rope_dim, f.interleaved, f.rope_col_offset) == (
        w.rope.table.data_ptr(), 2, 64, 64, 1, -1)
    c = _obj(a[8])
    _check_cache(c, w.cache, storage, 3 if cache_dtype == "fp8" else 0)
    if cache_dtype == "fp8":
        assert (c.k_scale, c.v_scale) == (w.cache.k_scale.data_ptr(), w.cache.v_scale.data_ptr())
    else:
        assert c.k_scale is None and c.v_scale is None
    assert a[9] == 1 and a[10] == w.q_out.data_ptr() and a[11] == w.q_out.stride(0)
    assert a[12] == {None: 0, "f32": 2}[q_out_dtype]
    assert a[13] == err.data_ptr() and a[14] is None and a[15] == 0


def test_norm_store_arguments(rs):
    w = W.ragged_store(2, lengths=[4, 2], cache_lengths=[1, 0], n_q_heads=2, n_kv_heads=1,
                       head_dim=128, page_size=16, rope_dim=64, theta=1e4, interleaved=False,
                       max_seq_len=64, norm=True, dtype="f16")
    rs.fused_qk_rmsnorm_rope_paged(w.qkv, 2, w.offsets, rs.Freqs(w.rope.table, False, 0),
                                   _paged(rs, w.cache, w.cache.storage), w.q_gamma, w.k_gamma,
                                   1e-5, 1.0, 0, w.q_out, multiply_before_cast=False,
                                   stream=0)
    (name, a), = rs.recorder.calls
    assert name == "fused_qk_rmsnorm_rope_paged"
    assert a[2] == 1 and a[3] == 6 and a[4] == 2 and a[6] == 2
    assert _obj(a[7]).rope_col_offset == 0 and _obj(a[7]).interleaved == 0
    assert a[9] == w.q_gamma.data_ptr() and a[10] == w.k_gamma.data_ptr()
    assert (a[11], a[12], a[13], a[14]) == (1e-5, 1.0, 0, 0)
    assert a[15] == w.q_out.data_ptr() and a[16] == w.q_out.stride(0)
    assert a[17] is None and a[18] is None and a[19] == 0


@pytest.mark.parametrize("single", [False, True])
def test_dual_band_arguments(rs, single):
    w = W.dual_band(3, lengths=[6, 1], cache_lengths=[0, 3], main_q_heads=4, main_kv_heads=2,
                    index_q_heads=2, index_kv_heads=1, head_dim=64, main_page_size=16,
                    index_page_size=8, rope_dim=32, theta=1e4, interleaved=True,
                    max_seq_len=64, single=single)
    g = w.gammas
    main = rs.NormBand(w.input, *w.main_cols, w.main_q_heads,
                       _paged(rs, w.main_cache, w.main_cache.storage), g[0], g[1], w.main_eps,
                       w.q_main_out)
    index = None
    if not single:
        index = rs.NormBand(w.input, *w.index_cols, w.index_q_heads,
                            _paged(rs, w.index_cache, w.index_cache.storage), g[2], g[3],
                            w.index_eps, w.q_index_out)
    rs.fused_dual_qk_rmsnorm_rope_paged(main, index, w.offsets, w.total_tokens,
                                        rs.Freqs(w.rope.table, True), 0.0, 1, stream=0)
    (name, a), = rs.recorder.calls
    assert name == "fused_dual_qk_rmsnorm_rope_paged"
    bands = [(_obj(a[0]), main, w.main_cache)]
    if single:
        assert a[1] is None
    else:
        bands.append((_obj(a[1]), index, w.index_cache))
    for b, nb, kv in bands:
        assert b.input == w.input.data_ptr() and b.input_row_stride == w.input.stride(0)
        assert (b.q_col, b.k_col, b.v_col, b.n_q_heads) == (nb.q_col, nb.k_col, nb.v_col,
                                                            nb.n_q_heads)
        _check_cache(b.cache.contents, kv, kv.storage, 0)
        assert b.q_gamma == nb.q_gamma.data_ptr() and b.k_gamma == nb.k_gamma.data_ptr()
        assert b.epsilon == pytest.approx(nb.epsilon)
        assert b.q_out == nb.q_out.data_ptr() and b.q_out_row_stride == nb.q_out.stride(0)
    assert a[2] == 0 and a[3] == w.offsets.data_ptr() and a[4] == 2 and a[5] == 7
    assert (a[7], a[8], a[9]) == (0.0, 1, 1)


def test_bshd_radd_and_gemv_arguments(rs):
    d = W.decode_bshd()
    kv = d.cache
    v = None if kv.v_offset is None else kv.storage[kv.v_offset:]
    cc = rs.ContCache(kv.storage[kv.k_offset:], v, kv.lookup_table, kv.cache_lengths,
                      kv.n_kv_heads, kv.head_dim, kv.num_slots, kv.num_layers, kv.max_seq_len,
                      kv.slot_stride, kv.layer_stride, kv.pos_stride, kv.head_stride)
    rs.qk_rope_bshd_continuous(d.q_proj, cc, rs.Freqs(d.rope.table, True), d.layer_idx,
                               d.valid_lengths, d.output, stream=0)
    r = W.radd(4, lengths=[3, 2], cache_lengths=[1, 4], n_kv_heads=2, head_dim=64,
               page_size=16, batch_offset=1)
    rs.kv_cache_radd(r.a, _paged(rs, r.cache, r.cache.storage), r.offsets, r.batch_offset,
                     r.layer_idx, stream=0)
    g = W.gemv_norm(5, n=24, k=64, n_normed=16)
    rs.matmul_fused_partial_rmsnorm(g.x, g.weight, g.gamma, g.epsilon, g.weight_offset,
                                    g.normed_output, g.unnormed_output, stream=0)
    (n1, a1), (n2, a2), (n3, a3) = rs.recorder.calls
    assert n1 == "qk_rope_bshd_continuous"
    assert a1[:5] == (d.q_proj.data_ptr(), *d.q_proj.shape)
    c = _obj(a1[5])
    assert (c.num_slots, c.max_seq_len, c.pos_stride, c.n_seqs) == (
        kv.num_slots, kv.max_seq_len, kv.pos_stride, kv.lookup_table.shape[0])
    assert a1[7] == d.layer_idx and a1[8] == d.valid_lengths.data_ptr()
    assert a1[9] == d.output.data_ptr()
    assert n2 == "kv_cache_radd"
    assert a2[0] == r.a.data_ptr() and a2[1] == r.a.stride(0) and a2[2] == r.a.shape[0]
    assert a2[5] == 2 and a2[6] == 1 and a2[7] == r.layer_idx
    assert n3 == "matmul_fused_partial_rmsnorm"
    assert a3[2:6] == (g.weight.stride(0), 24, 64, 1)
    assert a3[10] == 16 and a3[12] == 0
    assert a3[14] is None and a3[15] == 0  # no workspace given


def test_gemv_without_normed_part_passes_null_pointers(rs):
    g = W.gemv_norm(6, n=8, k=64, n_normed=0)
    rs.matmul_fused_partial_rmsnorm(g.x, g.weight, g.gamma, g.epsilon, 0.0, g.normed_output,
                                    g.unnormed_output, stream=0)
    (name, a), = rs.recorder.calls
    assert a[6] is None and a[9] is None and a[10] == 0 and a[11] == g.unnormed_output.data_ptr()
