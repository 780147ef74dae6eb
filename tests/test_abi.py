"""The C-ABI library loads on a machine without a GPU, exports every function that
include/rope_store.h declares, and rejects bad host arguments before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def rs():
    from conftest import build_library
    build_library()
    import rope_paged_kv_b200
    return rope_paged_kv_b200


def _declared():
    text = open(os.path.join(ROOT, "include", "rope_store.h")).read()
    return re.findall(r"^(?:rope_status_t|int32_t|const char \*)\s*(\w+)\(", text, re.M)


def test_header_declares_the_entry_points():
    names = set(_declared())
    assert {"rope_split_store_paged_ragged", "fused_qk_rmsnorm_rope_paged",
            "fused_dual_qk_rmsnorm_rope_paged", "qk_rope_bshd_continuous",
            "kv_cache_radd", "rope_status_string", "rope_set_launch_overlap",
            "rope_get_launch_overlap"} <= names


def test_library_exports_every_declared_symbol(rs):
    lib = rs.raw_library()
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", rs.LIBRARY_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(_declared()) <= exported
    assert set(rs.header_functions()) == set(_declared())


def test_binding_mirrors_header_structs(rs):
    # field order and sizes of the descriptors, against the header text
    text = open(os.path.join(ROOT, "include", "rope_store.h")).read()
    for cname, pyname in (("rope_freqs_t", "c_freqs"), ("rope_paged_cache_t", "c_paged_cache"),
                          ("rope_cont_cache_t", "c_cont_cache"),
                          ("rope_norm_band_t", "c_norm_band")):
        body = re.search(r"typedef struct \{([^}]*)\}\s*" + cname, text).group(1)
        body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
        fields = []
        for decl in body.split(";"):
            decl = decl.strip()
            if not decl:
                continue
            names = decl.split(None, 1)[1] if not decl.startswith("const") else \
                decl.split(None, 2)[2]
            for n in names.split(","):
                fields.append(n.strip().lstrip("*").strip())
        py = [f[0] for f in getattr(rs, pyname)._fields_]
        assert py == fields, (cname, py, fields)


def test_status_strings(rs):
    lib = rs.raw_library()
    for code in range(4):
        assert lib.rope_status_string(code)


def test_host_argument_checks_need_no_gpu(rs):
    lib = rs.raw_library()
    fake = 1 << 20   # a non-null, 16-byte aligned address; never dereferenced here
    f = rs.c_freqs(fake, 2, 64, 64, 1, -1)
    kv = rs.c_paged_cache(fake, fake, 0, 2, 64, 16, 8, 2, 4096, 2048, 128, 64, fake, 4, 4,
                          fake, 2)
    def call(*a):  # the store with the input and q_out in the cache's element type
        return lib.rope_split_store_paged_ragged(*a[:2], -1, *a[2:11], -1, *a[11:])
    # NULL descriptors / pointers
    assert call(fake, 512, 8, 4, fake, 2, None, ctypes.byref(kv), 1, fake, 256, None, None,
                None) == rs.ERR_INVALID_ARG
    assert call(fake, 512, 8, 4, None, 2, ctypes.byref(f), ctypes.byref(kv), 1, fake, 256,
                None, None, None) == rs.ERR_INVALID_ARG
    # layer past num_layers
    assert call(fake, 512, 8, 4, fake, 2, ctypes.byref(f), ctypes.byref(kv), 2, fake, 256,
                None, None, None) == rs.ERR_INVALID_ARG
    # odd rope_dim, rope_dim > head_dim
    for bad in (rs.c_freqs(fake, 2, 64, 63, 1, -1), rs.c_freqs(fake, 2, 64, 66, 1, -1)):
        assert call(fake, 512, 8, 4, fake, 2, ctypes.byref(bad), ctypes.byref(kv), 1, fake,
                    256, None, None, None) == rs.ERR_INVALID_ARG
    # half-split pairs that straddle a 16-byte vector
    bad = rs.c_freqs(fake, 2, 64, 8, 0, -1)
    assert call(fake, 512, 8, 4, fake, 2, ctypes.byref(bad), ctypes.byref(kv), 1, fake, 256,
                None, None, None) == rs.ERR_UNSUPPORTED
    # unsupported head_dim, misaligned row stride, misaligned base
    kv96 = rs.c_paged_cache(fake, fake, 0, 2, 96, 16, 8, 2, 4096, 2048, 192, 96, fake, 4, 4,
                            fake, 2)
    assert call(fake, 768, 8, 4, fake, 2, ctypes.byref(f), ctypes.byref(kv96), 1, fake, 384,
                None, None, None) == rs.ERR_UNSUPPORTED
    assert call(fake, 515, 8, 4, fake, 2, ctypes.byref(f), ctypes.byref(kv), 1, fake, 256,
                None, None, None) == rs.ERR_UNSUPPORTED
    assert call(fake + 2, 512, 8, 4, fake, 2, ctypes.byref(f), ctypes.byref(kv), 1, fake, 256,
                None, None, None) == rs.ERR_UNSUPPORTED
    # more sequences than the cache describes; tokens without sequences
    assert call(fake, 512, 8, 4, fake, 3, ctypes.byref(f), ctypes.byref(kv), 1, fake, 256,
                None, None, None) == rs.ERR_INVALID_ARG
    assert call(fake, 512, 8, 4, fake, 0, ctypes.byref(f), ctypes.byref(kv), 1, fake, 256,
                None, None, None) == rs.ERR_INVALID_ARG
    # empty work: OK without a launch
    assert call(fake, 512, 0, 4, fake, 2, ctypes.byref(f), ctypes.byref(kv), 1, fake, 256,
                None, None, None) == rs.OK
    # the norm op needs both gammas (checked before any launch)
    assert lib.fused_qk_rmsnorm_rope_paged(fake, 512, -1, 8, 4, fake, 2, ctypes.byref(f),
                                           ctypes.byref(kv), None, fake, 1e-6, 0.0, 0, 1, fake,
                                           256, None, None, None) == rs.ERR_INVALID_ARG
    # a q_out element type that does not exist
    assert lib.rope_split_store_paged_ragged(fake, 512, -1, 8, 4, fake, 2, ctypes.byref(f),
                                             ctypes.byref(kv), 1, fake, 256, 7, None, None,
                                             None) == rs.ERR_UNSUPPORTED
    # dual band: geometry must agree across bands
    kv128 = rs.c_paged_cache(fake, None, 0, 1, 128, 16, 8, 2, 4096, 2048, 128, 128, fake, 4,
                             4, fake, 2)
    mb = rs.c_norm_band(fake, 1024, 0, 256, 384, 2, ctypes.pointer(kv), fake, fake, 1e-6,
                        fake, 128)
    ib = rs.c_norm_band(fake, 1024, 512, 768, -1, 1, ctypes.pointer(kv128), fake, fake, 1e-6,
                        fake, 128)
    assert lib.fused_dual_qk_rmsnorm_rope_paged(ctypes.byref(mb), ctypes.byref(ib), -1, fake,
                                                2, 8,
                                                ctypes.byref(f), 0.0, 1, 1, None, None,
                                                None) == rs.ERR_INVALID_ARG
    # radd needs a V plane
    kvk = rs.c_paged_cache(fake, None, 0, 2, 64, 16, 8, 2, 4096, 2048, 128, 64, fake, 4, 4,
                           fake, 2)
    assert lib.kv_cache_radd(fake, 256, 8, ctypes.byref(kvk), fake, 2, 0, 1, None, None,
                             None) == rs.ERR_INVALID_ARG
    # BSHD: head_dim must match the cache
    cc = rs.c_cont_cache(fake, None, 0, 2, 64, 4, 1, 64, 8192, 8192, 128, 64, fake, fake, 4)
    assert lib.qk_rope_bshd_continuous(fake, 2, 1, 4, 128, ctypes.byref(cc), ctypes.byref(f),
                                       0, fake, fake, None, None) == rs.ERR_INVALID_ARG

    # a scheduling workspace must hold aligned uint32 words
    assert call(fake, 512, 8, 4, fake, 2, ctypes.byref(f), ctypes.byref(kv), 1, fake, 256,
                None, fake + 2, None) == rs.ERR_INVALID_ARG
    assert lib.kv_cache_radd(fake, 256, 8, ctypes.byref(kvk), fake, 2, 0, 1, None, fake + 1,
                             None) == rs.ERR_INVALID_ARG


def test_launch_overlap_mode(rs):
    lib = rs.raw_library()
    before = lib.rope_get_launch_overlap()
    assert before == rs.OVERLAP_PDL  # the default
    try:
        for mode in (rs.OVERLAP_OFF, rs.OVERLAP_PDL_EARLY_METADATA, rs.OVERLAP_PDL):
            assert lib.rope_set_launch_overlap(mode) == rs.OK
            assert lib.rope_get_launch_overlap() == mode
        assert lib.rope_set_launch_overlap(3) == rs.ERR_INVALID_ARG
        assert lib.rope_set_launch_overlap(-1) == rs.ERR_INVALID_ARG
        assert lib.rope_get_launch_overlap() == rs.OVERLAP_PDL
    finally:
        lib.rope_set_launch_overlap(before)


def test_gemv_host_checks_need_no_gpu(rs):
    lib = rs.raw_library()
    fake = 1 << 20
    call = lib.matmul_fused_partial_rmsnorm
    args = [fake, fake, 64, 8, 64, 1, fake, 1e-6, 0.0, fake, 8, None, 0, None, fake, 48, None]
    bad = list(args); bad[10] = 9          # n_normed > n
    assert call(*bad) == rs.ERR_INVALID_ARG
    bad = list(args); bad[5] = 0           # weight stored [k, n] (transpose_b = False)
    assert call(*bad) == rs.ERR_UNSUPPORTED
    bad = list(args); bad[3] = 0; bad[10] = 0  # no output at all: OK without a launch
    assert call(*bad) == rs.OK
    bad = list(args); bad[15] = 16         # workspace smaller than ROPE_GEMV_WORKSPACE_BYTES
    assert call(*bad) == rs.ERR_INVALID_ARG
    bad = list(args); bad[12] = 7          # unknown element type
    assert call(*bad) == rs.ERR_UNSUPPORTED


def test_fp8_cache_host_checks_need_no_gpu(rs):
    lib = rs.raw_library()
    fake = 1 << 20
    f = rs.c_freqs(fake, 2, 64, 64, 1, -1)
    # an E4M3 cache (dtype 3) needs its scales
    kv8 = rs.c_paged_cache(fake, fake, 3, 2, 64, 16, 8, 2, 4096, 2048, 128, 64, fake, 4, 4,
                           fake, 2, None, None)
    assert lib.rope_split_store_paged_ragged(fake, 512, 0, 8, 4, fake, 2, ctypes.byref(f),
                                             ctypes.byref(kv8), 1, fake, 256, -1, None, None,
                                             None) == rs.ERR_INVALID_ARG
    # an FP8 cache does not say what the input is
    assert lib.rope_split_store_paged_ragged(fake, 512, -1, 8, 4, fake, 2, ctypes.byref(f),
                                             ctypes.byref(kv8), 1, fake, 256, -1, None, None,
                                             None) == rs.ERR_UNSUPPORTED
    kv8s = rs.c_paged_cache(fake, fake, 3, 2, 64, 16, 8, 2, 4096, 2048, 128, 64, fake, 4, 4,
                            fake, 2, fake, fake)
    # radd does not read FP8 caches
    assert lib.kv_cache_radd(fake, 256, 8, ctypes.byref(kv8s), fake, 2, 0, 1, None, None,
                             None) == rs.ERR_UNSUPPORTED
    # K updated in place would have to be decoded: not built
    mb = rs.c_norm_band(fake, 1024, 0, -1, -1, 2, ctypes.pointer(kv8s), fake, fake, 1e-6,
                        fake, 128)
    assert lib.fused_dual_qk_rmsnorm_rope_paged(ctypes.byref(mb), None, 0, fake, 2, 8,
                                                ctypes.byref(f), 0.0, 1, 1, None, None,
                                                None) == rs.ERR_UNSUPPORTED


def test_binding_rejects_element_types_before_any_call(rs):
    # marshalling errors raise in Python before the library is entered (CPU tensors here are
    # never handed to it)
    import torch
    w = torch.zeros(8, 64, dtype=torch.bfloat16)
    x16 = torch.zeros(64, dtype=torch.float16)
    out = torch.zeros(8, dtype=torch.bfloat16)
    g = torch.zeros(8, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="input must have the weight's element type"):
        rs.matmul_fused_partial_rmsnorm(x16, w, g, 1e-6, 0.0, out, out[:0])
    with pytest.raises(ValueError, match="gamma"):
        rs.matmul_fused_partial_rmsnorm(torch.zeros(64, dtype=torch.bfloat16), w,
                                        g.float(), 1e-6, 0.0, out, out[:0])
    with pytest.raises(ValueError, match="unsupported element type"):
        rs.matmul_fused_partial_rmsnorm(torch.zeros(64, dtype=torch.int16),
                                        w.to(torch.int16), g, 1e-6, 0.0, out, out[:0])
    table = torch.zeros(16, 64, dtype=torch.float64)
    with pytest.raises(ValueError, match="unsupported element type"):
        rs.Freqs(table, True).c()
