"""The oracle's pins have teeth: each plausible mistake, planted in a copy of the C oracle
on the CPU, makes the pin suite fail.

Each mutant is a one-line edit of rope_oracle.c (a flipped sign, swapped cos/sin, a wrong
pair partner, a dropped cache length, epsilon outside the root, a sum instead of a mean, a
dropped weight_offset, a weight_offset left unrounded, a shifted slot, swapped K/V halves,
an off-by-one valid length, the wrong rotated columns, the normalised value rounded after
gamma or not at all under
multiply_before_cast = 0, and in the GEMV + partial RMSNorm: epsilon outside the root, the
mean over every column, the norm over the tail, a consumed weight_offset; and in the FP8
cache: no saturation, a wrong exponent bias, the scale applied the wrong way).  The copy is
built in a temporary directory and the pin suite runs against it in a subprocess; the test
passes when that run fails.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "rotation sign": ("y[ia] = a * c - b * s;", "y[ia] = a * c + b * s;"),
    "cos/sin swapped": ("double c = cs[2 * i], s = cs[2 * i + 1];",
                        "double s = cs[2 * i], c = cs[2 * i + 1];"),
    "half-split partner": ("int32_t ib = rope->interleaved ? o + 2 * i + 1 : o + i + half;",
                           "int32_t ib = rope->interleaved ? o + 2 * i + 1 : o + i + half - 1 "
                           "+ (i == 0);"),
    "position ignores cache length": ("int64_t pos = (int64_t)c->cache_lengths[b] + t;",
                                      "int64_t pos = t;"),
    "epsilon outside the root": ("double r = 1.0 / sqrt(ss / D + eps);",
                                 "double r = 1.0 / sqrt(ss / D) + eps;"),
    "sum instead of mean": ("double r = 1.0 / sqrt(ss / D + eps);",
                            "double r = 1.0 / sqrt(ss + eps);"),
    "weight_offset dropped": ("double g = orc_decode(dtype, gamma, d) + weight_offset;",
                              "double g = orc_decode(dtype, gamma, d);"),
    "weight_offset not rounded to the element type": (
        "double wo = requantize(dtype, weight_offset);", "double wo = weight_offset;"),
    "slot shifted": ("int64_t slot = pos % c->page_size;",
                     "int64_t slot = (pos + 1) % c->page_size;"),
    "radd halves swapped": ("double ak = orc_decode(dtype, a, row * a_row_stride + h * D + d);",
                            "double ak = orc_decode(dtype, a, row * a_row_stride + hidden + "
                            "h * D + d);"),
    "valid length off by one": ("if (s >= (int64_t)valid_lengths[b]) {",
                                "if (s > (int64_t)valid_lengths[b]) {"),
    "partial rope on the leading columns": (
        "return rope->rope_col_offset < 0 ? head_dim - rope->rope_dim : rope->rope_col_offset;",
        "return rope->rope_col_offset < 0 ? 0 : rope->rope_col_offset;"),
    "gemv epsilon outside the root": (
        "const double r = n_normed > 0 ? 1.0 / sqrt(ss / n_normed + eps) : 0.0;",
        "const double r = n_normed > 0 ? 1.0 / sqrt(ss / n_normed) + eps : 0.0;"),
    "gemv mean over every column": (
        "const double r = n_normed > 0 ? 1.0 / sqrt(ss / n_normed + eps) : 0.0;",
        "const double r = n_normed > 0 ? 1.0 / sqrt(ss / n + eps) : 0.0;"),
    "gemv norm taken over the tail": (
        "for (int64_t i = 0; i < n_normed; ++i) ss += y[i] * y[i];",
        "for (int64_t i = n - n_normed; i < n; ++i) ss += y[i] * y[i];"),
    "multiply after cast rounds after gamma": (
        "y[d] = multiply_before_cast ? y[d] * r * g : requantize(dtype, y[d] * r) * g;",
        "y[d] = multiply_before_cast ? y[d] * r * g : requantize(dtype, y[d] * r * g);"),
    "multiply after cast ignored": (
        "y[d] = multiply_before_cast ? y[d] * r * g : requantize(dtype, y[d] * r) * g;",
        "y[d] = y[d] * r * g;"),
    "e4m3 without saturation": ("  if (r > 448.0) r = 448.0;\n", "\n"),
    "e4m3 exponent bias": ("return sign | (uint8_t)((e - 1 + 7) << 3) | m;",
                           "return sign | (uint8_t)((e - 1 + 8) << 3) | m;"),
    "fp8 scale multiplied instead of divided": (
        "orc_encode(c->dtype, plane ? c->v : c->k, i, v / cache_scale(c, plane));",
        "orc_encode(c->dtype, plane ? c->v : c->k, i, v * cache_scale(c, plane));"),
    "gemv weight_offset consumed": (
        "orc_encode(dtype, normed_output, i, y[i] * r * orc_decode(dtype, gamma, i));",
        "orc_encode(dtype, normed_output, i, y[i] * r * (orc_decode(dtype, gamma, i) + "
        "weight_offset));"),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    src = open(os.path.join(ROOT, "oracle", "rope_oracle.c")).read()
    old, new = MUTANTS[name]
    assert old in src, f"mutation site for {name!r} not found"
    ign = shutil.ignore_patterns("*.so", "*.tmp", "__pycache__")
    for d in ("oracle", "workloads"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d, ignore=ign)
    os.makedirs(tmp_path / "tests")
    for f in ("conftest.py", "helpers.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), tmp_path / "tests" / f)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), tmp_path / "tests" / "golden")
    shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp_path / "pytest.ini")
    (tmp_path / "oracle" / "rope_oracle.c").write_text(src.replace(old, new, 1))
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py"], cwd=tmp_path, capture_output=True,
                       text=True, timeout=300)
    assert p.returncode == 1 and " failed" in p.stdout, (
        f"mutant {name!r} was not caught:\n{p.stdout[-2000:]}\n{p.stderr[-2000:]}")
