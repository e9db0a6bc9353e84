"""Plant a mistake in a copy of the oracle and check that the pins catch it.

Each case rewrites one line of ``oracle/moe_oracle.cpp`` in a temporary copy
of the repository (CPU only), rebuilds the copy's oracle and runs
``tests/test_oracle_pins.py`` against it in a subprocess. The pins must FAIL
for every planted mistake; the unmodified copy must pass.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "no_chunking": ("constexpr int64_t kChunk = 128;", "constexpr int64_t kChunk = 1 << 30;"),
    "mul_then_add": ("p[e] = std::fma(xi, w[e], p[e]);", "p[e] = xi * w[e] + p[e];"),
    "ties_to_higher_index": ("order[e] = static_cast<int32_t>(e);",
                             "order[e] = static_cast<int32_t>(E - 1 - e);"),
    "weights_renormalised": ("w[t * k + j] = std::exp(static_cast<double>(l[e]) - m) / s;",
                             "w[t * k + j] = std::exp(static_cast<double>(l[e]) - m) / (s * 0.0 + 1.0 + "
                             "std::exp(static_cast<double>(l[order[k - 1]]) - m));"),
    "gate_up_swapped": ("const double g = gu[r * f2 + j], u = gu[r * f2 + f + j];",
                        "const double u = gu[r * f2 + j], g = gu[r * f2 + f + j];"),
    "silu_sign": ("const double silu = g / (1.0 + std::exp(-g));",
                  "const double silu = g / (1.0 + std::exp(g));"),
    "down_transposed": ("wrow[c] = bf16_to_double(Wd[j * d + c]);",
                        "wrow[c] = bf16_to_double(Wd[(c % f) * d + (j + c / f) % d]);"),
    "combine_drops_last_slot": ("for (int64_t j = 0; j < k; ++j) {\n      const double* yr = y_rows",
                                "for (int64_t j = 0; j < k - 1; ++j) {\n      const double* yr = y_rows"),
    "permute_descending_tokens": ("const int32_t r = cursor[e]++;",
                                  "const int32_t r = offsets[e + 1] - 1 - (cursor[e]++ - offsets[e]);"),
    "bias_dropped": ("l[e] = l[e] + bias[e];", "l[e] = l[e] + 0.0f * bias[e];"),
    "mxfp4_ties_to_odd_code": ("kE2M1Mag[c]);\n    if (dist < bd || (dist == bd && (c & 1) == 0)) {",
                               "kE2M1Mag[c]);\n    if (dist < bd || (dist == bd && (c & 1) == 1)) {"),
    "mxfp8_ties_to_odd_code": ("e4m3_mag(c));\n    if (dist < bd || (dist == bd && (c & 1) == 0)) {",
                               "e4m3_mag(c));\n    if (dist < bd || (dist == bd && (c & 1) == 1)) {"),
    "mxfp4_scale_one_too_small": ("s = std::min(127, std::max(-127, e - 1 - 2));",
                                  "s = std::min(127, std::max(-127, e - 1 - 1));"),
    "mxfp4_sign_dropped": ("static_cast<uint8_t>((std::signbit(v) ? 8 : 0) | mag);",
                           "static_cast<uint8_t>(mag);"),
    "mxfp4_subnormal_value": ("const double kE2M1Mag[8] = {0.0, 0.5, 1.0,",
                              "const double kE2M1Mag[8] = {0.0, 0.25, 1.0,"),
    "mxfp8_scale_one_too_large": ("s = std::min(127, std::max(-127, e - 1 - 8));",
                                  "s = std::min(127, std::max(-127, e - 1 - 7));"),
    "mxfp8_subnormal_exponent": ("return e == 0 ? std::ldexp(m / 8.0, -6)", "return e == 0 ? std::ldexp(m / 8.0, -7)"),
    "mx_ffn_h_not_requantised": ("if (!st) st = oracle_mxfp8_dequantize(hc.data(), hs.data(), 1, f, hrow.data());",
                                 "if (!st) st = 0;"),
    "mx_ffn_gate_up_swapped": ("const double g = gu[j], u = gu[f + j];", "const double u = gu[j], g = gu[f + j];"),
    "mxfp8_nan_code_allowed": ("for (int c = 1; c < 127; ++c) {", "for (int c = 1; c < 128; ++c) {"),
    "mxfp8_dequant_scale_off_by_one": ("std::ldexp(e4m3_mag(c & 0x7f), static_cast<int>(q) - 127)",
                                       "std::ldexp(e4m3_mag(c & 0x7f), static_cast<int>(q) - 126)"),
    "qb_cutoff_is_kth_not_k_plus_first": ("std::greater<double>());\n    alpha[i] = v[k];",
                                          "std::greater<double>());\n    alpha[i] = v[k - 1];"),
    "qb_quantile_rank_floor": ("int64_t r = (m * k + n - 1) / n;", "int64_t r = (m * k) / n;"),
    "qb_bias_sign": ("b_new[j] = -mu[r - 1];", "b_new[j] = mu[r - 1];"),
    "qb_histogram_upper_edge": ("b_new[j] = -(lo + static_cast<double>(bin) * width);",
                                "b_new[j] = -(lo + static_cast<double>(bin + 1) * width);"),
    "situ_cap_ignored": ("if (act == 0) return silu(g) * v;", "if (act >= 0) return silu(g) * v;"),
    "situ_gate_without_sigmoid": ("return b1 * std::tanh(silu(g) / b1) * (b2 * std::tanh(v / b2));",
                                  "return b1 * std::tanh(g / b1) * (b2 * std::tanh(v / b2));"),
    "rmsnorm_without_sqrt": ("const double den = std::sqrt(ss / static_cast<double>(l) + eps);",
                             "const double den = ss / static_cast<double>(l) + eps;"),
    "latent_down_projection_shifted": ("z[t * l + c] += xi * bf16_to_double(Wdn[i * l + c]);",
                                       "z[t * l + c] += xi * bf16_to_double(Wdn[((i + 1) % d) * l + c]);"),
    "latent_combine_unweighted": ("u[t * l + c] += w[t * k + j] * yr[c];", "u[t * l + c] += yr[c];"),
    "latent_shared_experts_dropped": ("for (int64_t q = 0; q < T * d; ++q) out[q] += ys[q];",
                                      "for (int64_t q = 0; q < T * d; ++q) out[q] += 0.0 * ys[q];"),
}


def _copy_repo(dst):
    for sub in ("oracle", "tests"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(dst, sub),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__", "*.tmp*"))
    pkg = os.path.join(dst, "sparse_mixture_experts_route_b200")
    os.makedirs(pkg)
    for fn in ("__init__.py", "inputs.py"):
        shutil.copy(os.path.join(ROOT, "sparse_mixture_experts_route_b200", fn), pkg)


def _run_pins(dst):
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1", OMP_NUM_THREADS="4")
    return subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                           os.path.join(dst, "tests", "test_oracle_pins.py")],
                          cwd=dst, env=env, capture_output=True, text=True, timeout=600)


def test_unmodified_copy_passes(tmp_path):
    _copy_repo(str(tmp_path))
    r = _run_pins(str(tmp_path))
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    _copy_repo(str(tmp_path))
    src = os.path.join(str(tmp_path), "oracle", "moe_oracle.cpp")
    text = open(src).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not unique/found"
    open(src, "w").write(text.replace(old, new))
    r = _run_pins(str(tmp_path))
    assert r.returncode != 0, f"planted mistake '{name}' was not caught by the pins"
    assert "failed" in r.stdout or "Error" in r.stdout, r.stdout[-2000:]
