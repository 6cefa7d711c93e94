"""The pins must catch plausible mistakes: each case below plants one mistake
in a copy of the oracle's C source (on the CPU), builds it, and runs the pin
tests against it; at least one pin has to fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ssmq_oracle.c")
PINS = ["tests/test_oracle_quantizers.py", "tests/test_oracle_scans.py",
        "tests/test_calibration.py", "tests/test_oracle_conv.py"]

MUTANTS = {
    "m1_drop_Dx": ("if (p->D) acc += (double)p->D[c] * x;\n    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[idx]));\n    if (o->y) o->y[k * L + t] = acc;",
                   "if (0) acc += (double)p->D[c] * x;\n    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[idx]));\n    if (o->y) o->y[k * L + t] = acc;"),
    "m1_decay_sign": ("h[n] = exp(delta * (double)p->A[c * N + n]) * h[n] + delta * Bv * x;\n      acc += Cv * h[n];\n    }\n    if (p->D) acc += (double)p->D[c] * x;\n    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[idx]));\n    if (o->y)",
                      "h[n] = exp(-delta * (double)p->A[c * N + n]) * h[n] + delta * Bv * x;\n      acc += Cv * h[n];\n    }\n    if (p->D) acc += (double)p->D[c] * x;\n    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[idx]));\n    if (o->y)"),
    "m1_swap_BC": ("const double Bv = (double)p->B[bi] * (double)p->B_scale[si];\n      const double Cv = (double)p->C[bi] * (double)p->C_scale[si];\n      h[n] = exp(delta * (double)p->A[c * N + n]) * h[n] + delta * Bv * x;\n      acc += Cv * h[n];\n    }\n    if (p->D) acc += (double)p->D[c] * x;\n    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[idx]));\n    if (o->y)",
                   "const double Cv = (double)p->B[bi] * (double)p->B_scale[si];\n      const double Bv = (double)p->C[bi] * (double)p->C_scale[si];\n      h[n] = exp(delta * (double)p->A[c * N + n]) * h[n] + delta * Bv * x;\n      acc += Cv * h[n];\n    }\n    if (p->D) acc += (double)p->D[c] * x;\n    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[idx]));\n    if (o->y)"),
    "m1_group_index": ("const int64_t b = u / d, c = u % d, g = c * G / d;\n  const int64_t spg = N / p->state_group_size;\n  double* h = (double*)malloc",
                       "const int64_t b = u / d, c = u % d, g = c % G;\n  const int64_t spg = N / p->state_group_size;\n  double* h = (double*)malloc"),
    "quant_round_exact_quotient": ("float r = (float)((double)v / (double)step);\n  double k = nearbyint((double)r);",
                                   "double r = (double)v / (double)step;\n  double k = nearbyint(r);"),
    "quant_round_half_away": ("double k = nearbyint((double)r);", "double k = round((double)r);"),
    "quant_clamp_128": ("if (k < -(double)lim) k = -(double)lim;", "if (k < -(double)lim - 1) k = -(double)lim - 1;"),
    "softedge_le_threshold": ("if (a < thr_lo)\n      mode = ORC_MODE_SMALL;", "if (a <= thr_lo)\n      mode = ORC_MODE_SMALL;"),
    "softedge_payload_7bit_small": ("c = (uint8_t)(0x80 | (qv & 0x3F));", "c = (uint8_t)(0x80 | (qv & 0x7F));"),
    "softedge_ratio_swapped": ("if (mode == ORC_MODE_SMALL) f = ldexp(1.0, -r);", "if (mode == ORC_MODE_SMALL) f = ldexp(1.0, r);"),
    "ssd_group_index": ("const int64_t b = u / H, hd = u % H, g = hd * G / H;\n  const int64_t spg = N / p->state_group_size;\n  double* h = (double*)malloc((size_t)(P * N) * sizeof(double));\n  double* Bv",
                        "const int64_t b = u / H, hd = u % H, g = hd % G;\n  const int64_t spg = N / p->state_group_size;\n  double* h = (double*)malloc((size_t)(P * N) * sizeof(double));\n  double* Bv"),
    "ssd_decay_after_input": ("h[pp * N + n] = dA * h[pp * N + n] + delta * Bv[n] * x;\n        acc += Cv[n] * h[pp * N + n];\n      }\n      if (p->D) acc += (double)p->D[hd] * x;\n      if (p->z) acc *= orc_silu(orc_half_to_double(p->z[xi]));\n      if (o->y) o->y[(k * L + t) * P + pp] = acc;",
                              "h[pp * N + n] = dA * (h[pp * N + n] + delta * Bv[n] * x);\n        acc += Cv[n] * h[pp * N + n];\n      }\n      if (p->D) acc += (double)p->D[hd] * x;\n      if (p->z) acc *= orc_silu(orc_half_to_double(p->z[xi]));\n      if (o->y) o->y[(k * L + t) * P + pp] = acc;"),
    "chunked_drop_carry_decay": ("double acc = yd + exp(S[t]) * yo;", "double acc = yd + yo;"),
    "silu_sign": ("return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    "softplus_dropped_log": ("return v > 0.0 ? v + log1p(exp(-v)) : log1p(exp(v));", "return v > 0.0 ? v : exp(v);"),
    "cluster_scale_from_min": ("scales[j] = (float)(a[hi - 1].v / 127.0);", "scales[j] = (float)(a[lo].v / 127.0);"),
    "percentile_no_interp": ("return vk + frac * (vk1 - vk);", "return vk;"),
    "decode_drop_D": ("if (p->D) acc += (double)p->D[hd] * x;\n    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[xi]));\n    if (o->y) o->y[k * P + pp] = acc;",
                      "if (0) acc += (double)p->D[hd] * x;\n    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[xi]));\n    if (o->y) o->y[k * P + pp] = acc;"),
    "half_subnormal": ("v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);"),
    "m1_output_before_update": ("h[n] = exp(delta * (double)p->A[c * N + n]) * h[n] + delta * Bv * x;\n      acc += Cv * h[n];",
                                "acc += Cv * h[n];\n      h[n] = exp(delta * (double)p->A[c * N + n]) * h[n] + delta * Bv * x;"),
    "ssd_bc_scale_index": ("const int64_t si = g * spg + n / p->state_group_size;\n      Bv[n] = (double)p->B[bi] * (double)p->B_scale[si];",
                           "const int64_t si = g * spg + n % p->state_group_size;\n      Bv[n] = (double)p->B[bi] * (double)p->B_scale[si];"),
    "softedge_ge_hi": ("else if (a > thr_hi)", "else if (a >= thr_hi)"),
    "absmax_div_128": ("scales[g] = (float)(amax[g] / 127.0);", "scales[g] = (float)(amax[g] / 128.0);"),
    "m1_gate_before_D": ("    if (p->D) acc += (double)p->D[c] * x;\n    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[idx]));\n    if (o->y) o->y[k * L + t] = acc;",
                         "    if (p->z) acc *= orc_silu(orc_half_to_double(p->z[idx]));\n    if (p->D) acc += (double)p->D[c] * x;\n    if (o->y) o->y[k * L + t] = acc;"),
    "bias_after_softplus": ("  double v = dtv + bias;\n  return softplus ? orc_softplus(v) : v;",
                            "  double v = dtv;\n  return (softplus ? orc_softplus(v) : v) + bias;"),
    "decode_group_index": ("  const int64_t b = u / H, hd = u % H, g = hd * G / H;\n  const int64_t spg = N / p->state_group_size;\n  const double delta = orc_delta(orc_half_to_double(p->dt[b * H + hd]),",
                           "  const int64_t b = u / H, hd = u % H, g = hd % G;\n  const int64_t spg = N / p->state_group_size;\n  const double delta = orc_delta(orc_half_to_double(p->dt[b * H + hd]),"),
    "percentile_signed": ("if (isfinite(f)) v[m++] = fabs((double)f);", "if (isfinite(f)) v[m++] = (double)f;"),
    "percentile_position_n": ("const double pos = (double)(m - 1) * (q / 100.0);",
                              "const double pos = (double)m * (q / 100.0);"),
    "conv_taps_reversed": ("a = fmaf(weight[c * W + k], xv, a);",
                           "a = fmaf(weight[c * W + (W - 1 - k)], xv, a);"),
    "conv_bias_dropped": ("float a = bias ? bias[c] : 0.0f;", "float a = 0.0f;"),
    "conv_state_order": ("xv = (float)orc_half_to_double(pr[S + s]);",
                         "xv = (float)orc_half_to_double(pr[-s - 1]);"),
    "conv_state_out_shift": ("const int64_t s = seqlen - S + j; /* time of state slot j */",
                             "const int64_t s = seqlen - S + j - 1; /* time of state slot j */"),
    "exp_taylor_coefficient": ("p = fmaf(p, r, (float)(1.0 / 120.0));",
                               "p = fmaf(p, r, (float)(1.0 / 100.0));"),
    "exp_ln2_lo_dropped": ("r = fmaf(-kf, ln2_lo, r);", "r = fmaf(-kf, 0.0f, r);"),
    "silu_f32_sign": ("const float e = orc_exp_f32(-a);", "const float e = orc_exp_f32(a);"),
    "ssd_bias_dropped": ("orc_delta(orc_half_to_double(p->dt[(b * L + t) * H + hd]),\n                                   p->dt_bias ? (double)p->dt_bias[hd] : 0.0, p->dt_softplus);\n    const double dA",
                         "orc_delta(orc_half_to_double(p->dt[(b * L + t) * H + hd]),\n                                   0.0, p->dt_softplus);\n    const double dA"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not unique / missing: " + name
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-I",
                           os.path.join(ROOT, "oracle"), "-o", str(lib), str(mut), "-lm",
                           "-lpthread"])
    env = dict(os.environ, SSMQ_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *PINS], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "pins did not catch mutant " + name
