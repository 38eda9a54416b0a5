"""Planted-mistake check of the oracle's pins (CPU only).

Each mutant is a copy of ``oracle/sla_oracle.c`` with one plausible mistake
(a dropped term, a wrong sign or index, a transposed operand, a wrong rounding
rule).  The copy is compiled into a temporary library and every pin of
``test_oracle_pins`` is run against it; at least one pin must fail.  The
mistakes are planted in the oracle only, on the CPU.
"""
from __future__ import annotations

import os
import subprocess
import tempfile

import pytest

import oracle
from test_oracle_pins import PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "sla_oracle.c")

MUTANTS = {
    "drop_inv_sqrt_d": ("double inv_sqrt_d = 1.0 / sqrt((double)d);", "double inv_sqrt_d = 1.0;"),
    "linear_over_selected": ("if (r < k_sel && sel[r] == J) { ++r; continue; }",
                             "if (!(r < k_sel && sel[r] == J)) continue; ++r;"),
    "transposed_state": ("num += pq[c] * HI[(size_t)c * d + e];", "num += pq[c] * HI[(size_t)e * d + c];"),
    "tie_prefers_higher_block": ("return (x->j > y->j) - (x->j < y->j);", "return (x->j < y->j) - (x->j > y->j);"),
    "ceil_count": ("double x = floor(topk * (double)n_kb + 1e-4);", "double x = ceil(topk * (double)n_kb - 1e-4);"),
    "pool_divides_by_block": ("mean[(size_t)J * d + c] = s / (double)(t1 - t0);", "mean[(size_t)J * d + c] = s / (double)blk;"),
    "scale_over_128": ("const float qmax = fp8 ? 448.0f : 127.0f;", "const float qmax = fp8 ? 448.0f : 128.0f;"),
    "fp8_scale_over_240": ("const float qmax = fp8 ? 448.0f : 127.0f;", "const float qmax = fp8 ? 240.0f : 127.0f;"),
    "e4m3_exponent_bias_8": ("int e = E - 1 + 7;", "int e = E - 1 + 8;"),
    "e4m3_round_half_up": ("double r = nearbyint(ldexp(a, -qexp));", "double r = floor(ldexp(a, -qexp) + 0.5);"),
    "e4m3_no_subnormals": ("int qexp = a < ldexp(1.0, -6) ? -9 : (E - 1) - 3;", "int qexp = (E - 1) - 3;"),
    "rowquant_sum_not_mean": ("float ms = (float)(ss / (double)cols);", "float ms = (float)ss;"),
    "rowquant_eps_outside_sqrt": ("float den = sqrtf(ms + eps);", "float den = sqrtf(ms) + eps;"),
    "rowquant_gamma_dropped": ("if (gamma) v = v * gamma[c];", "(void)gamma;"),
    "w8a8_weight_scale_dropped": ("double v = (double)acc * (double)sx[m] * (double)sw[n];", "double v = (double)acc * (double)sx[m];"),
    "w8a8_bias_subtracted": ("if (bias) v += (double)bias[n];", "if (bias) v -= (double)bias[n];"),
    "fp8_logits_raw_bytes": ("acc += e4m3_value((uint8_t)q8[(size_t)i * d + c]) * e4m3_value((uint8_t)k8[(size_t)j * d + c]);",
                             "acc += (double)q8[(size_t)i * d + c] * e4m3_value((uint8_t)k8[(size_t)j * d + c]);"),
    "no_smoothing": ("mu[c] = (float)(s / (double)N);", "mu[c] = 0.0f;"),
    "softmax_unnormalised": ("for (int e = 0; e < d; ++e) os[e] /= den;", "(void)den;"),
    "elu_without_plus_one": ("return x > 0.0 ? x + 1.0 : exp(x);", "return x > 0.0 ? x : exp(x) - 1.0;"),
    "combine_minus": ("out[(size_t)o * d + e] = os[e] + ol[e];", "out[(size_t)o * d + e] = os[e] - ol[e];"),
    "drop_key_scale": ("l = (double)acc * (double)sq[I] * (double)sk[J] * inv_sqrt_d;",
                       "l = (double)acc * (double)sq[I] * inv_sqrt_d;"),
    "truncating_round": ("float r = rintf(x / s);", "float r = truncf(x / s);"),
    "score_key_index_swap": ("s = fma(qm[(size_t)I * d + c], km[(size_t)J * d + c], s);",
                             "s = fma(qm[(size_t)I * d + c], km[(size_t)((J + 1) % n_kb) * d + c], s);"),
    "bwd_softmax_drops_D": ("double ds = p[n] * (dp - D);", "double ds = p[n] * dp;"),
    "bwd_dk_unscaled": ("dk[(size_t)j * d + c] += ds * qi[c] * rsd;", "dk[(size_t)j * d + c] += ds * qi[c];"),
    "bwd_db_sign": ("double db = -dol / b;", "double db = dol / b;"),
    "bwd_dH_transposed": ("dHI[(size_t)c * d + e] += f[c] * da[e];", "dHI[(size_t)e * d + c] += f[c] * da[e];"),
    "bwd_key_side_over_selected": ("if (selected[(size_t)I * n_kb + J]) continue;",
                                   "if (!selected[(size_t)I * n_kb + J]) continue;"),
    "bwd_dv_linear_transposed": ("dv[(size_t)j * d + e] += G[(size_t)c * d + e] * fk;",
                                 "dv[(size_t)j * d + e] += G[(size_t)e * d + c] * fk;"),
    "bwd_elu_derivative_one": ("return x > 0.0 ? 1.0 : exp(x);\n}\n\nstatic int backward_head",
                               "return 1.0;\n}\n\nstatic int backward_head"),
    "bwd_dq_linear_without_dphi": ("dq[(size_t)i * d + c] += df * dphi_f(qi[c], phi);", "dq[(size_t)i * d + c] += df;"),
    "bwd_dz_dropped": ("double dfk = gz[c];", "double dfk = 0.0;"),
    "ragged_tail_dropped": ("int t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;\n        for (int j = t0; j < t1; ++j) {\n            double l;",
                            "int t0 = J * blk_k, t1 = t0 + blk_k <= N ? t0 + blk_k : t0;\n        for (int j = t0; j < t1; ++j) {\n            double l;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    search, replace = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(search) == 1, f"mutation site for {name} not unique in the oracle"
    mutated = src.replace(search, replace)
    with tempfile.TemporaryDirectory() as tmp:
        c_path = os.path.join(tmp, "mutant.c")
        so_path = os.path.join(tmp, "mutant.so")
        with open(c_path, "w") as f:
            f.write(mutated)
        subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", so_path, c_path, "-lm"])
        lib = oracle.load(so_path)
        caught = []
        for pin in PINS:
            try:
                pin(lib)
            except AssertionError:
                caught.append(pin.__name__)
            except (ValueError, IndexError, MemoryError, FloatingPointError):
                caught.append(pin.__name__)
        assert caught, f"no pin catches the planted mistake {name}"
