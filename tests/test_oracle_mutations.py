"""Each plausible mistake planted in a copy of the oracle must fail a pin.

The mutants are built from oracle/milo_oracle.c with one textual change each
(a dropped term, a wrong sign, a swapped index, a wrong tie-break ...), compiled
into a temporary directory, and the pin suite is run against them in a child
process.  The real oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "milo_oracle.c")

MUTANTS = {
    "dequant_sign": ("wrow[k] = ((double)codes[k] - z) * s;", "wrow[k] = (z - (double)codes[k]) * s;"),
    "drop_lorc": ("J->Y[(size_t)m * J->N + n] = acc + lorc;", "J->Y[(size_t)m * J->N + n] = acc;"),
    "transposed_U": ("milo_ref_h2d(P->U[(size_t)n * r + p])", "milo_ref_h2d(P->U[(size_t)p * N + n])"),
    "int3_u_scale_zero_swapped": ("dequant_row(P->Uq, P->Us, P->Uz, r, N, group, p, urow);",
                                  "dequant_row(P->Uq, P->Uz, P->Us, r, N, group, p, urow);"),
    "int3_v_not_quantised": ("dequant_row(P->Vq, P->Vs, P->Vz, r, K, group, p, Vd + (size_t)p * K);",
                             "for (int k = 0; k < K; ++k) Vd[(size_t)p * K + k] = milo_ref_h2d(P->V[(size_t)p * K + k]);"),
    "int3_u_untransposed": ("for (int n = 0; n < N; ++n) Ud[(size_t)n * r + p] = urow[n];",
                            "for (int n = 0; n < N; ++n) Ud[(size_t)n * r + p] = urow[(size_t)(n * r + p) % N];"),
    "zero_not_negated": ("float z_f = -mn / s;", "float z_f = mn / s;"),
    "scale_by_8": ("float s_f = range / 7.0f;", "float s_f = range / 8.0f;"),
    "round_half_up": ("float r = nearbyintf(v);    /* ties to even */", "float r = floorf(v + 0.5f);"),
    "tie_to_higher_id": ("milo_ref_h2d(l[e]) > milo_ref_h2d(l[best])", "milo_ref_h2d(l[e]) >= milo_ref_h2d(l[best])"),
    "renorm_over_all": ("if (renorm) {", "if (0) {"),
    "unit_group_swap": ("int c = rr / 16, m = rr % 16 + 16 * half;", "int c = rr / 16, m = rr % 16 + 16 * (1 - half);"),
    "spare_bits_swapped": ("pos = (m == 30) ? 15 : 31;", "pos = (m == 30) ? 31 : 15;"),
    "hi_lo_swapped": ("pos = 16 * (within % 2) + 3 * (within / 2) + beta;", "pos = 16 * (1 - within % 2) + 3 * (within / 2) + beta;"),
    "scale_index_transposed": ("scale[(size_t)j * J->N + n]", "scale[(size_t)n * (J->K / J->group) + j]"),
    "silu_sign": ("return a / (1.0 + exp(-a));", "return a / (1.0 + exp(a));"),
    "h_not_rounded": ("h[i] = milo_ref_h2d(h_bits[i]);", "h[i] = milo_ref_silu(a[i]) * b[i];"),
    "combine_drops_weight": ("acc += w[f] * y_slot[(size_t)f * H + n];", "acc += y_slot[(size_t)f * H + n];"),
    "shared_dropped": ("for (int s = 0; s < S; ++s) acc += y_sh[((size_t)s * T + t) * H + n];", ""),
    "gather_wrong_token": ("X + (size_t)(rows[m] / k) * H", "X + (size_t)(rows[m] % T) * H"),
    "perm_descending": ("int p = offsets[e] + count[e]++;", "int p = offsets[e + 1] - 1 - count[e]++;"),
    "f2h_truncate": ("double m = nearbyint(ldexp(a, 10 - e));", "double m = floor(ldexp(a, 10 - e));"),
    "hqq_shrink_without_sqrt": ("float d = sqrtf(a);", "float d = a;"),
    "hqq_shrink_sign": ("if (m > 0.0f) w_e = e < 0.0f ? -m : m;", "if (m > 0.0f) w_e = e < 0.0f ? m : -m;"),
    "hqq_kappa_ignored": ("beta = beta * kappa;", "beta = beta * 1.0f;"),
    "hqq_mean_over_63": ("z = acc * 0.015625f;", "z = acc / 63.0f;"),
    "hqq_best_zero_not_kept": ("best_err = err;\n            best_z = z;", "best_err = err;"),
    "hqq_l2_error": ("err = err + a;", "err = err + a * a;"),
    "hqq_scale_index_transposed": ("sz = (size_t)j * J->N + n;", "sz = (size_t)n * (J->K / 64) + j;"),
    "swiglu_gate_swapped": ("double v = milo_ref_silu(a[i]) * b[i];", "double v = milo_ref_silu(b[i]) * a[i];"),
    "bf16_read_as_fp16": ("X[i] = x_is_bf16 ? milo_ref_bf2d(x[i]) : milo_ref_h2d(x[i]);",
                          "X[i] = milo_ref_h2d(x[i]);"),
    "h_overflow_not_flagged": ("else if (!isfinite(h[i])) status |= REF_FP16_RANGE;", ";"),
    "d2h_binade_carry_lost": ("if (m == 2048.0) { m = 1024.0; e += 1; }", "if (m == 2048.0) { m = 2047.0; }"),
    "codes_clamped_at_6": ("/* also maps NaN to 0 */\n                if (r > 7.0f) r = 7.0f;",
                           "/* also maps NaN to 0 */\n                if (r > 6.0f) r = 6.0f;"),
    "zero_point_unrounded": ("float z = h2f(z_h);", "float z = z_f;"),
    "tile_pack_rows_j_and_j8_swapped": ("int q = i * 128 + ((r / 16) * 8 + r % 8) * 4 + ((r % 16) / 8) * 2;",
                                        "int q = i * 128 + ((r / 16) * 8 + r % 8) * 4 + (1 - (r % 16) / 8) * 2;"),
    "tile_pack_scale_zero_swapped": ("groups[q] = scale[(size_t)g * N + n];\n                    groups[q + 1] = zero[(size_t)g * N + n];",
                                     "groups[q] = zero[(size_t)g * N + n];\n                    groups[q + 1] = scale[(size_t)g * N + n];"),
    "int3_compensator_scale_index_transposed": ("double s = milo_ref_h2d(sc[(size_t)j * R + p]);",
                                                "double s = milo_ref_h2d(sc[(size_t)p * (Cc / group) + j]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found once"
    mutated = src.replace(old, new)
    c_path = tmp_path / "mutant.c"
    so_path = tmp_path / "mutant.so"
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fPIC",
                           "-shared", "-pthread", str(c_path), "-o", str(so_path), "-lm"])
    env = dict(os.environ, MILO_ORACLE_LIB=str(so_path))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        os.path.join(ROOT, "tests", "test_oracle_lorc_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
