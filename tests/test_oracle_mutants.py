"""The pins must catch plausible mistakes in the oracle.

Each case compiles a copy of the oracle's C source with one deliberate,
plausible mistake planted (on the CPU, in a temporary directory) and checks
that at least one pin of ``test_oracle_pins`` fails against it.  The pinned
oracle itself is untouched.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
from tests import test_oracle_pins as pins
from tests import test_oracle_variants as var

SRC = os.path.join(os.path.dirname(oracle.__file__), "tri_oracle.c")

# (name, text in the source, replacement)
MUTANTS = [
    ("omega exponent -f/d", "pow(theta, -2.0 * (double)f / (double)d)",
     "pow(theta, -1.0 * (double)f / (double)d)"),
    ("half-split pairing", "*y = ora_decode(base, dtype, row + 2 * f + 1);",
     "*y = ora_decode(base, dtype, row + (2 * f + 1 + d / 2) % d);"),
    ("phase sign", "const double phi = qarg[f] - karg[f];", "const double phi = karg[f] - qarg[f];"),
    ("de-rotation direction", "const double x = c * xr + s * yr;", "const double x = c * xr - s * yr;"),
    ("Delta sign", "(double)(p_cur - (int64_t)pos[j] + offsets[o])",
     "(double)((int64_t)pos[j] - p_cur + offsets[o])"),
    ("no 1/|D|", "use_max ? best : total / (double)n_off;", "use_max ? best : total;"),
    ("R weight on the wrong side", "(use_r ? 1.0 - st[f * 4 + 3] : 1.0)",
     "(use_r ? st[f * 4 + 3] : 1.0)"),
    # method variants
    ("no-trig keeps S_trig", "if (use_trig) s_trig +=", "if (1) s_trig +="),
    ("no-R keeps the R factor", "(use_r ? 1.0 - st[f * 4 + 3] : 1.0)",
     "(1.0 - st[f * 4 + 3])"),
    ("max over offsets takes the min", "if (s_trig + s_norm > best) best = s_trig + s_norm;",
     "if (best == -INFINITY || s_trig + s_norm < best) best = s_trig + s_norm;"),
    ("max over offsets drops S_norm", "if (s_trig + s_norm > best) best = s_trig + s_norm;",
     "if (s_trig > best) best = s_trig;"),
    ("half-split pairs f with f + d/2 - 1", "*y = ora_decode(base, dtype, row + f + d / 2);",
     "*y = ora_decode(base, dtype, row + (f + d / 2 - 1 + d) % d);"),
    ("post-RoPE calibration rotates forward", "const double xr = c * x + sn_ * y;",
     "const double xr = c * x - sn_ * y;"),
    ("recent window one short", "if (j < n_sink || j >= n - n_recent) kept[p++] = (int32_t)j;",
     "if (j < n_sink || j > n - n_recent) kept[p++] = (int32_t)j;"),
    ("protected keys ignored", "const int64_t rest = m - p;", "const int64_t rest = m - p; p = 0;"),
    ("attention skips the max shift", "const double w = exp(sc[j] - mx);",
     "const double w = exp(sc[j] - mx) * (j == 0 ? 2.0 : 1.0);"),
    ("attention scale dropped", "sc[j] = scale * dot;", "sc[j] = dot;"),
    ("attention over one row too few", "for (int64_t j = 0; j < n; ++j) {\n                const int64_t krow",
     "for (int64_t j = 0; j + 1 < n; ++j) {\n                const int64_t krow"),
    ("reconstruction phase sign", "- atan2(ks[f * 4 + 1], ks[f * 4]);",
     "+ atan2(ks[f * 4 + 1], ks[f * 4]);"),
    ("curve pairs the key after the query", "ora_decode(k, dtype, (kh * n_tok + t - D) * (int64_t)d + e);",
     "ora_decode(k, dtype, (kh * n_tok + (t - D + 1 < n_tok ? t - D + 1 : t - D)) * (int64_t)d + e);"),
    ("curve uses KV head h", "const int64_t kh = h / G;", "const int64_t kh = h % (n_qheads / G);"),
    ("pearson without centring", "sxy += (x[i] - mx) * (y[i] - my);", "sxy += x[i] * y[i];"),
    ("layer budget of the next layer", "const int64_t Bu = layer_budget ? layer_budget[layer] : B;",
     "const int64_t Bu = layer_budget ? layer_budget[(layer + 1) % n_layers] : B;"),
    ("sample sigma", "sqrt(ss / (double)n)", "sqrt(ss / (double)(n > 1 ? n - 1 : 1))"),
    ("mean over heads", "for (int h = 1; h < G; ++h) m = fmax(m, z[(int64_t)h * n + j]);",
     "for (int h = 1; h < G; ++h) m += z[(int64_t)h * n + j]; m /= G;"),
    ("ties to highest index", "return (a->idx < b->idx) ? -1 : (a->idx > b->idx);",
     "return (a->idx > b->idx) ? -1 : (a->idx < b->idx);"),
    ("NaN ranks highest", "if (a->nan != b->nan) return a->nan ? 1 : -1;",
     "if (a->nan != b->nan) return a->nan ? -1 : 1;"),
    ("gather off by one", "const int64_t src = u * cap + kp[rr];",
     "const int64_t src = u * cap + kp[rr] + (kp[rr] + 1 < n ? 1 : 0);"),
    ("mean norm uses |mean|", "sn += hypot(x, y);", "sn += fabs(x) + fabs(y);"),
    ("head max keeps a leading NaN", "for (int h = 1; h < G; ++h) m = fmax(m, z[(int64_t)h * n + j]);",
     "for (int h = 1; h < G; ++h) m = (z[(int64_t)h * n + j] > m) ? z[(int64_t)h * n + j] : m;"),
    ("head max takes a later NaN", "for (int h = 1; h < G; ++h) m = fmax(m, z[(int64_t)h * n + j]);",
     "for (int h = 1; h < G; ++h) m = (m > z[(int64_t)h * n + j]) ? m : z[(int64_t)h * n + j];"),
]

PIN_TESTS = [
    lambda: pins.test_zero_noise_calibration_recovers_centre_and_R1(),
    lambda: [pins.test_strig_equals_explicit_rope_logit(o) for o in [(1,), (65536,), (3, 1000), oracle.OFFSETS]],
    lambda: pins.test_strig_single_band_closed_form(),
    lambda: pins.test_R_zero_gives_pure_norm_score(),
    lambda: pins.test_offset_fold_equals_direct_sum(),
    lambda: pins.test_linear_offsets_geometric_closed_form(),
    lambda: pins.test_znorm_population_moments_and_max(),
    lambda: pins.test_znorm_max_skips_a_nan_head(),
    lambda: [pins.test_select_matches_brute_force(s) for s in range(12)],
    lambda: pins.test_select_order_and_threshold(),
    lambda: [pins.test_prune_gather_is_bitwise_and_ascending(dt) for dt in ("f32", "bf16")],
    lambda: pins.test_unit_phasor_MRL_matches_R(),
    lambda: var.test_no_trig_is_blind_to_band_phases(),
    lambda: var.test_no_trig_with_concentrated_queries_is_zero(),
    lambda: var.test_no_r_score_bounds(),
    lambda: var.test_no_r_equals_default_for_centreless_queries(),
    lambda: [var.test_max_over_offsets_equals_explicit_rope_logit_max(o)
             for o in [(1,), (3, 1000), oracle.OFFSETS]],
    lambda: var.test_max_over_offsets_bounds_the_mean(),
    lambda: var.test_half_split_is_a_relabelling_of_interleaved(),
    lambda: var.test_post_rope_calibration_recovers_pre_rope_stats(),
    lambda: [var.test_protected_selection_matches_brute_force(s) for s in range(8)],
    lambda: var.test_layer_budgets_equal_single_budget_runs(),
    lambda: var.test_decode_attention_matches_library_sdpa(),
    lambda: var.test_decode_attention_special_cases(),
    lambda: var.test_logit_reconstruction_is_the_rotated_centres_dot_product(),
    lambda: var.test_logit_curve_of_centred_sequences_equals_reconstruction(),
    lambda: var.test_pearson_matches_numpy(),
]


def test_unmutated_source_passes_every_pin():
    for t in PIN_TESTS:
        t()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique for {name}"
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", str(so), str(path),
                    "-lm"], check=True)
    failed = 0
    with oracle.using_library(str(so)):
        for t in PIN_TESTS:
            try:
                t()
            except AssertionError:
                failed += 1
    assert failed > 0, f"no pin caught the mutant '{name}'"
