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

SRC = os.path.join(os.path.dirname(oracle.__file__), "tri_oracle.c")

# (name, text in the source, replacement)
MUTANTS = [
    ("omega exponent -f/d", "pow(theta, -2.0 * (double)f / (double)d)",
     "pow(theta, -1.0 * (double)f / (double)d)"),
    ("half-split pairing", "const double yr = ora_decode(k, dtype, j * d + 2 * f + 1);",
     "const double yr = ora_decode(k, dtype, j * d + (2 * f + 1 + d / 2) % d);"),
    ("phase sign", "const double phi = qarg[f] - karg[f];", "const double phi = karg[f] - qarg[f];"),
    ("de-rotation direction", "const double x = c * xr + s * yr;", "const double x = c * xr - s * yr;"),
    ("Delta sign", "(double)(p_cur - (int64_t)pos[j] + offsets[o])",
     "(double)((int64_t)pos[j] - p_cur + offsets[o])"),
    ("no 1/|D|", "raw[(int64_t)h * n + j] = total / (double)n_off;", "raw[(int64_t)h * n + j] = total;"),
    ("R weight on the wrong side", "qnw[f] = (1.0 - st[f * 4 + 3]) * st[f * 4 + 2];",
     "qnw[f] = st[f * 4 + 3] * st[f * 4 + 2];"),
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
