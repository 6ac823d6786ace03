"""The folded weight record layout (CPU, nvcc only).

The fold writes, per query head and 16-byte key chunk, the offset-averaged
rotated centre A_f = E[q_f] e^{i w_f p_cur} C_f and the norm weight
c_f = (1 - R_f) E|q_f| of four bands (talk page: S_trig, S_norm and the
offset-averaged score); the score loops read them back as packed pairs.
This builds tests/host/wrec_layout_check.cu for the host and runs it: every
band's real part, imaginary part and norm weight must sit where both the
bf16 and the float32 score loops read them, and the 3 x 64 slots must tile
the 192-float record exactly.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def _nvcc():
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return cand if os.path.exists(cand) else None


def test_weight_record_layout(tmp_path):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not available")
    exe = str(tmp_path / "wrec_layout_check")
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    os.path.join(HERE, "host", "wrec_layout_check.cu"), "-o", exe],
                   check=True, capture_output=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"
