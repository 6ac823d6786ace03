"""The synthetic inputs have the structure the workloads state (no GPU):
positions, concentration R_f, heavy-norm outliers, determinism."""
import numpy as np
import pytest
import torch

import oracle
import synth


def test_dense_and_scattered_positions():
    dense = synth.make_positions(synth.SPECS["c2"], 2, 0, "cpu")
    assert torch.equal(dense[1], torch.arange(32768, dtype=torch.int32))
    c3 = synth.SPECS["c3"]
    pos = synth.make_positions(c3, 3, 0, "cpu").numpy()
    assert pos.shape == (3, c3.n_valid)
    assert np.all(np.diff(pos, axis=1) > 0)                    # strictly ascending
    assert pos.min() >= 0 and pos.max() == c3.p_cur - 1
    win = synth.STREAM_WINDOW
    assert np.array_equal(pos[:, -win:], np.tile(np.arange(c3.p_cur - win, c3.p_cur), (3, 1)))
    assert np.all(pos[:, :-win] < c3.p_cur - win)              # older keys before the window
    assert not np.array_equal(pos[0], pos[1])                   # units differ


def test_stream_window_positions():
    spec = synth.SPECS["c5"].scaled(n_seq=1, n_layers=1)
    hp = synth.head_params(spec)
    k, v, pos = synth.stream_window(spec, hp, 20, "cpu")
    assert k.shape == (spec.n_units, synth.STREAM_WINDOW, 128) and v.shape == k.shape
    assert torch.equal(pos[0], torch.arange(20 * 128, 21 * 128, dtype=torch.int32))


def test_concentration_matches_the_target_range():
    """c2: R_f ~ U[0.6, 1] per (head, band) through the Rician inversion of
    the noise; the oracle's calibration of the generated queries recovers it."""
    spec = synth.SPECS["c2"]
    hp = synth.head_params(spec)
    q = synth.calib_queries(spec, hp, 0, "cpu")
    R = oracle.calibrate(synth.host_elems(q))[..., 3]            # [Hq, 64]
    mag = np.abs(hp.q_centre[0])
    target = np.vectorize(synth.rician_R)(mag / hp.q_sigma[0])
    assert np.all((target >= 0.6 - 1e-9) & (target <= 1.0))
    assert np.max(np.abs(R - target)) < 0.05
    assert abs(R.mean() - 0.8) < 0.02


def test_heavy_norm_outliers_of_the_prefill_workload():
    """c4: 5 % of the keys are scaled x4 in norm (RoPE keeps norms)."""
    spec = synth.SPECS["c4"].scaled(n_layers=1)                # one layer's heads suffice
    hp = synth.head_params(spec)
    n = 20000
    pos = torch.arange(n, dtype=torch.int32).expand(2, n).contiguous()
    k, _ = synth.keys_values(spec, hp, 0, 2, pos, "cpu")
    norm = k.float().norm(dim=-1)
    frac = (norm > 2.5 * norm.median(dim=1, keepdim=True).values).float().mean().item()
    assert frac == pytest.approx(0.05, abs=0.006)


def test_generation_is_seeded():
    spec = synth.SPECS["c1"]
    a = synth.make_workload(spec, "cpu")
    b = synth.make_workload(spec, "cpu")
    assert torch.equal(a.k, b.k) and torch.equal(a.v, b.v) and torch.equal(a.pos, b.pos)
    c = synth.make_workload(spec.scaled(stream=spec.stream + 1), "cpu")
    assert not torch.equal(a.k, c.k)
