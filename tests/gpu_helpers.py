"""Shared helpers of the GPU parity tests: run the library, run the oracle on
the same bytes, and compare with the tolerances the acceptance criteria fix.

Tolerances (floating point, float32 accumulation on the GPU vs float64):
  raw per-head S~:  |gpu - ora| <= 1e-4 * max(|ora|, rms_j ora)   (scores cross 0)
  final z-max:      |gpu - ora| <= 1e-4 * max(1, |ora|)
Kept sets are compared exactly except for keys whose oracle final score lies
within 1e-4 * max(|T|, 1) of the B-th score T (the exempt band); the gathered
K/V/position rows must be the source rows at the GPU's own kept indices, bit
for bit.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import rope_aware_kv_b200 as tri
import synth

RAW_RTOL = 1e-4
Z_RTOL = 1e-4
BAND_RTOL = 1e-4


def stats_for(spec, wl, device="cuda"):
    """GPU calibration of every layer: [L, Hq, 64, 4] float32 (library), and the
    oracle's float64 calibration of the same queries."""
    gst = torch.empty((spec.n_layers, spec.n_qheads, 64, 4), dtype=torch.float32, device=device)
    ost = np.empty((spec.n_layers, spec.n_qheads, 64, 4))
    for layer in range(spec.n_layers):
        q = synth.calib_queries(spec, wl.hp, layer, device)
        tri.tri_calibrate(q, stats=gst[layer])
        ost[layer] = oracle.calibrate(synth.host_elems(q))
    torch.cuda.synchronize()
    return gst, ost


def check_raw(gpu_raw, ora_raw, n):
    """gpu_raw, ora_raw [G, >=n]."""
    g = gpu_raw[:, :n].astype(np.float64)
    o = ora_raw[:, :n]
    rms = np.sqrt(np.mean(o * o, axis=1, keepdims=True)) if n else np.ones((o.shape[0], 1))
    scale = np.maximum(np.abs(o), rms)
    err = np.abs(g - o) / scale
    return float(err.max()) if n else 0.0


def check_final(gpu_fin, ora_fin, n):
    g = gpu_fin[:n].astype(np.float64)
    o = ora_fin[:n]
    if n == 0:
        return 0.0
    both_nan = np.isnan(g) & np.isnan(o)
    err = np.where(both_nan, 0.0, np.abs(g - o) / np.maximum(1.0, np.abs(o)))
    return float(np.nan_to_num(err, nan=np.inf).max())


def check_kept(gpu_kept, ora_fin, ora_kept, n, B):
    """Compare kept sets with the exempt band.  Returns the number of keys on
    which the two sets differ (all of them inside the band)."""
    m = min(n, B)
    gk = np.asarray(gpu_kept[:m])
    assert len(gk) == m
    assert np.all(np.diff(gk) > 0), "kept indices not strictly ascending"
    assert m == 0 or (gk[0] >= 0 and gk[-1] < n)
    if m == n:
        assert np.array_equal(gk, np.arange(n))
        return 0
    ok = np.asarray(ora_kept[:m])
    fin = ora_fin[:n]
    T = fin[ok].min() if not np.isnan(fin[ok]).all() else np.nan
    if np.isnan(T):
        # every kept score is NaN: ranking is by index alone
        assert np.array_equal(gk, ok)
        return 0
    band = np.abs(fin - T) <= BAND_RTOL * max(abs(T), 1.0)
    gset = np.zeros(n, bool)
    gset[gk] = True
    oset = np.zeros(n, bool)
    oset[ok] = True
    diff = gset != oset
    assert not np.any(diff & ~band), (
        f"kept sets differ outside the exempt band at {np.nonzero(diff & ~band)[0][:10]}")
    return int(diff.sum())


def rows_equal(dst, src, idx):
    """dst [m, d] rows equal src[idx] bit for bit (tensors on any device)."""
    a = dst.contiguous().cpu().view(torch.uint8).numpy() if isinstance(dst, torch.Tensor) else dst
    b = src.contiguous().cpu() if isinstance(src, torch.Tensor) else torch.as_tensor(src)
    b = b[torch.as_tensor(np.asarray(idx, np.int64))].view(torch.uint8).numpy()
    return np.array_equal(a, b)
