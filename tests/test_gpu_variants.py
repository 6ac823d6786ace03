"""Method variants on the GPU against the oracle's variants, through the C ABI.

Ablations (shibing624 paper reading, ablation section): the score without
S_trig, without the concentration weight; the maximum over the future offsets
(its future-offset paragraph); half-split band pairing; protected sink /
recent keys (jaedaily.cn tutorial, streaming section); per-layer budgets
(same tutorial, budget paragraph); calibration of post-RoPE queries.
Same tolerances as the main parity tests: final scores 1e-4 relative, kept
sets exact outside the exempt band, gathered rows bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import rope_aware_kv_b200 as tri
import synth
from rope_aware_kv_b200 import build as tri_build
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tri_build.build()
    tri.load()
    oracle.build()
    yield
    torch.cuda.empty_cache()


def _spec(dtype="bf16", G=3, n_seq=2, n_layers=2, n_kvheads=2, cap=700, B=300, stream=31):
    return synth.Spec("t", n_seq, n_layers, n_kvheads, G, cap, cap, B, dtype, 3000, cap,
                      R_range=(0.6, 1.0), stream=stream)


def _ragged(spec, B):
    choices = [spec.cap, spec.cap - 1, 0, 1, B, B + 1, 257, spec.cap // 2]
    return np.clip(np.array([choices[u % len(choices)] for u in range(spec.n_units)], np.int32),
                   0, spec.cap)


def _stats(spec, wl, half=False):
    """GPU calibration with the config's pairing, and the oracle's."""
    cfg = tri.config(variant=tri.VAR_HALF_SPLIT if half else 0)
    gst = torch.empty((spec.n_layers, spec.n_qheads, 64, 4), dtype=torch.float32, device="cuda")
    ost = np.empty((spec.n_layers, spec.n_qheads, 64, 4))
    for layer in range(spec.n_layers):
        q = synth.calib_queries(spec, wl.hp, layer, "cuda")
        tri.tri_calibrate_ex(cfg, q, stats=gst[layer])
        ost[layer] = oracle.calibrate(synth.host_elems(q), half=half)
    torch.cuda.synchronize()
    return gst, ost


def _prune(spec, wl, gst, B, cfg, nv):
    U = spec.n_units
    kd = torch.zeros((U, B, 128), dtype=wl.k.dtype, device="cuda")
    vd = torch.zeros_like(kd)
    pd = torch.full((U, B), -1, dtype=torch.int32, device="cuda")
    kept = torch.empty((U, B), dtype=torch.int32, device="cuda")
    nk = torch.empty((U,), dtype=torch.int32, device="cuda")
    fin = torch.full((U, spec.cap), float("nan"), device="cuda")
    ws = tri.workspace(tri.tri_prune_workspace_bytes(spec.n_seq, spec.n_layers, spec.n_kvheads,
                                                     spec.G, spec.cap, B))
    tri.tri_prune(cfg, wl.k, wl.v, wl.pos, spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G,
                  wl.p_cur, gst, B, kd, vd, pd, nk, n_valid=torch.as_tensor(nv, device="cuda"),
                  kept=kept, ws=ws, final=fin)
    flags = tri.tri_check_device_error(ws)
    return dict(k=kd, v=vd, pos=pd, kept=kept.cpu().numpy(), n_kept=nk.cpu().numpy(),
                final=fin.cpu().numpy(), flags=flags)


def _check(spec, wl, out, o, B, nv, budgets=None, n_sink=0, n_recent=0):
    """Kept sets (protected keys as +inf in the oracle's final), final scores
    of the unprotected keys, the gathered rows."""
    mismatched = 0
    for u in range(spec.n_units):
        n = int(nv[u])
        Bu = B if budgets is None else min(B, budgets[(u // spec.n_kvheads) % spec.n_layers])
        m = min(n, Bu)
        assert out["n_kept"][u] == m, f"unit {u}"
        gk = out["kept"][u, :m]
        assert np.all(out["kept"][u, m:] == -1)
        fo = o["final"][u].copy()
        prot = np.zeros(spec.cap, bool)
        prot[:min(n_sink, n)] = True
        prot[max(n - n_recent, 0):n] = True
        if n > Bu and Bu > 0:
            free = ~prot[:n]
            g = out["final"][u, :n]
            assert H.check_final(g[free], fo[:n][free], int(free.sum())) <= H.Z_RTOL, f"unit {u}"
            assert np.all(np.isposinf(g[prot[:n]]))
        fo[prot] = np.inf
        mismatched += H.check_kept(gk, fo, o["kept"][u], n, Bu)
        assert H.rows_equal(out["k"][u, :m], wl.k[u], gk)
        assert H.rows_equal(out["v"][u, :m], wl.v[u], gk)
        assert np.array_equal(out["pos"][u, :m].cpu().numpy(), wl.pos[u].cpu().numpy()[gk])
    return mismatched


@pytest.mark.parametrize("path", [tri.PATH_PIPE, tri.PATH_FUSED, tri.PATH_COOP, tri.PATH_SPLIT])
@pytest.mark.parametrize("variant", [tri.VAR_NO_TRIG, tri.VAR_NO_R, tri.VAR_NO_TRIG | tri.VAR_NO_R])
def test_ablations_every_path(path, variant):
    B = 300
    spec = _spec(G=3, cap=700, B=B)
    wl = synth.make_workload(spec, "cuda")
    gst, ost = _stats(spec, wl)
    nv = _ragged(spec, B)
    out = _prune(spec, wl, gst, B, tri.config(path=path, variant=variant), nv)
    assert out["flags"] == 0
    o = oracle.prune(synth.host_elems(wl.k), None, wl.pos.cpu().numpy(), spec.n_seq,
                     spec.n_layers, spec.n_kvheads, spec.G, ost, wl.p_cur.cpu().numpy(), B,
                     n_valid=nv, want_gather=False, want_raw=False, variant=variant)
    assert _check(spec, wl, out, o, B, nv) <= 2 * spec.n_units


@pytest.mark.parametrize("dtype,G", [("bf16", 4), ("f32", 2)])
@pytest.mark.parametrize("variant", [tri.VAR_MAX_OFFSET, tri.VAR_HALF_SPLIT,
                                     tri.VAR_MAX_OFFSET | tri.VAR_HALF_SPLIT,
                                     tri.VAR_MAX_OFFSET | tri.VAR_NO_R])
def test_score_variants_split_path(dtype, G, variant):
    """Max over the offsets and half-split pairing (the split path): raw
    per-head scores of tri_score and the whole prune step, against the oracle."""
    B = 300
    spec = _spec(dtype=dtype, G=G, cap=700, B=B)
    wl = synth.make_workload(spec, "cuda")
    half = bool(variant & tri.VAR_HALF_SPLIT)
    gst, ost = _stats(spec, wl, half=half)
    nv = _ragged(spec, B)
    offsets = (1, 2, 4, 8, 16, 64, 512, 4096, 65536) if variant & tri.VAR_MAX_OFFSET else None
    cfg = tri.config(variant=variant, offsets=offsets)
    U = spec.n_units
    raw = torch.full((U, G, spec.cap), float("nan"), device="cuda")
    fin = torch.full((U, spec.cap), float("nan"), device="cuda")
    nvt = torch.as_tensor(nv, device="cuda")
    tri.tri_score(cfg, wl.k, spec.n_seq, spec.n_layers, spec.n_kvheads, G, wl.p_cur, gst,
                  final=fin, raw=raw, n_valid=nvt)
    offs = offsets if offsets is not None else oracle.OFFSETS
    o = oracle.prune(synth.host_elems(wl.k), None, wl.pos.cpu().numpy(), spec.n_seq,
                     spec.n_layers, spec.n_kvheads, G, ost, wl.p_cur.cpu().numpy(), B,
                     n_valid=nv, want_gather=False, want_raw=True, variant=variant, offsets=offs)
    raw_h = raw.cpu().numpy()
    for u in range(U):
        n = int(nv[u])
        assert H.check_raw(raw_h[u], o["raw"][u], n) <= H.RAW_RTOL, f"unit {u}"
    out = _prune(spec, wl, gst, B, cfg, nv)
    assert out["flags"] == 0
    assert _check(spec, wl, out, o, B, nv) <= 2 * U
    # a forced path without these variants is refused
    for path in (tri.PATH_PIPE, tri.PATH_FUSED, tri.PATH_COOP):
        with pytest.raises(tri.TriError):
            _prune(spec, wl, gst, B, tri.config(variant=variant, offsets=offsets, path=path), nv)


@pytest.mark.parametrize("path", [tri.PATH_PIPE, tri.PATH_SPLIT, tri.PATH_AUTO])
@pytest.mark.parametrize("n_sink,n_recent", [(4, 128), (0, 300), (7, 0)])
def test_protected_keys(path, n_sink, n_recent):
    B = 300
    spec = _spec(G=7, cap=700, B=B)
    wl = synth.make_workload(spec, "cuda")
    gst, ost = _stats(spec, wl)
    nv = _ragged(spec, B)
    cfg = tri.config(path=path, n_sink=n_sink, n_recent=n_recent)
    out = _prune(spec, wl, gst, B, cfg, nv)
    assert out["flags"] == 0
    o = oracle.prune(synth.host_elems(wl.k), None, wl.pos.cpu().numpy(), spec.n_seq,
                     spec.n_layers, spec.n_kvheads, spec.G, ost, wl.p_cur.cpu().numpy(), B,
                     n_valid=nv, want_gather=False, want_raw=False, n_sink=n_sink,
                     n_recent=n_recent)
    assert _check(spec, wl, out, o, B, nv, n_sink=n_sink, n_recent=n_recent) <= 2 * spec.n_units
    for u in range(spec.n_units):
        n, m = int(nv[u]), int(out["n_kept"][u])
        prot = [j for j in range(n) if j < n_sink or j >= n - n_recent]
        assert set(prot[:m]) <= set(out["kept"][u, :m].tolist())
    for bad in (tri.PATH_FUSED, tri.PATH_COOP):
        with pytest.raises(tri.TriError):
            _prune(spec, wl, gst, B, tri.config(path=bad, n_sink=n_sink, n_recent=n_recent), nv)


@pytest.mark.parametrize("path", [tri.PATH_PIPE, tri.PATH_SPLIT])
@pytest.mark.parametrize("cap,B", [(700, 300), (70000, 1500)])
def test_layer_budgets(path, cap, B):
    n_layers = 3
    budgets = [B, 37, 0]
    n_seq = 1 if cap > 10000 else 2
    spec = _spec(G=4, n_seq=n_seq, n_layers=n_layers, n_kvheads=1, cap=cap, B=B)
    wl = synth.make_workload(spec, "cuda")
    gst, ost = _stats(spec, wl)
    nv = _ragged(spec, B) if cap < 10000 else np.array([cap, cap - 1, cap - 7], np.int32)
    lb = torch.tensor(budgets, dtype=torch.int32, device="cuda")
    cfg = tri.config(path=path, layer_budget=lb)
    out = _prune(spec, wl, gst, B, cfg, nv)
    assert out["flags"] == 0
    o = oracle.prune(synth.host_elems(wl.k), None, wl.pos.cpu().numpy(), spec.n_seq, n_layers,
                     spec.n_kvheads, spec.G, ost, wl.p_cur.cpu().numpy(), B, n_valid=nv,
                     want_gather=False, want_raw=False, layer_budget=budgets)
    assert _check(spec, wl, out, o, B, nv, budgets=budgets) <= 2 * spec.n_units


def test_calibrate_post_rope_and_half_split():
    """Post-RoPE queries with their positions give the pre-RoPE statistics
    (oracle: rotated back in float64); half-split pairing as the oracle's."""
    spec = _spec(G=2, n_layers=1, n_kvheads=2)
    hp = synth.head_params(spec)
    q = synth.calib_queries(spec, hp, 0, "cuda")               # [Hq, n, 128] pre-RoPE
    n = q.shape[1]
    pos = torch.randint(0, 30000, (n,), generator=torch.Generator(device="cuda").manual_seed(2),
                        device="cuda", dtype=torch.int32)
    qpost = synth.rope_rotate(q.double(), pos.expand(q.shape[0], n)).to(q.dtype)
    for half in (False, True):
        cfg = tri.config(variant=tri.VAR_HALF_SPLIT if half else 0)
        g = tri.tri_calibrate_ex(cfg, qpost, q_pos=pos).cpu().numpy().astype(np.float64)
        o = oracle.calibrate(synth.host_elems(qpost), pos=pos.cpu().numpy(), half=half)
        scale = o[..., 2:3]
        assert np.max(np.abs(g[..., :3] - o[..., :3]) / scale) < 1e-5
        assert np.max(np.abs(g[..., 3] - o[..., 3])) < 1e-5
