"""GPU parity: every libtri entry point against the float64 oracle on the
same seeded inputs.  Calls go through the C ABI (ctypes binding).

Small cases span several key tiles and a ragged tail; the workload configs
run at their full sizes in the launch configuration the benchmark times, with
the oracle checking every unit where it finishes in seconds and a fixed
sample of units otherwise.
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


def _spec(dtype="bf16", G=3, n_seq=2, n_layers=2, n_kvheads=2, cap=700, B=300, n_cal=3000,
          positions="dense", p_cur=None, R_range=(0.6, 1.0), stream=11, **kw):
    return synth.Spec("t", n_seq, n_layers, n_kvheads, G, cap, cap, B, dtype, n_cal,
                      p_cur if p_cur is not None else cap, positions=positions, R_range=R_range,
                      stream=stream, **kw)


def _ragged_nvalid(spec, B):
    U = spec.n_units
    choices = [spec.cap, spec.cap - 1, 0, 1, B, B + 1, 255, 256, 257, 513, spec.cap // 2]
    nv = np.array([choices[u % len(choices)] for u in range(U)], np.int32)
    return np.clip(nv, 0, spec.cap)


# ---------------------------------------------------------------------------
# calibration
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_calibrate_parity(dtype):
    spec = _spec(dtype=dtype, G=3, n_layers=2, n_kvheads=1, n_cal=3000)
    wl = synth.make_workload(spec, "cuda")
    gst, ost = H.stats_for(spec, wl)
    g = gst.cpu().numpy().astype(np.float64)
    scale = ost[..., 2:3]
    assert np.max(np.abs(g[..., :3] - ost[..., :3]) / scale) < 1e-6
    assert np.max(np.abs(g[..., 3] - ost[..., 3])) < 1e-6


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_calibrate_from_shard_sums(dtype):
    """Calibration tokens split over data-parallel shards (uneven, one shard
    smaller than a reduction chunk): the shards' float64 sums, added as an
    all-reduce would, give the statistics of the whole batch (oracle and
    tri_calibrate)."""
    spec = _spec(dtype=dtype, G=3, n_layers=2, n_kvheads=1, n_cal=3000)
    wl = synth.make_workload(spec, "cuda")
    q = synth.calib_queries(spec, wl.hp, 1, "cuda")          # [Hq, 3000, 128]
    whole = tri.tri_calibrate(q)
    cuts = [0, 700, 1337, 1337 + 500, 3000]
    total = sum(tri.tri_calibrate_sums(q[:, a:b].contiguous())
                for a, b in zip(cuts[:-1], cuts[1:]))
    stats = tri.tri_calibrate_finish(total, q.shape[1]).cpu().numpy().astype(np.float64)
    ost = oracle.calibrate(synth.host_elems(q))
    scale = ost[..., 2:3]
    assert np.max(np.abs(stats[..., :3] - ost[..., :3]) / scale) < 1e-6
    assert np.max(np.abs(stats[..., 3] - ost[..., 3])) < 1e-6
    w = whole.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(stats[..., :3] - w[..., :3]) / w[..., 2:3]) < 1e-6
    assert np.max(np.abs(stats[..., 3] - w[..., 3])) < 1e-6


def test_calibrate_data_parallel_over_nccl_one_rank():
    """The data-parallel helper through a real NCCL all-reduce (one rank on
    this GPU): the statistics equal tri_calibrate's."""
    import os
    import socket

    import torch.distributed as dist

    spec = _spec(dtype="bf16", G=3, n_layers=1, n_kvheads=1, n_cal=2048)
    wl = synth.make_workload(spec, "cuda")
    q = synth.calib_queries(spec, wl.hp, 0, "cuda")
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        got = tri.calibrate_data_parallel(q)
    finally:
        dist.destroy_process_group()
    ref = tri.tri_calibrate(q).cpu().numpy().astype(np.float64)
    got = got.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got[..., :3] - ref[..., :3]) / ref[..., 2:3]) < 1e-6
    assert np.max(np.abs(got[..., 3] - ref[..., 3])) < 1e-6


# ---------------------------------------------------------------------------
# score
# ---------------------------------------------------------------------------
def _score_case(spec, n_valid=None):
    wl = synth.make_workload(spec, "cuda")
    gst, ost = H.stats_for(spec, wl)
    nv = torch.as_tensor(n_valid if n_valid is not None else wl.n_valid.cpu().numpy(),
                         dtype=torch.int32, device="cuda")
    raw = torch.full((spec.n_units, spec.G, spec.cap), float("nan"), device="cuda")
    cfg = tri.config()
    _, fin = tri.tri_score(cfg, wl.k, spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G, wl.p_cur,
                           gst, n_valid=nv, raw=raw)
    torch.cuda.synchronize()
    return wl, ost, nv.cpu().numpy(), raw.cpu().numpy(), fin.cpu().numpy()


@pytest.mark.parametrize("dtype,G", [("bf16", 1), ("bf16", 3), ("bf16", 7), ("bf16", 8),
                                     ("f32", 1), ("f32", 4)])
def test_score_parity_ragged(dtype, G):
    spec = _spec(dtype=dtype, G=G, cap=700)
    nv = _ragged_nvalid(spec, 300)
    wl, ost, nv, raw, fin = _score_case(spec, nv)
    o = oracle.prune(synth.host_elems(wl.k), None, wl.pos.cpu().numpy(), spec.n_seq,
                     spec.n_layers, spec.n_kvheads, G, ost, wl.p_cur.cpu().numpy(), 300,
                     n_valid=nv, want_gather=False)
    for u in range(spec.n_units):
        n = int(nv[u])
        assert H.check_raw(raw[u], o["raw"][u], n) <= H.RAW_RTOL
        assert H.check_final(fin[u], o["final"][u], n) <= H.Z_RTOL


@pytest.mark.parametrize("name", ["c1", "c2"])
def test_score_parity_config(name):
    spec = synth.SPECS[name]
    wl, ost, nv, raw, fin = _score_case(spec)
    o = oracle.prune(synth.host_elems(wl.k), None, wl.pos.cpu().numpy(), spec.n_seq,
                     spec.n_layers, spec.n_kvheads, spec.G, ost, wl.p_cur.cpu().numpy(), spec.B,
                     n_valid=nv, want_gather=False)
    for u in range(spec.n_units):
        n = int(nv[u])
        assert H.check_raw(raw[u], o["raw"][u], n) <= H.RAW_RTOL
        assert H.check_final(fin[u], o["final"][u], n) <= H.Z_RTOL


# ---------------------------------------------------------------------------
# select
# ---------------------------------------------------------------------------
def _select_inputs(U, cap, seed):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(U, cap)).astype(np.float32)
    # Heavy ties and special values in some units.
    x[1] = np.round(x[1] * 2) / 2
    x[2, ::7] = np.nan
    x[2, 1::7] = -0.0
    x[2, 2::7] = 0.0
    x[3] = 1.5
    x[4, : cap // 2] = -np.inf
    return x


@pytest.mark.parametrize("B", [1, 7, 100, 2048, 4999, 5000, 6000])
def test_select_parity(B):
    U, cap = 6, 5000
    x = _select_inputs(U, cap, B)
    nv = np.array([cap, cap, cap, cap, cap, 3001], np.int32)
    fin = torch.as_tensor(x, device="cuda")
    kept, nk = tri.tri_select_topB(fin, B, n_valid=torch.as_tensor(nv, device="cuda"))
    kept, nk = kept.cpu().numpy(), nk.cpu().numpy()
    for u in range(U):
        n = int(nv[u])
        ok, _ = oracle.select(x[u, :n].astype(np.float64), B)
        assert nk[u] == len(ok)
        np.testing.assert_array_equal(kept[u, :len(ok)], ok)
        assert np.all(kept[u, len(ok):] == -1)


def test_select_large_units_exact():
    """Several CTAs per unit (the split path's chunking) with quantised ties."""
    U, cap, B = 3, 131072 + 77, 4096
    rng = np.random.default_rng(5)
    x = (np.round(rng.normal(size=(U, cap)) * 64) / 64).astype(np.float32)
    fin = torch.as_tensor(x, device="cuda")
    kept, nk = tri.tri_select_topB(fin, B)
    kept = kept.cpu().numpy()
    for u in range(U):
        ok, _ = oracle.select(x[u].astype(np.float64), B)
        np.testing.assert_array_equal(kept[u], ok)


# ---------------------------------------------------------------------------
# compact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_compact_bitwise(dtype):
    U, cap, B = 5, 1000, 333
    g = torch.Generator(device="cuda").manual_seed(3)
    k = torch.randn((U, cap, 128), generator=g, device="cuda").to(dtype)
    v = torch.randn((U, cap, 128), generator=g, device="cuda").to(dtype)
    pos = torch.randint(0, 1 << 30, (U, cap), generator=g, device="cuda", dtype=torch.int32)
    rng = np.random.default_rng(4)
    kept = np.full((U, B), -1, np.int32)
    nk = np.array([B, B, 0, 1, 200], np.int32)
    for u in range(U):
        kept[u, :nk[u]] = np.sort(rng.choice(cap, nk[u], replace=False))
    kd = torch.zeros((U, B, 128), dtype=dtype, device="cuda")
    vd = torch.zeros_like(kd)
    pd = torch.full((U, B), -7, dtype=torch.int32, device="cuda")
    tri.tri_compact(k, v, pos, torch.as_tensor(kept, device="cuda"), torch.as_tensor(nk, device="cuda"),
                    kd, vd, pd)
    torch.cuda.synchronize()
    for u in range(U):
        m = int(nk[u])
        assert H.rows_equal(kd[u, :m], k[u], kept[u, :m])
        assert H.rows_equal(vd[u, :m], v[u], kept[u, :m])
        assert torch.equal(pd[u, :m].cpu(), pos[u].cpu()[torch.as_tensor(kept[u, :m], dtype=torch.long)])
        assert torch.all(pd[u, m:] == -7)


# ---------------------------------------------------------------------------
# prune (score + select + compact)
# ---------------------------------------------------------------------------
ALL_PATHS = [tri.PATH_PIPE, tri.PATH_FUSED, tri.PATH_SPLIT, tri.PATH_COOP]


def _run_prune(spec, wl, gst, B, path=tri.PATH_AUTO, n_valid=None, cap_dst=None, cfg=None):
    U = spec.n_units
    cap_dst = cap_dst or B
    nv = n_valid if n_valid is not None else wl.n_valid
    kd = torch.zeros((U, cap_dst, 128), dtype=wl.k.dtype, device="cuda")
    vd = torch.zeros_like(kd)
    pd = torch.full((U, cap_dst), -1, dtype=torch.int32, device="cuda")
    kept = torch.empty((U, B), dtype=torch.int32, device="cuda")
    nk = torch.empty((U,), dtype=torch.int32, device="cuda")
    fin = torch.full((U, spec.cap), float("nan"), device="cuda")
    ws = tri.workspace(tri.tri_prune_workspace_bytes(spec.n_seq, spec.n_layers, spec.n_kvheads,
                                                     spec.G, spec.cap, B))
    cfg = cfg if cfg is not None else tri.config(path=path)
    if cfg.path != path:
        cfg.path = path
    tri.tri_prune(cfg, wl.k, wl.v, wl.pos, spec.n_seq, spec.n_layers,
                  spec.n_kvheads, spec.G, wl.p_cur, gst, B, kd, vd, pd, nk, n_valid=nv, kept=kept,
                  ws=ws, final=fin)
    flags = tri.tri_check_device_error(ws)
    return dict(k=kd, v=vd, pos=pd, kept=kept.cpu().numpy(), n_kept=nk.cpu().numpy(), flags=flags,
                final=fin.cpu().numpy())


def _check_prune(spec, wl, ost, out, B, nv, units, offsets=oracle.OFFSETS):
    if len(units) == spec.n_units:
        o = oracle.prune(synth.host_elems(wl.k), None, wl.pos.cpu().numpy(), spec.n_seq,
                         spec.n_layers, spec.n_kvheads, spec.G, ost, wl.p_cur.cpu().numpy(), B,
                         n_valid=nv, want_gather=False, want_raw=False, offsets=offsets)
    else:
        o = _oracle_units(spec, wl, ost, B, nv, units, offsets=offsets)
    mismatched = 0
    for u in units:
        n = int(nv[u])
        m = min(n, B)
        assert out["n_kept"][u] == m
        gk = out["kept"][u, :m]
        if n > B:
            # Final scores of every pruned unit: the stated 1e-4 relative bound.
            assert H.check_final(out["final"][u], o["final"][u], n) <= H.Z_RTOL, f"unit {u}"
        mismatched += H.check_kept(gk, o["final"][u], o["kept"][u], n, B)
        assert np.all(out["kept"][u, m:] == -1)
        assert H.rows_equal(out["k"][u, :m], wl.k[u], gk)
        assert H.rows_equal(out["v"][u, :m], wl.v[u], gk)
        assert np.array_equal(out["pos"][u, :m].cpu().numpy(), wl.pos[u].cpu().numpy()[gk])
    return mismatched


def _oracle_units(spec, wl, ost, B, nv, units, offsets=oracle.OFFSETS):
    """Oracle on a sample of units without copying the whole cache to the host:
    the sampled units that share a current position go to one oracle call as
    a stack of single-head "layers" (each with its own statistics), so the
    oracle's threads run over them."""
    U, cap = spec.n_units, spec.cap
    fin = np.full((U, cap), np.nan)
    kept = np.full((U, B), -1, np.int32)
    pc = wl.p_cur.cpu().numpy()
    Lh = spec.n_layers * spec.n_kvheads
    by_pcur = {}
    for u in units:
        by_pcur.setdefault(int(pc[u // Lh]), []).append(u)
    for p_cur, us in by_pcur.items():
        idx = torch.as_tensor(us, device=wl.k.device)
        kk = synth.host_elems(wl.k[idx])
        pp = wl.pos[idx].cpu().numpy()
        st = np.stack([ost[(u // spec.n_kvheads) % spec.n_layers,
                           (u % spec.n_kvheads) * spec.G:(u % spec.n_kvheads + 1) * spec.G]
                       for u in us])
        o = oracle.prune(kk, None, pp, 1, len(us), 1, spec.G, st, np.asarray([p_cur]), B,
                         n_valid=np.asarray([nv[u] for u in us]), want_gather=False,
                         want_raw=False, offsets=offsets)
        for i, u in enumerate(us):
            fin[u] = o["final"][i]
            kept[u] = o["kept"][i]
    return dict(final=fin, kept=kept)


@pytest.mark.parametrize("path", ALL_PATHS)
@pytest.mark.parametrize("dtype,G", [("bf16", 7), ("bf16", 4), ("bf16", 1), ("f32", 2)])
def test_prune_parity_ragged(path, dtype, G):
    B = 300
    spec = _spec(dtype=dtype, G=G, cap=700, B=B)
    wl = synth.make_workload(spec, "cuda")
    gst, ost = H.stats_for(spec, wl)
    nv = _ragged_nvalid(spec, B)
    out = _run_prune(spec, wl, gst, B, path=path, n_valid=torch.as_tensor(nv, device="cuda"))
    assert out["flags"] == 0
    mismatched = _check_prune(spec, wl, ost, out, B, nv, list(range(spec.n_units)))
    assert mismatched <= 2 * spec.n_units


def test_prune_paths_agree():
    """Every path computes the same per-key scores; their moment sums run in
    different fixed orders, so the kept sets may differ only on keys inside
    the oracle's exempt band around the B-th score, and gathered rows follow
    each path's own indices."""
    B = 900
    spec = _spec(dtype="bf16", G=7, cap=3200, B=B, n_seq=2, n_layers=2, n_kvheads=4,
                 positions="scattered", p_cur=32768)
    wl = synth.make_workload(spec, "cuda")
    gst, ost = H.stats_for(spec, wl)
    outs = [_run_prune(spec, wl, gst, B, path=p) for p in ALL_PATHS]
    o = oracle.prune(synth.host_elems(wl.k), None, wl.pos.cpu().numpy(), spec.n_seq,
                     spec.n_layers, spec.n_kvheads, spec.G, ost, wl.p_cur.cpu().numpy(), B,
                     want_gather=False, want_raw=False)
    for u in range(spec.n_units):
        fin = o["final"][u]
        T = fin[o["kept"][u]].min()
        band = np.abs(fin - T) <= H.BAND_RTOL * max(abs(T), 1.0)
        for other in outs[1:]:
            diff = np.setxor1d(outs[0]["kept"][u], other["kept"][u])
            assert np.all(band[diff]), f"unit {u}: paths differ outside the exempt band"
        for other in outs:
            assert H.rows_equal(other["k"][u], wl.k[u], other["kept"][u])
            assert H.rows_equal(other["v"][u], wl.v[u], other["kept"][u])
            assert H.check_final(other["final"][u], fin, spec.cap) <= H.Z_RTOL


def _heavy_units(wl, count):
    """Units with the most heavy-norm keys (norm above twice the unit's median)."""
    norms = wl.k.float().norm(dim=-1)
    med = norms.median(dim=1, keepdim=True).values
    heavy = (norms > 2.0 * med).sum(dim=1)
    return torch.topk(heavy, count).indices.cpu().tolist()


@pytest.mark.parametrize("name,sample", [("c1", None), ("c2", None), ("c3", 48), ("c5", 32),
                                         ("c4", 32)])
def test_prune_parity_config(name, sample):
    """Every workload configuration at its full size, in the launch the bench
    times (the path tri_prune picks); units sampled where the oracle would
    take too long on all of them: spread over sequences, layers and heads,
    and for the long-prefill workload a quarter of them the units with the
    most heavy-norm keys.  Final scores are compared on every sampled unit."""
    spec = synth.SPECS[name]
    wl = synth.make_workload(spec, "cuda")
    gst, ost = H.stats_for(spec, wl)
    out = _run_prune(spec, wl, gst, spec.B)
    assert out["flags"] == 0
    nv = wl.n_valid.cpu().numpy()
    if sample is None:
        units = list(range(spec.n_units))
    else:
        spread = sample - sample // 4 if spec.outlier_frac > 0 else sample
        units = set(np.linspace(0, spec.n_units - 1, spread).astype(int).tolist())
        if spec.outlier_frac > 0:
            units |= set(_heavy_units(wl, sample - len(units)))
        units = sorted(units)
    mismatched = _check_prune(spec, wl, ost, out, spec.B, nv, units)
    assert mismatched <= 2 * len(units)


def test_prune_default_paths():
    """The path tri_prune takes for each workload configuration."""
    want = {"c1": tri.PATH_COOP, "c2": tri.PATH_COOP, "c3": tri.PATH_PIPE, "c4": tri.PATH_SPLIT,
            "c5": tri.PATH_PIPE}
    for name, path in want.items():
        s = synth.SPECS[name]
        assert tri.tri_prune_path(s.n_seq, s.n_layers, s.n_kvheads, s.G, s.cap, s.B,
                                  s.torch_dtype) == path, name


@pytest.mark.parametrize("dtype,G", [("bf16", 4), ("bf16", 7), ("f32", 3)])
def test_prune_parity_pipe_large_units(dtype, G):
    """Units too large for one CTA's shared memory: the pipelined kernel
    scores them in chunks spread over all CTAs, and the CTA that completes a
    unit selects it.  Ragged valid counts: a full unit, one key short, one
    kept whole (n_valid <= B), an empty one, and one ending inside a chunk."""
    B = 1000
    cap = 30000
    spec = _spec(dtype=dtype, G=G, n_seq=1, n_layers=2, n_kvheads=3, cap=cap, B=B, n_cal=2048)
    wl = synth.make_workload(spec, "cuda")
    gst, ost = H.stats_for(spec, wl)
    nv = np.array([cap, cap - 1, B, 0, 25001, 1793], np.int32)
    out = _run_prune(spec, wl, gst, B, path=tri.PATH_PIPE, n_valid=torch.as_tensor(nv, device="cuda"))
    assert out["flags"] == 0
    mismatched = _check_prune(spec, wl, ost, out, B, nv, list(range(spec.n_units)))
    assert mismatched <= 2 * spec.n_units


@pytest.mark.parametrize("path", ALL_PATHS)
def test_prune_parity_linear_offsets(path):
    """A non-default offset set (linear offsets 1..37, the paper reading's
    ablation of the offset range): every path against the oracle evaluated
    with the same offsets."""
    B = 400
    offs = list(range(1, 38))
    spec = _spec(dtype="bf16", G=7, cap=1500, B=B, n_seq=2, n_layers=1, n_kvheads=2,
                 positions="scattered", p_cur=20000)
    wl = synth.make_workload(spec, "cuda")
    gst, ost = H.stats_for(spec, wl)
    out = _run_prune(spec, wl, gst, B, path=path, cfg=tri.config(offsets=offs))
    assert out["flags"] == 0
    nv = wl.n_valid.cpu().numpy()
    mismatched = _check_prune(spec, wl, ost, out, B, nv, list(range(spec.n_units)), offsets=offs)
    assert mismatched <= 2 * spec.n_units


@pytest.mark.parametrize("name,path", [("c2", tri.PATH_AUTO), ("c2", tri.PATH_SPLIT),
                                       ("c3", tri.PATH_AUTO)])
def test_prune_deterministic(name, path):
    spec = synth.SPECS[name]
    wl = synth.make_workload(spec, "cuda")
    gst, _ = H.stats_for(spec, wl)
    a = _run_prune(spec, wl, gst, spec.B, path=path)
    b = _run_prune(spec, wl, gst, spec.B, path=path)
    np.testing.assert_array_equal(a["kept"], b["kept"])
    assert torch.equal(a["k"], b["k"]) and torch.equal(a["v"], b["v"]) and torch.equal(a["pos"], b["pos"])


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("path", ALL_PATHS)
def test_identical_keys_keep_lowest_indices(path):
    """All keys equal: every head has sigma = 0, every z is 0, all scores tie,
    and the lowest B indices are kept."""
    spec = _spec(dtype="bf16", G=3, cap=1000, B=123)
    wl = synth.make_workload(spec, "cuda")
    wl.k[:] = wl.k[:, :1]
    gst, _ = H.stats_for(spec, wl)
    out = _run_prune(spec, wl, gst, 123, path=path)
    assert np.all(out["kept"] == np.arange(123)[None, :])


@pytest.mark.parametrize("path", [tri.PATH_COOP, tri.PATH_SPLIT, tri.PATH_PIPE])
def test_threshold_tie_group_beyond_candidate_list(path):
    """Keys alternate between two vectors, so with one head the z-scores take
    two values and the B-th key sits in a group of 9000 equal scores: more
    than the cooperative kernel's candidate list holds (8192), which sends it
    down its unit-wide radix path.  The keys of a group are equal, so their
    scores are equal (the key position cancels); the lowest-index keys of
    the higher group are kept.  The oracle evaluates each key's score at its
    own position and so differs inside a group only by float64 rounding: it
    fixes which group is higher, and that each group's scores agree."""
    B = 5000
    spec = _spec(dtype="bf16", G=1, n_seq=1, n_layers=1, n_kvheads=2, cap=18000, B=B)
    wl = synth.make_workload(spec, "cuda")
    wl.k[:, 0::2] = wl.k[:, :1]
    wl.k[:, 1::2] = wl.k[:, 1:2]
    gst, ost = H.stats_for(spec, wl)
    out = _run_prune(spec, wl, gst, B, path=path)
    assert out["flags"] == 0
    o = _oracle_units(spec, wl, ost, B, wl.n_valid.cpu().numpy(), list(range(spec.n_units)))
    for u in range(spec.n_units):
        even, odd = o["final"][u, 0::2], o["final"][u, 1::2]
        assert np.ptp(even) <= 1e-9 and np.ptp(odd) <= 1e-9 and abs(even[0] - odd[0]) > 1.0
        first = 0 if even[0] > odd[0] else 1
        np.testing.assert_array_equal(out["kept"][u], first + 2 * np.arange(B))
        assert H.rows_equal(out["k"][u], wl.k[u], out["kept"][u])
        assert H.rows_equal(out["v"][u], wl.v[u], out["kept"][u])


@pytest.mark.parametrize("path", ALL_PATHS)
def test_identical_keys_beyond_every_candidate_list(path):
    """17000 equal keys (sigma = 0, every score 0, one z-bin): more than the
    fused kernel's candidate list in a four-stage ring (15360) and the
    cooperative kernel's (8192), so both rank the tie in place; the lowest B
    indices are kept."""
    B = 6000
    spec = _spec(dtype="bf16", G=1, n_seq=1, n_layers=1, n_kvheads=1, cap=17000, B=B)
    wl = synth.make_workload(spec, "cuda")
    wl.k[:] = wl.k[:, :1]
    gst, _ = H.stats_for(spec, wl)
    out = _run_prune(spec, wl, gst, B, path=path)
    assert out["flags"] == 0
    np.testing.assert_array_equal(out["kept"][0], np.arange(B))
    assert H.rows_equal(out["v"][0], wl.v[0], np.arange(B))


@pytest.mark.parametrize("path", ALL_PATHS)
def test_nan_key_poisons_unit_and_flags(path):
    """A NaN key makes that unit's moments NaN: every final score is NaN,
    NaN ranks last and ties go to the lowest indices; the flag is raised.
    Other units are unaffected."""
    B = 50
    spec = _spec(dtype="bf16", G=2, cap=400, B=B)
    wl = synth.make_workload(spec, "cuda")
    wl.k[1, 17, 5] = float("nan")
    gst, ost = H.stats_for(spec, wl)
    out = _run_prune(spec, wl, gst, B, path=path)
    assert out["flags"] & tri.FLAG_NONFINITE
    assert np.array_equal(out["kept"][1], np.arange(B))
    o = _oracle_units(spec, wl, ost, B, wl.n_valid.cpu().numpy(), [0, 1])
    np.testing.assert_array_equal(o["kept"][1], np.arange(B))
    H.check_kept(out["kept"][0], o["final"][0], o["kept"][0], spec.cap, B)


def test_nvalid_out_of_range_is_flagged_and_clamped():
    spec = _spec(dtype="bf16", G=2, cap=400, B=50)
    wl = synth.make_workload(spec, "cuda")
    gst, _ = H.stats_for(spec, wl)
    nv = torch.full((spec.n_units,), 400, dtype=torch.int32, device="cuda")
    nv[3] = 401
    out = _run_prune(spec, wl, gst, 50, n_valid=nv)
    assert out["flags"] & tri.FLAG_NVALID_RANGE
    assert out["n_kept"][3] == 50


def test_budget_at_least_cache_keeps_everything():
    spec = _spec(dtype="bf16", G=7, cap=512, B=512)
    wl = synth.make_workload(spec, "cuda")
    gst, _ = H.stats_for(spec, wl)
    out = _run_prune(spec, wl, gst, 600, cap_dst=600)
    assert np.all(out["n_kept"] == 512)
    assert np.all(out["kept"][:, :512] == np.arange(512)[None])
    assert np.all(out["kept"][:, 512:] == -1)
    assert torch.equal(out["k"][:, :512], wl.k)
