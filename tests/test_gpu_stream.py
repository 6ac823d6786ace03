"""The windowed driver: append each window of 128 generated tokens, prune the
cache back to B, swap the two cache buffers (hyper.ai summary, Method
section: prune every 128 generated tokens).

tri_append is checked for exact placement, n_valid / p_cur bookkeeping and
the overflow flag; a short stream shaped like the streaming workload (B 2048,
cap B + 128, GQA 28/4 with G = 7) is checked against the oracle at every
prune step, on the very cache state the GPU pruned.
"""
import numpy as np
import pytest
import torch

import oracle
import rope_aware_kv_b200 as tri
import synth
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from rope_aware_kv_b200 import build

    build.build()
    tri.load()
    oracle.build()


def test_append_places_rows_and_flags_overflow():
    n_seq, U, cap, n_new = 2, 6, 300, 5
    g = torch.Generator(device="cuda").manual_seed(5)
    k = torch.randn((U, cap, 128), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((U, cap, 128), generator=g, device="cuda").to(torch.bfloat16)
    pos = torch.randint(0, 1 << 20, (U, cap), generator=g, device="cuda", dtype=torch.int32)
    k0, v0, pos0 = k.clone(), v.clone(), pos.clone()
    nv0 = [10, 0, 296, 295, 150, 1]           # unit 2 would overflow (296 + 5 > 300)
    nv = torch.tensor(nv0, dtype=torch.int32, device="cuda")
    k_new = torch.randn((U, n_new, 128), generator=g, device="cuda").to(torch.bfloat16)
    v_new = torch.randn((U, n_new, 128), generator=g, device="cuda").to(torch.bfloat16)
    pos_new = (4000 + torch.arange(n_new, device="cuda", dtype=torch.int32))[None, :].repeat(U, 1)
    pos_new[4, 2] = 7000                       # the largest position of sequence 1
    p_cur = torch.zeros((n_seq,), dtype=torch.int64, device="cuda")
    ws = tri.workspace(256)
    tri.tri_append(k, v, pos, n_seq, nv, k_new, v_new, pos_new, p_cur=p_cur, ws=ws)
    flags = tri.tri_check_device_error(ws)
    assert flags & tri.FLAG_NVALID_RANGE
    nv_out = nv.cpu().tolist()
    for u in range(U):
        n = nv0[u]
        if u == 2:
            assert nv_out[u] == n
            assert torch.equal(k[u], k0[u]) and torch.equal(v[u], v0[u])
            assert torch.equal(pos[u], pos0[u])
            continue
        assert nv_out[u] == n + n_new
        assert torch.equal(k[u, n:n + n_new], k_new[u]) and torch.equal(v[u, n:n + n_new], v_new[u])
        assert torch.equal(pos[u, n:n + n_new], pos_new[u])
        assert torch.equal(k[u, :n], k0[u, :n]) and torch.equal(k[u, n + n_new:], k0[u, n + n_new:])
        assert torch.equal(v[u, :n], v0[u, :n]) and torch.equal(pos[u, :n], pos0[u, :n])
    assert p_cur.cpu().tolist() == [4000 + n_new, 7001]


def test_append_nothing_is_a_no_op():
    U, cap = 2, 16
    k = torch.zeros((U, cap, 128), dtype=torch.bfloat16, device="cuda")
    nv = torch.tensor([3, 4], dtype=torch.int32, device="cuda")
    empty = torch.zeros((U, 0, 128), dtype=torch.bfloat16, device="cuda")
    ws = tri.workspace(256)
    tri.tri_append(k, None, None, 1, nv, empty, None, None, ws=ws)
    assert tri.tri_check_device_error(ws) == 0
    assert nv.cpu().tolist() == [3, 4]
    assert not torch.any(k.view(torch.int16))


def test_stream_windows_match_oracle():
    """Three windows of the streaming workload's shape (2 sequences x 2 layers
    x 4 KV heads, G = 7, cap 2176, B 2048): each step appends 128 new tokens
    to the pruned cache and prunes it again; every step's kept sets and rows
    are checked against the oracle run on the cache the GPU pruned."""
    spec = synth.SPECS["c5"].scaled(n_seq=2, n_layers=2)
    U, cap, B, G = spec.n_units, spec.cap, spec.B, spec.G
    wl = synth.make_workload(spec, "cuda")
    gst, ost = H.stats_for(spec, wl)
    cur = dict(k=wl.k, v=wl.v, pos=wl.pos, nv=wl.n_valid.clone(), p_cur=wl.p_cur.clone())
    nxt = dict(k=torch.zeros_like(wl.k), v=torch.zeros_like(wl.v),
               pos=torch.full_like(wl.pos, -1))
    n_kept = torch.empty((U,), dtype=torch.int32, device="cuda")
    kept = torch.empty((U, B), dtype=torch.int32, device="cuda")
    ws = tri.workspace(tri.tri_prune_workspace_bytes(spec.n_seq, spec.n_layers, spec.n_kvheads,
                                                     G, cap, B))
    first_window = cap // synth.STREAM_WINDOW      # positions 0 .. cap-1 are windows 0 .. 16
    for step in range(3):
        nv_host = cur["nv"].cpu().numpy()
        assert np.all(nv_host == cap)
        tri.tri_prune(tri.config(), cur["k"], cur["v"], cur["pos"], spec.n_seq, spec.n_layers,
                      spec.n_kvheads, G, cur["p_cur"], gst, B, nxt["k"], nxt["v"], nxt["pos"],
                      n_kept, n_valid=cur["nv"], kept=kept, ws=ws)
        assert tri.tri_check_device_error(ws) == 0
        o = oracle.prune(synth.host_elems(cur["k"]), None, cur["pos"].cpu().numpy(), spec.n_seq,
                         spec.n_layers, spec.n_kvheads, G, ost, cur["p_cur"].cpu().numpy(), B,
                         n_valid=nv_host, want_gather=False, want_raw=False)
        gk_all = kept.cpu().numpy()
        mismatched = 0
        for u in range(U):
            gk = gk_all[u]
            mismatched += H.check_kept(gk, o["final"][u], o["kept"][u], cap, B)
            assert H.rows_equal(nxt["k"][u, :B], cur["k"][u], gk)
            assert H.rows_equal(nxt["v"][u, :B], cur["v"][u], gk)
            assert np.array_equal(nxt["pos"][u, :B].cpu().numpy(), cur["pos"][u].cpu().numpy()[gk])
        assert mismatched <= 2 * U
        assert np.all(n_kept.cpu().numpy() == B)
        # the next window of generated tokens goes after the kept rows
        k_new, v_new, pos_new = synth.stream_window(spec, wl.hp, first_window + step, "cuda")
        nv_next = n_kept.clone()
        p_next = torch.empty_like(cur["p_cur"])
        tri.tri_append(nxt["k"], nxt["v"], nxt["pos"], spec.n_seq, nv_next, k_new, v_new,
                       pos_new, p_cur=p_next, ws=ws)
        assert tri.tri_check_device_error(ws) == 0
        assert np.all(p_next.cpu().numpy() == (first_window + step + 1) * synth.STREAM_WINDOW)
        # kept positions stay ascending, then the new window follows
        pp = nxt["pos"].cpu().numpy()
        assert np.all(np.diff(pp[:, :cap], axis=1) > 0)
        nxt["nv"], nxt["p_cur"] = nv_next, p_next
        cur, nxt = nxt, dict(k=cur["k"], v=cur["v"], pos=cur["pos"])


@pytest.mark.parametrize("inplace,path", [(False, tri.PATH_PIPE), (True, tri.PATH_PIPE),
                                          (False, tri.PATH_AUTO), (True, tri.PATH_SPLIT)])
def test_stream_full_run(inplace, path):
    """The streaming workload's whole stream at reduced width (1 sequence x 1
    layer x 4 KV heads, G = 7, B 2048, window 128): 256 windows of generated
    tokens appended, a prune whenever the cache holds B + 128 rows (240
    prunes, the last at p_cur = 32768), through the window driver on two
    cache buffers or one buffer compacted in place.  Prune steps 1, 2, 60,
    120 and 240 are checked against the oracle run on the cache the GPU
    pruned (kept sets, final scores, the gathered rows)."""
    from types import SimpleNamespace

    from rope_aware_kv_b200.window import WindowDriver

    spec = synth.SPECS["c5"].scaled(n_seq=1, n_layers=1)
    U, cap, B, G = spec.n_units, spec.cap, spec.B, spec.G
    hp = synth.head_params(spec)
    gst, ost = H.stats_for(spec, SimpleNamespace(hp=hp))
    drv = WindowDriver(spec.n_seq, spec.n_layers, spec.n_kvheads, G, B, gst,
                       window=synth.STREAM_WINDOW, inplace=inplace, cfg=tri.config(path=path))
    assert drv.cap == cap
    checks = {1, 2, 60, 120, 240}
    seen = []
    for w in range(synth.STREAM_TOKENS // synth.STREAM_WINDOW):
        k_new, v_new, pos_new = synth.stream_window(spec, hp, w, "cuda")
        drv.append(k_new, v_new, pos_new, auto_prune=False)
        if not drv.full:
            continue
        step = drv.prunes + 1
        if step not in checks:
            drv.prune()
            continue
        # the cache about to be pruned
        k0, v0, p0 = drv.k_cache.clone(), drv.v_cache.clone(), drv.pos_cache.clone()
        nv0 = drv.n_valid.cpu().numpy()
        pc0 = drv.p_cur.cpu().numpy()
        assert np.all(nv0 == cap)
        assert np.all(pc0 == synth.STREAM_WINDOW * (w + 1))
        fin = torch.full((U, cap), float("nan"), device="cuda")
        drv.prune(final=fin)
        assert tri.tri_check_device_error(drv.ws) == 0
        o = oracle.prune(synth.host_elems(k0), None, p0.cpu().numpy(), spec.n_seq, spec.n_layers,
                         spec.n_kvheads, G, ost, pc0, B, n_valid=nv0, want_gather=False,
                         want_raw=False)
        gk_all = drv.kept.cpu().numpy()
        fin_h = fin.cpu().numpy()
        assert np.all(drv.n_valid.cpu().numpy() == B)
        mismatched = 0
        for u in range(U):
            gk = gk_all[u]
            assert H.check_final(fin_h[u], o["final"][u], cap) <= H.Z_RTOL, f"step {step} unit {u}"
            mismatched += H.check_kept(gk, o["final"][u], o["kept"][u], cap, B)
            assert H.rows_equal(drv.k_cache[u, :B], k0[u], gk)
            assert H.rows_equal(drv.v_cache[u, :B], v0[u], gk)
            assert np.array_equal(drv.pos_cache[u, :B].cpu().numpy(), p0[u].cpu().numpy()[gk])
        assert mismatched <= 2 * U
        seen.append(step)
    assert seen == sorted(checks)
    assert drv.prunes == 240
    assert drv.tokens == synth.STREAM_TOKENS
    assert np.all(drv.p_cur.cpu().numpy() == synth.STREAM_TOKENS)
    # kept positions stay ascending through the whole stream
    pp = drv.pos_cache.cpu().numpy()[:, :B]
    assert np.all(np.diff(pp, axis=1) > 0)
