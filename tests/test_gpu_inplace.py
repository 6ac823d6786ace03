"""In-place, order-preserving compaction (jaedaily.cn tutorial, eviction step:
keys[idx] / values[idx] with idx ascending) through the C ABI.

tri_compact_inplace must leave rows 0 .. n_kept-1 of the one buffer equal, bit
for bit, to the rows the kept indices named before the call, and every other
row untouched.  tri_prune_inplace must produce exactly what tri_prune writes
into a separate destination on the same path (same kept indices, counts and
final scores, the same rows), and match the oracle.
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


def _kept_lists(U, cap, B, seed):
    """Ascending kept lists of every shape the compaction meets: nothing kept,
    the identity (nothing moves), a long unmoved prefix, drops spread over
    the unit, one drop at row 0, every row kept of a short unit."""
    rng = np.random.default_rng(seed)
    kept = np.full((U, B), -1, np.int32)
    nk = np.zeros(U, np.int32)
    for u in range(U):
        kind = u % 6
        if kind == 0:
            m, idx = 0, np.zeros(0, np.int64)
        elif kind == 1:
            m = min(B, cap)
            idx = np.arange(m)
        elif kind == 2:
            m = min(B, cap)
            head = m // 2
            idx = np.concatenate([np.arange(head),
                                  np.sort(rng.choice(np.arange(head, cap), m - head, replace=False))])
        elif kind == 3:
            m = min(B, cap)
            idx = np.sort(rng.choice(cap, m, replace=False))
        elif kind == 4:
            m = min(B, cap - 1)
            idx = np.arange(1, m + 1)
        else:
            m = min(B, 37)
            idx = np.sort(rng.choice(cap, m, replace=False))
        kept[u, :m] = idx
        nk[u] = m
    return kept, nk


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("cap,B", [(700, 300), (2176, 2048), (130, 200)])
def test_compact_inplace_bitwise(dtype, cap, B):
    U = 12
    g = torch.Generator(device="cuda").manual_seed(cap + B)
    k = torch.randn((U, cap, 128), generator=g, device="cuda").to(dtype)
    v = torch.randn((U, cap, 128), generator=g, device="cuda").to(dtype)
    pos = torch.randint(0, 1 << 30, (U, cap), generator=g, device="cuda", dtype=torch.int32)
    k0, v0, p0 = k.clone(), v.clone(), pos.clone()
    kept_h, nk_h = _kept_lists(U, cap, B, seed=cap)
    kept = torch.as_tensor(kept_h, device="cuda")
    nk = torch.as_tensor(nk_h, device="cuda")
    ws = tri.workspace(256)
    tri.tri_compact_inplace(k, v, pos, kept, nk, ws=ws)
    assert tri.tri_check_device_error(ws) == 0
    for u in range(U):
        m = int(nk_h[u])
        idx = kept_h[u, :m]
        assert H.rows_equal(k[u, :m], k0[u], idx)
        assert H.rows_equal(v[u, :m], v0[u], idx)
        assert np.array_equal(pos[u, :m].cpu().numpy(), p0[u].cpu().numpy()[idx])
        assert torch.equal(k[u, m:], k0[u, m:]) and torch.equal(v[u, m:], v0[u, m:])
        assert torch.equal(pos[u, m:], p0[u, m:])


def test_compact_inplace_keys_only_and_bad_index():
    """V and positions may be absent; an index below its destination row (it
    would read a row already overwritten) or past the cache is skipped and
    flagged, every other row still moves."""
    U, cap, B = 3, 200, 64
    g = torch.Generator(device="cuda").manual_seed(3)
    k = torch.randn((U, cap, 128), generator=g, device="cuda").to(torch.bfloat16)
    k0 = k.clone()
    kept_h = np.stack([np.arange(0, 2 * B, 2) for _ in range(U)]).astype(np.int32)
    kept_h[1, 10] = 5            # below row 10
    kept_h[2, 20] = cap + 7      # outside the cache
    nk_h = np.full(U, B, np.int32)
    kept = torch.as_tensor(kept_h, device="cuda")
    ws = tri.workspace(256)
    tri.tri_compact_inplace(k, None, None, kept, torch.as_tensor(nk_h, device="cuda"), ws=ws)
    assert tri.tri_check_device_error(ws) & tri.FLAG_INDEX_RANGE
    assert H.rows_equal(k[0, :B], k0[0], kept_h[0])
    for u, bad in ((1, 10), (2, 20)):
        good = [r for r in range(B) if r != bad]
        assert H.rows_equal(k[u, good], k0[u], kept_h[u, good])


def test_compact_inplace_rejects_overlap():
    U, cap = 2, 64
    buf = torch.zeros((2 * U * cap * 128,), dtype=torch.bfloat16, device="cuda")
    k = buf[: U * cap * 128].view(U, cap, 128)
    v = buf[U * cap * 64: U * cap * 64 + U * cap * 128].view(U, cap, 128)
    kept = torch.zeros((U, 8), dtype=torch.int32, device="cuda")
    nk = torch.zeros((U,), dtype=torch.int32, device="cuda")
    with pytest.raises(tri.TriError):
        tri.tri_compact_inplace(k, v, None, kept, nk)


def _spec(dtype="bf16", G=3, n_seq=2, n_layers=2, n_kvheads=2, cap=700, B=300, stream=21):
    return synth.Spec("t", n_seq, n_layers, n_kvheads, G, cap, cap, B, dtype, 3000, cap,
                      R_range=(0.6, 1.0), stream=stream)


def _ragged(spec, B):
    choices = [spec.cap, spec.cap - 1, 0, 1, B, B + 1, 257, spec.cap // 2]
    return np.clip(np.array([choices[u % len(choices)] for u in range(spec.n_units)], np.int32),
                   0, spec.cap)


CASES = [
    # (dtype, G, cap, B, path): whole units per CTA (pipe, small mode), the
    # split kernels, units scored in chunks (pipe, large mode), AUTO.
    ("bf16", 7, 700, 300, tri.PATH_PIPE),
    ("f32", 2, 700, 300, tri.PATH_PIPE),
    ("bf16", 4, 700, 300, tri.PATH_SPLIT),
    ("f32", 3, 700, 300, tri.PATH_SPLIT),
    ("bf16", 4, 70000, 1500, tri.PATH_PIPE),
    ("bf16", 7, 2176, 2048, tri.PATH_AUTO),
]


@pytest.mark.parametrize("dtype,G,cap,B,path", CASES)
def test_prune_inplace_equals_pingpong_and_oracle(dtype, G, cap, B, path):
    n_seq, n_layers = (1, 1) if cap > 10000 else (2, 2)
    spec = _spec(dtype=dtype, G=G, n_seq=n_seq, n_layers=n_layers, cap=cap, B=B)
    U = spec.n_units
    wl = synth.make_workload(spec, "cuda")
    gst, ost = H.stats_for(spec, wl)
    nv_h = _ragged(spec, B)
    nv = torch.as_tensor(nv_h, device="cuda")
    cfg = tri.config(path=path)
    expect = tri.tri_prune_path(spec.n_seq, spec.n_layers, spec.n_kvheads, G, cap, B,
                                spec.torch_dtype, path, inplace=True)
    assert expect in (tri.PATH_PIPE, tri.PATH_SPLIT)
    ws = tri.workspace(tri.tri_prune_workspace_bytes(spec.n_seq, spec.n_layers, spec.n_kvheads, G,
                                                     cap, B))
    # Ping-pong reference on the same path.
    kd = torch.zeros((U, B, 128), dtype=wl.k.dtype, device="cuda")
    vd = torch.zeros_like(kd)
    pd = torch.full((U, B), -1, dtype=torch.int32, device="cuda")
    kept_a = torch.empty((U, B), dtype=torch.int32, device="cuda")
    nk_a = torch.empty((U,), dtype=torch.int32, device="cuda")
    fin_a = torch.full((U, cap), float("nan"), device="cuda")
    pp_cfg = tri.config(path=expect)
    tri.tri_prune(pp_cfg, wl.k, wl.v, wl.pos, spec.n_seq, spec.n_layers, spec.n_kvheads, G,
                  wl.p_cur, gst, B, kd, vd, pd, nk_a, n_valid=nv, kept=kept_a, ws=ws, final=fin_a)
    assert tri.tri_check_device_error(ws) == 0
    # In place on copies of the cache.
    k, v, pos = wl.k.clone(), wl.v.clone(), wl.pos.clone()
    kept_b = torch.empty((U, B), dtype=torch.int32, device="cuda")
    nk_b = torch.empty((U,), dtype=torch.int32, device="cuda")
    fin_b = torch.full((U, cap), float("nan"), device="cuda")
    tri.tri_prune_inplace(cfg, k, v, pos, spec.n_seq, spec.n_layers, spec.n_kvheads, G, wl.p_cur,
                          gst, B, nk_b, n_valid=nv, kept=kept_b, ws=ws, final=fin_b)
    assert tri.tri_check_device_error(ws) == 0
    assert torch.equal(kept_a, kept_b) and torch.equal(nk_a, nk_b)
    for u in range(U):
        if nv_h[u] > B:
            n = int(nv_h[u])
            assert torch.equal(fin_a[u, :n], fin_b[u, :n]), f"unit {u}"
    nk_h = nk_b.cpu().numpy()
    for u in range(U):
        m = int(nk_h[u])
        assert torch.equal(k[u, :m], kd[u, :m]) and torch.equal(v[u, :m], vd[u, :m])
        assert torch.equal(pos[u, :m], pd[u, :m])
        # rows past the kept ones are not written
        assert torch.equal(k[u, m:], wl.k[u, m:]) and torch.equal(pos[u, m:], wl.pos[u, m:])
    # Against the oracle (kept sets outside the exempt band, final scores).
    o = oracle.prune(synth.host_elems(wl.k), None, wl.pos.cpu().numpy(), spec.n_seq,
                     spec.n_layers, spec.n_kvheads, G, ost, wl.p_cur.cpu().numpy(), B,
                     n_valid=nv_h, want_gather=False, want_raw=False)
    gk_all = kept_b.cpu().numpy()
    fin = fin_b.cpu().numpy()
    mismatched = 0
    for u in range(U):
        n, m = int(nv_h[u]), int(nk_h[u])
        assert m == min(n, B)
        if n > B:
            assert H.check_final(fin[u], o["final"][u], n) <= H.Z_RTOL
        mismatched += H.check_kept(gk_all[u, :m], o["final"][u], o["kept"][u], n, B)
        assert H.rows_equal(k[u, :m], wl.k[u], gk_all[u, :m])
    assert mismatched <= 2 * U


@pytest.mark.parametrize("path", [tri.PATH_FUSED, tri.PATH_COOP])
def test_prune_inplace_refuses_paths_without_it(path):
    spec = _spec(G=3, cap=700, B=300)
    wl = synth.make_workload(spec, "cuda")
    gst, _ = H.stats_for(spec, wl)
    nk = torch.empty((spec.n_units,), dtype=torch.int32, device="cuda")
    assert tri.tri_prune_path(spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G, spec.cap,
                              spec.B, path=path, inplace=True) == -1
    with pytest.raises(tri.TriError):
        tri.tri_prune_inplace(tri.config(path=path), wl.k, wl.v, wl.pos, spec.n_seq,
                              spec.n_layers, spec.n_kvheads, spec.G, wl.p_cur, gst, spec.B, nk,
                              n_valid=wl.n_valid)
    # n_kept may not be the n_valid it reads
    nv = wl.n_valid.clone()
    with pytest.raises(tri.TriError):
        tri.tri_prune_inplace(tri.config(), wl.k, wl.v, wl.pos, spec.n_seq, spec.n_layers,
                              spec.n_kvheads, spec.G, wl.p_cur, gst, spec.B, nv, n_valid=nv)


@pytest.mark.parametrize("dtype,variant", [("bf16", 0), ("f32", 0), ("bf16", tri.VAR_MAX_OFFSET)])
def test_prune_paged_inplace_equals_contiguous(dtype, variant):
    """A paged cache (128-row pages in a shuffled pool, one page table row per
    unit) pruned in place gives the contiguous prune's kept indices, counts
    and final scores, and its logical rows 0 .. n_kept-1 hold the same rows."""
    B, cap, page = 300, 700, 128
    spec = _spec(dtype=dtype, G=4, cap=cap, B=B)
    U = spec.n_units
    wl = synth.make_workload(spec, "cuda")
    gst, _ = H.stats_for(spec, wl)
    nv_h = _ragged(spec, B)
    nv = torch.as_tensor(nv_h, device="cuda")
    ppu = (cap + page - 1) // page
    n_pages = U * ppu + 5
    rng = np.random.default_rng(9)
    table_h = rng.permutation(n_pages)[:U * ppu].reshape(U, ppu).astype(np.int32)
    table = torch.as_tensor(table_h, device="cuda")
    k_pool = torch.zeros((n_pages, page, 128), dtype=wl.k.dtype, device="cuda")
    v_pool = torch.zeros_like(k_pool)
    for u in range(U):
        for p in range(ppu):
            rows = min(page, cap - p * page)
            k_pool[table_h[u, p], :rows] = wl.k[u, p * page:p * page + rows]
            v_pool[table_h[u, p], :rows] = wl.v[u, p * page:p * page + rows]
    pos = wl.pos.clone()
    cfg = tri.config(variant=variant, path=tri.PATH_SPLIT)
    ws = tri.workspace(tri.tri_prune_workspace_bytes(spec.n_seq, spec.n_layers, spec.n_kvheads, 4,
                                                     cap, B))
    kd = torch.zeros((U, B, 128), dtype=wl.k.dtype, device="cuda")
    vd = torch.zeros_like(kd)
    pd = torch.full((U, B), -1, dtype=torch.int32, device="cuda")
    kept_a = torch.empty((U, B), dtype=torch.int32, device="cuda")
    nk_a = torch.empty((U,), dtype=torch.int32, device="cuda")
    fin_a = torch.full((U, cap), float("nan"), device="cuda")
    tri.tri_prune(cfg, wl.k, wl.v, wl.pos, spec.n_seq, spec.n_layers, spec.n_kvheads, 4,
                  wl.p_cur, gst, B, kd, vd, pd, nk_a, n_valid=nv, kept=kept_a, ws=ws, final=fin_a)
    assert tri.tri_check_device_error(ws) == 0
    kept_b = torch.empty((U, B), dtype=torch.int32, device="cuda")
    nk_b = torch.empty((U,), dtype=torch.int32, device="cuda")
    fin_b = torch.full((U, cap), float("nan"), device="cuda")
    tri.tri_prune_paged_inplace(cfg, k_pool, v_pool, pos, table, cap, spec.n_seq, spec.n_layers,
                                spec.n_kvheads, 4, wl.p_cur, gst, B, nk_b, n_valid=nv,
                                kept=kept_b, ws=ws, final=fin_b)
    assert tri.tri_check_device_error(ws) == 0
    assert torch.equal(kept_a, kept_b) and torch.equal(nk_a, nk_b)
    for u in range(U):
        n = int(nv_h[u])
        if n > B:
            assert torch.equal(fin_a[u, :n], fin_b[u, :n])
        m = int(nk_b[u])
        logical_k = torch.cat([k_pool[table_h[u, p]] for p in range(ppu)])[:cap]
        logical_v = torch.cat([v_pool[table_h[u, p]] for p in range(ppu)])[:cap]
        assert torch.equal(logical_k[:m], kd[u, :m]) and torch.equal(logical_v[:m], vd[u, :m])
        assert torch.equal(pos[u, :m], pd[u, :m])
        assert torch.equal(logical_k[m:], wl.k[u, m:])
    with pytest.raises(tri.TriError):
        tri.tri_prune_paged_inplace(tri.config(path=tri.PATH_PIPE), k_pool, v_pool, pos, table, cap,
                                    spec.n_seq, spec.n_layers, spec.n_kvheads, 4, wl.p_cur, gst, B,
                                    nk_b, n_valid=nv)
