"""A bounded wait that runs out is reported, and the library stays usable.

The cooperative path's unit-wide barriers wait (bounded) for every CTA of a
unit.  With the bound set to 1 ns most CTAs give up at the first barrier: the
call must still return, the device flag must carry TRI_FLAG_TIMEOUT, and the
next call with the default bound must produce the oracle's result.  No copy
is in flight into a CTA's shared memory at any unit barrier, so the CTAs that
give up exit cleanly.  Nothing here faults, traps or hangs the GPU: the wait
simply stops after its bound.
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


def test_coop_barrier_timeout_then_clean_call():
    spec = synth.Spec("t", 1, 1, 4, 7, 8192, 8192, 1024, "bf16", 3000, 8192,
                      R_range=(0.6, 1.0), stream=41)
    U, B = spec.n_units, spec.B
    assert tri.tri_prune_path(spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G, spec.cap, B,
                              path=tri.PATH_COOP) == tri.PATH_COOP
    wl = synth.make_workload(spec, "cuda")
    gst, ost = H.stats_for(spec, wl)
    kd = torch.zeros((U, B, 128), dtype=wl.k.dtype, device="cuda")
    vd = torch.zeros_like(kd)
    pd = torch.zeros((U, B), dtype=torch.int32, device="cuda")
    kept = torch.empty((U, B), dtype=torch.int32, device="cuda")
    nk = torch.empty((U,), dtype=torch.int32, device="cuda")
    ws = tri.workspace(tri.tri_prune_workspace_bytes(spec.n_seq, spec.n_layers, spec.n_kvheads,
                                                     spec.G, spec.cap, B))

    def run(cfg):
        tri.tri_prune(cfg, wl.k, wl.v, wl.pos, spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G,
                      wl.p_cur, gst, B, kd, vd, pd, nk, n_valid=wl.n_valid, kept=kept, ws=ws)
        return tri.tri_check_device_error(ws)

    flags = run(tri.config(path=tri.PATH_COOP, barrier_wait_ns=1))
    assert flags & tri.FLAG_TIMEOUT
    flags = run(tri.config(path=tri.PATH_COOP))
    assert flags == 0
    o = oracle.prune(synth.host_elems(wl.k), None, wl.pos.cpu().numpy(), spec.n_seq,
                     spec.n_layers, spec.n_kvheads, spec.G, ost, wl.p_cur.cpu().numpy(), B,
                     want_gather=False, want_raw=False)
    gk_all = kept.cpu().numpy()
    mismatched = 0
    for u in range(U):
        assert int(nk[u]) == B
        mismatched += H.check_kept(gk_all[u], o["final"][u], o["kept"][u], spec.cap, B)
        assert H.rows_equal(kd[u], wl.k[u], gk_all[u])
    assert mismatched <= 2 * U
