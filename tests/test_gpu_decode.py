"""Decode attention over the (compacted) cache against the oracle, through the
C ABI (jaedaily.cn tutorial, KV-compression objective: the next token attends
over the kept rows with the softmax renormalised over them).

Outputs are compared element-wise: |gpu - oracle| <= 1e-4 * max(1, |oracle|)
(float32 accumulation and exp2 against float64).  Covers ragged n_valid
(including 0 and 1), both dtypes, G = 1..8, units split over several CTAs
(the chunk merge), and the cache a prune step leaves behind.
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
TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tri_build.build()
    tri.load()
    oracle.build()
    yield
    torch.cuda.empty_cache()


def _check(out, ref):
    err = np.abs(out.astype(np.float64) - ref) / np.maximum(1.0, np.abs(ref))
    assert float(err.max()) <= TOL, float(err.max())


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("G,U,cap", [(7, 6, 700), (4, 3, 5000), (1, 2, 300), (8, 2, 20000)])
def test_decode_attention_parity(dtype, G, U, cap):
    g = torch.Generator(device="cuda").manual_seed(G * 1000 + cap)
    q = (torch.randn((U, G, 128), generator=g, device="cuda") * 0.3).to(dtype)
    k = torch.randn((U, cap, 128), generator=g, device="cuda").to(dtype)
    v = torch.randn((U, cap, 128), generator=g, device="cuda").to(dtype)
    choices = [cap, 0, 1, cap - 1, 257, cap // 3]
    nv = np.array([choices[u % len(choices)] for u in range(U)], np.int32)
    out = tri.tri_decode_attention(q, k, v, n_valid=torch.as_tensor(nv, device="cuda"))
    ref = oracle.decode_attention(synth.host_elems(q), synth.host_elems(k), synth.host_elems(v),
                                  n_valid=nv)
    _check(out.cpu().numpy(), ref)
    # another scale, every row valid
    out2 = tri.tri_decode_attention(q, k, v, scale=0.02)
    ref2 = oracle.decode_attention(synth.host_elems(q), synth.host_elems(k), synth.host_elems(v),
                                   scale=0.02)
    _check(out2.cpu().numpy(), ref2)


def test_decode_after_prune():
    """The next token attends over what a prune step kept: decode over the
    destination cache with n_kept rows equals the oracle on those rows."""
    spec = synth.SPECS["c5"].scaled(n_seq=1, n_layers=2)
    U, B, G = spec.n_units, spec.B, spec.G
    wl = synth.make_workload(spec, "cuda")
    gst, _ = H.stats_for(spec, wl)
    kd = torch.zeros((U, B, 128), dtype=wl.k.dtype, device="cuda")
    vd = torch.zeros_like(kd)
    pd = torch.zeros((U, B), dtype=torch.int32, device="cuda")
    nk = torch.empty((U,), dtype=torch.int32, device="cuda")
    tri.tri_prune(tri.config(), wl.k, wl.v, wl.pos, spec.n_seq, spec.n_layers, spec.n_kvheads, G,
                  wl.p_cur, gst, B, kd, vd, pd, nk, n_valid=wl.n_valid)
    q = synth.stream_window(spec, wl.hp, 17, "cuda")[0][:, :G].contiguous()  # some post-RoPE rows
    out = tri.tri_decode_attention(q, kd, vd, n_valid=nk)
    ref = oracle.decode_attention(synth.host_elems(q), synth.host_elems(kd), synth.host_elems(vd),
                                  n_valid=nk.cpu().numpy())
    _check(out.cpu().numpy(), ref)


def test_decode_rejects_bad_arguments():
    q = torch.zeros((2, 4, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((2, 16, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tri.TriError):
        tri.tri_decode_attention(q, k, k, scale=-1.0)
    q9 = torch.zeros((2, 9, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tri.TriError):
        tri.tri_decode_attention(q9, k, k)
