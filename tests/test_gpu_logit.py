"""The centre approximation's check on the GPU against the oracle: the
trigonometric-series logit(Delta) from the Q and K centres (talk page, centre
approximation), the measured mean post-RoPE logit at each distance, their
Pearson correlation (shibing624 paper reading, Fig. 1(D)), and the K centres
from post-RoPE keys calibrated with their positions.
"""
import numpy as np
import pytest
import torch

import oracle
import rope_aware_kv_b200 as tri
import synth
from rope_aware_kv_b200 import build as tri_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tri_build.build()
    tri.load()
    oracle.build()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_logit_reconstruction_curve_and_pearson(dtype):
    n = 2048
    spec = synth.Spec("t", 1, 1, 4, 2, n, n, 256, dtype, n, n, R_range=(0.6, 1.0), stream=51)
    G, Hq, Hkv = spec.G, spec.n_qheads, spec.n_kvheads
    hp = synth.head_params(spec)
    pos = torch.arange(n, device="cuda", dtype=torch.int32)
    q_pre = synth.calib_queries(spec, hp, 0, "cuda")[:, :n]
    q_post = synth.rope_rotate(q_pre.double(), pos.expand(Hq, n)).to(q_pre.dtype).contiguous()
    k_post, _ = synth.keys_values(spec, hp, 0, Hkv, pos.expand(Hkv, n), "cuda")
    cfg = tri.config()
    # centres from the post-RoPE rows rotated back by their positions
    qs = tri.tri_calibrate_ex(cfg, q_post, q_pos=pos)
    ks = tri.tri_calibrate_ex(cfg, k_post, q_pos=pos)
    oqs = oracle.calibrate(synth.host_elems(q_post), pos=pos.cpu().numpy())
    oks = oracle.calibrate(synth.host_elems(k_post), pos=pos.cpu().numpy())
    for g, o in ((qs, oqs), (ks, oks)):
        g = g.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(g[..., :3] - o[..., :3]) / o[..., 2:3]) < 1e-5
    deltas_h = np.arange(0, n + 64, 8, dtype=np.int64)
    deltas = torch.as_tensor(deltas_h, device="cuda")
    recon = tri.tri_logit_reconstruct(cfg, qs, ks, G, deltas).cpu().numpy()
    ref = oracle.logit_reconstruct(qs.cpu().numpy().astype(np.float64),
                                   ks.cpu().numpy().astype(np.float64), G, deltas_h)
    assert np.max(np.abs(recon - ref)) <= 1e-5 * np.abs(ref).max()
    curve = tri.tri_logit_curve(q_post, k_post, G, deltas).cpu().numpy()
    cref = oracle.logit_curve(synth.host_elems(q_post), synth.host_elems(k_post), G, deltas_h)
    assert np.max(np.abs(curve - cref)) <= 1e-4 * np.abs(cref).max()
    assert np.all(curve[:, deltas_h >= n] == 0.0)
    inside = torch.as_tensor(deltas_h < n, device="cuda")
    a = torch.as_tensor(curve, device="cuda")[:, inside].contiguous()
    b = torch.as_tensor(recon, device="cuda")[:, inside].contiguous()
    r = tri.tri_pearson(a, b).cpu().numpy()
    rref = oracle.pearson(a.cpu().numpy(), b.cpu().numpy())
    np.testing.assert_allclose(r, rref, atol=1e-5)
    assert np.all(np.abs(r) <= 1.0 + 1e-6)
