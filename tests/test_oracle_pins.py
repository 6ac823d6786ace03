"""Pins of the float64 oracle against what the pages and the mathematics fix.

No GPU.  Each test checks the oracle against something other than itself:
the explicit RoPE attention logit (rotate-then-dot with the talk page's 2x2
matrix), closed forms, brute force on tiny inputs, and invariants.  A
plausible mistake anywhere in the oracle (a wrong omega exponent, swapped
pairing, a phase sign, the de-rotation direction, a dropped 1/|D|, (1-R)
applied to the wrong term, sample instead of population sigma, mean instead
of max over heads, the wrong tie order, a gather off by one) fails at least
one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_constants.txt")
D = 128
F = D // 2


def _golden():
    vals = {}
    with open(GOLDEN) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    return vals


def _rope_matrix_rotate(x, p, theta=10000.0):
    """Explicit RoPE: per band f the 2x2 matrix [[cos, -sin], [sin, cos]] of
    angle omega_f * p applied to (x_2f, x_2f+1) (talk page, RoPE rotation)."""
    x = np.asarray(x, np.float64)
    out = np.empty_like(x)
    for f in range(x.shape[-1] // 2):
        a = theta ** (-2.0 * f / x.shape[-1]) * p
        M = np.array([[math.cos(a), -math.sin(a)], [math.sin(a), math.cos(a)]])
        out[..., 2 * f:2 * f + 2] = x[..., 2 * f:2 * f + 2] @ M.T
    return out


def _stats_identical(qbar, n=4):
    """Calibrate on n identical queries (zero noise)."""
    q = np.repeat(np.asarray(qbar, np.float32)[None, None, :], n, axis=1)
    return oracle.calibrate(q)


def test_page_constants():
    g = _golden()
    assert float(g["theta"]) == oracle.THETA
    assert tuple(int(x) for x in g["offsets"].split()) == oracle.OFFSETS
    assert len(oracle.OFFSETS) == 17


def test_zero_noise_calibration_recovers_centre_and_R1():
    rng = np.random.default_rng(0)
    qbar = rng.normal(size=D).astype(np.float32)
    st = _stats_identical(qbar, n=5)
    assert st.shape == (1, F, 4)
    np.testing.assert_array_equal(st[0, :, 0], qbar[0::2].astype(np.float64))
    np.testing.assert_array_equal(st[0, :, 1], qbar[1::2].astype(np.float64))
    np.testing.assert_allclose(st[0, :, 2], np.hypot(qbar[0::2].astype(np.float64), qbar[1::2]), rtol=1e-15)
    np.testing.assert_allclose(st[0, :, 3], 1.0, atol=1e-12)


@pytest.mark.parametrize("offsets", [(1,), (65536,), (3, 1000), oracle.OFFSETS])
def test_strig_equals_explicit_rope_logit(offsets):
    """(1) With every query at its centre, S~ is the mean over the future query
    positions p_cur + delta of the explicit post-RoPE dot product."""
    rng = np.random.default_rng(1)
    qbar = rng.normal(size=D).astype(np.float32)
    st = _stats_identical(qbar)
    n = 40
    pos = np.sort(rng.choice(200000, size=n, replace=False)).astype(np.int32)
    kpre = rng.normal(size=(n, D))
    kpost = np.stack([_rope_matrix_rotate(kpre[j], pos[j]) for j in range(n)]).astype(np.float32)
    p_cur = 200001
    got = oracle.score(kpost, pos, p_cur, st, offsets=offsets)[0]
    want = np.zeros(n)
    for dlt in offsets:
        qrot = _rope_matrix_rotate(qbar.astype(np.float64), p_cur + dlt)
        want += kpost.astype(np.float64) @ qrot
    want /= len(offsets)
    scale = np.abs(kpost).sum(1) * np.abs(qbar).sum()
    assert np.max(np.abs(got - want) / scale) < 1e-12


def test_strig_single_band_closed_form():
    """d = 2, omega_0 = 1: centre (1, 0), key (0, 1) at position 0, p_cur 0:
    S_trig(Delta) = cos(Delta - pi/2) = sin(Delta)."""
    st = _stats_identical(np.array([1.0, 0.0], np.float32))
    k = np.array([[0.0, 1.0]], np.float32)
    pos = np.array([0], np.int32)
    assert oracle.score(k, pos, 0, st, offsets=(1,))[0, 0] == pytest.approx(math.sin(1.0), abs=1e-15)
    got = oracle.score(k, pos, 0, st, offsets=(1, 2))[0, 0]
    assert got == pytest.approx(0.5 * (math.sin(1.0) + math.sin(2.0)), abs=1e-15)


def test_R_zero_gives_pure_norm_score():
    """(2) Symmetric queries {q, -q}: E[q_f] = 0, R_f = 0, so S_trig = 0 and
    S~ = sum_f E|q_f| |k_f|, with |k_f| = |k'_f| (rotation keeps norms)."""
    rng = np.random.default_rng(2)
    qbar = rng.normal(size=D).astype(np.float32)
    q = np.stack([qbar, -qbar])[None]
    st = oracle.calibrate(q)
    np.testing.assert_allclose(st[0, :, 3], 0.0, atol=1e-15)
    n = 16
    kpost = rng.normal(size=(n, D)).astype(np.float32)
    pos = rng.integers(0, 50000, size=n).astype(np.int32)
    got = oracle.score(kpost, pos, 60000, st)[0]
    qn = np.hypot(qbar[0::2].astype(np.float64), qbar[1::2])
    kn = np.hypot(kpost[:, 0::2].astype(np.float64), kpost[:, 1::2])
    np.testing.assert_allclose(got, kn @ qn, rtol=1e-13)


def _folded_score(kpost, st, p_cur, offsets, theta=10000.0):
    """Closed form of the offset average: the key position cancels and
    S~ = sum_f Re(A_f conj(k'_f)) + sum_f (1-R_f) E|q_f| |k'_f| with
    A_f = E[q_f] e^{i w_f p_cur} C_f and C_f = mean_delta e^{i w_f delta}."""
    f = np.arange(F)
    w = theta ** (-2.0 * f / D)
    C = np.mean([np.exp(1j * w * dl) for dl in offsets], axis=0)
    m = st[..., 0] + 1j * st[..., 1]
    A = m * np.exp(1j * w * p_cur) * C
    kc = kpost[:, 0::2].astype(np.float64) + 1j * kpost[:, 1::2]
    trig = np.real(kc.conj() @ A.T)
    norm = np.abs(kc) @ ((1.0 - st[..., 3]) * st[..., 2]).T
    return (trig + norm).T


def test_offset_fold_equals_direct_sum():
    """(3) The folded complex factor per band gives the same S~ as the
    direct 17-offset sum, with noisy (R < 1) calibration and G = 3."""
    rng = np.random.default_rng(3)
    G = 3
    q = rng.normal(size=(G, 64, D)).astype(np.float32) + rng.normal(size=(G, 1, D)).astype(np.float32)
    st = oracle.calibrate(q)
    assert np.all(st[..., 3] < 1.0)
    n = 50
    pos = np.sort(rng.choice(32768, n, replace=False)).astype(np.int32)
    kpost = rng.normal(size=(n, D)).astype(np.float32)
    got = oracle.score(kpost, pos, 32768, st)
    want = _folded_score(kpost, st, 32768, oracle.OFFSETS)
    assert np.max(np.abs(got - want)) < 1e-10 * np.max(np.abs(want))


def test_linear_offsets_geometric_closed_form():
    """(3b) For linear offsets 1..n the average factor has the geometric-sum
    closed form e^{iw}(1 - e^{iwn}) / (n (1 - e^{iw}))."""
    rng = np.random.default_rng(4)
    qbar = rng.normal(size=D).astype(np.float32)
    st = _stats_identical(qbar)
    n_off = 37
    kpost = rng.normal(size=(8, D)).astype(np.float32)
    pos = np.arange(8, dtype=np.int32) * 1000
    got = oracle.score(kpost, pos, 9000, st, offsets=tuple(range(1, n_off + 1)))[0]
    w = 10000.0 ** (-2.0 * np.arange(F) / D)
    z = np.exp(1j * w)
    C = z * (1 - z ** n_off) / (n_off * (1 - z))
    A = (st[0, :, 0] + 1j * st[0, :, 1]) * np.exp(1j * w * 9000) * C
    kc = kpost[:, 0::2].astype(np.float64) + 1j * kpost[:, 1::2]
    want = np.real(kc.conj() @ A)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_uniform_position_shift_invariance():
    """Only Delta = p_cur - p_k matters: shifting every key position and p_cur
    by c (and rotating the keys accordingly) leaves S~ unchanged."""
    rng = np.random.default_rng(5)
    q = rng.normal(size=(2, 32, D)).astype(np.float32) + 2.0
    st = oracle.calibrate(q)
    n = 24
    kpre = rng.normal(size=(n, D))
    pos = np.sort(rng.choice(10000, n, replace=False)).astype(np.int32)
    k0 = np.stack([_rope_matrix_rotate(kpre[j], pos[j]) for j in range(n)])
    c = 12345
    k1 = np.stack([_rope_matrix_rotate(kpre[j], pos[j] + c) for j in range(n)])
    s0 = oracle.score(k0.astype(np.float32), pos, 10000, st)
    s1 = oracle.score(k1.astype(np.float32), pos + c, 10000 + c, st)
    assert np.max(np.abs(s0 - s1)) < 1e-5 * np.max(np.abs(s0))


def test_znorm_population_moments_and_max():
    """z per head has mean 0 and population variance 1; the final score is the
    largest z of the group; sigma = 0 gives z = 0."""
    rng = np.random.default_rng(6)
    raw = rng.normal(size=(4, 301)) * np.array([[1.0], [3.0], [0.1], [7.0]]) + 5.0
    raw[2] = 2.5  # a constant head
    z, fin, mu, sd = oracle.znorm_max(raw)
    for h in (0, 1, 3):
        assert abs(z[h].mean()) < 1e-13
        assert abs((z[h] ** 2).mean() - 1.0) < 1e-12
    assert sd[2] == 0.0 and np.all(z[2] == 0.0)
    assert np.all(fin >= z.max(axis=0)) and np.all(fin <= z.max(axis=0))
    assert np.all([fin[j] in z[:, j] for j in range(raw.shape[1])])


def test_znorm_max_skips_a_nan_head():
    """Reading of the head maximum (the pages are silent on NaN): a head whose
    scores are NaN (its moments are NaN, so every z of it is NaN) is skipped
    by the maximum, wherever it sits in the group; the final score is NaN
    only when every head is NaN.  Expected values are the largest finite z
    of each key, formed here from the z the oracle returns."""
    rng = np.random.default_rng(16)
    for nan_head in (0, 2):
        raw = rng.normal(size=(3, 50)) * np.array([[1.0], [2.0], [0.5]])
        raw[nan_head, 7] = np.nan  # one NaN score poisons that head's moments
        z, fin, mu, sd = oracle.znorm_max(raw)
        assert np.isnan(mu[nan_head]) and np.all(np.isnan(z[nan_head]))
        others = [h for h in range(3) if h != nan_head]
        assert not np.any(np.isnan(fin))
        np.testing.assert_array_equal(fin, np.max(z[others], axis=0))
    raw = np.full((2, 5), np.nan)
    _, fin, _, _ = oracle.znorm_max(raw)
    assert np.all(np.isnan(fin))


def _brute_force_topB(vals, B):
    n = len(vals)
    m = min(B, n)

    def beats(a, b):  # a ranks above b: larger score, NaN lowest, ties by index
        va, vb = vals[a], vals[b]
        na, nb = math.isnan(va), math.isnan(vb)
        if na != nb:
            return nb
        if not na and va != vb:
            return va > vb
        return a < b

    found = []
    for S in itertools.combinations(range(n), m):
        rest = [j for j in range(n) if j not in S]
        if all(beats(a, b) for a in S for b in rest):
            found.append(list(S))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(12))
def test_select_matches_brute_force(seed):
    """(4) Top-B equals the unique subset whose every member outranks every
    non-member; quantised scores force ties, so the index rule is pinned."""
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 10))
    vals = rng.choice([-1.0, -0.0, 0.0, 0.5, 1.0, 2.0, np.nan], size=n,
                      p=[0.15, 0.1, 0.15, 0.2, 0.2, 0.1, 0.1])
    for B in range(0, n + 2):
        kept, _ = oracle.select(vals, B)
        assert list(kept) == _brute_force_topB(list(vals), B)


def test_select_order_and_threshold():
    """(5) Kept indices are strictly ascending, unique, in range, min(B, n) of them."""
    rng = np.random.default_rng(7)
    vals = rng.normal(size=1000)
    kept, thr = oracle.select(vals, 100)
    assert len(kept) == 100
    assert np.all(np.diff(kept) > 0) and kept[0] >= 0 and kept[-1] < 1000
    assert thr == np.sort(vals)[-100]
    assert set(kept) == set(np.argsort(-vals, kind="stable")[:100])


def _small_case(G=2, dtype="f32", seed=8, n=300, cap=320, B=100):
    rng = np.random.default_rng(seed)
    n_seq, L, Hkv = 2, 2, 2
    U = n_seq * L * Hkv
    q = rng.normal(size=(L * Hkv * G, 48, D)).astype(np.float32) + rng.normal(size=(L * Hkv * G, 1, D)).astype(np.float32)
    st = oracle.calibrate(q).reshape(L, Hkv * G, F, 4)
    kf = rng.normal(size=(U, cap, D)).astype(np.float32)
    vf = rng.normal(size=(U, cap, D)).astype(np.float32)
    if dtype == "bf16":
        k = (kf.view(np.uint32) >> 16).astype(np.uint16)
        v = (vf.view(np.uint32) >> 16).astype(np.uint16)
    else:
        k, v = kf, vf
    pos = np.tile(np.sort(rng.choice(5000, cap, replace=False)).astype(np.int32), (U, 1))
    n_valid = np.array([n, cap, 0, 1, B, B + 1, 7, n], np.int32)
    p_cur = np.array([5000, 6000], np.int64)
    return dict(k=k, v=v, pos=pos, n_seq=n_seq, L=L, Hkv=Hkv, G=G, st=st, p_cur=p_cur,
                n_valid=n_valid, B=B, U=U, cap=cap)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_prune_gather_is_bitwise_and_ascending(dtype):
    """(5) Gathered K, V and position rows are the source rows at the kept
    indices, bit for bit, in ascending order; n_kept = min(B, n_valid)."""
    c = _small_case(dtype=dtype)
    out = oracle.prune(c["k"], c["v"], c["pos"], c["n_seq"], c["L"], c["Hkv"], c["G"], c["st"],
                       c["p_cur"], c["B"], n_valid=c["n_valid"])
    for u in range(c["U"]):
        m = int(out["n_kept"][u])
        assert m == min(c["B"], c["n_valid"][u])
        kept = out["kept"][u, :m]
        assert np.all(np.diff(kept) > 0)
        assert np.all(kept < c["n_valid"][u])
        assert np.array_equal(out["k_dst"][u, :m].view(np.uint8), c["k"][u, kept].view(np.uint8))
        assert np.array_equal(out["v_dst"][u, :m].view(np.uint8), c["v"][u, kept].view(np.uint8))
        assert np.array_equal(out["pos_dst"][u, :m], c["pos"][u, kept])


def test_prune_unit_consistency_with_parts():
    """The batched prune equals score -> z-max -> select run unit by unit
    (unit order (seq, layer, kv head) and the group's query heads)."""
    c = _small_case(G=3, seed=9)
    out = oracle.prune(c["k"], c["v"], c["pos"], c["n_seq"], c["L"], c["Hkv"], c["G"], c["st"],
                       c["p_cur"], c["B"], n_valid=c["n_valid"])
    for u in range(c["U"]):
        seq, layer, kvh = u // (c["L"] * c["Hkv"]), (u // c["Hkv"]) % c["L"], u % c["Hkv"]
        n = int(c["n_valid"][u])
        st = c["st"][layer, kvh * c["G"]:(kvh + 1) * c["G"]]
        raw = oracle.score(c["k"][u, :n], c["pos"][u, :n], int(c["p_cur"][seq]), st)
        np.testing.assert_array_equal(raw, out["raw"][u, :, :n])
        _, fin, _, _ = oracle.znorm_max(raw)
        kept, _ = oracle.select(fin, c["B"])
        np.testing.assert_array_equal(kept, out["kept"][u, :len(kept)])


def test_G1_keeps_raw_topB():
    """G = 1: the z-map is increasing, so the kept set is the raw top-B."""
    c = _small_case(G=1, seed=10)
    out = oracle.prune(c["k"], c["v"], c["pos"], c["n_seq"], c["L"], c["Hkv"], 1, c["st"],
                       c["p_cur"], c["B"], n_valid=c["n_valid"])
    for u in range(c["U"]):
        n = int(c["n_valid"][u])
        kept_raw, _ = oracle.select(out["raw"][u, 0, :n], c["B"])
        np.testing.assert_array_equal(kept_raw, out["kept"][u, :len(kept_raw)])


def test_key_scaling_keeps_set():
    """Scaling every key by alpha > 0 scales S~ by alpha (both terms are
    linear in |k|); z-scores and the kept set are unchanged."""
    c = _small_case(seed=11)
    out1 = oracle.prune(c["k"], c["v"], c["pos"], c["n_seq"], c["L"], c["Hkv"], c["G"], c["st"],
                        c["p_cur"], c["B"], n_valid=c["n_valid"])
    out2 = oracle.prune(c["k"] * np.float32(4.0), c["v"], c["pos"], c["n_seq"], c["L"], c["Hkv"],
                        c["G"], c["st"], c["p_cur"], c["B"], n_valid=c["n_valid"])
    np.testing.assert_array_equal(out1["kept"], out2["kept"])
    ok = ~np.isnan(out1["raw"])
    np.testing.assert_allclose(out2["raw"][ok], 4.0 * out1["raw"][ok], rtol=1e-12, atol=1e-12)


def test_duplicated_heads_equal_single_head():
    """A group of identical query heads gives the same final score as one head."""
    rng = np.random.default_rng(12)
    q = rng.normal(size=(1, 40, D)).astype(np.float32) + 1.0
    st1 = oracle.calibrate(q)
    st3 = np.repeat(st1, 3, axis=0)
    k = rng.normal(size=(200, D)).astype(np.float32)
    pos = np.arange(200, dtype=np.int32)
    _, f1, _, _ = oracle.znorm_max(oracle.score(k, pos, 200, st1))
    _, f3, _, _ = oracle.znorm_max(oracle.score(k, pos, 200, st3))
    np.testing.assert_array_equal(f1, f3)


def test_unit_phasor_MRL_matches_R():
    """With every |q_f| equal, R_f is the mean resultant length of unit
    phasors |mean_i e^{j theta_i}| (paper reading, MRL definition)."""
    rng = np.random.default_rng(13)
    n = 500
    ang = rng.vonmises(0.3, 2.0, size=(n, F))
    q = np.empty((1, n, D), np.float32)
    q[0, :, 0::2] = 2.0 * np.cos(ang)
    q[0, :, 1::2] = 2.0 * np.sin(ang)
    st = oracle.calibrate(q)
    a = np.arctan2(q[0, :, 1::2].astype(np.float64), q[0, :, 0::2])
    mrl = np.abs(np.mean(np.exp(1j * a), axis=0))
    np.testing.assert_allclose(st[0, :, 3], mrl, rtol=1e-6)


def test_measured_R_matches_rician_closed_form():
    """Centre + Gaussian noise with sigma from the Rician inversion gives the
    target R on average (statistical, +-0.01)."""
    import torch

    targets = np.array([0.6, 0.7, 0.8, 0.9, 0.95, 0.99])
    rng = np.random.default_rng(14)
    n = 40000
    g = torch.Generator().manual_seed(14)
    q = np.empty((len(targets), n, D), np.float32)
    for i, R in enumerate(targets):
        mag = 1.0 + rng.random(F)
        ph = rng.uniform(0, 2 * np.pi, F)
        s = synth.sigma_for_R(R) * mag
        noise = torch.randn((n, F, 2), generator=g, dtype=torch.float64).numpy()
        q[i, :, 0::2] = mag * np.cos(ph) + s * noise[..., 0]
        q[i, :, 1::2] = mag * np.sin(ph) + s * noise[..., 1]
    st = oracle.calibrate(q)
    meas = st[..., 3].mean(axis=1)
    np.testing.assert_allclose(meas, targets, atol=0.01)


def test_rician_inversion_round_trip():
    for R in (0.3, 0.6, 0.75, 0.9, 0.98, 0.999):
        assert synth.rician_R(1.0 / synth.sigma_for_R(R)) == pytest.approx(R, abs=1e-9)
