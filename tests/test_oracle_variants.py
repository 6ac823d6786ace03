"""Pins of the oracle's method variants (no GPU).

Each variant is checked against something other than the oracle's own
formula: the explicit rotate-then-dot RoPE logit, invariants that follow from
the definitions (rotation invariance of a norm-only score, the sign of the
norm weight, max >= mean), a pure relabelling of vector components, brute
force on tiny inputs, and per-layer runs with a single budget.

Variants (shibing624 paper reading, ablation and future-offset sections;
jaedaily.cn tutorial, streaming and budget paragraphs): the score without
S_trig, without the concentration weight R, the maximum over the offsets,
half-split band pairing, protected sink / recent keys, per-layer budgets;
plus the calibration of post-RoPE queries (rotated back by their positions).
"""
import itertools
import math

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import _rope_matrix_rotate, _stats_identical

D = 128
F = D // 2


def _case(seed=3, n=24, noisy=True):
    rng = np.random.default_rng(seed)
    qbar = rng.normal(size=D).astype(np.float32)
    if noisy:
        q = (qbar[None, None, :] + 0.7 * rng.normal(size=(1, 64, D))).astype(np.float32)
        st = oracle.calibrate(q)
    else:
        st = _stats_identical(qbar)
    pos = np.sort(rng.choice(100000, size=n, replace=False)).astype(np.int32)
    kpre = rng.normal(size=(n, D))
    kpost = np.stack([_rope_matrix_rotate(kpre[j], pos[j]) for j in range(n)]).astype(np.float32)
    return qbar, st, kpost, pos, 100001


# ---------------------------------------------------------------------------
# without S_trig
# ---------------------------------------------------------------------------
def test_no_trig_is_blind_to_band_phases():
    """The score without S_trig depends on each band's norm only: turning any
    band of any key by any angle leaves it unchanged (the full score moves)."""
    _, st, k, pos, p_cur = _case()
    rng = np.random.default_rng(4)
    k2 = k.astype(np.float64).copy()
    for f in range(F):
        a = rng.uniform(0, 2 * math.pi, size=k.shape[0])
        x, y = k2[:, 2 * f].copy(), k2[:, 2 * f + 1].copy()
        k2[:, 2 * f] = np.cos(a) * x - np.sin(a) * y
        k2[:, 2 * f + 1] = np.sin(a) * x + np.cos(a) * y
    k2 = k2.astype(np.float32)
    s1 = oracle.score(k, pos, p_cur, st, variant=oracle.VAR_NO_TRIG)
    s2 = oracle.score(k2, pos, p_cur, st, variant=oracle.VAR_NO_TRIG)
    np.testing.assert_allclose(s1, s2, rtol=1e-6)
    full1 = oracle.score(k, pos, p_cur, st)
    full2 = oracle.score(k2, pos, p_cur, st)
    assert np.max(np.abs(full1 - full2)) > 1e-2 * np.max(np.abs(full1))


def test_no_trig_with_concentrated_queries_is_zero():
    """Identical calibration queries give R_f = 1, so the norm weight
    (1 - R_f) E|q_f| vanishes and nothing is left without S_trig."""
    _, st, k, pos, p_cur = _case(noisy=False)
    s = oracle.score(k, pos, p_cur, st, variant=oracle.VAR_NO_TRIG)
    assert np.max(np.abs(s)) < 1e-10 * np.abs(k).sum()


# ---------------------------------------------------------------------------
# without the concentration weight R
# ---------------------------------------------------------------------------
def test_no_r_score_bounds():
    """E|q_f| >= |E q_f| (mean of norms >= norm of the mean), so every
    offset's S_trig + E|q_f| |k_f| is >= 0: the score without R is never
    negative.  Dropping the (1 - R_f) factor adds R_f E|q_f| |k_f| >= 0, so it
    is never below the default score either (which may be negative)."""
    _, st, k, pos, p_cur = _case()
    base = oracle.score(k, pos, p_cur, st)
    nor = oracle.score(k, pos, p_cur, st, variant=oracle.VAR_NO_R)
    scale = np.abs(k).sum() * np.abs(st[..., 2]).sum()
    assert np.all(nor >= -1e-12 * scale)
    assert np.all(nor - base >= -1e-12 * scale)
    assert np.max(nor - base) > 1e-3 * np.max(np.abs(base))


def test_no_r_equals_default_for_centreless_queries():
    """Symmetric queries {q, -q}: E[q_f] = 0, R_f = 0, so the weight is E|q_f|
    either way and the two scores agree."""
    rng = np.random.default_rng(5)
    qbar = rng.normal(size=D).astype(np.float32)
    st = oracle.calibrate(np.stack([qbar, -qbar])[None])
    k = rng.normal(size=(12, D)).astype(np.float32)
    pos = rng.integers(0, 9000, size=12).astype(np.int32)
    np.testing.assert_array_equal(oracle.score(k, pos, 9000, st),
                                  oracle.score(k, pos, 9000, st, variant=oracle.VAR_NO_R))


# ---------------------------------------------------------------------------
# maximum over the offsets
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("offsets", [(1,), (3, 1000), oracle.OFFSETS])
def test_max_over_offsets_equals_explicit_rope_logit_max(offsets):
    """With every query at its centre (R = 1, no norm term), the variant is
    the maximum over the future query positions p_cur + delta of the explicit
    post-RoPE dot product."""
    qbar, st, k, pos, p_cur = _case(noisy=False)
    got = oracle.score(k, pos, p_cur, st, offsets=offsets, variant=oracle.VAR_MAX_OFFSET)[0]
    want = np.full(k.shape[0], -np.inf)
    for dlt in offsets:
        qrot = _rope_matrix_rotate(qbar.astype(np.float64), p_cur + dlt)
        want = np.maximum(want, k.astype(np.float64) @ qrot)
    scale = np.abs(k).sum(1) * np.abs(qbar).sum()
    assert np.max(np.abs(got - want) / scale) < 1e-12


def test_max_over_offsets_bounds_the_mean():
    _, st, k, pos, p_cur = _case()
    mean = oracle.score(k, pos, p_cur, st)
    mx = oracle.score(k, pos, p_cur, st, variant=oracle.VAR_MAX_OFFSET)
    assert np.all(mx >= mean - 1e-12 * np.abs(mean).max())
    assert np.max(mx - mean) > 1e-3 * np.abs(mean).max()


# ---------------------------------------------------------------------------
# half-split band pairing
# ---------------------------------------------------------------------------
def _half_to_interleaved(x):
    """Relabel components: (x_f, x_{f+d/2}) -> (x_2f, x_2f+1)."""
    out = np.empty_like(x)
    out[..., 0::2] = x[..., :F]
    out[..., 1::2] = x[..., F:]
    return out


def test_half_split_is_a_relabelling_of_interleaved():
    rng = np.random.default_rng(6)
    q = (rng.normal(size=(2, 40, D)) + rng.normal(size=(2, 1, D))).astype(np.float32)
    k = rng.normal(size=(30, D)).astype(np.float32)
    pos = np.sort(rng.choice(40000, 30, replace=False)).astype(np.int32)
    st_h = oracle.calibrate(q, half=True)
    st_i = oracle.calibrate(_half_to_interleaved(q))
    np.testing.assert_array_equal(st_h, st_i)
    for var in (0, oracle.VAR_MAX_OFFSET):
        got = oracle.score(k, pos, 40001, st_h, variant=var | oracle.VAR_HALF_SPLIT)
        want = oracle.score(_half_to_interleaved(k), pos, 40001, st_i, variant=var)
        np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------------------
# calibration from post-RoPE queries
# ---------------------------------------------------------------------------
def test_post_rope_calibration_recovers_pre_rope_stats():
    """Queries rotated by their positions (explicit RoPE matrices), then
    calibrated with those positions, give the statistics of the unrotated
    queries; without the positions they do not."""
    rng = np.random.default_rng(7)
    n = 50
    qpre = (rng.normal(size=(1, n, D)) * 0.4 + rng.normal(size=(1, 1, D)))
    pos = rng.integers(0, 30000, size=n).astype(np.int32)
    qpost = np.stack([_rope_matrix_rotate(qpre[0, j], pos[j]) for j in range(n)])[None]
    st_pre = oracle.calibrate(qpre.astype(np.float32))
    st_post = oracle.calibrate(qpost.astype(np.float32), pos=pos)
    scale = st_pre[..., 2:3]
    assert np.max(np.abs(st_post[..., :3] - st_pre[..., :3]) / scale) < 1e-5
    assert np.max(np.abs(st_post[..., 3] - st_pre[..., 3])) < 1e-5
    st_raw = oracle.calibrate(qpost.astype(np.float32))
    assert np.max(np.abs(st_raw[..., 3] - st_pre[..., 3])) > 0.05


# ---------------------------------------------------------------------------
# protected sink / recent keys
# ---------------------------------------------------------------------------
def _beats(vals, a, b):
    va, vb = vals[a], vals[b]
    na, nb = math.isnan(va), math.isnan(vb)
    if na != nb:
        return nb
    if not na and va != vb:
        return va > vb
    return a < b


@pytest.mark.parametrize("seed", range(8))
def test_protected_selection_matches_brute_force(seed):
    """Kept = every protected key (the lowest-indexed ones if they exceed B)
    plus the unique set of unprotected keys of the right size whose every
    member outranks every unprotected non-member."""
    rng = np.random.default_rng(300 + seed)
    n = int(rng.integers(1, 10))
    vals = list(rng.choice([-1.0, 0.0, 0.5, 1.0, 2.0, np.nan], size=n))
    for n_sink, n_recent in [(0, 0), (1, 0), (0, 2), (2, 3), (5, 5)]:
        prot = [j for j in range(n) if j < n_sink or j >= n - n_recent]
        free = [j for j in range(n) if j not in prot]
        for B in range(0, n + 2):
            m = min(B, n)
            if len(prot) >= m:
                want = prot[:m]
            else:
                found = [list(S) for S in itertools.combinations(free, m - len(prot))
                         if all(_beats(vals, a, b) for a in S for b in free if b not in S)]
                assert len(found) == 1
                want = sorted(prot + found[0])
            kept, _ = oracle.select_protected(np.asarray(vals), B, n_sink, n_recent)
            assert list(kept) == want, (n_sink, n_recent, B)
    kept0, t0 = oracle.select_protected(np.asarray(vals), 3, 0, 0)
    kept1, t1 = oracle.select(np.asarray(vals), 3)
    assert list(kept0) == list(kept1)


# ---------------------------------------------------------------------------
# per-layer budgets
# ---------------------------------------------------------------------------
def test_layer_budgets_equal_single_budget_runs():
    from tests.test_oracle_pins import _small_case

    c = _small_case()
    budgets = [37, c["B"]]
    out = oracle.prune(c["k"], c["v"], c["pos"], c["n_seq"], c["L"], c["Hkv"], c["G"], c["st"],
                       c["p_cur"], c["B"], n_valid=c["n_valid"], layer_budget=budgets)
    for layer, Bl in enumerate(budgets):
        ref = oracle.prune(c["k"], c["v"], c["pos"], c["n_seq"], c["L"], c["Hkv"], c["G"], c["st"],
                           c["p_cur"], Bl, n_valid=c["n_valid"])
        for u in range(c["U"]):
            if (u // c["Hkv"]) % c["L"] != layer:
                continue
            m = int(ref["n_kept"][u])
            assert out["n_kept"][u] == m
            np.testing.assert_array_equal(out["kept"][u, :m], ref["kept"][u, :m])
            np.testing.assert_array_equal(out["k_dst"][u, :m], ref["k_dst"][u, :m])
    with pytest.raises(ValueError):
        oracle.prune(c["k"], c["v"], c["pos"], c["n_seq"], c["L"], c["Hkv"], c["G"], c["st"],
                     c["p_cur"], c["B"], n_valid=c["n_valid"], layer_budget=[c["B"] + 1, 1])


# ---------------------------------------------------------------------------
# decode attention over the kept keys
# ---------------------------------------------------------------------------
def test_decode_attention_matches_library_sdpa():
    """Against torch's scaled_dot_product_attention in float64 on the CPU (a
    library routine), per unit and head, over the first n_valid rows."""
    import torch

    rng = np.random.default_rng(11)
    U, G, cap = 3, 4, 50
    q = rng.normal(size=(U, G, D)).astype(np.float32)
    k = rng.normal(size=(U, cap, D)).astype(np.float32)
    v = rng.normal(size=(U, cap, D)).astype(np.float32)
    nv = np.array([50, 17, 1], np.int32)
    got = oracle.decode_attention(q, k, v, n_valid=nv)
    for u in range(U):
        n = int(nv[u])
        qq = torch.from_numpy(q[u].astype(np.float64))[:, None, :]          # [G, 1, d]
        kk = torch.from_numpy(k[u, :n].astype(np.float64))[None].expand(G, n, D)
        vv = torch.from_numpy(v[u, :n].astype(np.float64))[None].expand(G, n, D)
        want = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[:, 0].numpy()
        np.testing.assert_allclose(got[u], want, rtol=1e-12, atol=1e-12)


def test_decode_attention_special_cases():
    """A zero query weighs every kept key equally (the mean of the values);
    one kept key returns its value; a key scored far above the others takes
    all the weight; no kept key gives zeros; reordering the keys changes
    nothing."""
    rng = np.random.default_rng(12)
    cap = 40
    k = rng.normal(size=(1, cap, D)).astype(np.float32)
    v = rng.normal(size=(1, cap, D)).astype(np.float32)
    q0 = np.zeros((1, 2, D), np.float32)
    np.testing.assert_allclose(oracle.decode_attention(q0, k, v)[0, 0],
                               v[0].astype(np.float64).mean(0), rtol=1e-12, atol=1e-13)
    q = rng.normal(size=(1, 2, D)).astype(np.float32)
    np.testing.assert_allclose(oracle.decode_attention(q, k, v, n_valid=[1])[0, 1], v[0, 0],
                               rtol=1e-15)
    assert not oracle.decode_attention(q, k, v, n_valid=[0]).any()
    k2 = k.copy()
    k2[0, 7] = 40.0 * q[0, 0] / np.linalg.norm(q[0, 0])
    np.testing.assert_allclose(oracle.decode_attention(q, k2, v, scale=1.0)[0, 0], v[0, 7],
                               rtol=1e-9, atol=1e-9)
    perm = rng.permutation(cap)
    np.testing.assert_allclose(oracle.decode_attention(q, k[:, perm], v[:, perm]),
                               oracle.decode_attention(q, k, v), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# logit(Delta) reconstruction from the centres, measured curve, Pearson
# ---------------------------------------------------------------------------
def test_logit_reconstruction_is_the_rotated_centres_dot_product():
    """The trig series in Delta equals the explicit post-RoPE dot product of
    the centres, the query centre at position p + Delta and the key centre at
    p (talk page, RoPE logit general form), for any p."""
    rng = np.random.default_rng(13)
    qbar = rng.normal(size=D)
    kbar = rng.normal(size=D)
    qs = _stats_identical(qbar.astype(np.float32))
    ks = _stats_identical(kbar.astype(np.float32))
    deltas = [0, 1, 7, 100, 4097, 30000]
    got = oracle.logit_reconstruct(qs, ks, 1, deltas)[0]
    q32, k32 = qbar.astype(np.float32).astype(np.float64), kbar.astype(np.float32).astype(np.float64)
    for p in (0, 12345):
        want = [_rope_matrix_rotate(q32, p + dl) @ _rope_matrix_rotate(k32, p) for dl in deltas]
        np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-10 * np.abs(q32).sum() * np.abs(k32).sum())


def test_logit_curve_of_centred_sequences_equals_reconstruction():
    """Every query and key at its centre (token t rotated to position t): the
    measured mean logit at each distance is exactly the reconstruction, and
    their Pearson correlation is 1; GQA maps query head h to KV head h / G."""
    rng = np.random.default_rng(14)
    n, G = 64, 2
    qbar = rng.normal(size=(2 * G, D)).astype(np.float32)
    kbar = rng.normal(size=(2, D)).astype(np.float32)
    pos = np.arange(n)
    q = np.stack([[_rope_matrix_rotate(qbar[h].astype(np.float64), t) for t in pos]
                  for h in range(2 * G)])
    k = np.stack([[_rope_matrix_rotate(kbar[h].astype(np.float64), t) for t in pos]
                  for h in range(2)])
    deltas = [0, 1, 2, 5, 17, 40, 63, 64]
    curve = oracle.logit_curve(q.astype(np.float32), k.astype(np.float32), G, deltas)
    qs = np.concatenate([_stats_identical(x) for x in qbar])
    ks = np.concatenate([_stats_identical(x) for x in kbar])
    recon = oracle.logit_reconstruct(qs, ks, G, deltas)
    scale = np.abs(qbar).sum() * np.abs(kbar).sum()
    np.testing.assert_allclose(curve[:, :-1], recon[:, :-1], atol=1e-5 * scale)
    assert np.all(curve[:, -1] == 0.0)       # no pair is 64 apart in 64 tokens
    r = oracle.pearson(curve[:, :-1], recon[:, :-1])
    np.testing.assert_allclose(r, 1.0, atol=1e-9)


def test_pearson_matches_numpy():
    rng = np.random.default_rng(15)
    a = rng.normal(size=(5, 40))
    b = 0.3 * a + rng.normal(size=(5, 40))
    want = [np.corrcoef(a[i], b[i])[0, 1] for i in range(5)]
    np.testing.assert_allclose(oracle.pearson(a, b), want, rtol=1e-12)
    assert oracle.pearson(np.ones((1, 8)), a[:1, :8])[0] == 0.0
