"""Float64 CPU oracle for TriAttention KV-cache pruning (test infrastructure).

This package is the correctness reference for the CUDA library.  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import it.  The library under ``rope_aware_kv_b200`` never imports,
links or calls anything here, and the two share no code.

The arithmetic lives in ``tri_oracle.c`` (plain C, double precision, OpenMP
over units); this module compiles it with gcc and marshals numpy arrays.
Every function follows the pages step by step:

* ``calibrate`` -- per-band query centre, mean norm and R_f = |E q_f| / E|q_f|
  (TriAttention talk announcement, qingkeai.online: S_norm equation and the
  R_f definition; hyper.ai summary of arXiv 2604.04921, Method section).
* ``score`` -- de-rotate each post-RoPE key by its position, then the explicit
  S_trig + S_norm sum averaged over the offsets D (talk page: RoPE rotation,
  RoPE logit general form, S_trig, S_norm and S~ equations).
* ``znorm_max`` -- z-score per query head, max over the GQA group (hyper.ai
  summary, Method section, "normalise then aggregate").
* ``select`` -- top-B by (score desc, index asc), returned ascending
  (jaedaily.cn KV-compression tutorial, eviction step).
* ``prune`` -- all of the above plus the bit-exact gather, over many units.
* ``logit_reconstruct`` / ``logit_curve`` / ``pearson`` -- the trig-series
  logit(Delta) from the Q/K centres, the measured mean logit at each distance,
  and their correlation (talk page, centre approximation; paper reading,
  Fig. 1(D)).
* ``decode_attention`` -- softmax attention of the next token's queries over
  the kept keys, renormalised over them (jaedaily.cn tutorial, compression
  objective), the consumer of the compacted cache.

Method variants (``variant`` bits, protection and per-layer budgets of
``prune``; ``calibrate`` with positions and pairing) follow the pages'
ablations and alternatives, see ``tri_oracle.c``.

Parity status: every function is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` against closed forms, brute force and
invariants; absolute score values at real-model scale are unpinned because the
pages print no worked example.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tri_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32 = 0
BF16 = 1

# The pages' constants: theta = 10000 and D = {1, 2, 4, ..., 2^16} (talk page,
# RoPE rotation and the offset-averaged score S~).
THETA = 10000.0
OFFSETS = tuple(1 << i for i in range(17))

# Variant bits (tri_oracle.c: ORA_VAR_*).
VAR_NO_TRIG = 1
VAR_NO_R = 2
VAR_MAX_OFFSET = 4
VAR_HALF_SPLIT = 8

_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source with gcc (IEEE math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fopenmp", "-shared", "-fPIC",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    if _lib is None:
        build()
        _bind(ctypes.CDLL(_LIB))
    return _lib


def _bind(lib):
    global _lib
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    i32 = ctypes.c_int
    d = ctypes.c_double
    lib.oracle_calibrate.argtypes = [P, i32, i64, i64, i32, P]
    lib.oracle_calibrate.restype = i32
    lib.oracle_calibrate_ex.argtypes = [P, i32, i64, i64, i32, P, d, i32, P]
    lib.oracle_calibrate_ex.restype = i32
    lib.oracle_select_protected.argtypes = [P, i64, i64, i64, i64, P, P]
    lib.oracle_select_protected.restype = i64
    lib.oracle_score.argtypes = [P, i32, i64, i32, P, i64, P, i32, d, P, i32, i32, P]
    lib.oracle_score.restype = i32
    lib.oracle_znorm_max.argtypes = [P, i32, i64, P, P, P, P]
    lib.oracle_znorm_max.restype = i32
    lib.oracle_select.argtypes = [P, i64, i64, P, P]
    lib.oracle_select.restype = i64
    lib.oracle_prune.argtypes = [P, P, P, i32, i64, i64, i64, i32, i64, i32, P, P, P, d, P,
                                 i32, i64, P, P, P, P, P, P, P, P, i64, P, i64, i32, i64, i64, P]
    lib.oracle_prune.restype = i32
    lib.oracle_decode_attention.argtypes = [P, P, P, i32, i64, i32, i64, i32, P, d, P]
    lib.oracle_decode_attention.restype = i32
    lib.oracle_logit_reconstruct.argtypes = [P, P, i64, i32, i32, d, P, i64, P]
    lib.oracle_logit_reconstruct.restype = i32
    lib.oracle_logit_curve.argtypes = [P, P, i32, i64, i32, i64, i32, P, i64, P]
    lib.oracle_logit_curve.restype = i32
    lib.oracle_pearson.argtypes = [P, P, i64, i64, P]
    lib.oracle_pearson.restype = i32
    lib.oracle_threads.argtypes = []
    lib.oracle_threads.restype = i32
    lib.oracle_set_threads.argtypes = [i32]
    lib.oracle_set_threads.restype = None
    _lib = lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _elem(a: np.ndarray):
    """Map a numpy key/query array to (contiguous array, oracle dtype code).

    float32 arrays are float32; uint16 arrays hold raw bfloat16 bit patterns.
    """
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"oracle takes float32 or raw-bf16 uint16 arrays, got {a.dtype}")


class using_library:
    """Temporarily route every call through another build of the oracle
    (used by the mutation tests, which compile deliberately broken copies)."""

    def __init__(self, path: str):
        self.path = path
        self.saved = None

    def __enter__(self):
        global _lib
        self.saved = _load()
        _lib = None
        _bind(ctypes.CDLL(self.path))
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def threads() -> int:
    return int(_load().oracle_threads())


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def calibrate(q: np.ndarray, pos=None, theta: float = THETA, half: bool = False) -> np.ndarray:
    """q: [H, n_tok, d] queries -> stats [H, d/2, 4] (re, im, mean|q_f|, R_f).

    Pre-RoPE queries by default; with ``pos`` ([n_tok] positions) the queries
    are post-RoPE and are rotated back first.  ``half``: half-split bands."""
    q, dt = _elem(q)
    H, n, d = q.shape
    out = np.empty((H, d // 2, 4), np.float64)
    if pos is None and not half:
        rc = _load().oracle_calibrate(_ptr(q), dt, H, n, d, _ptr(out))
    else:
        pp = None if pos is None else np.ascontiguousarray(np.asarray(pos, np.int32))
        rc = _load().oracle_calibrate_ex(_ptr(q), dt, H, n, d, _ptr(pp), float(theta),
                                         1 if half else 0, _ptr(out))
    if rc:
        raise ValueError(f"oracle_calibrate failed ({rc})")
    return out


def score(k: np.ndarray, pos: np.ndarray, p_cur: int, stats: np.ndarray,
          theta: float = THETA, offsets=OFFSETS, variant: int = 0) -> np.ndarray:
    """Per-head S~ for one unit: k [n, d] post-RoPE, pos [n], stats [G, d/2, 4] -> [G, n]."""
    k, dt = _elem(k)
    n, d = k.shape
    pos = np.ascontiguousarray(pos, np.int32)
    st = np.ascontiguousarray(stats, np.float64)
    G = st.shape[0]
    off = np.ascontiguousarray(np.asarray(offsets, np.int64))
    out = np.empty((G, n), np.float64)
    rc = _load().oracle_score(_ptr(k), dt, n, d, _ptr(pos), int(p_cur), _ptr(st), G,
                              float(theta), _ptr(off), len(off), int(variant), _ptr(out))
    if rc:
        raise ValueError(f"oracle_score failed ({rc})")
    return out


def znorm_max(raw: np.ndarray):
    """raw [G, n] -> (z [G, n], final [n], mu [G], sigma [G])."""
    raw = np.ascontiguousarray(raw, np.float64)
    G, n = raw.shape
    z = np.empty((G, n), np.float64)
    fin = np.empty((n,), np.float64)
    mu = np.empty((G,), np.float64)
    sd = np.empty((G,), np.float64)
    rc = _load().oracle_znorm_max(_ptr(raw), G, n, _ptr(z), _ptr(fin), _ptr(mu), _ptr(sd))
    if rc:
        raise ValueError(f"oracle_znorm_max failed ({rc})")
    return z, fin, mu, sd


def select(final: np.ndarray, B: int):
    """final [n] -> (kept indices ascending [min(B, n)], B-th score)."""
    fin = np.ascontiguousarray(final, np.float64)
    n = fin.shape[0]
    kept = np.empty((max(min(B, n), 1),), np.int32)
    thr = ctypes.c_double(0.0)
    m = _load().oracle_select(_ptr(fin), n, int(B), _ptr(kept), ctypes.byref(thr))
    if m < 0:
        raise ValueError("oracle_select failed")
    return kept[:m].copy(), thr.value


def select_protected(final: np.ndarray, B: int, n_sink: int, n_recent: int):
    """Top-B with the first n_sink and last n_recent keys always kept ->
    (kept ascending, score of the last unprotected key kept)."""
    fin = np.ascontiguousarray(final, np.float64)
    n = fin.shape[0]
    kept = np.empty((max(min(B, n), 1),), np.int32)
    thr = ctypes.c_double(0.0)
    m = _load().oracle_select_protected(_ptr(fin), n, int(B), int(n_sink), int(n_recent),
                                        _ptr(kept), ctypes.byref(thr))
    if m < 0:
        raise ValueError("oracle_select_protected failed")
    return kept[:m].copy(), thr.value


def prune(k, v, pos, n_seq, n_layers, n_kvheads, G, stats, p_cur, B, n_valid=None,
          theta=THETA, offsets=OFFSETS, units=None, want_raw=True, want_gather=True,
          variant=0, n_sink=0, n_recent=0, layer_budget=None):
    """Whole prune step on [U, cap, d] caches (see tri_oracle.c: oracle_prune).

    stats: [n_layers, n_kvheads*G, d/2, 4] float64.  Returns a dict with
    raw [U, G, cap], final [U, cap], kept [U, B], n_kept [U], thr [U] and,
    when ``want_gather``, k_dst / v_dst [U, B, d] and pos_dst [U, B].  Rows of
    units not in ``units`` are left as NaN / -1 / zero.
    """
    k, dt = _elem(k)
    v2, dtv = _elem(v) if v is not None else (None, dt)
    if v2 is not None and dtv != dt:
        raise TypeError("k and v must share a dtype")
    U, cap, d = k.shape
    if U != n_seq * n_layers * n_kvheads:
        raise ValueError("k.shape[0] must equal n_seq * n_layers * n_kvheads")
    pos = np.ascontiguousarray(pos, np.int32)
    st = np.ascontiguousarray(stats, np.float64)
    pc = np.ascontiguousarray(np.asarray(p_cur, np.int64).reshape(-1))
    nv = None if n_valid is None else np.ascontiguousarray(np.asarray(n_valid, np.int32))
    off = np.ascontiguousarray(np.asarray(offsets, np.int64))
    ul = None if units is None else np.ascontiguousarray(np.asarray(units, np.int64))
    lb = None if layer_budget is None else np.ascontiguousarray(np.asarray(layer_budget, np.int64))
    raw = np.full((U, G, cap), np.nan) if want_raw else None
    fin = np.full((U, cap), np.nan)
    kept = np.full((U, max(B, 1)), -1, np.int32)
    nk = np.zeros((U,), np.int64)
    thr = np.full((U,), np.nan)
    kd = vd = pd = None
    if want_gather:
        kd = np.zeros((U, B, d), k.dtype)
        vd = np.zeros((U, B, d), k.dtype) if v2 is not None else None
        pd = np.full((U, B), -1, np.int32)
    rc = _load().oracle_prune(
        _ptr(k), _ptr(v2), _ptr(pos), dt, n_seq, n_layers, n_kvheads, G, cap, d, _ptr(nv),
        _ptr(pc), _ptr(st), float(theta), _ptr(off), len(off), int(B), _ptr(raw), _ptr(fin),
        _ptr(kept), _ptr(nk), _ptr(thr), _ptr(kd), _ptr(vd), _ptr(pd), B if want_gather else 0,
        _ptr(ul), 0 if ul is None else len(ul), int(variant), int(n_sink), int(n_recent),
        _ptr(lb))
    if rc:
        raise ValueError(f"oracle_prune failed ({rc})")
    out = dict(final=fin, kept=kept[:, :B], n_kept=nk, thr=thr)
    if want_raw:
        out["raw"] = raw
    if want_gather:
        out.update(k_dst=kd, v_dst=vd, pos_dst=pd)
    return out


def decode_attention(q, k, v, n_valid=None, scale=None):
    """Attention of one query token per head over a cache (tri_oracle.c:
    oracle_decode_attention).  q [U, G, d], k / v [U, cap, d] (float32 or raw
    bf16 uint16, one type) -> out [U, G, d] float64."""
    q, dt = _elem(q)
    k, dtk = _elem(k)
    v, dtv = _elem(v)
    if not dt == dtk == dtv:
        raise TypeError("q, k and v must share a dtype")
    U, G, d = q.shape
    cap = k.shape[1]
    nv = None if n_valid is None else np.ascontiguousarray(np.asarray(n_valid, np.int32))
    sc = 1.0 / np.sqrt(d) if scale is None else float(scale)
    out = np.empty((U, G, d), np.float64)
    rc = _load().oracle_decode_attention(_ptr(q), _ptr(k), _ptr(v), dt, U, G, cap, d, _ptr(nv),
                                         sc, _ptr(out))
    if rc:
        raise ValueError(f"oracle_decode_attention failed ({rc})")
    return out


def logit_reconstruct(qstats, kstats, G, deltas, theta=THETA):
    """Trig-series logit(Delta) from the Q and K centres: qstats [Hq, d/2, 4],
    kstats [Hq/G, d/2, 4] -> [Hq, len(deltas)] (tri_oracle.c)."""
    qs = np.ascontiguousarray(qstats, np.float64)
    ks = np.ascontiguousarray(kstats, np.float64)
    Hq, F = qs.shape[0], qs.shape[1]
    dl = np.ascontiguousarray(np.asarray(deltas, np.int64))
    out = np.empty((Hq, len(dl)), np.float64)
    rc = _load().oracle_logit_reconstruct(_ptr(qs), _ptr(ks), Hq, int(G), 2 * F, float(theta),
                                          _ptr(dl), len(dl), _ptr(out))
    if rc:
        raise ValueError(f"oracle_logit_reconstruct failed ({rc})")
    return out


def logit_curve(q, k, G, deltas):
    """Mean post-RoPE logit at each distance: q [Hq, n, d], k [Hq/G, n, d]
    -> [Hq, len(deltas)] (tri_oracle.c)."""
    q, dt = _elem(q)
    k, dtk = _elem(k)
    if dt != dtk:
        raise TypeError("q and k must share a dtype")
    Hq, n, d = q.shape
    dl = np.ascontiguousarray(np.asarray(deltas, np.int64))
    out = np.empty((Hq, len(dl)), np.float64)
    rc = _load().oracle_logit_curve(_ptr(q), _ptr(k), dt, Hq, int(G), n, d, _ptr(dl), len(dl),
                                    _ptr(out))
    if rc:
        raise ValueError(f"oracle_logit_curve failed ({rc})")
    return out


def pearson(a, b):
    """Row-wise Pearson correlation of a and b [rows, n] -> [rows]."""
    a = np.ascontiguousarray(a, np.float64)
    b = np.ascontiguousarray(b, np.float64)
    rows, n = a.shape
    out = np.empty((rows,), np.float64)
    rc = _load().oracle_pearson(_ptr(a), _ptr(b), rows, n, _ptr(out))
    if rc:
        raise ValueError(f"oracle_pearson failed ({rc})")
    return out
