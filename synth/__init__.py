"""Seeded synthetic KV-cache workloads shaped like the pages' workloads.

This module only makes inputs.  It holds none of the pruning arithmetic: no
score, no normalisation, no selection.  Both the oracle side and the CUDA side
of every test take their inputs from here, and nothing here depends on either.

The data model follows the workloads described with the method: in the
pre-RoPE space every query head and key head concentrates around a fixed
per-band centre (TriAttention paper reading, shibing624 blog, section on the
pre-RoPE Q/K concentration: most heads have R > 0.9), keys are then rotated by
RoPE at their positions (talk announcement, qingkeai.online, RoPE rotation
equation, theta = 10000, interleaved pairs (x_2f, x_2f+1)), and values are
standard normal.  The pages' own workloads (32K-token reasoning traces from
AIME / MATH500 runs) are not available; these shapes stand in for them.

Noise level.  With a complex centre c_f of magnitude nu and independent
N(0, s^2) noise on each real component, |q_f| is Rician, and the expected
concentration E|.|-ratio R = nu / E|q_f| has the closed form
    R(r) = r / (sqrt(pi/2) * L_{1/2}(-r^2/2)),  r = nu / s,
with the Laguerre function L_{1/2}(-x) = e^{-x/2}[(1+x) I0(x/2) + x I1(x/2)].
``sigma_for_R`` inverts it, so a target R_f ~ U[lo, hi] per (head, band) can
be met by choosing s.  Random numbers come from seeded numpy / torch
generators; the bulk tensors are drawn on the device they are used on.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Sequence

import numpy as np
import torch

ROPE_THETA = 10000.0


# --------------------------------------------------------------------------
# Rician concentration
# --------------------------------------------------------------------------

def rician_R(r: float) -> float:
    """Expected |E[q]| / E[|q|] for centre magnitude / per-component sigma = r."""
    from scipy.special import i0e, i1e

    if r <= 0.0:
        return 0.0
    x = 0.5 * r * r
    # L_{1/2}(-x) e^{...} written with exponentially scaled Bessel functions.
    lag = (1.0 + x) * i0e(0.5 * x) + x * i1e(0.5 * x)
    return float(r / (math.sqrt(math.pi / 2.0) * lag))


def sigma_for_R(R: float) -> float:
    """Per-component noise sigma / centre magnitude that gives expected R."""
    if R >= 1.0 - 1e-12:
        return 0.0
    if R <= 0.0:
        return math.inf
    lo, hi = math.log(1e-6), math.log(1e6)
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if rician_R(math.exp(mid)) < R:
            lo = mid
        else:
            hi = mid
    return 1.0 / math.exp(0.5 * (lo + hi))


# --------------------------------------------------------------------------
# Specs of the five workloads
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    n_seq: int
    n_layers: int
    n_kvheads: int
    G: int
    cap: int            # rows per unit in the cache buffer
    n_valid: int        # valid keys per unit
    B: int              # budget
    dtype: str          # "bf16" or "f32"
    n_cal: int          # calibration query tokens per head
    p_cur: int          # current position (the next query position)
    positions: str = "dense"       # "dense" 0..n-1, or "scattered" (see make_positions)
    R_range: Optional[tuple] = None  # per-band target R ~ U[lo, hi]; None: sigma = 0.2|c|
    outlier_frac: float = 0.0
    outlier_scale: float = 4.0
    d: int = 128
    seed: int = 0
    stream: int = 0

    @property
    def n_units(self) -> int:
        return self.n_seq * self.n_layers * self.n_kvheads

    @property
    def n_qheads(self) -> int:
        return self.n_kvheads * self.G

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def esize(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def scaled(self, **kw) -> "Spec":
        return dataclasses.replace(self, **kw)


# Config strings as stated with the workloads; seeds: 0, stream = config number.
SPECS: Dict[str, Spec] = {
    # single head, fp32, 4096 keys at positions 0..4095, p_cur 4096, B 512,
    # centre magnitude ~N(1,0.3), sigma = 0.2 |centre| per component, 8192 cal queries.
    "c1": Spec("c1", 1, 1, 1, 1, 4096, 4096, 512, "f32", 8192, 4096, stream=1),
    # one layer, 28 query / 4 KV heads, 32768 bf16 keys, B 2048, R_f ~ U[0.6, 1].
    "c2": Spec("c2", 1, 1, 4, 7, 32768, 32768, 2048, "bf16", 10240, 32768,
               R_range=(0.6, 1.0), stream=2),
    # windowed decode step: 28 layers x 4 KV heads x 16 sequences, 3072 kept + 128
    # new keys at scattered ascending positions up to 32768, B 3072.
    "c3": Spec("c3", 16, 28, 4, 7, 3200, 3200, 3072, "bf16", 10240, 32768,
               positions="scattered", R_range=(0.6, 1.0), stream=3),
    # long prefill compaction: 32 layers x 8 KV heads x 4 sequences, 131072 keys,
    # B 4096, 5% heavy-norm outliers (x4).
    "c4": Spec("c4", 4, 32, 8, 4, 131072, 131072, 4096, "bf16", 10240, 131072,
               R_range=(0.6, 1.0), outlier_frac=0.05, stream=4),
    # streaming: 28 layers x 4 KV heads x 64 sequences, B 2048, prune every 128
    # generated tokens up to 32768 tokens (cap = B + 128).
    "c5": Spec("c5", 64, 28, 4, 7, 2176, 2176, 2048, "bf16", 10240, 2176,
               R_range=(0.6, 1.0), stream=5),
}

STREAM_WINDOW = 128          # prune every 128 generated tokens
STREAM_TOKENS = 32768        # tokens generated in the streaming workload


# --------------------------------------------------------------------------
# Head parameters (small, numpy float64)
# --------------------------------------------------------------------------

@dataclasses.dataclass
class HeadParams:
    q_centre: np.ndarray   # [L, Hq, F] complex128
    q_sigma: np.ndarray    # [L, Hq, F] float64 (per real component)
    k_centre: np.ndarray   # [L, Hkv, F] complex128
    k_sigma: np.ndarray    # [L, Hkv, F]


def _centres(rng: np.random.Generator, shape) -> np.ndarray:
    mag = np.abs(rng.normal(1.0, 0.3, size=shape))
    ph = rng.uniform(0.0, 2.0 * math.pi, size=shape)
    return mag * np.exp(1j * ph)


def _sigmas(rng: np.random.Generator, centre: np.ndarray, R_range) -> np.ndarray:
    mag = np.abs(centre)
    if R_range is None:
        return 0.2 * mag
    R = rng.uniform(R_range[0], R_range[1], size=centre.shape)
    ratio = np.vectorize(sigma_for_R)(R)
    return ratio * mag


def head_params(spec: Spec) -> HeadParams:
    rng = np.random.default_rng([spec.seed, spec.stream, 1])
    F = spec.d // 2
    qc = _centres(rng, (spec.n_layers, spec.n_qheads, F))
    kc = _centres(rng, (spec.n_layers, spec.n_kvheads, F))
    qs = _sigmas(rng, qc, spec.R_range)
    ks = _sigmas(rng, kc, spec.R_range)
    return HeadParams(qc, qs, kc, ks)


# --------------------------------------------------------------------------
# Bulk tensors
# --------------------------------------------------------------------------

def _gen(device, *key: int) -> torch.Generator:
    g = torch.Generator(device=device)
    h = 0
    for k in key:
        h = (h * 1000003 + int(k) + 1) % (2 ** 62)
    g.manual_seed(h)
    return g


def rope_rotate(x: torch.Tensor, pos: torch.Tensor, theta: float = ROPE_THETA) -> torch.Tensor:
    """Rotate interleaved pairs of x [..., n, d] (float64) by RoPE at positions pos [..., n]."""
    d = x.shape[-1]
    f = torch.arange(d // 2, device=x.device, dtype=torch.float64)
    w = theta ** (-2.0 * f / d)
    ang = pos.to(torch.float64).unsqueeze(-1) * w
    c, s = torch.cos(ang), torch.sin(ang)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = torch.empty_like(x)
    out[..., 0::2] = c * xe - s * xo
    out[..., 1::2] = s * xe + c * xo
    return out


def _pre_rope(g, centre: np.ndarray, sigma: np.ndarray, n: int, device) -> torch.Tensor:
    """centre/sigma [H, F] -> samples [H, n, d] float64 (interleaved re/im)."""
    H, F = centre.shape
    cre = torch.as_tensor(centre.real, device=device).unsqueeze(1)
    cim = torch.as_tensor(centre.imag, device=device).unsqueeze(1)
    sg = torch.as_tensor(sigma, device=device).unsqueeze(1)
    noise = torch.randn((H, n, F, 2), generator=g, device=device, dtype=torch.float32).double()
    out = torch.empty((H, n, 2 * F), device=device, dtype=torch.float64)
    out[..., 0::2] = cre + sg * noise[..., 0]
    out[..., 1::2] = cim + sg * noise[..., 1]
    return out


def calib_queries(spec: Spec, hp: HeadParams, layer: int, device) -> torch.Tensor:
    """Pre-RoPE calibration queries of one layer: [Hq, n_cal, d] in the spec dtype."""
    g = _gen(device, spec.seed, spec.stream, 2, layer)
    q = _pre_rope(g, hp.q_centre[layer], hp.q_sigma[layer], spec.n_cal, device)
    return q.to(spec.torch_dtype)


def make_positions(spec: Spec, units: int, unit0: int, device) -> torch.Tensor:
    """Positions [units, n_valid] int32 for units unit0..unit0+units-1."""
    n = spec.n_valid
    if spec.positions == "dense":
        return torch.arange(n, device=device, dtype=torch.int32).expand(units, n).contiguous()
    # scattered: the last 128 positions are the newest window, the rest are a
    # sorted random subset of [0, p_cur - 128) (a cache already pruned before).
    new = STREAM_WINDOW
    old = n - new
    span = spec.p_cur - new
    g = _gen(device, spec.seed, spec.stream, 3, unit0)
    keys = torch.rand((units, span), generator=g, device=device)
    pick = torch.topk(keys, old, dim=1).indices
    pick, _ = torch.sort(pick, dim=1)
    tail = torch.arange(span, spec.p_cur, device=device).expand(units, new)
    return torch.cat([pick, tail], dim=1).to(torch.int32).contiguous()


def keys_values(spec: Spec, hp: HeadParams, unit0: int, units: int, pos: torch.Tensor,
                device, tag: int = 4):
    """Post-RoPE keys and values [units, n, d] for a run of consecutive units."""
    n = pos.shape[1]
    F = spec.d // 2
    L, Hkv = spec.n_layers, spec.n_kvheads
    u = torch.arange(unit0, unit0 + units)
    layer = ((u // Hkv) % L).numpy()
    kvh = (u % Hkv).numpy()
    centre = hp.k_centre[layer, kvh]       # [units, F]
    sigma = hp.k_sigma[layer, kvh]
    g = _gen(device, spec.seed, spec.stream, tag, unit0, units)
    pre = _pre_rope(g, centre, sigma, n, device)
    if spec.outlier_frac > 0:
        mask = torch.rand((units, n), generator=g, device=device) < spec.outlier_frac
        pre = torch.where(mask.unsqueeze(-1), pre * spec.outlier_scale, pre)
    k = rope_rotate(pre, pos).to(spec.torch_dtype)
    v = torch.randn((units, n, spec.d), generator=g, device=device,
                    dtype=torch.float32).to(spec.torch_dtype)
    return k, v


@dataclasses.dataclass
class Workload:
    spec: Spec
    hp: HeadParams
    k: torch.Tensor        # [U, cap, d]
    v: torch.Tensor        # [U, cap, d]
    pos: torch.Tensor      # [U, cap] int32
    n_valid: torch.Tensor  # [U] int32
    p_cur: torch.Tensor    # [n_seq] int64


def make_workload(spec: Spec, device, chunk_units: int = 32) -> Workload:
    """Full cache of a spec, drawn on ``device`` in chunks of units."""
    hp = head_params(spec)
    U, cap, d = spec.n_units, spec.cap, spec.d
    k = torch.zeros((U, cap, d), dtype=spec.torch_dtype, device=device)
    v = torch.zeros((U, cap, d), dtype=spec.torch_dtype, device=device)
    pos = torch.zeros((U, cap), dtype=torch.int32, device=device)
    for u0 in range(0, U, chunk_units):
        nu = min(chunk_units, U - u0)
        p = make_positions(spec, nu, u0, device)
        kk, vv = keys_values(spec, hp, u0, nu, p, device)
        k[u0:u0 + nu, :spec.n_valid] = kk
        v[u0:u0 + nu, :spec.n_valid] = vv
        pos[u0:u0 + nu, :spec.n_valid] = p
        del kk, vv, p
    n_valid = torch.full((U,), spec.n_valid, dtype=torch.int32, device=device)
    p_cur = torch.full((spec.n_seq,), spec.p_cur, dtype=torch.int64, device=device)
    return Workload(spec, hp, k, v, pos, n_valid, p_cur)


def stream_window(spec: Spec, hp: HeadParams, w: int, device, units: Optional[Sequence[int]] = None):
    """Keys, values and positions of generated-token window w (positions 128w..128w+127).

    Drawn for all units at once (so a unit's rows do not depend on which other
    units are requested), then optionally sliced to ``units``.
    """
    U = spec.n_units
    n = STREAM_WINDOW
    pos = torch.arange(w * n, (w + 1) * n, device=device, dtype=torch.int32).expand(U, n)
    k, v = keys_values(spec, hp, 0, U, pos, device, tag=1000 + w)
    if units is not None:
        idx = torch.as_tensor(list(units), device=device, dtype=torch.long)
        return k[idx], v[idx], pos[idx].contiguous()
    return k, v, pos.contiguous()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bfloat16 bit patterns of a tensor as a host uint16 array (for the oracle)."""
    if t.dtype != torch.bfloat16:
        raise TypeError("bf16_bits wants a bfloat16 tensor")
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def host_elems(t: torch.Tensor) -> np.ndarray:
    """Host copy of a key/query tensor in the form the oracle takes."""
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.detach().contiguous().cpu().numpy().astype(np.float32, copy=False)
