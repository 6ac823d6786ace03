"""Python binding of libtri, the sm_100a TriAttention KV-pruning library.

Argument marshalling only: every function here checks tensor shapes and
dtypes, passes raw device pointers and sizes to the C ABI of
``include/tri.h`` through ctypes, and raises on a non-zero status.  Every
step of the method runs in the library's CUDA kernels.  PyTorch supplies the
device memory (tensors and workspaces) and the current CUDA stream.

There is no CPU fallback: importing works without a GPU (so the library can
be inspected and its symbols checked), but calling any entry point without
the built ``libtri.so`` or without a CUDA device raises.

Names follow the C ABI: ``tri_calibrate``, ``tri_score``, ``tri_select_topB``,
``tri_compact``, ``tri_prune``, ``tri_append``, ``tri_check_device_error`` and
the ``*_workspace_bytes`` queries.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtri.so")

TRI_F32 = 0
TRI_BF16 = 1

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape or type",
          3: "workspace missing or too small", 4: "CUDA error", 5: "device-side flag set",
          6: "request exceeds the static scratch"}

FLAG_NVALID_RANGE = 0x1
FLAG_INDEX_RANGE = 0x2
FLAG_NONFINITE = 0x4
FLAG_TIMEOUT = 0x8

MAX_OFFSETS = 64
HEAD_DIM = 128

PATH_AUTO = 0
PATH_FUSED = 1
PATH_SPLIT = 2
PATH_COOP = 3
PATH_PIPE = 4

# Symbols include/tri.h declares (checked by the ABI tests).
EXPORTS = (
    "tri_config_default", "tri_status_str", "tri_version",
    "tri_calibrate_workspace_bytes", "tri_calibrate", "tri_calibrate_sums", "tri_calibrate_finish",
    "tri_score_workspace_bytes", "tri_score",
    "tri_select_workspace_bytes", "tri_select_topB",
    "tri_compact_workspace_bytes", "tri_compact",
    "tri_prune_workspace_bytes", "tri_prune",
    "tri_append", "tri_check_device_error",
    "tri_set_timing_events", "tri_last_launch_count", "tri_set_phase_trace",
    "tri_select_topB_static", "tri_select_static_scratch_bytes", "tri_prune_path",
    "tri_compact_inplace", "tri_prune_inplace", "tri_calibrate_ex",
    "tri_decode_workspace_bytes", "tri_decode_attention",
    "tri_logit_reconstruct", "tri_logit_curve", "tri_pearson", "tri_prune_paged_inplace",
)


class TriError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {STATUS.get(code, 'unknown')} (status {code})")
        self.code = code


VAR_NO_TRIG = 0x1
VAR_NO_R = 0x2
VAR_MAX_OFFSET = 0x4
VAR_HALF_SPLIT = 0x8


class TriConfig(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int), ("theta", ctypes.c_double),
                ("n_offsets", ctypes.c_int), ("offsets", ctypes.c_int64 * MAX_OFFSETS),
                ("path", ctypes.c_int), ("variant", ctypes.c_int),
                ("n_sink", ctypes.c_int64), ("n_recent", ctypes.c_int64),
                ("layer_budget", ctypes.c_void_p), ("barrier_wait_ns", ctypes.c_int64)]


_lib = None


def library_path() -> str:
    return LIB_PATH


def load(path: Optional[str] = None):
    """Load libtri.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libtri.so not built at {p}; run `python -m rope_aware_kv_b200.build`")
    lib = ctypes.CDLL(p)
    P, i64, i32, sz, d = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_double
    u32p = ctypes.POINTER(ctypes.c_uint32)
    sig = {
        "tri_config_default": (None, [ctypes.POINTER(TriConfig), i32]),
        "tri_status_str": (ctypes.c_char_p, [i32]),
        "tri_version": (ctypes.c_char_p, []),
        "tri_calibrate_workspace_bytes": (sz, [i64, i64, i32]),
        "tri_calibrate": (i32, [P, i32, i64, i64, i32, P, P, sz, P]),
        "tri_calibrate_sums": (i32, [P, i32, i64, i64, i32, P, P, sz, P]),
        "tri_calibrate_finish": (i32, [P, i64, i64, i32, P, P]),
        "tri_prune_paged_inplace": (i32, [ctypes.POINTER(TriConfig), P, P, P, i32, i64, i64, i64,
                                          i32, i64, P, P, P, i64, P, i64, i64, i64, P, P, P, P, sz,
                                          P]),
        "tri_logit_reconstruct": (i32, [ctypes.POINTER(TriConfig), P, P, i64, i32, P, i64, P, P]),
        "tri_logit_curve": (i32, [P, P, i32, i64, i32, i64, i32, P, i64, P, P]),
        "tri_pearson": (i32, [P, P, i64, i64, P, P]),
        "tri_decode_workspace_bytes": (sz, [i64, i32, i64]),
        "tri_decode_attention": (i32, [P, P, P, i32, i64, i32, i64, i32, P, ctypes.c_float, P, P,
                                       sz, P]),
        "tri_calibrate_ex": (i32, [ctypes.POINTER(TriConfig), P, i32, i64, i64, i32, P, P, P, sz,
                                   P]),
        "tri_score_workspace_bytes": (sz, [i64, i64, i64, i32, i64, i32]),
        "tri_score": (i32, [ctypes.POINTER(TriConfig), P, i32, i64, i64, i64, i32, i64, P, P, P, P,
                            P, P, sz, P]),
        "tri_select_workspace_bytes": (sz, [i64, i64, i64]),
        "tri_select_topB": (i32, [P, i64, i64, P, i64, P, P, P, sz, P]),
        "tri_compact_workspace_bytes": (sz, []),
        "tri_compact": (i32, [P, P, P, i32, i64, i64, i32, P, P, i64, P, P, P, i64, P, sz, P]),
        "tri_prune_workspace_bytes": (sz, [i64, i64, i64, i32, i64, i64, i32]),
        "tri_prune": (i32, [ctypes.POINTER(TriConfig), P, P, P, i32, i64, i64, i64, i32, i64, P, P,
                            P, i64, P, P, P, i64, P, P, P, P, sz, P]),
        "tri_append": (i32, [P, P, P, i32, i64, i64, i64, i32, P, P, P, P, P, i64, P, sz, P]),
        "tri_check_device_error": (i32, [P, P, u32p]),
        "tri_set_timing_events": (i32, [ctypes.POINTER(ctypes.c_void_p), i32]),
        "tri_last_launch_count": (i32, []),
        "tri_set_phase_trace": (i32, [P, sz]),
        "tri_select_topB_static": (i32, [P, i64, i64, P, i64, P, P, P]),
        "tri_select_static_scratch_bytes": (sz, []),
        "tri_prune_path": (i32, [i64, i64, i64, i32, i64, i64, i32, i32, i32]),
        "tri_compact_inplace": (i32, [P, P, P, i32, i64, i64, i32, P, P, i64, P, sz, P]),
        "tri_prune_inplace": (i32, [ctypes.POINTER(TriConfig), P, P, P, i32, i64, i64, i64, i32,
                                    i64, P, P, P, i64, P, P, P, P, sz, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


# ---------------------------------------------------------------------------
# helpers (marshalling only)
# ---------------------------------------------------------------------------

def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TRI_BF16
    if t.dtype == torch.float32:
        return TRI_F32
    raise TypeError(f"keys/queries must be bfloat16 or float32, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libtri takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libtri takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, code: int):
    if code != 0:
        raise TriError(fn, code)


def config(theta: float = 10000.0, offsets: Optional[Sequence[int]] = None,
           head_dim: int = HEAD_DIM, path: int = PATH_AUTO, variant: int = 0,
           n_sink: int = 0, n_recent: int = 0,
           layer_budget: Optional[torch.Tensor] = None,
           barrier_wait_ns: int = 0) -> TriConfig:
    """Method parameters (tri.h: tri_config).  ``variant``: VAR_* bits;
    ``n_sink`` / ``n_recent``: protected first / last keys of every unit;
    ``layer_budget``: int32 CUDA tensor [n_layers] of per-layer budgets (the
    config keeps its pointer only: keep the tensor alive while it is used);
    ``barrier_wait_ns``: bound of the cooperative path's unit-barrier waits
    (0: 2 s; a short bound exists to test the timeout path)."""
    cfg = TriConfig()
    load().tri_config_default(ctypes.byref(cfg), head_dim)
    cfg.theta = float(theta)
    cfg.path = int(path)
    cfg.variant = int(variant)
    cfg.n_sink = int(n_sink)
    cfg.n_recent = int(n_recent)
    cfg.barrier_wait_ns = int(barrier_wait_ns)
    if layer_budget is not None:
        if layer_budget.dtype != torch.int32 or not layer_budget.is_cuda:
            raise TypeError("layer_budget must be an int32 CUDA tensor")
        cfg.layer_budget = layer_budget.data_ptr()
    if offsets is not None:
        offs = list(offsets)
        if not 1 <= len(offs) <= MAX_OFFSETS:
            raise ValueError("1..64 offsets")
        cfg.n_offsets = len(offs)
        for i, o in enumerate(offs):
            cfg.offsets[i] = int(o)
    return cfg


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A device byte buffer for the ``ws`` argument (256-byte aligned by torch)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------

def tri_calibrate_workspace_bytes(n_heads: int, n_tok: int, head_dim: int = HEAD_DIM) -> int:
    return load().tri_calibrate_workspace_bytes(n_heads, n_tok, head_dim)


def tri_calibrate(q_pre: torch.Tensor, stats: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """q_pre [..., n_tok, d] pre-RoPE queries -> stats [..., d/2, 4] float32."""
    *lead, n_tok, d = q_pre.shape
    H = 1
    for x in lead:
        H *= x
    if stats is None:
        stats = torch.empty((*lead, d // 2, 4), dtype=torch.float32, device=q_pre.device)
    need = tri_calibrate_workspace_bytes(H, n_tok, d)
    if ws is None:
        ws = workspace(need, q_pre.device)
    _check("tri_calibrate", load().tri_calibrate(_ptr(q_pre), _dt(q_pre), H, n_tok, d, _ptr(stats),
                                                _ptr(ws), ws.numel(), _stream(stream)))
    return stats


def tri_calibrate_ex(cfg: TriConfig, q: torch.Tensor, q_pos: Optional[torch.Tensor] = None,
                     stats: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Calibration with the config's band pairing; with ``q_pos`` ([n_tok]
    int32 positions) q holds post-RoPE rows that are rotated back first.
    q [..., n_tok, d] -> stats [..., d/2, 4] float32."""
    *lead, n_tok, d = q.shape
    H = 1
    for x in lead:
        H *= x
    if stats is None:
        stats = torch.empty((*lead, d // 2, 4), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(tri_calibrate_workspace_bytes(H, n_tok, d), q.device)
    _check("tri_calibrate_ex", load().tri_calibrate_ex(
        ctypes.byref(cfg), _ptr(q), _dt(q), H, n_tok, d, _ptr(q_pos), _ptr(stats), _ptr(ws),
        ws.numel(), _stream(stream)))
    return stats


def tri_calibrate_sums(q_pre: torch.Tensor, sums: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """q_pre [..., n_tok, d] (one shard's tokens) -> float64 sums [..., d/2, 3]."""
    *lead, n_tok, d = q_pre.shape
    H = 1
    for x in lead:
        H *= x
    if sums is None:
        sums = torch.empty((*lead, d // 2, 3), dtype=torch.float64, device=q_pre.device)
    need = tri_calibrate_workspace_bytes(H, n_tok, d)
    if ws is None:
        ws = workspace(need, q_pre.device)
    _check("tri_calibrate_sums", load().tri_calibrate_sums(
        _ptr(q_pre), _dt(q_pre), H, n_tok, d, _ptr(sums), _ptr(ws), ws.numel(), _stream(stream)))
    return sums


def tri_calibrate_finish(sums: torch.Tensor, n_tok_total: int,
                         stats: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """float64 sums [..., d/2, 3] over n_tok_total tokens -> stats [..., d/2, 4]."""
    *lead, F, _ = sums.shape
    H = 1
    for x in lead:
        H *= x
    if stats is None:
        stats = torch.empty((*lead, F, 4), dtype=torch.float32, device=sums.device)
    _check("tri_calibrate_finish", load().tri_calibrate_finish(
        _ptr(sums), H, int(n_tok_total), 2 * F, _ptr(stats), _stream(stream)))
    return stats


def calibrate_data_parallel(q_shard: torch.Tensor, group=None) -> torch.Tensor:
    """Calibration over the calibration tokens of all data-parallel ranks:
    each rank reduces its own shard q_shard [..., n_tok_rank, d] to float64
    sums, one all-reduce adds the sums and the token counts over the process
    group, and every rank forms the same statistics [..., d/2, 4]."""
    import torch.distributed as dist

    sums = tri_calibrate_sums(q_shard)
    n = torch.tensor([q_shard.shape[-2]], dtype=torch.float64, device=sums.device)
    both = torch.cat([sums.reshape(-1), n])
    dist.all_reduce(both, op=dist.ReduceOp.SUM, group=group)
    total = int(round(both[-1].item()))
    return tri_calibrate_finish(both[:-1].reshape(sums.shape).contiguous(), total)


def tri_score_workspace_bytes(n_seq, n_layers, n_kvheads, G, cap, head_dim=HEAD_DIM) -> int:
    return load().tri_score_workspace_bytes(n_seq, n_layers, n_kvheads, G, cap, head_dim)


def tri_score(cfg: TriConfig, k_post: torch.Tensor, n_seq: int, n_layers: int, n_kvheads: int,
              G: int, p_cur: torch.Tensor, stats: torch.Tensor, n_valid: Optional[torch.Tensor] = None,
              raw: Optional[torch.Tensor] = None, final: Optional[torch.Tensor] = None,
              ws: Optional[torch.Tensor] = None, stream=None):
    """k_post [U, cap, d] -> (raw [U, G, cap] or None, final [U, cap])."""
    U, cap, d = k_post.shape
    if final is None:
        final = torch.empty((U, cap), dtype=torch.float32, device=k_post.device)
    if ws is None:
        ws = workspace(tri_score_workspace_bytes(n_seq, n_layers, n_kvheads, G, cap, d), k_post.device)
    _check("tri_score", load().tri_score(
        ctypes.byref(cfg), _ptr(k_post), _dt(k_post), n_seq, n_layers, n_kvheads, G, cap,
        _ptr(n_valid), _ptr(p_cur), _ptr(stats), _ptr(raw), _ptr(final), _ptr(ws), ws.numel(),
        _stream(stream)))
    return raw, final


def tri_select_workspace_bytes(n_units: int, cap: int, B: int) -> int:
    return load().tri_select_workspace_bytes(n_units, cap, B)


def tri_select_topB(final: torch.Tensor, B: int, n_valid: Optional[torch.Tensor] = None,
                    kept: Optional[torch.Tensor] = None, n_kept: Optional[torch.Tensor] = None,
                    ws: Optional[torch.Tensor] = None, stream=None):
    """final [U, cap] float32 -> (kept [U, B] int32 ascending, -1 padded; n_kept [U])."""
    U, cap = final.shape
    dev = final.device
    if kept is None:
        kept = torch.empty((U, B), dtype=torch.int32, device=dev)
    if n_kept is None:
        n_kept = torch.empty((U,), dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(tri_select_workspace_bytes(U, cap, B), dev)
    _check("tri_select_topB", load().tri_select_topB(
        _ptr(final), U, cap, _ptr(n_valid), B, _ptr(kept), _ptr(n_kept), _ptr(ws), ws.numel(),
        _stream(stream)))
    return kept, n_kept


def tri_select_topB_static(final: torch.Tensor, B: int, n_valid: Optional[torch.Tensor] = None,
                           kept: Optional[torch.Tensor] = None,
                           n_kept: Optional[torch.Tensor] = None, stream=None):
    """tri_select_topB with the library's static device scratch instead of a
    workspace (for callers that cannot allocate device memory; see tri.h).
    Overlapping calls race on the shared scratch."""
    U, cap = final.shape
    dev = final.device
    if kept is None:
        kept = torch.empty((U, B), dtype=torch.int32, device=dev)
    if n_kept is None:
        n_kept = torch.empty((U,), dtype=torch.int32, device=dev)
    _check("tri_select_topB_static", load().tri_select_topB_static(
        _ptr(final), U, cap, _ptr(n_valid), B, _ptr(kept), _ptr(n_kept), _stream(stream)))
    return kept, n_kept


def tri_compact(k_src: torch.Tensor, v_src: Optional[torch.Tensor], pos_src: Optional[torch.Tensor],
                kept: torch.Tensor, n_kept: torch.Tensor, k_dst: torch.Tensor,
                v_dst: Optional[torch.Tensor] = None, pos_dst: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, stream=None):
    U, cap_src, d = k_src.shape
    B = kept.shape[1]
    cap_dst = k_dst.shape[1]
    if ws is None:
        ws = workspace(load().tri_compact_workspace_bytes(), k_src.device)
    _check("tri_compact", load().tri_compact(
        _ptr(k_src), _ptr(v_src), _ptr(pos_src), _dt(k_src), U, cap_src, d, _ptr(kept),
        _ptr(n_kept), B, _ptr(k_dst), _ptr(v_dst), _ptr(pos_dst), cap_dst, _ptr(ws), ws.numel(),
        _stream(stream)))


def tri_compact_inplace(k: torch.Tensor, v: Optional[torch.Tensor], pos: Optional[torch.Tensor],
                        kept: torch.Tensor, n_kept: torch.Tensor,
                        ws: Optional[torch.Tensor] = None, stream=None):
    """Move row kept[u][r] to row r of the same buffers (r < n_kept[u])."""
    U, cap, d = k.shape
    B = kept.shape[1]
    if ws is None:
        ws = workspace(load().tri_compact_workspace_bytes(), k.device)
    _check("tri_compact_inplace", load().tri_compact_inplace(
        _ptr(k), _ptr(v), _ptr(pos), _dt(k), U, cap, d, _ptr(kept), _ptr(n_kept), B, _ptr(ws),
        ws.numel(), _stream(stream)))


def tri_prune_workspace_bytes(n_seq, n_layers, n_kvheads, G, cap, B, head_dim=HEAD_DIM) -> int:
    return load().tri_prune_workspace_bytes(n_seq, n_layers, n_kvheads, G, cap, B, head_dim)


def tri_prune_path(n_seq, n_layers, n_kvheads, G, cap, B, dtype=torch.bfloat16,
                   path: int = PATH_AUTO, inplace: bool = False) -> int:
    """Kernel path tri_prune (or tri_prune_inplace) takes for these shapes
    (PATH_PIPE / COOP / FUSED / SPLIT; -1 if none)."""
    dt = TRI_BF16 if dtype == torch.bfloat16 else TRI_F32
    return int(load().tri_prune_path(n_seq, n_layers, n_kvheads, G, cap, B, dt, path,
                                     1 if inplace else 0))


def tri_prune(cfg: TriConfig, k_src: torch.Tensor, v_src: Optional[torch.Tensor],
              pos_src: Optional[torch.Tensor], n_seq: int, n_layers: int, n_kvheads: int, G: int,
              p_cur: torch.Tensor, stats: torch.Tensor, B: int, k_dst: torch.Tensor,
              v_dst: Optional[torch.Tensor], pos_dst: Optional[torch.Tensor],
              n_kept: torch.Tensor, n_valid: Optional[torch.Tensor] = None,
              kept: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None,
              final: Optional[torch.Tensor] = None):
    """One prune step: score, select the top-B, gather into the destination
    cache.  ``final`` (optional, [U, cap_src] float32) receives the final
    scores of the units that were pruned."""
    U, cap_src, d = k_src.shape
    cap_dst = k_dst.shape[1]
    if ws is None:
        ws = workspace(tri_prune_workspace_bytes(n_seq, n_layers, n_kvheads, G, cap_src, B, d),
                       k_src.device)
    _check("tri_prune", load().tri_prune(
        ctypes.byref(cfg), _ptr(k_src), _ptr(v_src), _ptr(pos_src), _dt(k_src), n_seq, n_layers,
        n_kvheads, G, cap_src, _ptr(n_valid), _ptr(p_cur), _ptr(stats), B, _ptr(k_dst), _ptr(v_dst),
        _ptr(pos_dst), cap_dst, _ptr(kept), _ptr(n_kept), _ptr(final), _ptr(ws), ws.numel(),
        _stream(stream)))


def tri_prune_inplace(cfg: TriConfig, k: torch.Tensor, v: Optional[torch.Tensor],
                      pos: Optional[torch.Tensor], n_seq: int, n_layers: int, n_kvheads: int,
                      G: int, p_cur: torch.Tensor, stats: torch.Tensor, B: int,
                      n_kept: torch.Tensor, n_valid: Optional[torch.Tensor] = None,
                      kept: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                      stream=None, final: Optional[torch.Tensor] = None):
    """One prune step that compacts the cache in place (kept rows move to the
    front of k, v and pos in temporal order)."""
    U, cap, d = k.shape
    if ws is None:
        ws = workspace(tri_prune_workspace_bytes(n_seq, n_layers, n_kvheads, G, cap, B, d),
                       k.device)
    _check("tri_prune_inplace", load().tri_prune_inplace(
        ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(pos), _dt(k), n_seq, n_layers, n_kvheads, G,
        cap, _ptr(n_valid), _ptr(p_cur), _ptr(stats), B, _ptr(kept), _ptr(n_kept), _ptr(final),
        _ptr(ws), ws.numel(), _stream(stream)))


def tri_logit_reconstruct(cfg: TriConfig, q_stats: torch.Tensor, k_stats: torch.Tensor, G: int,
                          deltas: torch.Tensor, stream=None) -> torch.Tensor:
    """Trig-series logit(Delta) from the centres: q_stats [Hq, 64, 4], k_stats
    [Hq/G, 64, 4], deltas int64 CUDA [n] -> [Hq, n] float32."""
    Hq = q_stats.shape[0]
    out = torch.empty((Hq, deltas.numel()), dtype=torch.float32, device=q_stats.device)
    _check("tri_logit_reconstruct", load().tri_logit_reconstruct(
        ctypes.byref(cfg), _ptr(q_stats), _ptr(k_stats), Hq, G, _ptr(deltas), deltas.numel(),
        _ptr(out), _stream(stream)))
    return out


def tri_logit_curve(q_post: torch.Tensor, k_post: torch.Tensor, G: int, deltas: torch.Tensor,
                    stream=None) -> torch.Tensor:
    """Mean post-RoPE logit at each distance: q [Hq, n, d], k [Hq/G, n, d],
    deltas int64 CUDA [m] -> [Hq, m] float32."""
    Hq, n, d = q_post.shape
    out = torch.empty((Hq, deltas.numel()), dtype=torch.float32, device=q_post.device)
    _check("tri_logit_curve", load().tri_logit_curve(
        _ptr(q_post), _ptr(k_post), _dt(q_post), Hq, G, n, d, _ptr(deltas), deltas.numel(),
        _ptr(out), _stream(stream)))
    return out


def tri_pearson(a: torch.Tensor, b: torch.Tensor, stream=None) -> torch.Tensor:
    """Row-wise Pearson correlation of two [rows, n] float32 CUDA tensors."""
    rows, n = a.shape
    out = torch.empty((rows,), dtype=torch.float32, device=a.device)
    _check("tri_pearson", load().tri_pearson(_ptr(a), _ptr(b), rows, n, _ptr(out),
                                             _stream(stream)))
    return out


def tri_decode_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         n_valid: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                         out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """Attention of one query token per head over each unit's first n_valid
    cache rows: q [U, G, d], k / v [U, cap, d] -> out [U, G, d] float32."""
    U, G, d = q.shape
    cap = k.shape[1]
    if out is None:
        out = torch.empty((U, G, d), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(load().tri_decode_workspace_bytes(U, G, cap), q.device)
    sc = (1.0 / d ** 0.5) if scale is None else float(scale)
    _check("tri_decode_attention", load().tri_decode_attention(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), U, G, cap, d, _ptr(n_valid), ctypes.c_float(sc),
        _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def tri_prune_paged_inplace(cfg: TriConfig, k_pool: torch.Tensor, v_pool: Optional[torch.Tensor],
                            pos: Optional[torch.Tensor], page_table: torch.Tensor, cap: int,
                            n_seq: int, n_layers: int, n_kvheads: int, G: int,
                            p_cur: torch.Tensor, stats: torch.Tensor, B: int,
                            n_kept: torch.Tensor, n_valid: Optional[torch.Tensor] = None,
                            kept: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                            stream=None, final: Optional[torch.Tensor] = None):
    """In-place prune of a paged cache: k_pool / v_pool [n_pages, page_rows, d],
    page_table int32 [U, pages_per_unit], pos [U, cap] (logical rows)."""
    n_pages, page_rows, d = k_pool.shape
    ppu = page_table.shape[1]
    if ws is None:
        ws = workspace(tri_prune_workspace_bytes(n_seq, n_layers, n_kvheads, G, cap, B, d),
                       k_pool.device)
    _check("tri_prune_paged_inplace", load().tri_prune_paged_inplace(
        ctypes.byref(cfg), _ptr(k_pool), _ptr(v_pool), _ptr(pos), _dt(k_pool), n_seq, n_layers,
        n_kvheads, G, cap, _ptr(n_valid), _ptr(p_cur), _ptr(stats), B, _ptr(page_table),
        page_rows, ppu, n_pages, _ptr(kept), _ptr(n_kept), _ptr(final), _ptr(ws), ws.numel(),
        _stream(stream)))


def tri_append(k_cache, v_cache, pos_cache, n_seq: int, n_valid: torch.Tensor,
               k_new, v_new, pos_new, p_cur: Optional[torch.Tensor] = None,
               ws: Optional[torch.Tensor] = None, stream=None):
    U, cap, d = k_cache.shape
    n_new = k_new.shape[1]
    if ws is None:
        ws = workspace(256, k_cache.device)
    _check("tri_append", load().tri_append(
        _ptr(k_cache), _ptr(v_cache), _ptr(pos_cache), _dt(k_cache), n_seq, U, cap, d,
        _ptr(n_valid), _ptr(p_cur), _ptr(k_new), _ptr(v_new), _ptr(pos_new), n_new, _ptr(ws),
        ws.numel(), _stream(stream)))


def tri_set_timing_events(events: Optional[Sequence["torch.cuda.Event"]]):
    """Record events[i] on the call's stream after the i-th kernel each
    following tri_* call launches (None stops).  Keeps the handles alive."""
    global _timing_keep
    if not events:
        _timing_keep = None
        _check("tri_set_timing_events", load().tri_set_timing_events(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _timing_keep = (arr, list(events))
    _check("tri_set_timing_events", load().tri_set_timing_events(arr, len(events)))


def tri_set_phase_trace(buf: Optional[torch.Tensor]):
    """Per-unit phase timestamps of the fused kernel into buf (int64 CUDA
    tensor of at least 8 * units entries), or None to stop."""
    if buf is None:
        _check("tri_set_phase_trace", load().tri_set_phase_trace(None, 0))
    else:
        _check("tri_set_phase_trace", load().tri_set_phase_trace(_ptr(buf), buf.numel() * buf.element_size()))


def tri_last_launch_count() -> int:
    return int(load().tri_last_launch_count())


_timing_keep = None


def tri_check_device_error(ws: torch.Tensor, stream=None) -> int:
    """Synchronise and return the device flag bits of the last call on ws (0 = none)."""
    flags = ctypes.c_uint32(0)
    code = load().tri_check_device_error(_ptr(ws), _stream(stream), ctypes.byref(flags))
    if code not in (0, 5):
        raise TriError("tri_check_device_error", code)
    return int(flags.value)
