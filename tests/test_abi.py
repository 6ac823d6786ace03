"""The C-ABI library builds, loads and exports every symbol include/tri.h
declares; host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

import rope_aware_kv_b200 as tri
from rope_aware_kv_b200 import build as tri_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tri.h")
GOLDEN = os.path.join(ROOT, "tests", "golden", "page_constants.txt")


@pytest.fixture(scope="module")
def lib():
    tri_build.build()
    return tri.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tri_[a-zA-Z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("tri_calibrate", "tri_score", "tri_select_topB", "tri_compact", "tri_prune"):
        assert n in names
    assert set(names) == set(tri.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_library_is_sm100a_only(lib):
    assert b"sm_100a" in lib.tri_version()


def test_default_config_matches_the_pages(lib):
    vals = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    cfg = tri.config()
    assert cfg.theta == float(vals["theta"])
    assert [cfg.offsets[i] for i in range(cfg.n_offsets)] == [int(x) for x in vals["offsets"].split()]
    assert cfg.head_dim == 128 and cfg.path == tri.PATH_AUTO


def test_status_strings(lib):
    for code in range(6):
        assert lib.tri_status_str(code).decode() == tri.STATUS[code]


def test_workspace_queries(lib):
    small = lib.tri_prune_workspace_bytes(1, 1, 4, 7, 4096, 512, 128)
    big = lib.tri_prune_workspace_bytes(1, 1, 4, 7, 32768, 2048, 128)
    assert 256 < small < big
    assert lib.tri_score_workspace_bytes(1, 1, 4, 7, 32768, 128) >= 4 * 7 * 32768 * 4
    assert lib.tri_select_workspace_bytes(4, 32768, 2048) >= 3 * 4 * 2048 * 4
    assert lib.tri_compact_workspace_bytes() == 256
    assert lib.tri_calibrate_workspace_bytes(28, 10240, 128) > 256


def _prune_status(lib, cfg, **over):
    args = dict(k_src=1 << 36, v_src=1 << 37, pos_src=1 << 38, dt=tri.TRI_BF16, n_seq=1,
                n_layers=1, n_kvheads=4, G=7, cap=4096, n_valid=None, p_cur=16, stats=16, B=512,
                k_dst=1 << 40, v_dst=1 << 41, pos_dst=1 << 42, cap_dst=512, kept=None, n_kept=16,
                final=None, ws=None, ws_bytes=0)
    args.update(over)
    P = lambda v: None if v is None else ctypes.c_void_p(v)
    return lib.tri_prune(ctypes.byref(cfg) if cfg is not None else None, P(args["k_src"]),
                         P(args["v_src"]), P(args["pos_src"]), args["dt"], args["n_seq"],
                         args["n_layers"], args["n_kvheads"], args["G"], args["cap"],
                         P(args["n_valid"]), P(args["p_cur"]), P(args["stats"]), args["B"],
                         P(args["k_dst"]), P(args["v_dst"]), P(args["pos_dst"]), args["cap_dst"],
                         P(args["kept"]), P(args["n_kept"]), P(args["final"]), P(args["ws"]),
                         args["ws_bytes"], None)


def test_host_validation_without_gpu(lib):
    """Bad arguments are refused on the host before anything is launched."""
    cfg = tri.config()
    assert _prune_status(lib, None) == 1                      # no config
    assert _prune_status(lib, cfg, G=9) == 2                  # group too large
    assert _prune_status(lib, cfg, G=0) == 2
    assert _prune_status(lib, cfg, dt=7) == 2                 # unknown dtype
    assert _prune_status(lib, cfg, B=0) == 1                  # empty budget
    assert _prune_status(lib, cfg, k_src=(1 << 36) + 2) == 1  # misaligned keys
    assert _prune_status(lib, cfg, v_dst=None) == 1           # v_src without v_dst
    assert _prune_status(lib, cfg, cap_dst=100) == 1          # destination too small
    assert _prune_status(lib, cfg) == 3                       # well formed: no workspace
    assert _prune_status(lib, cfg, k_dst=(1 << 36) + 4096) == 1  # K destination overlaps K
    assert _prune_status(lib, cfg, v_dst=(1 << 37) + 256) == 1   # V destination overlaps V
    assert _prune_status(lib, cfg, k_dst=(1 << 37) + 512) == 1   # K destination overlaps V
    assert _prune_status(lib, cfg, pos_dst=(1 << 38) + 64) == 1  # positions overlap
    assert _prune_status(lib, cfg, final=(1 << 43) + 2) == 1     # misaligned final scores
    assert _prune_status(lib, cfg, final=1 << 43) == 3           # well formed: no workspace
    bad = tri.config(head_dim=64)
    assert _prune_status(lib, bad) == 2
    cfg2 = tri.config()
    cfg2.n_offsets = 0
    assert _prune_status(lib, cfg2) == 1
    cfg3 = tri.config(path=7)
    assert _prune_status(lib, cfg3) == 1
    assert _prune_status(lib, tri.config(path=tri.PATH_PIPE)) in (2, 3)  # no device here: 2


def test_calibration_split_validation_without_gpu(lib):
    """The data-parallel calibration entry points refuse bad arguments on
    the host (fake, never dereferenced addresses)."""
    q, sums, stats, ws = 4096, 8192, 12288, 16384
    wsb = tri.tri_calibrate_workspace_bytes(2, 100)
    assert lib.tri_calibrate_sums(None, 0, 2, 100, 128, sums, ws, wsb, None) == 1
    assert lib.tri_calibrate_sums(q, 0, 2, 100, 128, None, ws, wsb, None) == 1
    assert lib.tri_calibrate_sums(q, 0, 0, 100, 128, sums, ws, wsb, None) == 1
    assert lib.tri_calibrate_sums(q, 0, 2, 100, 64, sums, ws, wsb, None) == 2
    assert lib.tri_calibrate_sums(q, 7, 2, 100, 128, sums, ws, wsb, None) == 2
    assert lib.tri_calibrate_sums(q + 4, 0, 2, 100, 128, sums, ws, wsb, None) == 1
    assert lib.tri_calibrate_sums(q, 0, 2, 100, 128, sums + 4, ws, wsb, None) == 1
    assert lib.tri_calibrate_sums(q, 0, 2, 100, 128, sums, ws, 16, None) == 3
    assert lib.tri_calibrate_finish(None, 2, 100, 128, stats, None) == 1
    assert lib.tri_calibrate_finish(sums, 2, 0, 128, stats, None) == 1
    assert lib.tri_calibrate_finish(sums, 2, 100, 64, stats, None) == 2
    assert lib.tri_calibrate_finish(sums + 4, 2, 100, 128, stats, None) == 1


def test_new_entry_points_validate_on_the_host(lib):
    """In-place / paged prune, decode attention, the logit(Delta) calls and
    the config's variant fields refuse bad arguments before any launch
    (fake, never dereferenced addresses)."""
    P = ctypes.c_void_p
    k, v, pos = P(1 << 36), P(1 << 37), P(1 << 38)
    cfg = tri.config()

    def inplace(c, **o):
        a = dict(k=k, v=v, pos=pos, n_valid=P(1 << 39), n_kept=P(1 << 40))
        a.update(o)
        return lib.tri_prune_inplace(ctypes.byref(c), a["k"], a["v"], a["pos"], tri.TRI_BF16, 1,
                                     1, 4, 7, 4096, a["n_valid"], P(16), P(16), 512, None,
                                     a["n_kept"], None, None, 0, None)
    assert inplace(cfg, n_kept=P(1 << 39)) == 1            # n_kept is n_valid
    assert inplace(cfg, v=P((1 << 36) + 4096)) == 1         # K and V overlap
    assert inplace(tri.config(path=tri.PATH_FUSED)) in (2, 1)
    assert inplace(tri.config(path=tri.PATH_COOP)) in (2, 1)
    assert inplace(tri.config(variant=0x10)) == 1           # unknown variant bit
    assert inplace(tri.config(n_sink=-1)) == 1
    assert inplace(tri.config(barrier_wait_ns=-5)) == 1

    def paged(rows, ppu=40, n_pages=200, table=P(1 << 41)):
        return lib.tri_prune_paged_inplace(ctypes.byref(cfg), k, v, pos, tri.TRI_BF16, 1, 1, 4,
                                           7, 4096, None, P(16), P(16), 512, table, rows, ppu,
                                           n_pages, None, P(1 << 40), None, None, 0, None)
    assert paged(100) == 1                                   # not whole score tiles
    assert paged(128, ppu=8) == 1                            # pages do not cover cap
    assert paged(128, table=None) == 1
    assert paged(128, n_pages=0) == 1

    q, out, ws = P(1 << 36), P(1 << 42), P(1 << 43)
    assert lib.tri_decode_attention(q, k, v, tri.TRI_BF16, 4, 7, 2048, 128, None,
                                    ctypes.c_float(0.0), out, ws, 1 << 20, None) == 1
    assert lib.tri_decode_attention(q, k, v, tri.TRI_BF16, 4, 9, 2048, 128, None,
                                    ctypes.c_float(0.1), out, ws, 1 << 20, None) == 2
    assert lib.tri_decode_attention(q, k, v, tri.TRI_BF16, 4, 7, 2048, 64, None,
                                    ctypes.c_float(0.1), out, ws, 1 << 20, None) == 2
    assert lib.tri_decode_attention(P((1 << 36) + 4), k, v, tri.TRI_BF16, 4, 7, 2048, 128, None,
                                    ctypes.c_float(0.1), out, ws, 1 << 20, None) == 1
    assert lib.tri_decode_workspace_bytes(4, 7, 2048) >= 256

    d = P(1 << 44)
    assert lib.tri_logit_curve(q, k, tri.TRI_BF16, 8, 3, 100, 128, d, 10, out, None) == 1  # 8 % 3
    assert lib.tri_logit_curve(q, k, tri.TRI_BF16, 8, 2, 100, 64, d, 10, out, None) == 2
    assert lib.tri_logit_curve(q, k, tri.TRI_BF16, 8, 2, 100, 128, P((1 << 44) + 4), 10, out,
                               None) == 1                    # deltas not 8-byte aligned
    assert lib.tri_logit_reconstruct(ctypes.byref(cfg), P(16), P(16), 8, 3, d, 10, out, None) == 1
    assert lib.tri_pearson(P(16), P(16), 0, 10, out, None) == 1
    assert lib.tri_calibrate_ex(ctypes.byref(tri.config(variant=0x40)), q, tri.TRI_BF16, 2, 100,
                                128, None, P(16), ws, 1 << 20, None) == 1
