"""tri_select_topB_static: the selection without a caller workspace.

Callers that cannot allocate device memory (a serving engine that owns all
device memory and gives a plugin only its inputs and outputs, or a path that
must never call cudaMalloc) use this entry point; its scratch is a static
device array inside the library.  These tests call it through the C ABI and
check that it returns exactly what tri_select_topB returns, on two calls in a
row (the second call must not see the first call's leftovers).  The file is
named so that pytest collects it last; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import rope_aware_kv_b200 as tri
from rope_aware_kv_b200 import build as tri_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    tri_build.build()
    tri.load()


def _inputs(U, cap, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn((U, cap), generator=g, device="cuda")
    x[0] = torch.round(x[0] * 4) / 4          # many ties
    x[1, ::5] = float("nan")                  # NaN ranks last
    x[1, 1::5] = -0.0
    nv = torch.full((U,), cap, dtype=torch.int32, device="cuda")
    nv[2] = cap // 3
    return x, nv


@pytest.mark.parametrize("U,cap,B", [(4, 32768, 2048), (6, 5000, 777)])
def test_static_select_matches_workspace_select_twice(U, cap, B):
    assert tri.load().tri_select_static_scratch_bytes() == 1 << 20
    for seed in (1, 2):  # two calls in a row on different inputs
        x, nv = _inputs(U, cap, seed)
        ref_kept, ref_n = tri.tri_select_topB(x, B, n_valid=nv)
        kept, n = tri.tri_select_topB_static(x, B, n_valid=nv)
        torch.cuda.synchronize()
        assert torch.equal(kept, ref_kept)
        assert torch.equal(n, ref_n)


def test_static_select_rejects_requests_beyond_the_scratch():
    U, cap, B = 64, 32768, 100   # 64 units need 1.5 MiB of histograms
    x = torch.zeros((U, cap), device="cuda")
    kept = torch.empty((U, B), dtype=torch.int32, device="cuda")
    n = torch.empty((U,), dtype=torch.int32, device="cuda")
    code = tri.load().tri_select_topB_static(ctypes.c_void_p(x.data_ptr()), U, cap, None, B,
                                             ctypes.c_void_p(kept.data_ptr()),
                                             ctypes.c_void_p(n.data_ptr()), None)
    assert code == 6
    assert tri.load().tri_status_str(6).decode() == "request exceeds the static scratch"
