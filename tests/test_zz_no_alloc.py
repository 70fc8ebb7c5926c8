"""The allocation-free forward entry point (ar_attn_fwd_noalloc).

Some callers cannot allocate device memory while they run (a CUDA-graph
capture that must not allocate, a host application that owns the allocator).
For them the library offers a forward pass whose scratch is a fixed array
built into the library.  These tests call it through the C ABI and check it
against the regular forward (ar_attn_fwd) with the same tolerances as the
other parity tests, on two calls in a row (the second reuses the array the
first one left behind).  This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from sliding_window_attention_rmsnorm_b200 import attn, build, synth

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2, LSE_ABS = 2e-2, 5e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    attn.lib()


def close(a, b, tol_abs):
    a, b = a.float().cpu().numpy().astype(np.float64), b.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(a).all()
    assert np.abs(a - b).max() <= tol_abs
    nb = np.linalg.norm(b)
    if nb > 0 and tol_abs == MAX_ABS:
        assert np.linalg.norm(a - b) / nb <= REL_L2


@pytest.mark.parametrize("B,T,H,window", [(2, 300, 3, 100), (8, 2048, 4, 1024)])
def test_noalloc_matches_regular_forward_twice(B, T, H, window):
    x = synth.layer_inputs(21, T, B, T, H, 128)
    q, k, v = (x[r].cuda() for r in ("q", "k", "v"))
    o_ref, lse_ref = attn.fwd(q, k, v, window)
    # a different problem first, so the shared scratch holds stale data
    y = synth.layer_inputs(22, 0, 1, 640, 2, 128)
    attn.fwd_noalloc(y["q"].cuda(), y["k"].cuda(), y["v"].cuda(), 64)
    for _ in range(2):
        o, lse = attn.fwd_noalloc(q, k, v, window)
        attn.sync_status()
        close(o, o_ref, MAX_ABS)
        close(lse, lse_ref, LSE_ABS)


def test_noalloc_rejects_problems_beyond_its_scratch():
    L = attn.lib()
    vp = ctypes.c_void_p
    # 9 * 1 * 2^17 key rows > 2^20: rejected before any pointer is touched
    B, T, H = 9, 1 << 17, 1
    p = vp(1 << 20)
    st = L.ar_attn_fwd_noalloc(p, p, p, p, p, B, T, H, 128, -1, ctypes.c_float(1e-6), ctypes.c_float(0.088), None)
    assert st == -10 and "scratch" in attn.strerror(st)
