"""C-ABI checks that need no GPU: the library loads, exports every declared
symbol, and its host-side logic (argument validation, window rule, pair
count, workspace sizes) behaves as the header states.

Validation tests always include at least one invalid argument that the
library checks before touching the device, so no kernel is ever launched on
the placeholder pointers used here.
"""
import ctypes
import os
import re

import pytest

from oracle import oracle as orc
from oracle.stack import layer_windows as oracle_windows
from sliding_window_attention_rmsnorm_b200 import attn, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return attn.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ar_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ar_attn_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("ar_attn_fwd", "ar_attn_bwd", "ar_attn_bwd_workspace_bytes", "ar_attn_sync_status",
              "ar_attn_strerror"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), n


def test_strerror(L):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -9, 12345):
        assert attn.strerror(code)
    assert attn.strerror(0) == "ok"


def test_layer_window_matches_oracle_rule(L):
    for n_layer in (1, 2, 4, 8, 12, 13):
        for T in (256, 2048, 8192):
            for pat in ("SSSL", "L", "SL", "SLLL", "SSSS", "sssl"):
                mine = [L.ar_attn_layer_window(l, n_layer, T, pat.encode()) for l in range(n_layer)]
                assert mine == oracle_windows(n_layer, T, pat), (n_layer, T, pat)
    assert L.ar_attn_layer_window(0, 8, 2048, b"SXSL") == 1024
    assert L.ar_attn_layer_window(1, 8, 2048, b"SXSL") == -5
    assert L.ar_attn_layer_window(8, 8, 2048, b"SSSL") == -5
    assert L.ar_attn_layer_window(0, 8, 2048, None) == -1


def test_unmasked_pairs_matches_oracle(L):
    for T in (1, 2, 7, 128, 129, 200, 256, 2048):
        for w in (-1, 0, 1, 5, 127, 128, 1024, T - 2, T - 1, T, 5 * T):
            assert L.ar_attn_unmasked_pairs(T, w) == orc.unmasked_pairs(T, w if w < T - 1 else -1), (T, w)


def test_workspace_sizes(L):
    B, T, H, D = 8, 2048, 4, 128
    # the forward needs no scratch: it has no workspace argument at all
    assert not hasattr(L, "ar_attn_fwd_workspace_bytes")
    # three per-token fp32 vectors + one 32 KB G tile per (query tile, key tile)
    # pair of the full causal band, nq (nq + 1) / 2 per head (nq = 16 here)
    assert attn.bwd_workspace_bytes(B, T, H, D) == 3 * B * H * T * 4 + B * H * 136 * 32768
    # ragged T rounds the per-token vectors up to whole 128-token tiles (nq = 2: 3 tiles)
    assert attn.bwd_workspace_bytes(1, 200, 1, 128) == 3 * 256 * 4 + 3 * 32768
    # heads are grouped so that the G tiles fit in 1 GiB: T = 8192 gives 2080 tiles per
    # head (68 MB), 15 heads per group
    assert attn.bwd_workspace_bytes(4, 8192, 8, 128) == 3 * 32 * 8192 * 4 + 15 * 2080 * 32768
    assert attn.bwd_workspace_bytes(0, 200, 1, 128) == 0
    # head dimension 64: the same per-token vectors and G tiles (queries x keys)
    assert attn.bwd_workspace_bytes(1, 200, 1, 64) == attn.bwd_workspace_bytes(1, 200, 1, 128)
    assert attn.bwd_workspace_bytes(1, 200, 1, 96) == 0
    # the RoPE paths take head dimension 128 only
    assert attn.bwd_rope_workspace_bytes(1, 200, 1, 64) == 0 and attn.fwd_rope_workspace_bytes(1, 200, 1, 64) == 0


P16 = 1 << 20  # a 16-byte aligned placeholder address; never dereferenced


def fwd_call(L, q=P16, k=P16, v=P16, o=P16, lse=P16, B=1, T=128, H=1, D=128, window=-1, eps=1e-6,
             scale=0.088):
    vp = ctypes.c_void_p
    return L.ar_attn_fwd(vp(q), vp(k), vp(v), vp(o), vp(lse), B, T, H, D, window, eps, scale, None)


def bwd_call(L, ptr=P16, dq=P16, B=1, T=128, H=1, D=128, eps=1e-6, scale=0.088, ws=None, ws_bytes=0):
    vp = ctypes.c_void_p
    return L.ar_attn_bwd(vp(ptr), vp(ptr), vp(ptr), vp(ptr), vp(ptr), vp(ptr), vp(dq), vp(ptr), vp(ptr),
                         B, T, H, D, -1, eps, scale, vp(ws), ws_bytes, None)


def test_fwd_argument_errors(L):
    assert fwd_call(L, q=0) == -1
    assert fwd_call(L, o=0) == -1
    # lse may be NULL (the forward-only use): validation goes on to the next check
    assert fwd_call(L, lse=0, B=0) == -2
    assert fwd_call(L, lse=0, k=P16 + 8) == -4
    assert fwd_call(L, lse=P16 + 2) == -4
    assert fwd_call(L, B=0) == -2
    assert fwd_call(L, T=-3) == -2
    assert fwd_call(L, H=0) == -2
    assert fwd_call(L, D=96) == -3
    assert fwd_call(L, D=256) == -3
    assert fwd_call(L, D=64, B=0) == -2  # 64 is a supported head dimension: validation goes on
    assert fwd_call(L, k=P16 + 8) == -4
    assert fwd_call(L, eps=-1.0) == -5
    assert fwd_call(L, eps=float("nan")) == -5
    assert fwd_call(L, scale=0.0) == -5
    assert fwd_call(L, scale=float("inf")) == -5


def test_bwd_argument_errors(L):
    assert bwd_call(L, dq=0) == -1
    assert bwd_call(L, B=-1) == -2
    assert bwd_call(L, D=256) == -3
    assert bwd_call(L, dq=P16 + 4) == -4
    assert bwd_call(L, scale=-0.5) == -5
    assert bwd_call(L, ws=P16, ws_bytes=100) == -9


def test_grouped_kv_head_arguments(L):
    vp = ctypes.c_void_p

    def fwd_gqa(H, Hkv, k=P16):
        return L.ar_attn_fwd_gqa(vp(P16), vp(k), vp(P16), vp(P16), vp(P16), 1, 128, H, Hkv, 128, -1, 1e-6, 0.088,
                                 None)

    def bwd_gqa(H, Hkv, ws=None, ws_bytes=0):
        p = vp(P16)
        return L.ar_attn_bwd_gqa(p, p, p, p, p, p, p, p, p, 1, 128, H, Hkv, 128, -1, 1e-6, 0.088, vp(ws),
                                 ws_bytes, None)

    # Hkv must divide H and lie in 1..H; checked before anything touches a device
    for H, Hkv in ((4, 3), (4, 0), (4, 5), (6, -2)):
        assert fwd_gqa(H, Hkv) == -2 and bwd_gqa(H, Hkv) == -2
        assert attn.bwd_workspace_bytes(1, 128, H, 128, Hkv) == 0
    assert fwd_gqa(4, 2, k=P16 + 8) == -4
    assert bwd_gqa(4, 2, ws=P16, ws_bytes=100) == -9
    # per query head as for multi-head attention: G tiles of whole groups, here all 4 query heads
    assert attn.bwd_workspace_bytes(1, 200, 4, 128, 2) == 3 * 4 * 256 * 4 + 4 * 3 * 32768
    assert attn.bwd_workspace_bytes(1, 200, 4, 128, 2) == attn.bwd_workspace_bytes(1, 200, 4, 128)
    # T = 8192: 15 query heads fit in 1 GiB of G tiles; groups of 4 round that down to 12
    assert attn.bwd_workspace_bytes(4, 8192, 8, 128, 2) == 3 * 32 * 8192 * 4 + 12 * 2080 * 32768
    assert attn.bwd_workspace_bytes(4, 8192, 8, 128, 8) == 3 * 32 * 8192 * 4 + 15 * 2080 * 32768


def test_stack_buffers_follow_kv_heads(L):
    """The stack driver sizes dk, dv like k, v and its backward scratch for the
    K/V head count (built on CPU tensors: nothing is launched here)."""
    import torch
    from sliding_window_attention_rmsnorm_b200 import stack
    B, T, H, D = 1, 200, 4, 128
    for Hkv in (4, 2, 1):
        layer = dict(q=torch.zeros(B, T, H, D, dtype=torch.bfloat16), dO=torch.zeros(B, T, H, D, dtype=torch.bfloat16),
                     k=torch.zeros(B, T, Hkv, D, dtype=torch.bfloat16), v=torch.zeros(B, T, Hkv, D, dtype=torch.bfloat16))
        st = stack.Stack([layer, layer], windows=[100, 200])
        assert st.out[0]["dk"].shape == (B, T, Hkv, D) and st.out[1]["dv"].shape == (B, T, Hkv, D)
        assert st.out[0]["dq"].shape == (B, T, H, D) and st.out[0]["lse"].shape == (B, H, T)
        assert st.ws_bwd.numel() == attn.bwd_workspace_bytes(B, T, H, D, Hkv) > 0


def test_stack_keeps_rope_forward_workspaces(L):
    """With RoPE each layer keeps its own forward workspace (its rotated k and
    mixed v) for its backward, sized by whether the layer has a value embedding."""
    import torch
    from sliding_window_attention_rmsnorm_b200 import stack
    B, T, H, Hkv, D = 1, 200, 4, 2, 128
    z = lambda h: torch.zeros(B, T, h, D, dtype=torch.bfloat16)  # noqa: E731
    plain = dict(q=z(H), dO=z(H), k=z(Hkv), v=z(Hkv))
    with_ve = dict(plain, ve=z(Hkv), g=torch.zeros(B, T, Hkv, dtype=torch.bfloat16))
    cos = torch.zeros(T, 64, dtype=torch.bfloat16)
    st = stack.Stack([plain, with_ve], windows=[100, 200], rope=(cos, cos))
    assert [w.numel() for w in st.ws_fwd] == [attn.fwd_rope_workspace_bytes(B, T, Hkv, D, False),
                                              attn.fwd_rope_workspace_bytes(B, T, Hkv, D, True)]
    assert st.ws_fwd[0].data_ptr() != st.ws_fwd[1].data_ptr()


def test_bwd_rope_saved_argument_errors(L):
    """ar_attn_bwd_rope_saved validates like ar_attn_bwd_rope, and `saved` must
    be 256-byte aligned; every call here fails before touching the device."""
    vp, P = ctypes.c_void_p, lambda a: ctypes.c_void_p(a)  # noqa: E731
    B, T, H, Hkv, D = 1, 256, 4, 2, 128
    args = dict(q=P(0x100000), k=P(0x200000), v=P(0x300000), o=P(0x400000), dO=P(0x500000), lse=P(0x600000),
                cos=P(0x700000), sin=P(0x800000), dq=P(0x900000), dk=P(0xa00000), dv=P(0xb00000))

    def call(saved, **over):
        a = dict(args, **over)
        return L.ar_attn_bwd_rope_saved(a["q"], a["k"], a["v"], a["o"], a["dO"], a["lse"], a["cos"], a["sin"], T,
                                        None, None, a["dq"], a["dk"], a["dv"], None, None, B, T, H, Hkv, D, 128,
                                        ctypes.c_float(1e-6), ctypes.c_float(0.088), saved, P(0xc00000),
                                        ctypes.c_size_t(1 << 40), None)
    assert call(P(0xd00010)) == -4                    # saved not 256-byte aligned
    assert call(P(0xd00000), q=None) == -1            # a required pointer missing
    assert call(P(0xd00000), dq=P(0x900008)) == -4    # an output not 16-byte aligned
    assert call(None, q=None) == -1                   # saved = NULL: ar_attn_bwd_rope's checks


def test_wait_limit_setter(L):
    """Host-side only: the setter accepts any limit and 0 restores the default."""
    assert L.ar_attn_set_wait_limit_ns(ctypes.c_ulonglong(1)) == 0
    assert L.ar_attn_set_wait_limit_ns(ctypes.c_ulonglong(0)) == 0
    attn.set_wait_limit_ns(0)


def test_binding_rejects_mismatched_outputs():
    """Caller-supplied outputs are checked against the tensors they are shaped
    after before anything reaches the library (CPU tensors: rejected as not on
    a CUDA device, whatever else is wrong)."""
    import torch
    q = torch.zeros(1, 4, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn._check_out(torch.zeros(1, 4, 1, 128, dtype=torch.bfloat16), q, "dq")
    with pytest.raises(ValueError):
        attn._check_out(q.float(), q, "out")
    with pytest.raises(ValueError):
        attn._check_lse(torch.zeros(1, 2, 4), 1, 2, 4, q.device)
