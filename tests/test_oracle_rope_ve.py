"""Pins of the RoPE and value-embedding oracle (oracle/rope_ve.py), CPU only.

Each test ties it to something other than itself:
* the rotation's sign convention to a closed form (a quarter turn maps the
  halves (a, b) to (b, -a), as the printed formula y1 = x1 cos + x2 sin,
  y2 = -x1 sin + x2 cos gives), position 0 to the identity;
* with exact cos/sin, the invariants of a rotation: row lengths kept, logits
  that depend only on the distance between positions, and the transpose as
  the inverse; with any table, the transpose as the adjoint;
* the tables to the angle definition within bf16 rounding;
* the whole composite (rotation, norm, windowed attention, gate) and all its
  gradients to torch fp64 autograd, and to central differences.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import rope_ve


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_quarter_turn_and_position_zero():
    x = rand((1, 3, 2, 8), 1)
    cos = np.zeros((3, 4))
    sin = np.ones((3, 4))
    y = rope_ve.rope(x, cos, sin)
    np.testing.assert_array_equal(y[..., :4], x[..., 4:])
    np.testing.assert_array_equal(y[..., 4:], -x[..., :4])
    c, s = rope_ve.rope_tables(16, 8)
    assert np.all(c[0] == 1.0) and np.all(s[0] == 0.0)
    y = rope_ve.rope(x, c, s)
    np.testing.assert_array_equal(y[:, 0], x[:, 0])
    assert not np.allclose(y[:, 1:], x[:, 1:])


def test_tables_follow_the_angle_definition():
    T, D = 2048, 128
    c, s = rope_ve.rope_tables(T, D)
    ce, se = rope_ve.rope_tables(T, D, rounding="none")
    # bf16 rounding (half an ulp, 2^-9 relative, at most 2^-9 absolute) plus the
    # fp32 angle t * inv_freq (relative error ~2^-24, t < 2048)
    tol = 2.0 ** -9 + 2.0 ** -24 * T * 2
    assert np.abs(c - ce).max() <= tol and np.abs(s - se).max() <= tol
    assert np.abs(c - ce).max() > 0  # really rounded


def test_rotation_invariants_with_exact_tables():
    T, D = 40, 16
    c, s = rope_ve.rope_tables(T, D, rounding="none")
    x = rand((2, T, 3, D), 2)
    y = rope_ve.rope(x, c, s)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(rope_ve.rope_transposed(y, c, s), x, atol=1e-13)
    # the same q and k at every position: the logits depend only on t - s
    qv, kv = rand((D,), 3), rand((D,), 4)
    qr = rope_ve.rope(np.broadcast_to(qv, (1, T, 1, D)), c, s)[0, :, 0]
    kr = rope_ve.rope(np.broadcast_to(kv, (1, T, 1, D)), c, s)[0, :, 0]
    L = qr @ kr.T
    for dlt in range(-5, 6):
        diag = np.diagonal(L, offset=dlt)
        np.testing.assert_allclose(diag, diag[0], atol=1e-12)
    assert abs(L[10, 10] - L[10, 3]) > 1e-3  # and it does depend on the distance


def test_transpose_is_the_adjoint_for_any_table():
    T, D = 30, 16
    c, s = rope_ve.rope_tables(T, D)
    x, y = rand((1, T, 2, D), 5), rand((1, T, 2, D), 6)
    lhs = np.sum(rope_ve.rope(x, c, s) * y)
    rhs = np.sum(x * rope_ve.rope_transposed(y, c, s))
    assert abs(lhs - rhs) <= 1e-12 * (abs(lhs) + 1)


def torch_composite(q, k, v, dO, ve, g, cos, sin, window, eps, scale):
    """fp64 torch: rotation, F.rms_norm, SDPA with the band mask, the gate;
    gradients by autograd."""
    t = {n: torch.tensor(a, dtype=torch.float64, requires_grad=True) for n, a in
         dict(q=q, k=k, v=v, ve=ve, g=g).items()}
    B, T, H, D = q.shape
    d = D // 2
    c = torch.tensor(cos[:T], dtype=torch.float64)[None, :, None, :]
    s = torch.tensor(sin[:T], dtype=torch.float64)[None, :, None, :]

    def rot(x):
        return torch.cat([x[..., :d] * c + x[..., d:] * s, -x[..., :d] * s + x[..., d:] * c], dim=-1)

    vm = t["v"] + 2 * torch.sigmoid(t["g"])[..., None] * t["ve"]
    Hkv = k.shape[2]
    kr, vr = rot(t["k"]), vm
    if Hkv != H:
        kr, vr = kr.repeat_interleave(H // Hkv, dim=2), vr.repeat_interleave(H // Hkv, dim=2)
    qh = F.rms_norm(rot(t["q"]), (D,), eps=eps).transpose(1, 2)
    kh = F.rms_norm(kr, (D,), eps=eps).transpose(1, 2)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = (j <= i) & ((i - j <= window) if window >= 0 else torch.ones_like(j <= i))
    o = F.scaled_dot_product_attention(qh, kh, vr.transpose(1, 2), attn_mask=mask, scale=scale).transpose(1, 2)
    (o * torch.tensor(dO)).sum().backward()
    return o.detach().numpy(), {n: x.grad.numpy() for n, x in t.items()}


@pytest.mark.parametrize("B,T,H,Hkv,D,window", [(1, 20, 2, 2, 16, 5), (2, 33, 4, 2, 32, -1), (1, 40, 2, 1, 128, 7)])
def test_composite_matches_torch_autograd(B, T, H, Hkv, D, window):
    eps, scale = 1e-6, 1.0 / math.sqrt(D)
    q, dO = rand((B, T, H, D), 10), rand((B, T, H, D), 11)
    k, v, ve = rand((B, T, Hkv, D), 12), rand((B, T, Hkv, D), 13), rand((B, T, Hkv, D), 14)
    g = rand((B, T, Hkv), 15)
    cos, sin = rope_ve.rope_tables(T + 7, D)  # a longer table, as the pages precompute
    ro, rg = torch_composite(q, k, v, dO, ve, g, cos, sin, window, eps, scale)
    o, _ = rope_ve.attn_fwd(q, k, v, cos, sin, window, eps, scale, ve=ve, g=g)
    gr = rope_ve.attn_bwd(q, k, v, dO, cos, sin, window, eps, scale, ve=ve, g=g)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-10)
    for mine, ref in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dve", "ve"), ("dg", "g")):
        np.testing.assert_allclose(gr[mine], rg[ref], rtol=0, atol=1e-10, err_msg=mine)


def test_finite_differences():
    B, T, H, D, window, eps = 1, 6, 1, 4, 3, 1e-6
    scale = 1.0 / math.sqrt(D)
    args = {n: rand((B, T, H, D), 20 + i) for i, n in enumerate(("q", "k", "v", "ve"))}
    args["g"] = rand((B, T, H), 25)
    dO = rand((B, T, H, D), 26)
    cos, sin = rope_ve.rope_tables(T, D)
    gr = rope_ve.attn_bwd(args["q"], args["k"], args["v"], dO, cos, sin, window, eps, scale, ve=args["ve"],
                          g=args["g"])

    def loss(a):
        o, _ = rope_ve.attn_fwd(a["q"], a["k"], a["v"], cos, sin, window, eps, scale, ve=a["ve"], g=a["g"])
        return float(np.sum(o * dO))

    h = 1e-6
    for name, grad in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("ve", "dve"), ("g", "dg")):
        an = gr[grad]
        for f in range(args[name].size):
            a = {n: x.copy() for n, x in args.items()}
            a[name].flat[f] += h
            lp = loss(a)
            a[name].flat[f] -= 2 * h
            fd = (lp - loss(a)) / (2 * h)
            assert abs(fd - an.flat[f]) <= 1e-6 * (abs(an.flat[f]) + np.abs(an).max()), (name, f)


def test_gate_limits():
    B, T, H, D, w = 1, 24, 2, 16, 6
    q, k, v = rand((B, T, H, D), 30), rand((B, T, H, D), 31), rand((B, T, H, D), 32)
    cos, sin = rope_ve.rope_tables(T, D)
    o_plain, _ = rope_ve.attn_fwd(q, k, v, cos, sin, w)
    # a closed gate (sigmoid -> 0) leaves v alone
    o_closed, _ = rope_ve.attn_fwd(q, k, v, cos, sin, w, ve=rand((B, T, H, D), 33), g=np.full((B, T, H), -40.0))
    np.testing.assert_allclose(o_closed, o_plain, atol=1e-12)
    # gate 2 sigmoid(0) = 1 with ve = -v cancels the values: o = 0
    o_zero, _ = rope_ve.attn_fwd(q, k, v, cos, sin, w, ve=-v, g=np.zeros((B, T, H)))
    np.testing.assert_allclose(o_zero, 0.0, atol=1e-13)


def test_bf16_round_matches_torch():
    x = rand(5000, 40) * np.exp(rand(5000, 41) * 5)
    x32 = x.astype(np.float32).astype(np.float64)
    ref = torch.tensor(x32, dtype=torch.float32).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(rope_ve.bf16_round(x32), ref)


def test_rounded_operands_only_change_the_operands():
    """With round_operands the core sees the rounded rotated q, k (and mixed v):
    identity rounding gives the exact result, and the forward on rounded
    operands is the plain oracle on those operands."""
    from oracle import oracle as orc
    B, T, H, D, w = 1, 30, 2, 16, 7
    q, k, v, ve = (rand((B, T, H, D), 50 + i) for i in range(4))
    g = rand((B, T, H), 55)
    cos, sin = rope_ve.rope_tables(T, D)
    o1, l1 = rope_ve.attn_fwd(q, k, v, cos, sin, w, ve=ve, g=g, round_operands=lambda a: a)
    o2, l2 = rope_ve.attn_fwd(q, k, v, cos, sin, w, ve=ve, g=g)
    np.testing.assert_array_equal(o1, o2)
    r = rope_ve.bf16_round
    o3, _ = rope_ve.attn_fwd(q, k, v, cos, sin, w, ve=ve, g=g, round_operands=r)
    o4, _ = orc.attn_fwd(r(rope_ve.rope(q, cos, sin)), r(rope_ve.rope(k, cos, sin)), r(rope_ve.mix_value(v, ve, g)), w)
    np.testing.assert_array_equal(o3, o4)
    assert np.abs(o3 - o2).max() > 0
