"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test ties the oracle to something the pages or the mathematics fix:
an independent library routine for the same special case, finite
differences of the oracle's own forward, closed forms, and invariants.
Together they catch a dropped term, a wrong sign, a wrong index or a
transposed operand anywhere in the forward, the softmax backward or the
RMSNorm backward.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import oracle as orc
from oracle.stack import layer_windows
from sliding_window_attention_rmsnorm_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape)


# ---------------------------------------------------------------- library check
def torch_reference(q, k, v, dO, window, eps, scale):
    """Textbook composition: F.rms_norm + SDPA with an explicit band mask, fp64 autograd."""
    q, k, v, dO = (torch.tensor(x, dtype=torch.float64) for x in (q, k, v, dO))
    q.requires_grad_(True); k.requires_grad_(True); v.requires_grad_(True)
    B, T, H, D = q.shape
    qh = F.rms_norm(q, (D,), eps=eps).transpose(1, 2)
    kh = F.rms_norm(k, (D,), eps=eps).transpose(1, 2)
    vt = v.transpose(1, 2)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = j <= i
    if window >= 0:
        mask = mask & (i - j <= window)
    o = F.scaled_dot_product_attention(qh, kh, vt, attn_mask=mask, scale=scale)
    scores = (qh @ kh.transpose(-1, -2)) * scale
    lse = torch.logsumexp(scores.masked_fill(~mask, float("-inf")), dim=-1)
    o = o.transpose(1, 2)
    (o * dO).sum().backward()
    return (o.detach().numpy(), lse.detach().numpy(), q.grad.numpy(), k.grad.numpy(),
            v.grad.numpy())


@pytest.mark.parametrize("B,T,H,D,window", [
    (1, 1, 1, 8, -1), (2, 7, 2, 16, 2), (1, 33, 3, 32, 5), (1, 40, 1, 128, 0),
    (1, 64, 2, 128, 17), (1, 64, 2, 128, -1), (2, 50, 1, 64, 63),
])
def test_matches_torch_sdpa_fp64(B, T, H, D, window):
    eps, scale = 1e-6, 1.0 / math.sqrt(D)
    q, k, v, dO = (rand((B, T, H, D), s) for s in range(4))
    ro, rlse, rdq, rdk, rdv = torch_reference(q, k, v, dO, window, eps, scale)
    o, lse = orc.attn_fwd(q, k, v, window, eps, scale)
    g = orc.attn_bwd(q, k, v, dO, window, eps, scale)
    for name, a, b in [("o", o, ro), ("lse", lse, rlse), ("dq", g["dq"], rdq),
                       ("dk", g["dk"], rdk), ("dv", g["dv"], rdv), ("lse_bwd", g["lse"], rlse)]:
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-10, err_msg=name)


def torch_reference_gqa(q, k, v, dO, window, eps, scale):
    """Grouped K/V heads through the same textbook composition: each K/V head is
    repeated for the query heads of its group (query head h reads K/V head
    h // (H // Hkv)), so autograd sums dk, dv over the group."""
    H, Hkv = q.shape[2], k.shape[2]
    kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (k, v))
    kr, vr = (x.repeat_interleave(H // Hkv, dim=2) for x in (kt, vt))
    qt, dOt = (torch.tensor(x, dtype=torch.float64) for x in (q, dO))
    qt.requires_grad_(True)
    B, T, _, D = q.shape
    qh = F.rms_norm(qt, (D,), eps=eps).transpose(1, 2)
    kh = F.rms_norm(kr, (D,), eps=eps).transpose(1, 2)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = (j <= i) & ((i - j <= window) if window >= 0 else torch.ones_like(j <= i))
    o = F.scaled_dot_product_attention(qh, kh, vr.transpose(1, 2), attn_mask=mask, scale=scale).transpose(1, 2)
    (o * dOt).sum().backward()
    return o.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("B,T,H,Hkv,D,window", [
    (1, 9, 2, 1, 8, -1), (2, 21, 4, 2, 16, 4), (1, 40, 6, 3, 128, 0), (1, 48, 4, 1, 64, 11),
])
def test_grouped_kv_heads_match_torch_sdpa_fp64(B, T, H, Hkv, D, window):
    eps, scale = 1e-6, 1.0 / math.sqrt(D)
    q, dO = rand((B, T, H, D), 40), rand((B, T, H, D), 41)
    k, v = rand((B, T, Hkv, D), 42), rand((B, T, Hkv, D), 43)
    ro, rdq, rdk, rdv = torch_reference_gqa(q, k, v, dO, window, eps, scale)
    o, _ = orc.attn_fwd(q, k, v, window, eps, scale)
    g = orc.attn_bwd(q, k, v, dO, window, eps, scale)
    for name, a, b in [("o", o, ro), ("dq", g["dq"], rdq), ("dk", g["dk"], rdk), ("dv", g["dv"], rdv)]:
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-10, err_msg=name)


def test_grouped_kv_heads_finite_differences():
    """dk, dv of a shared K/V head against central differences of the forward."""
    B, T, H, Hkv, D, window, eps = 1, 7, 4, 2, 4, 3, 1e-6
    scale = 1.0 / math.sqrt(D)
    q, dO = rand((B, T, H, D), 50), rand((B, T, H, D), 51)
    k, v = rand((B, T, Hkv, D), 52), rand((B, T, Hkv, D), 53)
    g = orc.attn_bwd(q, k, v, dO, window, eps, scale)

    def loss(k_, v_):
        o, _ = orc.attn_fwd(q, k_, v_, window, eps, scale)
        return float(np.sum(o * dO))

    h = 1e-6
    for name, src in (("dk", 0), ("dv", 1)):
        an = g[name]
        gmax = np.abs(an).max()
        for f in range(k.size):
            args = [k.copy(), v.copy()]
            args[src].flat[f] += h
            lp = loss(*args)
            args[src].flat[f] -= 2 * h
            lm = loss(*args)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - an.flat[f]) <= 1e-6 * (abs(an.flat[f]) + gmax), (name, f, fd, an.flat[f])


def test_grouped_kv_heads_equal_duplicated_heads():
    """Grouped K/V heads give the multi-head result on K/V duplicated per query
    head, with dk, dv summed over each group; a K/V-head subset matches."""
    B, T, H, Hkv, D, w = 2, 30, 6, 2, 16, 9
    q, dO = rand((B, T, H, D), 60), rand((B, T, H, D), 61)
    k, v = rand((B, T, Hkv, D), 62), rand((B, T, Hkv, D), 63)
    kd, vd = np.repeat(k, H // Hkv, axis=2), np.repeat(v, H // Hkv, axis=2)
    o, lse = orc.attn_fwd(q, k, v, w)
    od, lsed = orc.attn_fwd(q, kd, vd, w)
    np.testing.assert_allclose(o, od, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lsed, rtol=0, atol=1e-13)
    g, gd = orc.attn_bwd(q, k, v, dO, w), orc.attn_bwd(q, kd, vd, dO, w)
    np.testing.assert_allclose(g["dq"], gd["dq"], rtol=0, atol=1e-12)
    for n in ("dk", "dv"):
        summed = gd[n].reshape(B, T, Hkv, H // Hkv, D).sum(axis=3)
        np.testing.assert_allclose(g[n], summed, rtol=0, atol=1e-12)
    sub = orc.attn_bwd(q, k, v, dO, w, heads=[1 * Hkv + 1])  # b = 1, K/V head 1
    np.testing.assert_array_equal(sub["dk"][1, :, 1], g["dk"][1, :, 1])
    np.testing.assert_array_equal(sub["dq"][1, :, 3:6], g["dq"][1, :, 3:6])
    assert np.isnan(sub["dk"][0]).all()


def test_delta_equals_rowsum_dO_o():
    """delta is computed as sum_j P dP; it must equal the row sum of dO*o."""
    B, T, H, D, w = 1, 30, 2, 16, 7
    q, k, v, dO = (rand((B, T, H, D), 10 + s) for s in range(4))
    o, _ = orc.attn_fwd(q, k, v, w)
    g = orc.attn_bwd(q, k, v, dO, w)
    ref = np.einsum("bthd,bthd->bht", dO, o)
    np.testing.assert_allclose(g["delta"], ref, atol=1e-12)


# ---------------------------------------------------------------- finite differences
@pytest.mark.parametrize("T,D,window", [(6, 4, 2), (8, 4, -1), (5, 128, 1), (8, 128, 3)])
def test_finite_differences(T, D, window):
    B, H, eps = 1, 1, 1e-6
    scale = 1.0 / math.sqrt(D)
    q, k, v, dO = (rand((B, T, H, D), 20 + s) for s in range(4))
    g = orc.attn_bwd(q, k, v, dO, window, eps, scale)

    def loss(q_, k_, v_):
        o, _ = orc.attn_fwd(q_, k_, v_, window, eps, scale)
        return float(np.sum(o * dO))

    h = 1e-6
    rng = np.random.default_rng(7)
    for name, idx_src in (("dq", 0), ("dk", 1), ("dv", 2)):
        an = g[name]
        gmax = np.abs(an).max()
        flat = list(range(q.size)) if D == 4 else list(rng.choice(q.size, 48, replace=False))
        for f in flat:
            args = [q.copy(), k.copy(), v.copy()]
            args[idx_src].flat[f] += h
            lp = loss(*args)
            args[idx_src].flat[f] -= 2 * h
            lm = loss(*args)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - an.flat[f]) <= 1e-6 * (abs(an.flat[f]) + gmax), (name, f, fd, an.flat[f])


# ---------------------------------------------------------------- closed forms
def test_full_window_equivalence_bitwise():
    """Any window >= T-1 is full causal: results are bit-identical."""
    B, T, H, D = 1, 24, 2, 32
    q, k, v, dO = (rand((B, T, H, D), 30 + s) for s in range(4))
    outs = []
    for w in (T - 1, T, 10 * T, -1):
        o, lse = orc.attn_fwd(q, k, v, w)
        g = orc.attn_bwd(q, k, v, dO, w)
        outs.append((o, lse, g["dq"], g["dk"], g["dv"]))
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert np.array_equal(a, b)
    # and a narrower window is really different
    o_s, _ = orc.attn_fwd(q, k, v, T - 2)
    assert not np.array_equal(o_s, outs[0][0])


@pytest.mark.parametrize("window", [-1, 0, 3])
def test_softmax_rows_sum_to_one(window):
    """A value column of ones comes out as exactly the softmax row sums."""
    B, T, H, D = 1, 40, 2, 16
    q, k, v = (rand((B, T, H, D), 40 + s) for s in range(3))
    v[..., 0] = 1.0
    o, _ = orc.attn_fwd(q, k, v, window)
    np.testing.assert_allclose(o[..., 0], 1.0, atol=1e-12)


@pytest.mark.parametrize("window", [-1, 5])
def test_lse_bounds(window):
    """|s_ij| <= scale*||qhat|| ||khat|| <= scale*D, so lse_i = log n_i +- scale*D."""
    B, T, H, D = 2, 64, 2, 128
    q, k, v = (rand((B, T, H, D), 50 + s) for s in range(3))
    scale = 1.0 / math.sqrt(D)
    _, lse = orc.attn_fwd(q, k, v, window, scale=scale)
    w = T if window < 0 else window
    n = np.array([min(i, w) + 1 for i in range(T)], dtype=np.float64)
    assert np.all(lse >= np.log(n) - scale * D - 1e-12)
    assert np.all(lse <= np.log(n) + scale * D + 1e-12)
    # peaked keys drive some logits near the bound: lse must still respect it
    qb = synth.normal_bf16((B, T, H, D), 1)
    kb = synth.peaked_keys(qb, 2)
    _, lse2 = orc.attn_fwd(qb, kb, v, window, scale=scale)
    assert np.all(np.abs(lse2 - np.log(n)) <= scale * D + 1e-12)


def test_row_zero_and_window_zero():
    B, T, H, D = 2, 20, 3, 16
    q, k, v, dO = (rand((B, T, H, D), 60 + s) for s in range(4))
    o, _ = orc.attn_fwd(q, k, v, -1)
    assert np.array_equal(o[:, 0], v[:, 0])            # row 0 sees only key 0
    o0, lse0 = orc.attn_fwd(q, k, v, 0)
    assert np.array_equal(o0, v)                        # w = 0: every row sees itself
    g = orc.attn_bwd(q, k, v, dO, 0)
    assert np.array_equal(g["dv"], dO)
    assert np.all(g["dq"] == 0.0) and np.all(g["dk"] == 0.0)


@pytest.mark.parametrize("window", [-1, 4])
def test_uniform_keys_give_window_mean(window):
    B, T, H, D = 1, 30, 2, 16
    q, v = rand((B, T, H, D), 70), rand((B, T, H, D), 71)
    k = np.broadcast_to(rand((B, 1, H, D), 72), (B, T, H, D)).copy()
    o, _ = orc.attn_fwd(q, k, v, window)
    w = T if window < 0 else window
    for i in range(T):
        j0 = max(0, i - w)
        np.testing.assert_allclose(o[:, i], v[:, j0:i + 1].mean(axis=1), atol=1e-12)


@pytest.mark.parametrize("window", [-1, 6])
def test_masked_positions_get_zero_gradient(window):
    B, T, H, D, i0 = 1, 32, 2, 16, 20
    q, k, v, dO = (rand((B, T, H, D), 80 + s) for s in range(4))
    dO[:, np.arange(T) != i0] = 0.0
    g = orc.attn_bwd(q, k, v, dO, window)
    w = T if window < 0 else window
    outside = [j for j in range(T) if not (i0 - w <= j <= i0)]
    assert np.all(g["dk"][:, outside] == 0.0) and np.all(g["dv"][:, outside] == 0.0)
    assert np.all(g["dq"][:, np.arange(T) != i0] == 0.0)
    inside = [j for j in range(T) if i0 - w <= j <= i0]
    assert np.all(np.abs(g["dv"][:, inside]).sum(axis=-1) > 0)


def test_norm_invariants():
    """eps = 0: o is invariant to a positive per-row scale of q and k, and the
    norm's gradient is orthogonal to its input row."""
    B, T, H, D = 1, 24, 2, 32
    q, k, v, dO = (rand((B, T, H, D), 90 + s) for s in range(4))
    c = np.exp(rand((B, T, H, 1), 95))
    o1, _ = orc.attn_fwd(q, k, v, 5, eps=0.0)
    o2, _ = orc.attn_fwd(q * c, k / c, v, 5, eps=0.0)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    g = orc.attn_bwd(q, k, v, dO, 5, eps=0.0)
    qq = np.einsum("bthd,bthd->bth", g["dq"], q)
    kk = np.einsum("bthd,bthd->bth", g["dk"], k)
    assert np.abs(qq).max() < 1e-12 * np.abs(g["dq"]).max() * np.abs(q).max() * D
    assert np.abs(kk).max() < 1e-12 * np.abs(g["dk"]).max() * np.abs(k).max() * D


def test_head_subset_equals_full():
    """Computing a subset of heads gives the same values as the full run."""
    B, T, H, D = 2, 20, 3, 16
    q, k, v, dO = (rand((B, T, H, D), 100 + s) for s in range(4))
    o, lse = orc.attn_fwd(q, k, v, 4)
    o2, lse2 = orc.attn_fwd(q, k, v, 4, heads=[4])
    b, h = divmod(4, H)
    assert np.array_equal(o[b, :, h], o2[b, :, h]) and np.array_equal(lse[b, h], lse2[b, h])
    g = orc.attn_bwd(q, k, v, dO, 4)
    g2 = orc.attn_bwd(q, k, v, dO, 4, heads=[4])
    for n in ("dq", "dk", "dv"):
        assert np.array_equal(g[n][b, :, h], g2[n][b, :, h])


# ---------------------------------------------------------------- pages' own numbers
def test_layer_windows_match_pages_flop_count():
    fx = json.load(open(os.path.join(GOLDEN, "pages_flops_per_token.json")))
    ws = layer_windows(fx["n_layer"], fx["seq_len"])
    flops = 6 * (fx["transformer_matrix_params"] + fx["lm_head_params"]) \
        + 12 * fx["n_embd"] * sum(ws)
    assert flops == fx["flops_per_token"]
    T = fx["seq_len"]
    assert [l for l, w in enumerate(ws) if w < T] == fx["local_layers"]
    assert [l for l, w in enumerate(ws) if w == T] == fx["global_layers"]


def test_unmasked_pair_counts():
    """Pair counts quoted for the workloads (window w allows i - j <= w)."""
    assert orc.unmasked_pairs(256, 128) == 24768
    assert orc.unmasked_pairs(256, -1) == 32896
    assert orc.unmasked_pairs(2048, 1024) == 1574400
    assert orc.unmasked_pairs(2048, 2048) == 2098176
