"""GPU parity of the fused RoPE / value-embedding path against the fp64 oracle.

The pages run two steps just before the attention core ("autoresearch" README
(gitee), section 7.4: rotary position embedding of q and k with bf16 cos/sin
tables; section 5.2.3: v + 2 sigmoid(g) ve on the layers that have a value
embedding).  ar_attn_fwd_rope rotates k and mixes v once per layer in a
pre-pass and rotates each Q tile inside the forward kernel;
ar_attn_bwd_rope runs the backward kernels on the pre-pass's rotated and mixed
operands and finishes the chain rule in their epilogues.

The kernels round the rotated q, k and the mixed v to bf16 once before their
products; in the pages' model those are bf16 tensors too (their rotation and
gate run under bf16 autocast).  So each case is compared twice:
(a) with the oracle given those operands rounded to bf16 once
    (oracle.rope_ve, round_operands=bf16_round): the bars of every other
    parity test, |err| <= 2e-2 + 2^-8 |ref| with relative L2 <= 5e-3, lse 1e-3;
(b) with the exact oracle: the operand rounding adds its own error, so
    relative L2 <= 1e-2 (two independent sources of about 0.3 % each), and
    lse within 1e-3 plus the rounding's bound on row i, the largest logit change
    it can cause, scale rq_i max_j rk_j 2^-8 sum_d |q_id| |k_jd| over the row's
    visible keys (q, k rotated).
"""
import numpy as np
import pytest
import torch

from oracle import rope_ve as orv
from sliding_window_attention_rmsnorm_b200 import attn, build, synth

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2, LSE_ABS, ULP = 2e-2, 5e-3, 1e-3, 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    attn.lib()


def inputs(cfg, B, T, H, Hkv, with_ve, rows=None):
    xq = synth.layer_inputs(cfg, 0, B, T, H, 128, roles=("q", "dO"))
    xk = synth.layer_inputs(cfg, 0, B, T, Hkv, 128, roles=("k", "v"))
    x = dict(q=xq["q"], dO=xq["dO"], k=xk["k"], v=xk["v"])
    if with_ve:
        x["ve"], x["g"] = synth.value_embedding(cfg, 0, B, T, Hkv, 128)
    c, s = orv.rope_tables(rows or T, 128)
    x["cos"] = torch.tensor(c, dtype=torch.float64).to(torch.bfloat16)  # exact: the values are bf16
    x["sin"] = torch.tensor(s, dtype=torch.float64).to(torch.bfloat16)
    return x


def check(a, b, name, tag, heads=None, nh=None):
    if heads is not None:
        if name == "lse":
            a = np.stack([a[h // nh, h % nh] for h in heads])
            b = np.stack([b[h // nh, h % nh] for h in heads])
        else:
            a = np.stack([a[h // nh, :, h % nh] for h in heads])
            b = np.stack([b[h // nh, :, h % nh] for h in heads])
    a = a.astype(np.float64)
    assert np.isfinite(a).all(), (tag, name)
    err = np.abs(a - b)
    if name == "lse":
        assert err.max() <= LSE_ABS, (tag, name, err.max())
        return
    assert (err - (MAX_ABS + ULP * np.abs(b))).max() <= 0, (tag, name, err.max())
    nb = np.linalg.norm(b)
    if nb > 0:
        assert np.linalg.norm(a - b) / nb <= REL_L2, (tag, name, np.linalg.norm(a - b) / nb)


def lse_rounding_bound(x, w, heads=None, H=None):
    """Per-row bound of the lse change from rounding the rotated q, k to bf16
    (half an ulp, 2^-9 relative, on each element): [B, H, T], or the listed heads."""
    qr, kr = orv.rope(x["q"], x["cos"], x["sin"]), orv.rope(x["k"], x["cos"], x["sin"])
    B, T, Hq, D = qr.shape
    grp = Hq // kr.shape[2]
    scale = 1.0 / np.sqrt(D)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    vis = (j <= i) & ((i - j <= w) if 0 <= w < T - 1 else True)
    out = {}
    for hh in (heads if heads is not None else range(B * Hq)):
        b, h = divmod(hh, Hq)
        q, k = qr[b, :, h], kr[b, :, h // grp]
        rq = 1.0 / np.sqrt(np.mean(q * q, axis=1) + 1e-6)
        rk = 1.0 / np.sqrt(np.mean(k * k, axis=1) + 1e-6)
        m = (np.abs(q) @ np.abs(k).T) * rk[None, :]
        out[hh] = 1e-3 + scale * 2.0 ** -8 * rq * np.where(vis, m, 0.0).max(axis=1)
    if heads is not None:
        return np.stack([out[hh] for hh in heads])
    return np.stack([out[hh] for hh in range(B * Hq)]).reshape(B, Hq, T)


def check_exact(a, b, name, tag):
    a = a.astype(np.float64)
    nb = np.linalg.norm(b)
    if nb > 0:
        assert np.linalg.norm(a - b) / nb <= 1e-2, (tag, name, "exact oracle rel l2", np.linalg.norm(a - b) / nb)


def gpu_fwd(x, w):
    d = {n: t.cuda() for n, t in x.items()}
    o, lse = attn.fwd_rope(d["q"], d["k"], d["v"], d["cos"], d["sin"], w, ve=d.get("ve"), ve_gate=d.get("g"))
    attn.sync_status()
    return o.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("B,T,H,Hkv,w,with_ve", [(2, 300, 4, 4, 100, False), (2, 300, 4, 2, 100, True),
                                                 (1, 1000, 2, 2, -1, True), (1, 129, 3, 1, 0, True),
                                                 (2, 640, 4, 4, 256, True)])
def test_forward_rope_ve(B, T, H, Hkv, w, with_ve):
    x = inputs(31, B, T, H, Hkv, with_ve, rows=T + 50)
    o, lse = gpu_fwd(x, w)
    tag = "rope B=%d T=%d H=%d Hkv=%d w=%d ve=%s" % (B, T, H, Hkv, w, with_ve)
    ro, rl = orv.attn_fwd(x["q"], x["k"], x["v"], x["cos"], x["sin"], w, ve=x.get("ve"), g=x.get("g"),
                          round_operands=orv.bf16_round)
    check(o, ro, "o", tag)
    check(lse, rl, "lse", tag)
    eo, el = orv.attn_fwd(x["q"], x["k"], x["v"], x["cos"], x["sin"], w, ve=x.get("ve"), g=x.get("g"))
    check_exact(o, eo, "o", tag)
    assert (np.abs(lse - el) - lse_rounding_bound(x, w)).max() <= 0, (tag, "lse beyond the rounding bound")


def test_forward_rope_ve_full_size_sampled():
    """B=8, T=2048, H=4, window 1024 (an S layer of the stack), RoPE and the
    value embedding, three whole heads against the oracle."""
    B, T, H, w = 8, 2048, 4, 1024
    x = inputs(32, B, T, H, H, True)
    o, lse = gpu_fwd(x, w)
    heads = [0, 13, B * H - 1]
    ro, rl = orv.attn_fwd(x["q"], x["k"], x["v"], x["cos"], x["sin"], w, ve=x["ve"], g=x["g"], heads=heads,
                          round_operands=orv.bf16_round)
    for n, a, b in (("o", o, ro), ("lse", lse, rl)):
        check(a, b, n, "rope full size", heads, H)
    eo, el = orv.attn_fwd(x["q"], x["k"], x["v"], x["cos"], x["sin"], w, ve=x["ve"], g=x["g"], heads=heads)
    sel = np.stack([lse[h // H, h % H] for h in heads])
    ref = np.stack([el[h // H, h % H] for h in heads])
    assert (np.abs(sel - ref) - lse_rounding_bound(x, w, heads, H)).max() <= 0
    check_exact(np.stack([o[h // H, :, h % H] for h in heads]), np.stack([eo[h // H, :, h % H] for h in heads]),
                "o", "rope full size")


def gpu_fwd_bwd(x, w):
    d = {n: t.cuda() for n, t in x.items()}
    o, lse = attn.fwd_rope(d["q"], d["k"], d["v"], d["cos"], d["sin"], w, ve=d.get("ve"), ve_gate=d.get("g"))
    g = attn.bwd_rope(d["q"], d["k"], d["v"], o, d["dO"], lse, d["cos"], d["sin"], w, ve=d.get("ve"),
                      ve_gate=d.get("g"))
    attn.sync_status()
    names = ("dq", "dk", "dv", "dve", "dg")[:len(g)]
    out = {n: t.float().cpu().numpy() for n, t in zip(names, g)}
    out["o"], out["lse"] = o.float().cpu().numpy(), lse.cpu().numpy()
    return out


@pytest.mark.parametrize("B,T,H,Hkv,w,with_ve", [(2, 300, 4, 4, 100, False), (2, 300, 4, 2, 100, True),
                                                 (1, 1000, 2, 2, -1, True), (1, 129, 3, 1, 0, True)])
def test_backward_rope_ve(B, T, H, Hkv, w, with_ve):
    """dq, dk, dv for the unrotated, unmixed inputs (and dve, dg with the value
    embedding) against the oracle's chain rule."""
    x = inputs(33, B, T, H, Hkv, with_ve, rows=T + 50)
    g = gpu_fwd_bwd(x, w)
    tag = "rope bwd B=%d T=%d H=%d Hkv=%d w=%d ve=%s" % (B, T, H, Hkv, w, with_ve)
    r = orv.attn_bwd(x["q"], x["k"], x["v"], x["dO"], x["cos"], x["sin"], w, ve=x.get("ve"), g=x.get("g"),
                     round_operands=orv.bf16_round)
    e = orv.attn_bwd(x["q"], x["k"], x["v"], x["dO"], x["cos"], x["sin"], w, ve=x.get("ve"), g=x.get("g"))
    for n in ("dq", "dk", "dv") + (("dve", "dg") if with_ve else ()):
        check(g[n], r[n], n, tag)
        check_exact(g[n], e[n], n, tag)


def test_backward_rope_ve_full_size_sampled():
    """B=8, T=2048, H=4, window 1024, RoPE and the value embedding: the
    backward on three whole heads against the oracle."""
    B, T, H, w = 8, 2048, 4, 1024
    x = inputs(34, B, T, H, H, True)
    g = gpu_fwd_bwd(x, w)
    heads = [1, 14, B * H - 2]
    r = orv.attn_bwd(x["q"], x["k"], x["v"], x["dO"], x["cos"], x["sin"], w, ve=x["ve"], g=x["g"], heads=heads,
                     round_operands=orv.bf16_round)
    for n in ("dq", "dk", "dv", "dve"):
        check(g[n], r[n], n, "rope bwd full size", heads, H)
    a = np.stack([g["dg"][h // H, :, h % H] for h in heads])
    b = np.stack([r["dg"][h // H, :, h % H] for h in heads])
    err = np.abs(a - b)
    assert (err - (MAX_ABS + ULP * np.abs(b))).max() <= 0 and np.linalg.norm(a - b) / np.linalg.norm(b) <= REL_L2


def test_backward_rope_ve_several_head_groups():
    """B=2, T=8192, H=8, Hkv=4, full causal, RoPE and the value embedding: the
    G tiles of all 16 query heads exceed the 1 GiB buffer, so the backward runs
    as two launches over disjoint K/V-head groups, on the rotated and mixed
    operands the pre-pass writes after the G buffer.  One K/V head from each
    launch (with its two query heads) against the oracle."""
    B, T, H, Hkv, w = 2, 8192, 8, 4, -1
    assert attn.bwd_workspace_bytes(B, T, H, 128, Hkv) < B * H * 2080 * 32768  # really split
    x = inputs(36, B, T, H, Hkv, True)
    g = gpu_fwd_bwd(x, w)
    heads = [1, B * Hkv - 2]  # first launch: K/V heads 0-3; second: 4-7
    grp = H // Hkv
    qheads = [hk // Hkv * H + (hk % Hkv) * grp + m for hk in heads for m in range(grp)]
    r = orv.attn_bwd(x["q"], x["k"], x["v"], x["dO"], x["cos"], x["sin"], w, ve=x["ve"], g=x["g"], heads=heads,
                     round_operands=orv.bf16_round)
    tag = "rope bwd head groups"
    check(g["dq"], r["dq"], "dq", tag, qheads, H)
    for n in ("dk", "dv", "dve"):
        check(g[n], r[n], n, tag, heads, Hkv)
    a = np.stack([g["dg"][h // Hkv, :, h % Hkv] for h in heads])
    b = np.stack([r["dg"][h // Hkv, :, h % Hkv] for h in heads])
    err = np.abs(a - b)
    assert (err - (MAX_ABS + ULP * np.abs(b))).max() <= 0 and np.linalg.norm(a - b) / np.linalg.norm(b) <= REL_L2


@pytest.mark.parametrize("B,T,H,Hkv,w,with_ve", [(2, 300, 4, 2, 100, True), (1, 640, 4, 4, 256, False),
                                                 (2, 2048, 4, 4, 1024, True)])
def test_backward_with_saved_forward_operands(B, T, H, Hkv, w, with_ve):
    """ar_attn_bwd_rope_saved, given the forward's workspace (its rotated k and
    mixed v), rotates only q and returns bitwise the outputs of ar_attn_bwd_rope,
    which forms them again."""
    x = inputs(38, B, T, H, Hkv, with_ve)
    d = {n: t.cuda() for n, t in x.items()}
    ws = torch.empty(attn.fwd_rope_workspace_bytes(B, T, Hkv, 128, with_ve), dtype=torch.uint8, device="cuda")
    o, lse = attn.fwd_rope(d["q"], d["k"], d["v"], d["cos"], d["sin"], w, ve=d.get("ve"), ve_gate=d.get("g"),
                           workspace=ws)
    a = attn.bwd_rope(d["q"], d["k"], d["v"], o, d["dO"], lse, d["cos"], d["sin"], w, ve=d.get("ve"),
                      ve_gate=d.get("g"))
    b = attn.bwd_rope(d["q"], d["k"], d["v"], o, d["dO"], lse, d["cos"], d["sin"], w, ve=d.get("ve"),
                      ve_gate=d.get("g"), saved=ws)
    attn.sync_status()
    assert len(a) == len(b) == (5 if with_ve else 3)
    for n, ta, tb in zip(("dq", "dk", "dv", "dve", "dg"), a, b):
        assert torch.equal(ta, tb), n
