"""fp64 oracle for the steps just before the attention core: rotary position
embedding of q and k, and the value-embedding gate on v.  TEST
INFRASTRUCTURE ONLY, like the rest of oracle/: the tests, the smoke check and
the benchmark's CPU-baseline leg may use it; the product never does.

What the pages compute ("autoresearch" README (gitee)):

* Section 7.4 "RoPE": the head dimension is split into two halves x1 = x[:D/2],
  x2 = x[D/2:], and each position t rotates them with cos_t, sin_t:
      y1 = x1 cos_t + x2 sin_t,   y2 = -x1 sin_t + x2 cos_t.
  The tables are precomputed once: inv_freq_c = 1 / base^(2c / D) for
  c = 0 .. D/2 - 1 (base 10000), angle = t * inv_freq_c, taken in fp32, and
  stored as bf16; row t of the table is position t.
* Section 5.2.3 "Value Embedding (ResFormer)": on the layers that have one, a
  per-token value embedding ve (same shape as v) is mixed in with a gate from a
  small linear layer over the first 32 channels of the block input:
      v <- v + 2 sigmoid(g) ve,   g = ve_gate(x[..., :32])   (one g per K/V head).
  The gate's linear layer is model state outside the attention core; the core
  takes its output g (the gate logits, [B, T, Hkv]).
* Section 7.3: q and k then go through the parameter-free RMSNorm before the
  attention product.  Rotation keeps a row's length, so rotating before or
  after the norm gives the same result; this oracle rotates first.

Everything here is the plain definition in fp64 on top of the attention
oracle (oracle.attn_fwd / attn_bwd), which sees the rotated q, k and the mixed
v.  The backward is the chain rule written out: the attention gradient of the
rotated / mixed inputs, then the transposed rotation (dx1 = dy1 cos - dy2 sin,
dx2 = dy1 sin + dy2 cos) and the gate's derivative.
"""
import numpy as np

from . import oracle as _attn


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def rope_tables(T: int, D: int, base: float = 10000.0, rounding: str = "bf16"):
    """cos, sin tables [T, D/2] as the pages precompute them: angles in fp32,
    cos and sin in fp32, then rounded to bf16 (rounding="bf16"; "none" keeps
    the exact fp64 cos and sin of the fp64 angles, for the invariance pins).
    Returned as fp64 arrays holding those values."""
    if rounding == "none":
        c = np.arange(0, D, 2, dtype=np.float64)
        inv = 1.0 / (base ** (c / D))
        ang = np.outer(np.arange(T, dtype=np.float64), inv)
        return np.cos(ang), np.sin(ang)
    import torch  # fp32 and bf16 rounding as the pages' tables get them
    c = torch.arange(0, D, 2, dtype=torch.float32)
    inv = 1.0 / (base ** (c / D))
    ang = torch.outer(torch.arange(T, dtype=torch.float32), inv)
    return (ang.cos().to(torch.bfloat16).double().numpy(), ang.sin().to(torch.bfloat16).double().numpy())


def rope(x, cos, sin):
    """Rotate the two halves of every row of x [B, T, H, D] by position:
    row t uses cos[t], sin[t] ([>= T, D/2])."""
    x = _f64(x)
    T, d = x.shape[1], x.shape[3] // 2
    c = _f64(cos)[None, :T, None, :]
    s = _f64(sin)[None, :T, None, :]
    x1, x2 = x[..., :d], x[..., d:]
    return np.concatenate([x1 * c + x2 * s, -x1 * s + x2 * c], axis=-1)


def rope_transposed(dy, cos, sin):
    """The transpose of rope (its gradient map): dx1 = dy1 cos - dy2 sin,
    dx2 = dy1 sin + dy2 cos."""
    dy = _f64(dy)
    T, d = dy.shape[1], dy.shape[3] // 2
    c = _f64(cos)[None, :T, None, :]
    s = _f64(sin)[None, :T, None, :]
    d1, d2 = dy[..., :d], dy[..., d:]
    return np.concatenate([d1 * c - d2 * s, d1 * s + d2 * c], axis=-1)


def _sigmoid(g):
    return 1.0 / (1.0 + np.exp(-g))


def mix_value(v, ve, g):
    """v + 2 sigmoid(g) ve, with g [B, T, Hkv] broadcast over the head dimension."""
    return _f64(v) + 2.0 * _sigmoid(_f64(g))[..., None] * _f64(ve)


def bf16_round(x):
    """fp64 values rounded to the nearest bf16 value (ties to even)."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    quantum = np.ldexp(1.0, e - 8)  # bf16 keeps 8 significant bits
    return np.round(x / quantum) * quantum


def _operands(q, k, v, cos, sin, ve, g, round_operands):
    qr, kr = rope(q, cos, sin), rope(k, cos, sin)
    vm = mix_value(v, ve, g) if ve is not None else _f64(v)
    if round_operands is not None:
        qr, kr = round_operands(qr), round_operands(kr)
        if ve is not None:
            vm = round_operands(vm)
    return qr, kr, vm


def attn_fwd(q, k, v, cos, sin, window, eps=1e-6, scale=None, ve=None, g=None, heads=None, round_operands=None):
    """Forward of the attention core with RoPE on q, k (and the value embedding
    on v when ve, g are given); returns (o, lse).  round_operands: None (exact),
    or a function applied to the rotated q, k and the mixed v before the core,
    e.g. bf16_round: in the pages' model those are bf16 tensors (the rotation
    and the gate run under bf16 autocast)."""
    qr, kr, vm = _operands(q, k, v, cos, sin, ve, g, round_operands)
    return _attn.attn_fwd(qr, kr, vm, window, eps, scale, heads=heads)


def attn_bwd(q, k, v, dO, cos, sin, window, eps=1e-6, scale=None, ve=None, g=None, heads=None,
             round_operands=None):
    """Backward of attn_fwd above: dict(dq, dk, dv[, dve, dg]) in fp64 (dg is the
    gradient with respect to the gate logits g).  heads: K/V heads, as for
    oracle.attn_bwd; round_operands as for attn_fwd (the chain rule through the
    rotation and the gate stays exact)."""
    qr, kr, vm = _operands(q, k, v, cos, sin, ve, g, round_operands)
    r = _attn.attn_bwd(qr, kr, vm, dO, window, eps, scale, heads=heads)
    out = dict(dq=rope_transposed(r["dq"], cos, sin), dk=rope_transposed(r["dk"], cos, sin), dv=r["dv"])
    if ve is not None:
        sg = _sigmoid(_f64(g))
        out["dve"] = 2.0 * sg[..., None] * r["dv"]
        out["dg"] = np.sum(r["dv"] * _f64(ve), axis=-1) * 2.0 * sg * (1.0 - sg)
    return out
