"""A model of the CUDA kernels' arithmetic, for the tests only.

The fp64 oracle (oracle/) computes the exact result.  The kernels round some
intermediate values to bf16, as FlashAttention-3 does (the kernel the pages'
trainer loads: "autoresearch" README (gitee), section 5.2.1), and their error
against the oracle comes from those roundings.  This module recomputes the
same quantities in fp64 with exactly those roundings and nothing else:

  forward   p_ij = 2^(s_ij log2 e - c_i) with c_i the softmax offset (the
            logit bound scale*D*log2 e when it is at most 32, else the row
            maximum); the PV product takes bf16(p); o = bf16(sum_j bf16(p_ij) v_j
            / n_i), n_i = sum_j bf16(p_ij) with the fixed offset and sum_j p_ij
            otherwise; lse_i = ln(sum_j exp(s_ij)), unrounded.
  backward  delta_i = dO_i . o_i with the bf16 o; P_ij = exp(s_ij - lse_i);
            dv_j = bf16(sum_i bf16(P_ij) dO_i); G_ij = P_ij (dO_i . v_j -
            delta_i) rq_i rk_j, and the products take bf16(G);
            dk_j = bf16(scale (sum_i bf16(G_ij) q_i - rk_j^2 / D sum_i G_ij
            (q_i . k_j) k_j)); dq_i = bf16(scale (a_i - (a_i . q_i) / D /
            (mean q_i^2 + eps) q_i)) with a_i = sum_j bf16(G_ij) k_j.

(rq, rk: 1/rms of the raw bf16 rows; the norm is applied to the logits and
gradients, never to rounded q or k.)  What remains between this model and the
GPU is fp32 accumulation order and the hardware exp2 approximation: a few
units in the last place of fp32, which can flip a bf16 rounding here and
there.  So the GPU must agree with this model far more tightly than with the
oracle, and the gap between this model and the oracle is the error that the
bf16 operands alone explain.

This is test infrastructure: it imports nothing from the product package or
from oracle/.
"""
import math

import numpy as np

LOG2E = 1.4426950408889634


def bf16(x):
    """Round fp64 values to the nearest bf16 value (ties to even)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    quantum = np.ldexp(1.0, e - 8)  # bf16 keeps 8 significant bits
    return np.round(x / quantum) * quantum


def _f64(t):
    if hasattr(t, "detach"):
        t = t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def _mask(T, window):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    vis = j <= i
    if 0 <= window < T - 1:
        vis &= (i - j) <= window
    return vis


def _rinv(x, eps):
    return 1.0 / np.sqrt(np.mean(x * x, axis=-1) + eps)


def _identity(x):
    return x


def forward(q, k, v, window, eps=1e-6, scale=None, rounding=True):
    """(o, lse) as the forward kernel computes them, in fp64 with its roundings
    (rounding=False: the same expressions without them, i.e. the exact result)."""
    rnd = bf16 if rounding else _identity
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    grp = H // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    vis = _mask(T, window)
    bound = scale * D * LOG2E
    o = np.zeros_like(q)
    lse = np.zeros((B, H, T))
    for b in range(B):
        for h in range(H):
            qi, kj, vj = q[b, :, h], k[b, :, h // grp], v[b, :, h // grp]
            rq, rk = _rinv(qi, eps), _rinv(kj, eps)
            x = (qi @ kj.T) * rq[:, None] * rk[None, :] * (scale * LOG2E)  # logits, log2 units
            x = np.where(vis, x, -np.inf)
            if bound <= 32.0:
                off = np.full(T, bound)
            else:
                off = x.max(axis=1)
            p = np.exp2(x - off[:, None])
            pb = rnd(p)
            l = p.sum(axis=1)
            norm = pb.sum(axis=1) if bound <= 32.0 else l
            o[b, :, h] = rnd((pb @ vj) / norm[:, None])
            lse[b, h] = (off + np.log2(l)) / LOG2E
    return o, lse


def backward(q, k, v, o, dO, lse, window, eps=1e-6, scale=None, rounding=True):
    """(dq, dk, dv) as the backward kernels compute them from the given o (bf16
    values) and lse, in fp64 with their roundings (rounding=False: without)."""
    rnd = bf16 if rounding else _identity
    q, k, v, o, dO, lse = (_f64(t) for t in (q, k, v, o, dO, lse))
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    grp = H // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    vis = _mask(T, window)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for hk in range(Hkv):
            kj, vj = k[b, :, hk], v[b, :, hk]
            rk = _rinv(kj, eps)
            dk_acc = np.zeros((T, D))
            dt = np.zeros(T)
            dv_acc = np.zeros((T, D))
            for h in range(hk * grp, (hk + 1) * grp):
                qi, dOi, oi = q[b, :, h], dO[b, :, h], o[b, :, h]
                rq = _rinv(qi, eps)
                S = qi @ kj.T  # raw logits q_i . k_j
                x = S * rq[:, None] * rk[None, :] * (scale * LOG2E)
                P = np.where(vis, np.exp2(x - (lse[b, h] * LOG2E)[:, None]), 0.0)
                delta = np.sum(dOi * oi, axis=1)
                dP = dOi @ vj.T
                G = P * (dP - delta[:, None]) * rq[:, None] * rk[None, :]
                Gb = rnd(G)
                dv_acc += rnd(P).T @ dOi
                dk_acc += Gb.T @ qi
                dt += np.sum(G * S, axis=0)
                a = Gb @ kj
                cq = np.sum(a * qi, axis=1) / D * rq * rq
                dq[b, :, h] = rnd(scale * (a - cq[:, None] * qi))
            ck = dt * rk * rk / D
            dk[b, :, hk] = rnd(scale * (dk_acc - ck[:, None] * kj))
            dv[b, :, hk] = rnd(dv_acc)
    return dq, dk, dv


def run(x, window, eps=1e-6, scale=None, rounding=True):
    """Forward and backward of the model on one input dict (q, k, v, dO)."""
    o, lse = forward(x["q"], x["k"], x["v"], window, eps, scale, rounding)
    dq, dk, dv = backward(x["q"], x["k"], x["v"], o, x["dO"], lse, window, eps, scale, rounding)
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv)
