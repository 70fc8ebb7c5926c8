"""CPU checks of the kernel-arithmetic model (tests/kernel_model.py).

The model is what makes the GPU tests' edge-case bound checkable: the GPU is
held to it within about one bf16 ulp, and here it is tied to the oracle.

* Without its bf16 roundings the model is the exact computation: it matches
  the fp64 oracle to rounding noise, for multi-head and grouped heads, for
  sliding and full windows, and for the running-max softmax offset.
* With them, its distance from the oracle is the error the precision model
  allows, and it stays inside the bound the GPU edge-case tests use
  (|err| <= 2e-2 + 2^-8 |ref|).
* For saturated softmax (keys close to their queries) the model's large
  relative error in dq and dk comes from one rounding only: o rounded to bf16
  before delta = rowsum(dO * o) (FlashAttention's convention).
"""
import math

import numpy as np
import pytest

import kernel_model as km
from oracle import oracle as orc
from sliding_window_attention_rmsnorm_b200 import synth

MAX_ABS, ULP_SLACK = 2e-2, 2.0 ** -8


def oracle_run(x, w, eps=1e-6, scale=None):
    o, lse = orc.attn_fwd(x["q"], x["k"], x["v"], w, eps, scale)
    g = orc.attn_bwd(x["q"], x["k"], x["v"], x["dO"], w, eps, scale)
    return dict(o=o, lse=lse, dq=g["dq"], dk=g["dk"], dv=g["dv"])


def gqa(seed, B, T, H, Hkv):
    xq = synth.layer_inputs(seed, 0, B, T, H, 128)
    xk = synth.layer_inputs(seed, 1, B, T, Hkv, 128)
    return dict(q=xq["q"], dO=xq["dO"], k=xk["k"], v=xk["v"])


def test_bf16_rounding():
    """Round to nearest, ties to even, 8 significant bits (torch agrees)."""
    import torch
    x = np.random.default_rng(3).standard_normal(20000) * np.exp(np.random.default_rng(4).uniform(-20, 20, 20000))
    ref = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).double().numpy()
    x32 = x.astype(np.float32).astype(np.float64)  # torch rounds from fp32
    np.testing.assert_array_equal(km.bf16(x32), ref)
    assert km.bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0      # tie to even
    assert km.bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6


@pytest.mark.parametrize("case", ["mha_ragged", "gqa_full", "running_max"])
def test_model_without_rounding_is_the_oracle(case):
    if case == "mha_ragged":
        x, w, eps, scale = synth.layer_inputs(7, 200, 2, 200, 3, 128), 130, 1e-6, None
    elif case == "gqa_full":
        x, w, eps, scale = gqa(18, 1, 160, 4, 2), -1, 1e-6, None
    else:  # logit bound 0.2 * 128 * log2 e = 36.9 > 32: running-max offset
        x, w, eps, scale = synth.layer_inputs(12, 0, 1, 150, 2, 128), 50, 1e-6, 0.2
    m = km.run(x, w, eps, scale, rounding=False)
    r = oracle_run(x, w, eps, scale)
    for n in ("o", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(m[n], r[n], rtol=0, atol=1e-11, err_msg=n)


@pytest.mark.parametrize("T,w", [(129, 64), (640, 256), (300, 255)])
def test_model_error_is_inside_the_edge_bound(T, w):
    x = synth.layer_inputs(7, T, 2, T, 3, 128)
    m, r = km.run(x, w), oracle_run(x, w)
    for n in ("o", "dq", "dk", "dv"):
        err = np.abs(m[n] - r[n])
        assert (err - (MAX_ABS + ULP_SLACK * np.abs(r[n]))).max() <= 0, (n, err.max())
        assert np.linalg.norm(m[n] - r[n]) / np.linalg.norm(r[n]) <= 5e-3, n
        assert err.max() > 1e-3, (n, "the roundings must show")  # the model is not the oracle


def test_saturated_softmax_error_comes_from_delta():
    x = synth.layer_inputs(9, 0, 1, 384, 2, 128)
    x["k"] = synth.peaked_keys(x["q"], 9999)
    w = 64
    r = oracle_run(x, w)
    o_exact, lse = km.forward(x["q"], x["k"], x["v"], w, rounding=False)

    def rel(dq):
        return np.linalg.norm(dq - r["dq"]) / np.linalg.norm(r["dq"])

    full = km.backward(x["q"], x["k"], x["v"], km.bf16(o_exact), x["dO"], lse, w)[0]
    no_delta_rounding = km.backward(x["q"], x["k"], x["v"], o_exact, x["dO"], lse, w)[0]
    only_delta_rounding = km.backward(x["q"], x["k"], x["v"], km.bf16(o_exact), x["dO"], lse, w,
                                      rounding=False)[0]
    assert rel(full) > 0.1 and rel(only_delta_rounding) > 0.1
    assert rel(no_delta_rounding) < 5e-3
    assert abs(rel(full) - rel(only_delta_rounding)) < 0.05 * rel(full)
