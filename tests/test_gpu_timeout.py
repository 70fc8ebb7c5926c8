"""Failure detection on the GPU: a device-side wait that runs out.

Every wait inside the kernels is bounded (by default 2 s of %globaltimer);
one that runs out makes its CTA abandon the work, let the copies and
tensor-core operations it started finish, free its tensor memory and exit,
and sets a status word that ar_attn_sync_status reports as AR_ERR_TIMEOUT.
The pages handle failures at the level of whole runs (the "autoresearch"
README (gitee), section 6.3: a run past its time budget is killed and logged
as a crash); this is the same idea for one call: nothing waits forever.

The test shortens the limit to 1 ns, so that waits which are not satisfied at
once run out during a normal forward and backward (nothing is broken: the
waits are the kernels' ordinary ones), checks that both calls report the
timeout, restores the default, and checks that the next calls on the same
context give exactly the results of a call made before the timeout.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from sliding_window_attention_rmsnorm_b200 import attn, build, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    attn.lib()


def _expect_timeout():
    with pytest.raises(attn.ArAttnError) as e:
        attn.sync_status()
    assert e.value.status == -8, e.value


def test_short_wait_limit_times_out_and_the_next_call_is_correct():
    # B=8, T=2048, H=4, window 1024: several units per CTA, so some waits span
    # whole units (tens of microseconds)
    B, T, H, w = 8, 2048, 4, 1024
    x = synth.layer_inputs(2, 0, B, T, H, 128)
    q, k, v, dO = (x[r].cuda() for r in ("q", "k", "v", "dO"))
    o_ref, lse_ref = attn.fwd(q, k, v, w)
    g_ref = attn.bwd(q, k, v, o_ref, dO, lse_ref, w)
    attn.sync_status()
    try:
        attn.set_wait_limit_ns(1)
        o_bad, lse_bad = attn.fwd(q, k, v, w)
        _expect_timeout()
        attn.bwd(q, k, v, o_ref, dO, lse_ref, w)
        _expect_timeout()
    finally:
        attn.set_wait_limit_ns(0)
    o, lse = attn.fwd(q, k, v, w)
    g = attn.bwd(q, k, v, o, dO, lse, w)
    attn.sync_status()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    for a, b in zip(g, g_ref):
        assert torch.equal(a, b)
    # and that result is the right one (one head against the oracle)
    head = 5
    b, h = divmod(head, H)
    ro, rl = orc.attn_fwd(x["q"], x["k"], x["v"], w, heads=[head])
    rg = orc.attn_bwd(x["q"], x["k"], x["v"], x["dO"], w, heads=[head])
    for got, ref in ((o, ro), (g[0], rg["dq"]), (g[1], rg["dk"]), (g[2], rg["dv"])):
        a = got[b, :, h].float().cpu().numpy().astype(np.float64)
        r = ref[b, :, h]
        assert np.abs(a - r).max() <= 2e-2 and np.linalg.norm(a - r) / np.linalg.norm(r) <= 5e-3
    assert np.abs(lse[b, h].cpu().numpy() - rl[b, h]).max() <= 1e-3
