"""GPU parity of the prefill gradients (gdn_chunk_bwd) against the fp64
gradient oracle (oracle/backward.py, pinned by finite differences of the
forward oracle).

Tolerance: max|got - ref| <= 1e-3 rms(ref) for every gradient (dq, dk, dv,
dg, dbeta and the initial state's): the kernels compute in fp32 from the
same bf16 / fp32 inputs, so the error is fp32 rounding carried through the
chunk chain -- the decode rule's bound, well above it.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as BW
from synth import grad_inputs, prefill_inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda")
TOL = 1e-3
NAMES = ("dq", "dk", "dv", "dg", "dbeta", "ds0")


def _run(gdn, x, do, dsT):
    d = {n: (None if t is None else t.to(DEV)) for n, t in x.items()}
    r = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["s0"], do.to(DEV),
                      None if dsT is None else dsT.to(DEV))
    torch.cuda.synchronize()
    assert gdn.check() == gdn.GDN_OK
    return {n: t.cpu() for n, t in r.items()}


def _compare(got, ref, where=""):
    for n in NAMES:
        e = oracle.rel_err(got[n], ref[n])
        assert e <= TOL, (where, n, e)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_gradients_match_oracle(gdn, dk, dv, gate):
    """77 tokens: two full 32-token chunks and a ragged one; an initial state
    and a gradient arriving at the final state."""
    x = prefill_inputs(2, 77, 3, dk, dv, gate=gate, s0_std=0.1, seed=80)
    do, dsT = grad_inputs(2, 77, 3, dk, dv, seed=81)
    got = _run(gdn, x, do, dsT)
    ref = BW.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], do, dsT,
                      per_channel=gate == "channel")
    _compare(got, ref)


@pytest.mark.parametrize("T", [1, 5, 31, 32, 33, 64])
def test_gradients_short_and_chunk_edge_lengths(gdn, T):
    x = prefill_inputs(2, T, 2, 128, 128, gate="channel", s0_std=0.1, seed=82 + T)
    do, dsT = grad_inputs(2, T, 2, 128, 128, seed=90 + T)
    got = _run(gdn, x, do, dsT)
    ref = BW.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], do, dsT, per_channel=True)
    _compare(got, ref, T)


def test_no_initial_state_no_final_gradient_and_strong_decay(gdn):
    """state_in = 0 and d_state_out = 0; a scalar gate down to -20 per token
    (any g <= 0 is allowed for it) and g = 0 tokens."""
    x = prefill_inputs(2, 70, 2, 128, 64, gate="scalar", seed=95)
    gen = torch.Generator().manual_seed(96)
    x["g"] = -20.0 * torch.rand(x["g"].shape, generator=gen) * (torch.rand(x["g"].shape, generator=gen) < 0.7)
    do, _ = grad_inputs(2, 70, 2, 128, 64, seed=97, d_state=False)
    got = _run(gdn, x, do, None)
    ref = BW.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], None, do, None, per_channel=False)
    _compare(got, ref)


def test_per_channel_gate_at_its_bound(gdn):
    """Per-channel g = -5 on many channels (the decay factors reach e^-80)."""
    x = prefill_inputs(1, 96, 2, 128, 128, gate="channel", s0_std=0.1, seed=98)
    gen = torch.Generator().manual_seed(99)
    x["g"] = torch.where(torch.rand(x["g"].shape, generator=gen) < 0.5, torch.full_like(x["g"], -5.0), x["g"])
    do, dsT = grad_inputs(1, 96, 2, 128, 128, seed=100)
    got = _run(gdn, x, do, dsT)
    ref = BW.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], do, dsT, per_channel=True)
    _compare(got, ref)


def test_zero_tokens_passes_the_state_gradient_through(gdn):
    x = prefill_inputs(2, 0, 2, 128, 128, gate="channel", s0_std=0.1, seed=101)
    _, dsT = grad_inputs(2, 0, 2, 128, 128, seed=102)
    dq = gdn.chunk_bwd(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), x["g"].to(DEV),
                       x["beta"].to(DEV), x["s0"].to(DEV), torch.empty(2, 0, 2, 128, device=DEV),
                       dsT.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(dq["ds0"].cpu(), dsT)


def test_gdn2_layer_shape_sampled_heads(gdn):
    """The GDN-2 layer shape (B8 H8 T2048 d128, per-channel gate): all
    gradients of two (b, h) pairs against the oracle, run per head."""
    B, T, H = 8, 2048, 8
    x = prefill_inputs(B, T, H, 128, 128, gate="channel", seed=2)
    do, dsT = grad_inputs(B, T, H, 128, 128, seed=103)
    got = _run(gdn, dict(x, s0=None), do, dsT)
    for b, h in ((0, 0), (7, 5)):
        sub = {n: x[n][b:b + 1, :, h:h + 1] for n in ("q", "k", "v", "g", "beta")}
        ref = BW.backward(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], None,
                          do[b:b + 1, :, h:h + 1], dsT[b:b + 1, h:h + 1], per_channel=True)
        sel = {n: got[n][b:b + 1, :, h:h + 1] for n in ("dq", "dk", "dv", "dg", "dbeta")}
        sel["ds0"] = got["ds0"][b:b + 1, h:h + 1]
        _compare(sel, ref, (b, h))
    assert all(np.isfinite(t.numpy()).all() for t in got.values())
