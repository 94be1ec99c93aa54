"""GPU parity of the token-serial fused recurrence against the fp64 oracle:
the decode step (gdn_recurrent_step) and the fp32 / token-serial prefill.

Tolerance rule: max|got - ref| <= tol * rms(ref) over the whole tensor.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import CONFIGS, config_inputs, decode_inputs, prefill_inputs

pytestmark = pytest.mark.gpu


def _decode_run(gdn, x, steps):
    dev = torch.device("cuda")
    state = x["s0"].to(dev).clone()
    q, k, v, g, beta = (x[n].to(dev) for n in ("q", "k", "v", "g", "beta"))
    outs = torch.empty(steps, *x["v"].shape[1:], dtype=torch.float32, device=dev)
    for t in range(steps):
        gdn.recurrent_step(q[t], k[t], v[t], g[t], beta[t], state, out=outs[t])
    torch.cuda.synchronize()
    return outs.cpu(), state.cpu()


@pytest.mark.parametrize("gate", ["channel", "scalar"])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_small(gdn, gate, d):
    x = decode_inputs(3, 5, d, d, 12, gate=gate, seed=11)
    got_o, got_s = _decode_run(gdn, x, 12)
    ref_o, ref_s = oracle.run_steps(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                                    per_channel=gate == "channel")
    assert oracle.rel_err(got_o, ref_o) <= 1e-3
    assert oracle.rel_err(got_s, ref_s) <= 1e-3


def test_decode_mixed_dims_fp32_io(gdn):
    x = decode_inputs(2, 3, 128, 64, 6, gate="channel", io=torch.float32, seed=12)
    got_o, got_s = _decode_run(gdn, x, 6)
    ref_o, ref_s = oracle.run_steps(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                                    per_channel=True)
    assert oracle.rel_err(got_o, ref_o) <= 1e-5
    assert oracle.rel_err(got_s, ref_s) <= 1e-5


def test_decode_full_config(gdn, oracle_threads):
    """B=64 sequences, H=16, d=128, 1024 successive steps, state in place;
    every step's output and the final state within 1e-3 * rms."""
    cfg = CONFIGS[4]
    x = config_inputs(cfg)
    got_o, got_s = _decode_run(gdn, x, cfg.steps)
    ref_o, ref_s = oracle.run_steps(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                                    per_channel=True, threads=oracle_threads)
    for t in (0, 1, cfg.steps // 2, cfg.steps - 1):
        assert oracle.rel_err(got_o[t], ref_o[t]) <= cfg.tol, t
    assert oracle.rel_err(got_o, ref_o) <= cfg.tol
    assert oracle.rel_err(got_s, ref_s) <= cfg.tol


def test_decode_out_of_place_leaves_input(gdn):
    x = decode_inputs(2, 2, 128, 128, 1, gate="scalar", seed=13)
    dev = torch.device("cuda")
    s_in = x["s0"].to(dev)
    s_keep = s_in.clone()
    s_out = torch.empty_like(s_in)
    gdn.recurrent_step(*(x[n][0].to(dev) for n in ("q", "k", "v", "g", "beta")), s_in,
                       state_out=s_out)
    torch.cuda.synchronize()
    assert torch.equal(s_in, s_keep)
    ref_o, ref_s = oracle.run_steps(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                                    per_channel=False)
    assert oracle.rel_err(s_out.cpu(), ref_s) <= 1e-3


def test_prefill_fp32_config1(gdn):
    """Oracle-scale prefill: fp32 I/O, B1 H2 T256 d64, scalar gate, tol 1e-4."""
    cfg = CONFIGS[1]
    x = config_inputs(cfg)
    dev = torch.device("cuda")
    out, s = gdn.chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta")), None)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], None, per_channel=False)
    assert oracle.rel_err(out.cpu(), ref_o) <= cfg.tol
    assert oracle.rel_err(s.cpu(), ref_s) <= cfg.tol


@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_prefill_token_serial_bf16(gdn, gate):
    x = prefill_inputs(2, 77, 3, 128, 128, gate=gate, s0_std=0.1, seed=14)
    dev = torch.device("cuda")
    out, s = gdn.chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta", "s0")),
                           chunk_size=1)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                              per_channel=gate == "channel")
    assert oracle.rel_err(out.cpu(), ref_o) <= 2e-2
    assert oracle.rel_err(s.cpu(), ref_s) <= 1e-3


def test_prefill_zero_length_copies_state(gdn):
    x = prefill_inputs(1, 0, 2, 128, 128, gate="scalar", s0_std=0.1, seed=15)
    dev = torch.device("cuda")
    out, s = gdn.chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta", "s0")))
    torch.cuda.synchronize()
    assert out.numel() == 0
    assert torch.equal(s.cpu(), x["s0"])
    _, s0 = gdn.chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta")), None)
    torch.cuda.synchronize()
    assert float(s0.abs().max()) == 0.0
