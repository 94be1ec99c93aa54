"""GPU parity of the segment-parallel long-sequence path (gdn_chunk_fwd_segments):
per-segment zero-start states and transitions, serial combine, second pass.

The state map of a stretch of tokens is affine in the start state (formula of
the Atomic-GDN2 model card, section 2.1), so any segmentation must give the
token-serial result; checked against the fp64 oracle and against the
unsegmented chunk path.
"""
import pytest
import torch

import oracle
from synth import CONFIGS, config_inputs, prefill_inputs

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _run(gdn, x, segments, state_out=None):
    dev = torch.device("cuda")
    args = [x[n].to(dev) for n in ("q", "k", "v", "g", "beta")]
    s0 = x["s0"].to(dev) if x["s0"] is not None else None
    out, s = gdn.chunk_fwd(*args, s0, segments=segments, state_out=state_out)
    torch.cuda.synchronize()
    return out.cpu(), s.cpu()


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("segments", [2, 3, 5, 16])
def test_segments_match_oracle_and_unsegmented(gdn, gate, segments):
    x = prefill_inputs(1, 1000, 2, 128, 128, gate=gate, s0_std=0.1, seed=300 + segments)
    o_seg, s_seg = _run(gdn, x, segments)
    o_one, s_one = _run(gdn, x, 1)
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                              per_channel=gate == "channel")
    assert oracle.rel_err(o_seg, ref_o) <= TOL
    assert oracle.rel_err(s_seg, ref_s) <= TOL
    assert oracle.rel_err(o_seg, o_one.double()) <= TOL / 2
    assert oracle.rel_err(s_seg, s_one.double()) <= TOL / 2


def test_segments_zero_initial_state_and_batch(gdn):
    x = prefill_inputs(2, 640, 3, 128, 128, gate="channel", seed=310)
    o_seg, s_seg = _run(gdn, x, 4)
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], None, per_channel=True)
    assert oracle.rel_err(o_seg, ref_o) <= TOL
    assert oracle.rel_err(s_seg, ref_s) <= TOL


def test_segments_in_place_state(gdn):
    x = prefill_inputs(1, 700, 2, 128, 128, gate="scalar", s0_std=0.1, seed=311)
    dev = torch.device("cuda")
    st = x["s0"].to(dev).clone()
    out, _ = gdn.chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta")), st,
                           state_out=st, segments=3)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], per_channel=False)
    assert oracle.rel_err(out.cpu(), ref_o) <= TOL
    assert oracle.rel_err(st.cpu(), ref_s) <= TOL


def test_segments_more_than_chunks_is_capped(gdn):
    x = prefill_inputs(1, 130, 1, 128, 128, gate="channel", s0_std=0.1, seed=312)
    o_seg, s_seg = _run(gdn, x, 50)          # 3 chunks: capped at 3 segments
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], per_channel=True)
    assert oracle.rel_err(o_seg, ref_o) <= TOL
    assert oracle.rel_err(s_seg, ref_s) <= TOL


def test_long_context_config_every_head(gdn, oracle_threads):
    """B=1, H=16, T=262,144, scalar gate with 10% g = 0; the default entry point
    (automatic segmentation, 9 segments per head).  Every head against the
    oracle, each held to the rule on its own (the oracle runs 8 heads at a
    time to bound its fp64 copies at about 9 GB)."""
    cfg = CONFIGS[5]
    x = config_inputs(cfg)
    dev = torch.device("cuda")
    out, s = gdn.chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta")), None)
    torch.cuda.synchronize()
    out, s = out.cpu(), s.cpu()
    for h0 in range(0, cfg.H, 8):
        sl = {n: x[n][:, :, h0:h0 + 8].contiguous() for n in ("q", "k", "v", "g", "beta")}
        ref_o, ref_s = oracle.run(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], None,
                                  per_channel=False, threads=oracle_threads)
        for j in range(8):
            eo = oracle.rel_err(out[:, :, h0 + j], ref_o[:, :, j])
            es = oracle.rel_err(s[:, h0 + j], ref_s[:, j])
            assert eo <= cfg.tol and es <= cfg.tol, (h0 + j, eo, es)
        del ref_o, ref_s, sl


@pytest.mark.parametrize("pattern", ["floor", "runs"])
def test_segments_channel_gate_at_its_bound(gdn, pattern):
    """Per-channel g at -5 (every token, or runs mixed with g = 0 inside a
    chunk): the transitions of the segments decay to (near) zero and the
    factored decay works at the edge of its range."""
    from tests.test_gpu_chunk import _gate_at_bound
    x = _gate_at_bound(prefill_inputs(1, 900, 2, 128, 128, gate="channel", s0_std=0.1, seed=320),
                       pattern)
    o_seg, s_seg = _run(gdn, x, 3)
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], per_channel=True)
    assert torch.isfinite(o_seg).all() and torch.isfinite(s_seg).all()
    assert oracle.rel_err(o_seg, ref_o) <= TOL
    assert oracle.rel_err(s_seg, ref_s) <= TOL


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_segments_without_decay_run_full_transitions(gdn, gate):
    """g = 0 and a small beta: the transition of a segment barely decays, so
    no transition may end early; the segmented result must still be exact."""
    x = prefill_inputs(1, 1200, 2, 128, 128, gate=gate, s0_std=0.1, seed=330)
    x["g"].zero_()
    x["beta"] = (0.02 * x["beta"]).contiguous()
    o_seg, s_seg = _run(gdn, x, 4)
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                              per_channel=gate == "channel")
    assert oracle.rel_err(o_seg, ref_o) <= TOL
    assert oracle.rel_err(s_seg, ref_s) <= TOL


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("late", ["beta_above_one", "positive_g"])
def test_segments_with_tokens_outside_the_contracting_domain(gdn, gate, late):
    """Fast decay first (the transitions would end after a chunk or two),
    then tokens outside the domain that makes every step a contraction
    (beta > 1, or g > 0 -- in one channel of a per-channel gate): the early
    end must not be taken, and the result must match the oracle."""
    x = prefill_inputs(1, 1024, 2, 128, 128, gate=gate, s0_std=0.1, seed=331)
    g, beta = x["g"].clone(), x["beta"].clone()
    g[...] = -3.0
    if late == "beta_above_one":
        beta[:, 600:610] = 1.8
    elif gate == "scalar":
        g[:, 600:610] = 0.05
    else:
        g[:, 600:610, :, 77] = 0.05
    x["g"], x["beta"] = g.contiguous(), beta.contiguous()
    o_seg, s_seg = _run(gdn, x, 3)
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                              per_channel=gate == "channel")
    assert oracle.rel_err(o_seg, ref_o) <= TOL
    assert oracle.rel_err(s_seg, ref_s) <= TOL


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("what", ["beta", "g"])
def test_segments_outside_the_domain_in_a_chunk_they_run(gdn, gate, what):
    """A token outside the domain inside the first chunk of every segment
    (token 5 of each: beta = 2.5, so beta |k|^2 > 2, or g = +0.05 -- in one
    channel of a per-channel gate), where the transition runs rather than
    skips it: the in-kernel checks on run tokens must keep the transitions
    in full."""
    x = prefill_inputs(1, 960, 2, 128, 128, gate=gate, s0_std=0.1, seed=332)
    beta, g = x["beta"].clone(), x["g"].clone()
    for t in (5, 325, 645):                   # 3 segments of 320 tokens
        if what == "beta":
            beta[:, t] = 2.5
        elif gate == "scalar":
            g[:, t] = 0.05
        else:
            g[:, t, :, 77] = 0.05
    x["beta"], x["g"] = beta.contiguous(), g.contiguous()
    o_seg, s_seg = _run(gdn, x, 3)
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                              per_channel=gate == "channel")
    assert oracle.rel_err(o_seg, ref_o) <= TOL
    assert oracle.rel_err(s_seg, ref_s) <= TOL
