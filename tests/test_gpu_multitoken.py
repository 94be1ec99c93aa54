"""GPU parity of the multi-token decode step (gdn_recurrent_steps: T draft
tokens per sequence with the state after every token kept) and of the
commit of an accepted prefix (gdn_state_select), against the fp64 oracle.

Tolerance: the decode rule, max|got - ref| <= 1e-3 rms(ref), for the outputs,
every snapshot and the final state; the snapshot after token t is compared
with the oracle run over the first t + 1 tokens.  Equality with T single
decode steps and the selection itself are bit-exact (same arithmetic in the
same order; a copy).
"""
import numpy as np
import pytest
import torch

import oracle
from synth import prefill_inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda")
TOL = 1e-3


def _dev(x):
    return {n: (None if t is None else t.to(DEV)) for n, t in x.items()}


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_steps_and_snapshots_match_oracle(gdn, dk, dv, gate):
    T = 5
    x = prefill_inputs(2, T, 3, dk, dv, gate=gate, s0_std=0.1, seed=70)
    d = _dev(x)
    state = d["s0"].clone()
    out, snap = gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], state,
                                    state_out=state)
    torch.cuda.synchronize()
    pc = gate == "channel"
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], per_channel=pc)
    assert oracle.rel_err(out.cpu(), ref_o) <= TOL
    assert oracle.rel_err(state.cpu(), ref_s) <= TOL
    for t in range(T):
        _, ref_t = oracle.run(x["q"][:, :t + 1], x["k"][:, :t + 1], x["v"][:, :t + 1],
                              x["g"][:, :t + 1], x["beta"][:, :t + 1], x["s0"], per_channel=pc)
        assert oracle.rel_err(snap[:, t].cpu(), ref_t) <= TOL, t
    assert torch.equal(snap[:, T - 1], state)


def test_steps_equal_single_decode_steps_bitwise(gdn):
    """The decode shape (B64 H16 d128, per-channel gate), 4 draft tokens: the
    same kernel tiling as the single step, so every result is identical."""
    B, T, H = 64, 4, 16
    x = prefill_inputs(B, T, H, 128, 128, gate="channel", s0_std=0.1, seed=71)
    d = _dev(x)
    out, snap = gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], d["s0"])
    state = d["s0"].clone()
    for t in range(T):
        o = gdn.recurrent_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                               d["v"][:, t].contiguous(), d["g"][:, t].contiguous(),
                               d["beta"][:, t].contiguous(), state)
        assert torch.equal(o, out[:, t]), t
        assert torch.equal(state, snap[:, t]), t
    assert torch.equal(d["s0"].cpu(), x["s0"])     # state_in read only without state_out


def test_state_select_commits_accepted_prefix(gdn):
    B, T, H = 6, 4, 2
    x = prefill_inputs(B, T, H, 128, 64, gate="scalar", s0_std=0.1, seed=72)
    d = _dev(x)
    _, snap = gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], d["s0"])
    nacc = torch.tensor([1, 4, 0, 2, 5, -1], dtype=torch.int32, device=DEV)
    state = torch.full_like(d["s0"], 7.0)
    gdn.state_select(snap, nacc, state)
    torch.cuda.synchronize()
    for b, n in enumerate(nacc.tolist()):
        if 1 <= n <= T:
            assert torch.equal(state[b], snap[b, n - 1]), b
        else:
            assert bool((state[b] == 7.0).all()), b          # count out of 1..T: untouched
    _, ref_s = oracle.run(x["q"][:, :2], x["k"][:, :2], x["v"][:, :2], x["g"][:, :2],
                          x["beta"][:, :2], x["s0"], per_channel=False)
    assert oracle.rel_err(state[3].cpu(), ref_s[3]) <= TOL


def test_steps_without_snapshots_in_place(gdn):
    x = prefill_inputs(3, 7, 2, 128, 128, gate="channel", s0_std=0.1, seed=73)
    d = _dev(x)
    state = d["s0"].clone()
    out, snap = gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], state,
                                    state_out=state, snapshots=None)
    torch.cuda.synchronize()
    assert snap is None
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"], per_channel=True)
    assert oracle.rel_err(out.cpu(), ref_o) <= TOL
    assert oracle.rel_err(state.cpu(), ref_s) <= TOL


def test_steps_decode_shape_sampled_rows(gdn, oracle_threads):
    """B64 H16 d128, per-channel gate, 8 draft tokens with snapshots: rows 0
    and 63 against the oracle (outputs, snapshots after tokens 1, 4 and 8)."""
    B, T, H = 64, 8, 16
    x = prefill_inputs(B, T, H, 128, 128, gate="channel", s0_std=0.1, seed=74)
    d = _dev(x)
    out, snap = gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], d["s0"])
    torch.cuda.synchronize()
    rows = [0, 63]
    sub = {n: x[n][rows] for n in ("q", "k", "v", "g", "beta", "s0")}
    ref_o, _ = oracle.run(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], sub["s0"],
                          per_channel=True, threads=oracle_threads)
    assert oracle.rel_err(out[rows].cpu(), ref_o) <= TOL
    for t in (0, 3, 7):
        _, ref_t = oracle.run(sub["q"][:, :t + 1], sub["k"][:, :t + 1], sub["v"][:, :t + 1],
                              sub["g"][:, :t + 1], sub["beta"][:, :t + 1], sub["s0"],
                              per_channel=True, threads=oracle_threads)
        assert oracle.rel_err(snap[rows, t].cpu(), ref_t) <= TOL, t
    assert np.isfinite(snap.cpu().numpy()).all()
