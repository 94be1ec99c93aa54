"""GPU parity of the decoupled erase / write form (gdn_recurrent_steps_decoupled)
against its fp64 oracle (oracle/decoupled.py).  The form is a reading of the
pages (no formula is given: parity unpinned as to the form); the arithmetic
of the reading is what is compared.

Tolerance: the decode rule, max|got - ref| <= 1e-3 rms(ref), on the outputs,
the snapshots and the final state (fp32 arithmetic, exact inputs).
"""
import pytest
import torch

import oracle
from oracle import decoupled as DC
from synth import prefill_inputs, write_gate

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda")
TOL = 1e-3


def _run(gdn, x, bw, snapshots=True):
    d = {n: x[n].to(DEV) for n in ("q", "k", "v", "g", "beta", "s0")}
    state = d["s0"].clone()
    out, snap = gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], state, state_out=state,
                                    snapshots=snapshots, beta_write=bw.to(DEV))
    torch.cuda.synchronize()
    return out.cpu(), None if snap is None else snap.cpu(), state.cpu()


@pytest.mark.parametrize("T", [1, 6, 150])
@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_decoupled_matches_oracle(gdn, gate, T):
    """One decode token, six draft tokens with snapshots, and a 150-token
    token-serial prefill."""
    x = prefill_inputs(2, T, 3, 128, 128, gate=gate, s0_std=0.1, seed=110 + T)
    bw = write_gate(2, T, 3, seed=111 + T)
    out, snap, state = _run(gdn, x, bw, snapshots=True if T <= 6 else None)
    pc = gate == "channel"
    ref_o, ref_s = DC.run(x["q"], x["k"], x["v"], x["g"], x["beta"], bw, x["s0"], per_channel=pc)
    assert oracle.rel_err(out, ref_o) <= TOL
    assert oracle.rel_err(state, ref_s) <= TOL
    if snap is not None:
        for t in range(T):
            _, ref_t = DC.run(x["q"][:, :t + 1], x["k"][:, :t + 1], x["v"][:, :t + 1],
                              x["g"][:, :t + 1], x["beta"][:, :t + 1], bw[:, :t + 1], x["s0"],
                              per_channel=pc)
            assert oracle.rel_err(snap[:, t], ref_t) <= TOL, t


def test_equal_gates_match_the_coupled_kernel(gdn):
    x = prefill_inputs(3, 5, 2, 64, 128, gate="channel", s0_std=0.1, seed=120)
    out_d, _, s_d = _run(gdn, x, x["beta"].clone(), snapshots=None)
    d = {n: x[n].to(DEV) for n in ("q", "k", "v", "g", "beta", "s0")}
    state = d["s0"].clone()
    out_c, _ = gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], state, state_out=state,
                                   snapshots=None)
    torch.cuda.synchronize()
    assert oracle.rel_err(out_d, out_c.cpu()) <= 1e-5
    assert oracle.rel_err(s_d, state.cpu()) <= 1e-5


def test_decoupled_decode_shape_sampled_rows(gdn, oracle_threads):
    """B64 H16 d128, per-channel gate, 4 tokens: rows 0 and 63."""
    B, T, H = 64, 4, 16
    x = prefill_inputs(B, T, H, 128, 128, gate="channel", s0_std=0.1, seed=121)
    bw = write_gate(B, T, H, seed=122)
    out, snap, state = _run(gdn, x, bw)
    rows = [0, 63]
    sub = {n: x[n][rows] for n in ("q", "k", "v", "g", "beta", "s0")}
    ref_o, ref_s = DC.run(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], bw[rows], sub["s0"],
                          per_channel=True)
    assert oracle.rel_err(out[rows], ref_o) <= TOL
    assert oracle.rel_err(state[rows], ref_s) <= TOL
    assert oracle.rel_err(snap[rows, T - 1], ref_s) <= TOL
