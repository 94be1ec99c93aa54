"""GPU parity of the layer's input prologue (gdn_prologue and the decode step
with the prologue fused in) against the fp64 prologue oracle, alone and
followed by the recurrence.

Tolerances:
  * prologue outputs q, k, v (bf16): |got - ref| <= 2^-8 |ref| + 1e-5 rms(ref)
    element by element -- one bf16 rounding (half an ulp is at most 2^-8 of
    the value) of an fp32 result whose own error is a few fp32 ulps;
  * g, beta (fp32): |got - ref| <= 1e-5 |ref| (+ 1e-30);
  * the history ring: bit-exact (it holds bf16 inputs as fp32 values);
  * prologue + prefill: the prefill rule max|got - ref| <= 2e-2 rms(ref),
    with the oracle recurrence run on the oracle prologue's outputs rounded
    to bf16 (round to nearest even), the dtype the prefill takes.  With the
    prologue's output statistics the output is a small difference of larger
    terms: rounding q, k, v to bf16 alone moves the fp64 output by 6-10% of
    its rms, so the fp64 prologue outputs themselves are no fair reference
    for any bf16 prefill;
    The final state after such a prefill is checked against max|S_ref|
    instead: S_T holds the last token's key at first order (beta_T k_T e_T^T),
    so a bf16 rounding of k_T that the fp32 kernel and the fp64 oracle decide
    on opposite sides of a tie moves a row of S_T by beta_T ulp(k) |e_T| --
    measured at 5% of rms(S_T) for one such element, with max|S| ~ 24 rms(S)
    on these statistics.  The chunk kernel's state on shared inputs is held
    to the rms rule by the prefill tests;
  * fused decode (fp32 throughout, no bf16 hand-off): 1e-3 rms(ref), the
    decode rule, against the unrounded oracle prologue.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import prologue as P
from synth import prologue_inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda")


def _dev(x):
    return None if x is None else x.to(DEV)


def _check_bf16(got, ref, name):
    got = got.float().cpu().double().numpy()
    rms = float(np.sqrt(np.mean(ref * ref)))
    bad = np.abs(got - ref) > 2.0 ** -8 * np.abs(ref) + 1e-5 * rms
    assert not bad.any(), f"{name}: {int(bad.sum())} elements out of tolerance, " \
                          f"first at {np.argwhere(bad)[0].tolist()}"


def _check_f32(got, ref, name, rtol=1e-5):
    got = got.cpu().double().numpy()
    bad = np.abs(got - ref) > rtol * np.abs(ref) + 1e-30
    assert not bad.any(), f"{name}: {int(bad.sum())} elements out of tolerance"


def _oracle(x, activation="silu", rows=None):
    sel = slice(None) if rows is None else rows
    ring = None if x["ring"] is None else x["ring"][sel]
    return P.prologue(x["q_raw"][sel], x["k_raw"][sel], x["v_raw"][sel], x["g_raw"][sel],
                      x["beta_raw"][sel], x["conv_w"], ring, x["pos0"][sel].numpy(),
                      activation=activation)


def _err_vs_max(got, ref):
    """max |got - ref| / max |ref| (the end-to-end state rule)."""
    got = np.asarray(got.cpu().double().numpy() if hasattr(got, "cpu") else got, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / np.max(np.abs(ref)))


def _bf16(a):
    """The oracle's fp64 values rounded to bf16 (RN-even), back in fp64."""
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def _gpu_prologue(gdn, x, activation="silu", use_pos=True):
    ring = _dev(x["ring"])
    outs = gdn.prologue(*(_dev(x[n]) for n in ("q_raw", "k_raw", "v_raw", "g_raw", "beta_raw",
                                              "conv_w")),
                        ring, _dev(x["pos0"]) if use_pos else None, activation=activation)
    torch.cuda.synchronize()
    return outs, ring


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_prologue_matches_oracle(gdn, dk, dv, gate):
    # T = 77: two full 32-token tiles and a ragged tail.
    x = prologue_inputs(2, 77, 3, dk, dv, gate=gate, seed=31)
    (q, k, v, g, beta), ring = _gpu_prologue(gdn, x)
    rq, rk, rv, rg, rb, rring = _oracle(x)
    _check_bf16(q, rq, "q")
    _check_bf16(k, rk, "k")
    _check_bf16(v, rv, "v")
    _check_f32(g, rg, "g")
    _check_f32(beta, rb, "beta", rtol=1e-6)
    assert torch.equal(ring.cpu(), torch.from_numpy(rring).float())


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 31, 32, 33])
def test_prologue_short_and_tile_edge_lengths(gdn, T):
    """Lengths below the convolution width (the ring supplies history and is
    only partly overwritten) and around the 32-token tile."""
    x = prologue_inputs(3, T, 2, 128, 128, gate="channel", seed=40 + T)
    (q, k, v, g, beta), ring = _gpu_prologue(gdn, x)
    rq, rk, rv, rg, rb, rring = _oracle(x)
    for got, ref, n in ((q, rq, "q"), (k, rk, "k"), (v, rv, "v")):
        _check_bf16(got, ref, n)
    _check_f32(g, rg, "g")
    assert torch.equal(ring.cpu(), torch.from_numpy(rring).float())


def test_prologue_without_ring_or_positions_and_no_activation(gdn):
    x = prologue_inputs(2, 40, 2, 128, 64, gate="scalar", ring=False, seed=50)
    (q, k, v, g, beta), ring = _gpu_prologue(gdn, x, activation="none", use_pos=False)
    assert ring is None
    x0 = dict(x, pos0=torch.zeros_like(x["pos0"]))
    rq, rk, rv, rg, rb, _ = _oracle(x0, activation="none")
    for got, ref, n in ((q, rq, "q"), (k, rk, "k"), (v, rv, "v")):
        _check_bf16(got, ref, n)
    # no history: token 0's output is tap 3 times its own input
    w3 = x["conv_w"][:, 2 * 128:, 3]
    np.testing.assert_allclose(rv[:, 0], (w3[None] * x["v_raw"][:, 0].float()).double().numpy())


def test_prologue_streaming_matches_one_pass(gdn):
    """Two calls that carry the ring (positions advanced) equal one call."""
    x = prologue_inputs(2, 70, 2, 128, 128, gate="channel", seed=51)
    (q1, k1, v1, g1, b1), _ = _gpu_prologue(gdn, x)
    ring = _dev(x["ring"])
    pos = _dev(x["pos0"])
    parts = []
    for t0, t1 in ((0, 29), (29, 70)):
        sl = {n: _dev(x[n][:, t0:t1].contiguous()) for n in ("q_raw", "k_raw", "v_raw", "g_raw",
                                                            "beta_raw")}
        parts.append(gdn.prologue(sl["q_raw"], sl["k_raw"], sl["v_raw"], sl["g_raw"],
                                  sl["beta_raw"], _dev(x["conv_w"]), ring, pos + t0))
    torch.cuda.synchronize()
    for i, whole in enumerate((q1, k1, v1, g1, b1)):
        assert torch.equal(torch.cat([parts[0][i], parts[1][i]], dim=1), whole), i


@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_prologue_then_prefill_matches_oracle(gdn, gate):
    """gdn_prologue -> gdn_chunk_fwd against the oracle recurrence on the
    oracle prologue's outputs (q, k, v rounded to bf16); 200 tokens: several
    chunks and a ragged tail."""
    x = prologue_inputs(2, 200, 3, 128, 128, gate=gate, seed=52)
    (q, k, v, g, beta), _ = _gpu_prologue(gdn, x)
    out, s_t = gdn.chunk_fwd(q, k, v, g, beta)
    torch.cuda.synchronize()
    rq, rk, rv, rg, rb, _ = _oracle(x)
    ref_o, ref_s = oracle.run(_bf16(rq), _bf16(rk), _bf16(rv), rg, rb,
                              per_channel=gate == "channel")
    assert oracle.rel_err(out.cpu(), ref_o) <= 2e-2
    assert _err_vs_max(s_t, ref_s) <= 2e-2


def _step_inputs(x, t):
    """Token t of prologue_inputs' [B, T, H, ...] tensors, as decode inputs."""
    return [_dev(x[n][:, t].contiguous()) for n in ("q_raw", "k_raw", "v_raw", "g_raw", "beta_raw")]


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_fused_decode_matches_oracle(gdn, dk, dv, gate):
    """Steps of the decode kernel with the prologue fused in, ring and
    positions carried, state in place, against the oracle prologue over the
    same tokens followed by the oracle recurrence."""
    steps = 9
    x = prologue_inputs(3, steps, 2, dk, dv, gate=gate, seed=60)
    s0 = torch.randn(3, 2, dk, dv, generator=torch.Generator().manual_seed(61)) * 0.1
    state = s0.to(DEV)
    ring = _dev(x["ring"])
    pos = _dev(x["pos0"])
    w = _dev(x["conv_w"])
    outs = []
    for t in range(steps):
        outs.append(gdn.recurrent_step_prologue(*_step_inputs(x, t), w, ring, state, pos + t))
    torch.cuda.synchronize()
    got = torch.stack(outs, 1).cpu()                   # [B, steps, H, dv]
    rq, rk, rv, rg, rb, rring = _oracle(x)
    ref_o, ref_s = oracle.run(rq, rk, rv, rg, rb, s0, per_channel=gate == "channel")
    assert oracle.rel_err(got, ref_o) <= 1e-3
    assert oracle.rel_err(state.cpu(), ref_s) <= 1e-3
    assert torch.equal(ring.cpu(), torch.from_numpy(rring).float())


def test_prefill_then_fused_decode_continues_the_sequence(gdn):
    """Prefill of 45 tokens (prologue + chunk), then 6 fused decode steps
    that read the ring the prefill left.  Reference: the oracle prologue over
    all 51 tokens; the oracle recurrence over the first 45 with q, k, v
    rounded to bf16 (the prefill's input dtype), continued over the last 6
    unrounded (the fused step keeps them in fp32)."""
    T0, steps = 45, 6
    x = prologue_inputs(2, T0 + steps, 4, 128, 128, gate="channel", seed=62)
    head = {n: _dev(x[n][:, :T0].contiguous()) for n in ("q_raw", "k_raw", "v_raw", "g_raw",
                                                         "beta_raw")}
    ring = _dev(x["ring"])
    pos = _dev(x["pos0"])
    w = _dev(x["conv_w"])
    q, k, v, g, beta = gdn.prologue(head["q_raw"], head["k_raw"], head["v_raw"], head["g_raw"],
                                    head["beta_raw"], w, ring, pos)
    out0, state = gdn.chunk_fwd(q, k, v, g, beta)
    outs = [gdn.recurrent_step_prologue(*_step_inputs(x, T0 + t), w, ring, state, pos + T0 + t)
            for t in range(steps)]
    torch.cuda.synchronize()
    rq, rk, rv, rg, rb, rring = _oracle(x)
    head_ref = [_bf16(a[:, :T0]) for a in (rq, rk, rv)] + [rg[:, :T0], rb[:, :T0]]
    ref_o0, ref_s0 = oracle.run(*head_ref, per_channel=True)
    ref_o1, ref_s = oracle.run(rq[:, T0:], rk[:, T0:], rv[:, T0:], rg[:, T0:], rb[:, T0:], ref_s0,
                               per_channel=True)
    assert oracle.rel_err(out0.cpu(), ref_o0) <= 2e-2
    assert oracle.rel_err(torch.stack(outs, 1).cpu(), ref_o1) <= 2e-2
    assert _err_vs_max(state, ref_s) <= 2e-2
    assert torch.equal(ring.cpu(), torch.from_numpy(rring).float())


def test_prologue_full_layer_size_sampled_rows(gdn, oracle_threads):
    """The GDN-2 layer shape (B8 H8 T2048 d128, per-channel gate), the launch
    the benchmark times: rows 0 and 7 checked element by element, then the
    prologue -> prefill chain for the same rows against the oracle."""
    x = prologue_inputs(8, 2048, 8, 128, 128, gate="channel", seed=2)
    (q, k, v, g, beta), ring = _gpu_prologue(gdn, x)
    out, s_t = gdn.chunk_fwd(q, k, v, g, beta)
    torch.cuda.synchronize()
    rows = [0, 7]
    rq, rk, rv, rg, rb, rring = _oracle(x, rows=rows)
    _check_bf16(q[rows], rq, "q")
    _check_bf16(k[rows], rk, "k")
    _check_bf16(v[rows], rv, "v")
    _check_f32(g[rows], rg, "g")
    assert torch.equal(ring[rows].cpu(), torch.from_numpy(rring).float())
    ref_o, ref_s = oracle.run(_bf16(rq), _bf16(rk), _bf16(rv), rg, rb, per_channel=True,
                              threads=oracle_threads)
    assert oracle.rel_err(out[rows].cpu(), ref_o) <= 2e-2
    assert _err_vs_max(s_t[rows], ref_s) <= 2e-2


def test_fused_decode_full_batch_sampled_rows(gdn, oracle_threads):
    """The decode shape (B64 H16 d128, per-channel gate), 256 successive fused
    steps, state in place; rows 0 and 63 against the oracle."""
    steps = 256
    x = prologue_inputs(64, steps, 16, 128, 128, gate="channel", seed=4)
    s0 = torch.randn(64, 16, 128, 128, generator=torch.Generator().manual_seed(5)) * 0.1
    state = s0.to(DEV)
    ring = _dev(x["ring"])
    pos = _dev(x["pos0"])
    w = _dev(x["conv_w"])
    dev_in = {n: _dev(x[n]) for n in ("q_raw", "k_raw", "v_raw", "g_raw", "beta_raw")}
    got = torch.empty(64, steps, 16, 128, dtype=torch.float32, device=DEV)
    for t in range(steps):
        got[:, t] = gdn.recurrent_step_prologue(
            *(dev_in[n][:, t].contiguous() for n in ("q_raw", "k_raw", "v_raw", "g_raw", "beta_raw")),
            w, ring, state, pos + t)
    torch.cuda.synchronize()
    rows = [0, 63]
    rq, rk, rv, rg, rb, rring = _oracle(x, rows=rows)
    ref_o, ref_s = oracle.run(rq, rk, rv, rg, rb, s0[rows], per_channel=True,
                              threads=oracle_threads)
    assert oracle.rel_err(got[rows].cpu(), ref_o) <= 1e-3
    assert oracle.rel_err(state[rows].cpu(), ref_s) <= 1e-3
    assert torch.equal(ring[rows].cpu(), torch.from_numpy(rring).float())


# ---- the prefill with the prologue applied while loading (gdn_chunk_fwd_prologue) ----
def _fused(gdn, x, s0=None, activation="silu", use_ring=True, use_pos=True, fused=True):
    ring = _dev(x["ring"]) if use_ring else None
    out, s_t = gdn.chunk_fwd_prologue(
        *(_dev(x[n]) for n in ("q_raw", "k_raw", "v_raw", "g_raw", "beta_raw", "conv_w")),
        ring, _dev(x["pos0"]) if use_pos else None, _dev(s0), activation=activation, fused=fused)
    torch.cuda.synchronize()
    return out, s_t, ring


@pytest.mark.parametrize("route", ["fused", "two_passes"])
@pytest.mark.parametrize("gate", ["channel", "scalar"])
@pytest.mark.parametrize("T", [1, 2, 63, 64, 200, 515])
def test_fused_prologue_prefill_matches_oracle(gdn, gate, T, route):
    """The prologue-plus-prefill call, on either route, against the oracle
    prologue (q, k, v rounded to bf16) followed by the oracle recurrence, with
    a history ring, random positions (the first tokens' convolution reads the
    ring) and S0 != 0; lengths from 1 token to several chunks with a ragged
    tail."""
    x = prologue_inputs(2, T, 3, 128, 128, gate=gate, seed=60 + T)
    s0 = torch.randn(2, 3, 128, 128, generator=torch.Generator().manual_seed(61)) * 0.1
    out, s_t, ring = _fused(gdn, x, s0, fused=route == "fused")
    rq, rk, rv, rg, rb, rring = _oracle(x)
    ref_o, ref_s = oracle.run(_bf16(rq), _bf16(rk), _bf16(rv), rg, rb, s0,
                              per_channel=gate == "channel")
    assert oracle.rel_err(out.cpu(), ref_o) <= 2e-2
    assert _err_vs_max(s_t, ref_s) <= 2e-2
    assert torch.equal(ring.cpu(), torch.from_numpy(rring).float())
    assert gdn.check() == gdn.GDN_OK


@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_fused_prologue_prefill_equals_the_two_passes(gdn, gate):
    """Fused against gdn_prologue then gdn_chunk_fwd on the same inputs: the
    same arithmetic except the order of the q/k sums of squares, which can
    flip the bf16 rounding of a q or k element; the output, a small
    difference of larger terms, then moves by a few 1e-3 of its rms.  Held to
    half the prefill tolerance, as the other cross-form checks."""
    x = prologue_inputs(2, 300, 4, 128, 128, gate=gate, seed=62)
    s0 = torch.randn(2, 4, 128, 128, generator=torch.Generator().manual_seed(63)) * 0.1
    out_f, s_f, ring_f = _fused(gdn, x, s0)
    (q, k, v, g, beta), ring_u = _gpu_prologue(gdn, x)
    out_u, s_u = gdn.chunk_fwd(q, k, v, g, beta, _dev(s0))
    torch.cuda.synchronize()
    assert oracle.rel_err(out_f.cpu(), out_u.cpu().double()) <= 1e-2
    assert _err_vs_max(s_f, s_u.cpu().double().numpy()) <= 1e-2
    assert torch.equal(ring_f.cpu(), ring_u.cpu())


def test_fused_prologue_without_ring_positions_or_activation(gdn):
    x = prologue_inputs(1, 150, 2, 128, 128, gate="channel", ring=False, seed=64)
    out, s_t, _ = _fused(gdn, x, activation="none", use_ring=False, use_pos=False)
    x0 = dict(x)
    x0["pos0"] = torch.zeros_like(x["pos0"])
    rq, rk, rv, rg, rb, _ = _oracle(x0, activation="none")
    ref_o, ref_s = oracle.run(_bf16(rq), _bf16(rk), _bf16(rv), rg, rb, per_channel=True)
    assert oracle.rel_err(out.cpu(), ref_o) <= 2e-2
    assert _err_vs_max(s_t, ref_s) <= 2e-2


def test_fused_prologue_other_shapes_take_the_two_passes(gdn):
    """dk = dv = 64 (not the fused kernel's shape) and a pair count above
    half the SMs run the prologue pass into scratch, then the prefill."""
    for B, T, H, d in ((1, 130, 2, 64), (2, 70, 40, 128)):
        x = prologue_inputs(B, T, H, d, d, gate="scalar", seed=65 + H)
        out, s_t, ring = _fused(gdn, x)
        rq, rk, rv, rg, rb, rring = _oracle(x)
        ref_o, ref_s = oracle.run(_bf16(rq), _bf16(rk), _bf16(rv), rg, rb, per_channel=False)
        assert oracle.rel_err(out.cpu(), ref_o) <= 2e-2, (B, T, H, d)
        assert _err_vs_max(s_t, ref_s) <= 2e-2, (B, T, H, d)
        assert torch.equal(ring.cpu(), torch.from_numpy(rring).float())


@pytest.mark.parametrize("route", ["fused", "two_passes"])
def test_fused_prologue_full_layer_size_sampled_rows(gdn, oracle_threads, route):
    """The GDN-2 layer shape (B8 H8 T2048 d128, per-channel gate) through the
    prologue-plus-prefill call; rows 0 and 7 against the oracle."""
    x = prologue_inputs(8, 2048, 8, 128, 128, gate="channel", seed=2)
    out, s_t, _ = _fused(gdn, x, fused=route == "fused")
    rows = [0, 7]
    rq, rk, rv, rg, rb, _ = _oracle(x, rows=rows)
    ref_o, ref_s = oracle.run(_bf16(rq), _bf16(rk), _bf16(rv), rg, rb, per_channel=True,
                              threads=oracle_threads)
    assert oracle.rel_err(out[rows].cpu(), ref_o) <= 2e-2
    assert _err_vs_max(s_t[rows], ref_s) <= 2e-2


@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_fused_prologue_prefill_is_repeatable(gdn, gate):
    """The fused route twice on the same inputs (the ring restored in
    between): the same bits, outputs, final state and ring alike."""
    x = prologue_inputs(2, 300, 4, 128, 128, gate=gate, seed=66)
    s0 = torch.randn(2, 4, 128, 128, generator=torch.Generator().manual_seed(67)) * 0.1
    runs = [_fused(gdn, x, s0) for _ in range(2)]
    for a, b in zip(runs[0], runs[1]):
        assert torch.equal(a.cpu(), b.cpu())
