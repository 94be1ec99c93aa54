"""GPU parity of the chunkwise tensor-core prefill (gdn_chunk_fwd, bf16 I/O,
dk = dv = 128) against the fp64 oracle.

Tolerance rule: max|got - ref| <= tol * rms(ref), tol = 2e-2 for bf16 I/O.
Full-size workloads are checked pair by pair: every (b, h) pair is held to
the rule on its own (the oracle computes pairs independently).
"""
import numpy as np
import pytest
import torch

import oracle
from synth import CONFIGS, config_inputs, prefill_inputs

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _gpu(gdn, x, chunk_size=0, with_s0=True):
    dev = torch.device("cuda")
    args = [x[n].to(dev) for n in ("q", "k", "v", "g", "beta")]
    s0 = x["s0"].to(dev) if (with_s0 and x["s0"] is not None) else None
    out, s = gdn.chunk_fwd(*args, s0, chunk_size=chunk_size)
    torch.cuda.synchronize()
    return out.float().cpu(), s.cpu()


def _ref(x, per_channel, heads=None, with_s0=True):
    s0 = x["s0"] if with_s0 else None
    return oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], s0, per_channel=per_channel,
                      heads=heads)


def _pairs(x, heads):
    H = x["q"].shape[2]
    return [divmod(bh, H) for bh in heads]


def _check_pairs(got_o, got_s, ref_o, ref_s, pairs, tol=TOL):
    for b, h in pairs:
        eo = oracle.rel_err(got_o[b, :, h], ref_o[b, :, h])
        es = oracle.rel_err(got_s[b, h], ref_s[b, h])
        assert eo <= tol and es <= tol, f"(b={b}, h={h}): out {eo:.3e} state {es:.3e}"


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 150, 256])
def test_small_shapes(gdn, gate, T):
    x = prefill_inputs(2, T, 3, 128, 128, gate=gate, s0_std=0.1, seed=200 + T)
    got_o, got_s = _gpu(gdn, x)
    ref_o, ref_s = _ref(x, gate == "channel")
    assert oracle.rel_err(got_o, ref_o) <= TOL
    assert oracle.rel_err(got_s, ref_s) <= TOL


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_zero_initial_state_and_no_state_out(gdn, gate):
    x = prefill_inputs(1, 200, 2, 128, 128, gate=gate, seed=210)
    dev = torch.device("cuda")
    out, s = gdn.chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta")), None,
                           return_state=False)
    torch.cuda.synchronize()
    assert s is None
    ref_o, _ = _ref(x, gate == "channel")
    assert oracle.rel_err(out.float().cpu(), ref_o) <= TOL


def test_in_place_state(gdn):
    x = prefill_inputs(2, 130, 2, 128, 128, gate="channel", s0_std=0.1, seed=211)
    dev = torch.device("cuda")
    st = x["s0"].to(dev).clone()
    out, s = gdn.chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta")), st, state_out=st)
    torch.cuda.synchronize()
    ref_o, ref_s = _ref(x, True)
    assert s.data_ptr() == st.data_ptr()
    assert oracle.rel_err(out.float().cpu(), ref_o) <= TOL
    assert oracle.rel_err(st.cpu(), ref_s) <= TOL


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_chunk_size_independence(gdn, gate):
    """Chunked (C = 64) and token-serial (C = 1) agree within tol/2 of each
    other and each within tol of the oracle."""
    x = prefill_inputs(2, 300, 2, 128, 128, gate=gate, s0_std=0.1, seed=212)
    o64, s64 = _gpu(gdn, x, chunk_size=64)
    o1, s1 = _gpu(gdn, x, chunk_size=1)
    ref_o, ref_s = _ref(x, gate == "channel")
    assert oracle.rel_err(o64, ref_o) <= TOL and oracle.rel_err(o1, ref_o) <= TOL
    assert oracle.rel_err(o64, o1.double()) <= TOL / 2
    assert oracle.rel_err(s64, s1.double()) <= TOL / 2


def test_channel_gate_equal_channels_equals_scalar(gdn):
    x = prefill_inputs(1, 192, 2, 128, 128, gate="scalar", s0_std=0.1, seed=213)
    xc = dict(x)
    xc["g"] = x["g"][..., None].expand(*x["g"].shape, 128).contiguous()
    o_s, s_s = _gpu(gdn, x)
    o_c, s_c = _gpu(gdn, xc)
    assert oracle.rel_err(o_c, o_s.double()) <= TOL / 2
    assert oracle.rel_err(s_c, s_s.double()) <= TOL / 2


def test_frozen_state_special_case(gdn):
    """beta = 0 and g = 0: the state is unchanged and o_t = S0^T q_t."""
    x = prefill_inputs(1, 100, 2, 128, 128, gate="channel", s0_std=0.1, seed=214)
    x["beta"].zero_()
    x["g"].zero_()
    got_o, got_s = _gpu(gdn, x)
    ref = torch.einsum("bhij,bthi->bthj", x["s0"].double(), x["q"].double())
    assert oracle.rel_err(got_o, ref) <= TOL
    assert oracle.rel_err(got_s, x["s0"].double()) <= 1e-2


def test_split_sequence_carries_state(gdn):
    x = prefill_inputs(1, 256, 2, 128, 128, gate="channel", s0_std=0.1, seed=215)
    o_all, s_all = _gpu(gdn, x)
    a = {n: (x[n][:, :100].contiguous() if n != "s0" else x[n]) for n in x}
    o1, s1 = _gpu(gdn, a)
    bpart = {n: (x[n][:, 100:].contiguous() if n != "s0" else s1) for n in x}
    o2, s2 = _gpu(gdn, bpart)
    assert oracle.rel_err(torch.cat([o1, o2], 1), o_all.double()) <= TOL / 2
    assert oracle.rel_err(s2, s_all.double()) <= TOL / 2


def test_prefill_equals_decode_steps(gdn):
    x = prefill_inputs(2, 70, 2, 128, 128, gate="channel", s0_std=0.1, seed=216)
    o_p, s_p = _gpu(gdn, x)
    dev = torch.device("cuda")
    st = x["s0"].to(dev).clone()
    outs = []
    for t in range(70):
        outs.append(gdn.recurrent_step(*(x[n][:, t].contiguous().to(dev)
                                         for n in ("q", "k", "v", "g", "beta")), st))
    torch.cuda.synchronize()
    o_d = torch.stack(outs, 1).cpu()
    assert oracle.rel_err(o_p, o_d.double()) <= TOL
    assert oracle.rel_err(s_p, st.cpu().double()) <= TOL


@pytest.mark.parametrize("index", [2, 3])
def test_full_config_every_pair(gdn, index, oracle_threads):
    """The GDN-2 layer workload (64 pairs, per-channel gate, prep pool) and the
    scalar training workload (48 pairs, S0 != 0, segment path): every (b, h)
    pair against the oracle, each held to the rule on its own."""
    cfg = CONFIGS[index]
    x = config_inputs(cfg)
    got_o, got_s = _gpu(gdn, x)
    BH = cfg.B * cfg.H
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                              per_channel=cfg.per_channel, threads=oracle_threads)
    _check_pairs(got_o, got_s, ref_o, ref_s, _pairs(x, range(BH)), cfg.tol)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("T", [50, 64, 200, 700])
def test_single_cta_pair_and_pool_kernels_agree(gdn, gate, T, monkeypatch):
    """The one-CTA kernel, the two-CTA cluster kernel (chunk-local work on one
    SM, state chain on the other) and the prep-pool kernel (chains fed by
    prep CTAs on every other SM through a global slot buffer) compute the same
    chunk algebra.  With 4 pairs and few chunks, most prep CTAs of the pool
    get no task at all.  The forms do not share an arithmetic order (the
    gate's prefix sums, T' = T Diag(beta) formed on different sides, the
    one-CTA kernel's U from Z = V - Y), so a bf16 operand can round the other
    way and they agree to the bf16 operands' error (tol / 2), not bit for bit;
    each form on its own is bit-for-bit repeatable (test_every_form_is_repeatable)."""
    x = prefill_inputs(2, T, 2, 128, 128, gate=gate, s0_std=0.1, seed=230 + T)
    got = {}
    for kernel in ("single", "pair", "pool"):
        monkeypatch.setenv("GDN_CHUNK_KERNEL", kernel)
        got[kernel] = _gpu(gdn, x)
    ref_o, ref_s = _ref(x, gate == "channel")
    for o, s in got.values():
        assert oracle.rel_err(o, ref_o) <= TOL and oracle.rel_err(s, ref_s) <= TOL
    o1, s1 = got["single"]
    for kernel in ("pair", "pool"):
        o2, s2 = got[kernel]
        assert oracle.rel_err(o2, o1.double()) <= TOL / 2, kernel
        assert oracle.rel_err(s2, s1.double()) <= TOL / 2, kernel
    assert gdn.check() == gdn.GDN_OK


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("B,H,T", [(2, 37, 300), (3, 5, 1000), (1, 1, 129)])
def test_pool_kernel_pair_counts(gdn, gate, B, H, T, monkeypatch):
    """Pool form at B*H = 74 (as many chains as prep CTAs on 148 SMs), at an
    odd pair count with many chunks per prep CTA, and with one pair: sampled
    pairs against the oracle, all pairs against the cluster kernel.  The two
    forms run the same products, but the gate's prefix sums are summed in
    another fp32 order, and a bf16 operand (K*E) can round the other way, so
    they agree to the bf16 operands' error, not bit for bit."""
    x = prefill_inputs(B, T, H, 128, 128, gate=gate, s0_std=0.1, seed=250 + B * H)
    monkeypatch.setenv("GDN_CHUNK_KERNEL", "pool")
    o_pool, s_pool = _gpu(gdn, x)
    monkeypatch.setenv("GDN_CHUNK_KERNEL", "pair")
    o_pair, s_pair = _gpu(gdn, x)
    BH = B * H
    heads = sorted({0, BH // 2, BH - 1})
    ref_o, ref_s = _ref(x, gate == "channel", heads=heads)
    _check_pairs(o_pool, s_pool, ref_o, ref_s, _pairs(x, heads))
    assert oracle.rel_err(o_pool, o_pair.double()) <= TOL / 2
    assert oracle.rel_err(s_pool, s_pair.double()) <= TOL / 2
    assert gdn.check() == gdn.GDN_OK


@pytest.mark.parametrize("kernel", ["single", "pair", "pool"])
def test_scalar_gate_beyond_the_bounded_domain(gdn, kernel, monkeypatch):
    """The scalar gate accepts any g <= 0: chunks whose total decay exceeds the
    range of the factored form take exact per-element exponentials."""
    x = prefill_inputs(1, 256, 2, 128, 128, gate="scalar", s0_std=0.1, seed=240)
    gen = torch.Generator().manual_seed(241)
    strong = -30.0 * torch.rand(x["g"].shape, generator=gen)
    x["g"] = torch.where(torch.arange(256)[None, :, None] < 128, strong, x["g"]).contiguous()
    monkeypatch.setenv("GDN_CHUNK_KERNEL", kernel)
    got_o, got_s = _gpu(gdn, x)
    ref_o, ref_s = _ref(x, False)
    assert oracle.rel_err(got_o, ref_o) <= TOL
    assert oracle.rel_err(got_s, ref_s) <= TOL


def _gate_at_bound(x, pattern):
    """Per-channel g at the edge of its domain [-5, 0] (model card, section 2.1:
    g = -min(softplus(.), 160 / bs2), bs2 = 32).  "floor": g = -5 on every token
    and channel, so a 64-token chunk decays by exp(-320) and every factor of
    the factored decay sits at exp(+-80) or below.  "runs": runs of 7 tokens
    alternate between -5 and 0, shifted per channel, so one chunk mixes full
    decay and no decay; channels 0-7 stay at -5 and channels 8-15 at 0."""
    B, T, H, dk = x["g"].shape
    if pattern == "floor":
        g = torch.full((B, T, H, dk), -5.0)
    else:
        t = torch.arange(T)[:, None]
        c = torch.arange(dk)[None, :]
        g = torch.where(((t // 7) + c) % 2 == 0, -5.0, 0.0)
        g[:, 0:8] = -5.0
        g[:, 8:16] = 0.0
        g = g[None, :, None, :].expand(B, T, H, dk)
    x["g"] = g.contiguous().float()
    return x


@pytest.mark.parametrize("kernel", ["single", "pair", "pool"])
@pytest.mark.parametrize("pattern", ["floor", "runs"])
def test_channel_gate_at_its_bound(gdn, kernel, pattern, monkeypatch):
    x = _gate_at_bound(prefill_inputs(2, 300, 2, 128, 128, gate="channel", s0_std=0.1, seed=260),
                       pattern)
    monkeypatch.setenv("GDN_CHUNK_KERNEL", kernel)
    got_o, got_s = _gpu(gdn, x)
    ref_o, ref_s = _ref(x, True)
    assert torch.isfinite(got_o).all() and torch.isfinite(got_s).all()
    assert oracle.rel_err(got_o, ref_o) <= TOL
    assert oracle.rel_err(got_s, ref_s) <= TOL
    assert gdn.check() == gdn.GDN_OK


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_second_device_in_the_same_process(gdn, gate):
    """Kernel attributes (the shared-memory limit) and the SM count belong to a
    device: a call on cuda:1 after one on cuda:0 in the same process must not
    rely on settings made while cuda:0 was current."""
    if torch.cuda.device_count() < 2:
        pytest.skip("one GPU visible")
    x = prefill_inputs(2, 300, 3, 128, 128, gate=gate, s0_std=0.1, seed=270)
    ref_o, ref_s = _ref(x, gate == "channel")
    for dev_index in (0, 1):
        dev = torch.device("cuda", dev_index)
        with torch.cuda.device(dev):
            args = [x[n].to(dev) for n in ("q", "k", "v", "g", "beta")]
            out, s = gdn.chunk_fwd(*args, x["s0"].to(dev))
            torch.cuda.synchronize(dev)
            assert oracle.rel_err(out.cpu(), ref_o) <= TOL, dev_index
            assert oracle.rel_err(s.cpu(), ref_s) <= TOL, dev_index
            assert gdn.check() == gdn.GDN_OK


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("form", ["single", "pair", "pool", "segments"])
def test_every_form_is_repeatable(gdn, gate, form, monkeypatch):
    """Two calls on the same inputs give the same bits, in every form of the
    prefill (no form reads a record, a slot or a staged tile before it is
    complete, and no reduction depends on timing).  A race between a producer
    and its consumer shows up here as a difference."""
    x = prefill_inputs(2, 700, 3, 128, 128, gate=gate, s0_std=0.1, seed=270)
    dev = torch.device("cuda")
    args = [x[n].to(dev) for n in ("q", "k", "v", "g", "beta")]
    s0 = x["s0"].to(dev)
    if form != "segments":
        monkeypatch.setenv("GDN_CHUNK_KERNEL", form)
    seg = 3 if form == "segments" else 1
    runs = []
    for _ in range(3):
        out, s = gdn.chunk_fwd(*args, s0, segments=seg)
        torch.cuda.synchronize()
        runs.append((out.cpu(), s.cpu()))
    assert gdn.check() == gdn.GDN_OK
    for out, s in runs[1:]:
        assert torch.equal(out, runs[0][0]) and torch.equal(s, runs[0][1])
