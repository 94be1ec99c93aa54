"""Seeded synthetic inputs for the Gated DeltaNet recurrence.

This module is the only code shared by the CUDA path's tests / benchmark and
the oracle.  It draws random numbers and applies the input recipe; it holds
none of the recurrence's arithmetic.

Recipe (the workloads the pages describe; no dataset is involved):
  * q, k ~ N(0, 1), L2-normalised over the key dimension for every
    (b, t, h) -- the mixer normalises q and k per head before the kernel
    (Atomic-GDN2 model card, section 2.1 layer description);
  * v ~ N(0, 1);
  * beta = sigmoid(N(0, 1));
  * g = -min(softplus(N(0, 1)), 5): the model card's log-decay
    parameterisation with bs2 = 32, i.e. g in [-5, 0] (section 2.1);
  * optional initial state S0 ~ N(0, std) in fp32;
  * optional "no forgetting" tokens: a Bernoulli(p) mask over (b, t, h)
    sets g = 0 exactly (alpha = 1).

Everything is drawn on the CPU from ``torch.Generator().manual_seed(seed)``
in the fixed order q, k, v, beta, g, S0, mask, in fp32, then q / k / v are
cast to the I/O dtype; both sides read the cast values.  Large tensors are
drawn in slices of ``SLICE_TOKENS`` tokens (same order) to bound host memory.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

SLICE_TOKENS = 4096


@dataclass(frozen=True)
class Config:
    """One workload of the benchmark / parity suite."""
    index: int
    name: str
    B: int
    H: int
    dk: int
    dv: int
    T: int = 0                 # prefill length (0 for decode)
    steps: int = 0             # decode: successive single-token steps
    io: str = "bf16"           # dtype of q, k, v (and prefill output)
    gate: str = "scalar"       # "scalar" (per head) or "channel" (per key channel)
    s0_std: float = 0.0        # 0 = zero initial state
    g_zero_frac: float = 0.0   # fraction of (b, t, h) with g = 0 exactly
    tol: float = 2e-2          # max|got - ref| <= tol * rms(ref)
    mode: str = "prefill"
    extra: dict = field(default_factory=dict)

    @property
    def per_channel(self) -> bool:
        return self.gate == "channel"

    @property
    def torch_io(self):
        return torch.float32 if self.io == "f32" else torch.bfloat16


CONFIGS = {
    1: Config(1, "oracle-scale prefill B1 H2 T256 d64 fp32 scalar gate",
              B=1, H=2, T=256, dk=64, dv=64, io="f32", gate="scalar", tol=1e-4),
    2: Config(2, "GDN-2 layer prefill B8 H8 T2048 d128 bf16 per-channel gate",
              B=8, H=8, T=2048, dk=128, dv=128, io="bf16", gate="channel", tol=2e-2),
    3: Config(3, "scalar-gate training-length prefill B4 H12 T8192 d128 bf16 S0~N(0,0.1)",
              B=4, H=12, T=8192, dk=128, dv=128, io="bf16", gate="scalar", s0_std=0.1, tol=2e-2),
    4: Config(4, "recurrent decode B64 H16 d128 1024 steps bf16 per-channel gate S0~N(0,0.1)",
              B=64, H=16, dk=128, dv=128, steps=1024, io="bf16", gate="channel", s0_std=0.1,
              tol=1e-3, mode="decode"),
    5: Config(5, "long-context prefill B1 H16 T262144 d128 bf16 scalar gate 10% g=0",
              B=1, H=16, T=262144, dk=128, dv=128, io="bf16", gate="scalar", g_zero_frac=0.1,
              tol=2e-2),
}


def _randn_sliced(gen, lead, tokens, tail, token_axis):
    """randn of shape lead + (tokens,) + tail, drawn slice by slice over tokens."""
    parts = []
    for t0 in range(0, tokens, SLICE_TOKENS):
        n = min(SLICE_TOKENS, tokens - t0)
        parts.append(torch.randn(*lead, n, *tail, generator=gen))
    if not parts:
        return torch.empty(*lead, 0, *tail)
    return torch.cat(parts, dim=token_axis)


def _unit(x):
    return x / x.norm(dim=-1, keepdim=True)


def _gate(raw):
    return -torch.clamp(torch.nn.functional.softplus(raw), max=5.0)


def prefill_inputs(B, T, H, dk, dv, *, gate="scalar", io=torch.bfloat16, s0_std=0.0,
                   g_zero_frac=0.0, seed=0):
    """Inputs for one prefill call (layout [B, T, H, ...]).

    Returns a dict of CPU tensors: q, k [B,T,H,dk] (io dtype), v [B,T,H,dv]
    (io dtype), g [B,T,H] or [B,T,H,dk] fp32, beta [B,T,H] fp32, s0
    [B,H,dk,dv] fp32 or None.
    """
    gen = torch.Generator().manual_seed(int(seed))
    q = _unit(_randn_sliced(gen, (B,), T, (H, dk), 1)).to(io)
    k = _unit(_randn_sliced(gen, (B,), T, (H, dk), 1)).to(io)
    v = _randn_sliced(gen, (B,), T, (H, dv), 1).to(io)
    beta = torch.sigmoid(_randn_sliced(gen, (B,), T, (H,), 1))
    g_tail = (H, dk) if gate == "channel" else (H,)
    g = _gate(_randn_sliced(gen, (B,), T, g_tail, 1))
    s0 = torch.randn(B, H, dk, dv, generator=gen) * s0_std if s0_std > 0 else None
    if g_zero_frac > 0:
        mask = torch.rand(B, T, H, generator=gen) < g_zero_frac
        if gate == "channel":
            g[mask] = 0.0
        else:
            g = torch.where(mask, torch.zeros_like(g), g)
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(), g=g.contiguous(),
                beta=beta.contiguous(), s0=None if s0 is None else s0.contiguous())


def decode_inputs(B, H, dk, dv, steps, *, gate="channel", io=torch.bfloat16, s0_std=0.1, seed=0):
    """Inputs for ``steps`` successive single-token decode calls.

    Returns q, k [N,B,H,dk], v [N,B,H,dv] (io dtype), g [N,B,H] or
    [N,B,H,dk] fp32, beta [N,B,H] fp32, s0 [B,H,dk,dv] fp32 (N = steps).
    """
    gen = torch.Generator().manual_seed(int(seed))
    q = _unit(torch.randn(steps, B, H, dk, generator=gen)).to(io)
    k = _unit(torch.randn(steps, B, H, dk, generator=gen)).to(io)
    v = torch.randn(steps, B, H, dv, generator=gen).to(io)
    beta = torch.sigmoid(torch.randn(steps, B, H, generator=gen))
    g_shape = (steps, B, H, dk) if gate == "channel" else (steps, B, H)
    g = _gate(torch.randn(*g_shape, generator=gen))
    s0 = torch.randn(B, H, dk, dv, generator=gen) * s0_std if s0_std > 0 else torch.zeros(B, H, dk, dv)
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(), g=g.contiguous(),
                beta=beta.contiguous(), s0=s0.contiguous())


def config_inputs(cfg: Config, seed: int | None = None, **overrides):
    """Inputs of a named workload; ``seed`` defaults to the config index.

    ``overrides`` may shrink a dimension (B, H, T, steps) for a reduced case
    of the same recipe.
    """
    seed = cfg.index if seed is None else seed
    B = overrides.get("B", cfg.B)
    H = overrides.get("H", cfg.H)
    if cfg.mode == "decode":
        return decode_inputs(B, H, cfg.dk, cfg.dv, overrides.get("steps", cfg.steps),
                             gate=cfg.gate, io=cfg.torch_io, s0_std=cfg.s0_std, seed=seed)
    return prefill_inputs(B, overrides.get("T", cfg.T), H, cfg.dk, cfg.dv, gate=cfg.gate,
                          io=cfg.torch_io, s0_std=cfg.s0_std, g_zero_frac=cfg.g_zero_frac,
                          seed=seed)


def prologue_inputs(B, T, H, dk, dv, *, gate="channel", ring=True, pos0_max=1000, seed=0):
    """Raw inputs of the layer's input prologue (layout [B, T, H, ...]).

    Recipe: q_raw, k_raw, v_raw ~ N(0, 1) rounded to bf16 (the projections'
    outputs); g_raw ~ N(0, 2) (so that the softplus bound of 5 is active on
    a fraction of tokens); beta_raw ~ N(0, 1); conv taps ~ U(-0.5, 0.5) (the
    default initialisation bound 1/sqrt(width) of a width-4 depthwise
    convolution); the history ring holds bf16-representable N(0, 1) values,
    and pos0 ~ U{0 .. pos0_max} (a ring position not a multiple of 4 in
    general).  Drawn in that order from ``manual_seed(seed)``.
    """
    gen = torch.Generator().manual_seed(int(seed))
    q = _randn_sliced(gen, (B,), T, (H, dk), 1).to(torch.bfloat16)
    k = _randn_sliced(gen, (B,), T, (H, dk), 1).to(torch.bfloat16)
    v = _randn_sliced(gen, (B,), T, (H, dv), 1).to(torch.bfloat16)
    g_tail = (H, dk) if gate == "channel" else (H,)
    g = _randn_sliced(gen, (B,), T, g_tail, 1) * 2.0
    beta = _randn_sliced(gen, (B,), T, (H,), 1)
    w = torch.rand(H, 2 * dk + dv, 4, generator=gen) - 0.5
    C = 2 * dk + dv
    r = torch.randn(B, H, 4, C, generator=gen).to(torch.bfloat16).float() if ring else None
    pos0 = torch.randint(0, pos0_max + 1, (B,), generator=gen, dtype=torch.int32)
    return dict(q_raw=q.contiguous(), k_raw=k.contiguous(), v_raw=v.contiguous(), g_raw=g.contiguous(),
                beta_raw=beta.contiguous(), conv_w=w.contiguous(), ring=r, pos0=pos0)


def grad_inputs(B, T, H, dk, dv, *, seed=0, d_state=True):
    """Incoming gradients of a prefill call: d_out [B, T, H, dv] ~ N(0, 1) and
    d_state_out [B, H, dk, dv] ~ N(0, 1) (or None), fp32, drawn in that order
    from ``manual_seed(seed)``."""
    gen = torch.Generator().manual_seed(int(seed))
    d_out = _randn_sliced(gen, (B,), T, (H, dv), 1)
    ds = torch.randn(B, H, dk, dv, generator=gen) if d_state else None
    return d_out.contiguous(), ds


def write_gate(B, T, H, *, seed=0):
    """A separate write gate for the decoupled form: sigmoid(N(0, 1)) per
    (b, t, h), fp32, from ``manual_seed(seed)`` (the erase gate is the
    recipe's beta)."""
    gen = torch.Generator().manual_seed(int(seed))
    return torch.sigmoid(_randn_sliced(gen, (B,), T, (H,), 1)).contiguous()

