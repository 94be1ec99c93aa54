"""fp64 oracle of the input prologue of a Gated DeltaNet layer -- TEST
INFRASTRUCTURE ONLY (same import rule as the rest of ``oracle/``).

What the prologue computes, per (batch, head), from the layer's projected
inputs to the recurrence's inputs:

* a causal depthwise convolution of width 4 over the token axis, applied to
  every channel of q, k and v (the DeltaNet layers' "kernel-4 convolution",
  Qwen3.5 27B page, section on the hybrid layout; "causal convolutions on ...
  q/k/v", HANDOFF timeline page, v2 entry):
      y_t[c] = sum_{j=0..3} w[c, j] x_{t-3+j}[c]     (tap 3 = the current token),
  with the inputs of the positions before the first token taken from a
  4-slot history ring (slot p mod 4 holds position p's input) or zero;
* an activation after the convolution: none, or SiLU y / (1 + exp(-y)) (the
  pages name none; SiLU is the usual short-convolution activation of GDN
  layers, and "none" is kept selectable);
* q and k L2-normalised over the head's channels, x (sum x^2 + 1e-6)^(-1/2);
* beta = sigmoid(beta_raw) and g = -min(softplus(g_raw), 5) (Atomic-GDN2 model
  card, section 2.1: the bound 160 / bs2 with bs2 = 32).

Layouts follow the library's: q_raw, k_raw [B, T, H, dk]; v_raw [B, T, H, dv];
g_raw [B, T, H] or [B, T, H, dk]; beta_raw [B, T, H]; conv_w [H, 2 dk + dv, 4]
(channels in the order q | k | v); ring [B, H, 4, 2 dk + dv]; pos0 [B] = the
position of token 0 of each row.  Everything is computed in fp64 with plain
NumPy loops over the four taps.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6
G_BOUND = 5.0


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if x.dtype.is_floating_point:
            x = x.double()
        return x.numpy()
    return np.asarray(x, dtype=np.float64)


def silu(y):
    return y / (1.0 + np.exp(-y))


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def softplus(x):
    """log(1 + exp(x)), written to stay finite for large |x|."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 30.0, x, np.log1p(np.exp(np.minimum(x, 30.0))))


def l2norm(x):
    """x / sqrt(sum over the last axis of x^2 + 1e-6)."""
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + EPS)


def causal_conv4(x, w, history):
    """x [B, T, H, C]; w [H, C, 4]; history [B, H, 3, C] = inputs at positions
    t0 - 3 .. t0 - 1.  Returns y [B, T, H, C] with tap 3 on the current token."""
    B, T, H, C = x.shape
    ext = np.concatenate([np.transpose(history, (0, 2, 1, 3)), x], axis=1)   # [B, T + 3, H, C]
    y = np.zeros_like(x)
    for j in range(4):
        y += w[None, None, :, :, j] * ext[:, j:j + T]
    return y


def ring_history(ring, pos0, B, H, C):
    """The three inputs before each row's first token, from a 4-slot ring
    (slot p mod 4 = position p), or zeros without a ring."""
    hist = np.zeros((B, H, 3, C))
    if ring is None:
        return hist
    for b in range(B):
        for i in range(3):
            p = int(pos0[b]) - 3 + i
            hist[b, :, i] = ring[b, :, p % 4] if p >= 0 else 0.0
    return hist


def ring_after(ring, pos0, x, B, H, C):
    """The ring after the T tokens of x: slot p mod 4 takes position p's input
    for the last min(T, 4) positions; the other slots keep their values."""
    T = x.shape[1]
    out = np.zeros((B, H, 4, C)) if ring is None else np.array(ring, dtype=np.float64, copy=True)
    for b in range(B):
        for t in range(max(0, T - 4), T):
            p = int(pos0[b]) + t
            out[b, :, p % 4] = x[b, t]
    return out


def prologue(q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring=None, pos0=None, *,
             activation: str = "silu"):
    """Returns (q, k, v, g, beta, ring_out) in fp64; ring_out is None without a ring."""
    q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring = (
        _f64(t) for t in (q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring))
    B, T, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    pos0 = np.zeros(B, dtype=np.int64) if pos0 is None else np.asarray(_f64(pos0)).astype(np.int64)
    x = np.concatenate([q_raw, k_raw, v_raw], axis=-1)                      # [B, T, H, 2dk + dv]
    C = x.shape[-1]
    y = causal_conv4(x, conv_w, ring_history(ring, pos0, B, H, C))
    if activation == "silu":
        y = silu(y)
    elif activation != "none":
        raise ValueError(activation)
    q = l2norm(y[..., :dk])
    k = l2norm(y[..., dk:2 * dk])
    v = y[..., 2 * dk:]
    g = -np.minimum(softplus(g_raw), G_BOUND)
    beta = sigmoid(beta_raw)
    ring_out = None if ring is None else ring_after(ring, pos0, x, B, H, C)
    return q, k, v, g, beta, ring_out
