"""Python binding of libgdn (Gated DeltaNet recurrence on B200, sm_100a).

Argument marshalling only: every step of the recurrence runs in the CUDA
kernels of ``libgdn.so`` behind the C ABI of ``include/gdn.h``.  PyTorch
provides device memory and streams.  There is no CPU fallback: if the native
library is missing or no CUDA device is present, the calls raise.

    out, s_final = chunk_fwd(q, k, v, g, beta, state_in)        # prefill
    o = recurrent_step(q, k, v, g, beta, state)                 # decode, in place

Gate mode is read from g's shape: [..., H] scalar per head, [..., H, dk] per
key channel.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libgdn.so"

GDN_OK = 0
GDN_ERR_INVALID_ARG = -1
GDN_ERR_UNSUPPORTED = -2
GDN_ERR_MISALIGNED = -3
GDN_ERR_CUDA = -4
GDN_ERR_NOMEM = -5
GDN_ERR_TIMEOUT = -6
GDN_ERR_SCRATCH_LIMIT = -7
GATE_SCALAR = 0
GATE_CHANNEL = 1
IO_BF16 = 0
IO_F32 = 1
ACT_NONE = 0
ACT_SILU = 1

SYMBOLS = ("gdn_chunk_fwd", "gdn_chunk_fwd_ex", "gdn_chunk_fwd_segments",
           "gdn_chunk_fwd_segments_noalloc", "gdn_recurrent_step", "gdn_recurrent_step_ex",
           "gdn_chunk_bwd", "gdn_recurrent_steps", "gdn_recurrent_steps_decoupled", "gdn_state_select",
           "gdn_prologue", "gdn_recurrent_step_prologue", "gdn_chunk_fwd_prologue",
           "gdn_check", "gdn_status_string")

_lib = None


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load() -> ctypes.CDLL:
    """Load libgdn.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise ImportError(f"{LIB_PATH} is missing; run `python -m gated_delta_rule_77_b200.build`")
    lib = ctypes.CDLL(str(LIB_PATH))
    vp, fp, i = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
    lib.gdn_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, i, i, i, i, i, i, vp]
    lib.gdn_chunk_fwd_ex.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, i, i, i, i, i, i, i, i, vp]
    lib.gdn_chunk_fwd_segments.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, i, i, i, i, i, i, i, vp]
    lib.gdn_chunk_fwd_segments_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, i, i, i, i, i, i, i,
                                                   vp]
    lib.gdn_recurrent_step.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, i, i, i, i, i, vp]
    lib.gdn_recurrent_step_ex.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, i, i, i, i, i, i, vp]
    lib.gdn_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, fp, fp, fp, fp, fp, fp, i, i, i,
                                  i, i, i, vp]
    lib.gdn_recurrent_steps.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, vp, i, i, i, i, i, i, vp]
    lib.gdn_recurrent_steps_decoupled.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, fp, vp, i, i, i, i,
                                                  i, i, vp]
    lib.gdn_state_select.argtypes = [fp, vp, fp, i, i, i, i, i, vp]
    lib.gdn_prologue.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, vp, vp, vp, fp, fp, i, i, i, i, i,
                                 i, i, vp]
    lib.gdn_recurrent_step_prologue.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, fp, fp, vp, i, i, i,
                                                i, i, i, vp]
    lib.gdn_chunk_fwd_prologue.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, fp, vp, fp, i, i, i, i,
                                           i, i, i, i, vp]
    lib.gdn_check.argtypes = [vp]
    lib.gdn_status_string.argtypes = [i]
    lib.gdn_status_string.restype = ctypes.c_char_p
    for name in SYMBOLS[:-1]:
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("every tensor must be a contiguous CUDA tensor")


def _io_code(dtype):
    if dtype == torch.bfloat16:
        return IO_BF16
    if dtype == torch.float32:
        return IO_F32
    raise ValueError(f"unsupported I/O dtype {dtype}")


def chunk_fwd(q, k, v, g, beta, state_in=None, *, out=None, state_out=None,
              return_state: bool = True, chunk_size: int = 0, segments=None, stream=None):
    """Chunkwise prefill.  q, k [B,T,H,dk]; v [B,T,H,dv]; g [B,T,H] or
    [B,T,H,dk] fp32; beta [B,T,H] fp32; state_in [B,H,dk,dv] fp32 or None.
    ``segments``: None = automatic; an int selects gdn_chunk_fwd_segments
    (1 = no sequence parallelism, n > 1 = n time segments).
    Returns (out [B,T,H,dv] fp32, final state or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gate = GATE_CHANNEL if g.dim() == 4 else GATE_SCALAR
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=torch.float32, device=v.device)
    if state_out is None and return_state:
        state_out = torch.empty(B, H, dk, dv, dtype=torch.float32, device=v.device)
    _check_cuda(q, k, v, g, beta, state_in, out, state_out)
    if segments is not None:
        rc = load().gdn_chunk_fwd_segments(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                           _ptr(state_in), _ptr(out), _ptr(state_out), B, T, H,
                                           dk, dv, gate, int(segments), _stream(stream))
        if rc != GDN_OK:
            raise GdnError(rc, "gdn_chunk_fwd_segments")
        return out, state_out
    rc = load().gdn_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in),
                                 _ptr(out), _ptr(state_out), B, T, H, dk, dv, gate,
                                 _io_code(q.dtype), int(chunk_size), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_fwd_ex")
    return out, state_out


def recurrent_step(q, k, v, g, beta, state, *, state_out=None, out=None, stream=None):
    """One decode step.  q, k [B,H,dk]; v [B,H,dv]; g [B,H] or [B,H,dk];
    beta [B,H]; state [B,H,dk,dv] fp32 (updated in place unless state_out is
    given).  Returns out [B,H,dv] fp32."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    gate = GATE_CHANNEL if g.dim() == 3 else GATE_SCALAR
    if state_out is None:
        state_out = state
    if out is None:
        out = torch.empty(B, H, dv, dtype=torch.float32, device=v.device)
    _check_cuda(q, k, v, g, beta, state, state_out, out)
    rc = load().gdn_recurrent_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                      _ptr(state), _ptr(state_out), _ptr(out), B, H, dk, dv,
                                      gate, _io_code(q.dtype), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_recurrent_step_ex")
    return out


def chunk_bwd(q, k, v, g, beta, state_in, d_out, d_state_out=None, *, stream=None):
    """Gradients of the prefill (gdn_chunk_bwd) for the loss
    sum(d_out * out) + sum(d_state_out * state_out).  Returns a dict of fp32
    tensors dq, dk, dv, dg, dbeta and ds0 (the initial state's gradient)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gate = GATE_CHANNEL if g.dim() == 4 else GATE_SCALAR
    dev = q.device
    out = dict(dq=torch.empty(B, T, H, dk, dtype=torch.float32, device=dev),
               dk=torch.empty(B, T, H, dk, dtype=torch.float32, device=dev),
               dv=torch.empty(B, T, H, dv, dtype=torch.float32, device=dev),
               dg=torch.empty(g.shape, dtype=torch.float32, device=dev),
               dbeta=torch.empty(B, T, H, dtype=torch.float32, device=dev),
               ds0=torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev))
    _check_cuda(q, k, v, g, beta, state_in, d_out, d_state_out)
    if q.dtype != torch.bfloat16:
        raise ValueError("q, k, v must be bf16")
    rc = load().gdn_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in),
                              _ptr(d_out), _ptr(d_state_out), _ptr(out["dq"]), _ptr(out["dk"]),
                              _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["ds0"]),
                              B, T, H, dk, dv, gate, _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_bwd")
    return out


def recurrent_steps(q, k, v, g, beta, state, *, state_out=None, snapshots=True, out=None,
                    beta_write=None, stream=None):
    """T successive decode tokens per sequence (speculative verification).
    q, k [B,T,H,dk] bf16; v [B,T,H,dv] bf16; g [B,T,H] or [B,T,H,dk];
    beta [B,T,H]; state [B,H,dk,dv] fp32, read only unless state_out is
    ``state`` itself.  ``snapshots``: True allocates [B,T,H,dk,dv], a tensor
    is written, None skips them.  ``beta_write`` [B,T,H]: a separate write
    gate (gdn_recurrent_steps_decoupled; ``beta`` is then the erase gate).
    Returns (out [B,T,H,dv] fp32, snapshots)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gate = GATE_CHANNEL if g.dim() == 4 else GATE_SCALAR
    if snapshots is True:
        snapshots = torch.empty(B, T, H, dk, dv, dtype=torch.float32, device=v.device)
    elif snapshots is False:
        snapshots = None
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=torch.float32, device=v.device)
    _check_cuda(q, k, v, g, beta, state, state_out, snapshots, out, beta_write)
    if beta_write is not None:
        rc = load().gdn_recurrent_steps_decoupled(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                                  _ptr(beta_write), _ptr(state), _ptr(state_out),
                                                  _ptr(snapshots), _ptr(out), B, T, H, dk, dv, gate,
                                                  _stream(stream))
        if rc != GDN_OK:
            raise GdnError(rc, "gdn_recurrent_steps_decoupled")
        return out, snapshots
    rc = load().gdn_recurrent_steps(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
                                    _ptr(state_out), _ptr(snapshots), _ptr(out), B, T, H, dk, dv,
                                    gate, _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_recurrent_steps")
    return out, snapshots


def state_select(snapshots, num_accepted, state, *, stream=None):
    """state[b] := snapshots[b, num_accepted[b] - 1] where 1 <= n_b <= T
    (num_accepted: int32 [B] on the device); other rows unchanged."""
    B, T, H, dk, dv = snapshots.shape
    _check_cuda(snapshots, num_accepted, state)
    if num_accepted.dtype != torch.int32:
        raise ValueError("num_accepted must be int32")
    rc = load().gdn_state_select(_ptr(snapshots), _ptr(num_accepted), _ptr(state), B, T, H, dk, dv,
                                 _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_state_select")
    return state


def _act_code(activation):
    if activation == "silu":
        return ACT_SILU
    if activation == "none":
        return ACT_NONE
    raise ValueError(f"unknown activation {activation!r}")


def prologue(q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring=None, pos0=None, *,
             activation: str = "silu", stream=None):
    """The layer's input prologue over T tokens (gdn_prologue).  q_raw, k_raw
    [B,T,H,dk] bf16; v_raw [B,T,H,dv] bf16; g_raw [B,T,H] or [B,T,H,dk] fp32;
    beta_raw [B,T,H] fp32; conv_w [H, 2dk+dv, 4] fp32; ring [B,H,4,2dk+dv]
    fp32 (updated in place) or None; pos0 [B] int32 or None.  Returns
    (q, k, v, g, beta), ready for chunk_fwd."""
    B, T, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    gate = GATE_CHANNEL if g_raw.dim() == 4 else GATE_SCALAR
    dev = q_raw.device
    q = torch.empty(B, T, H, dk, dtype=torch.bfloat16, device=dev)
    k = torch.empty_like(q)
    v = torch.empty(B, T, H, dv, dtype=torch.bfloat16, device=dev)
    g = torch.empty(g_raw.shape, dtype=torch.float32, device=dev)
    beta = torch.empty(B, T, H, dtype=torch.float32, device=dev)
    _check_cuda(q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring, pos0)
    if q_raw.dtype != torch.bfloat16 or v_raw.dtype != torch.bfloat16:
        raise ValueError("q_raw, k_raw and v_raw must be bf16")
    if pos0 is not None and pos0.dtype != torch.int32:
        raise ValueError("pos0 must be int32")
    rc = load().gdn_prologue(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(g_raw), _ptr(beta_raw),
                             _ptr(conv_w), _ptr(ring), _ptr(pos0), _ptr(q), _ptr(k), _ptr(v),
                             _ptr(g), _ptr(beta), B, T, H, dk, dv, gate, _act_code(activation),
                             _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_prologue")
    return q, k, v, g, beta


def recurrent_step_prologue(q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring, state, pos=None, *,
                            activation: str = "silu", state_out=None, out=None, stream=None):
    """One decode step with the prologue fused in (gdn_recurrent_step_prologue).
    q_raw, k_raw [B,H,dk] bf16; v_raw [B,H,dv] bf16; g_raw [B,H] or [B,H,dk];
    beta_raw [B,H]; ring [B,H,4,2dk+dv] fp32 (slot pos mod 4 written);
    state [B,H,dk,dv] fp32 (in place unless state_out); pos [B] int32 or
    None.  Returns out [B,H,dv] fp32."""
    B, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    gate = GATE_CHANNEL if g_raw.dim() == 3 else GATE_SCALAR
    if state_out is None:
        state_out = state
    if out is None:
        out = torch.empty(B, H, dv, dtype=torch.float32, device=v_raw.device)
    _check_cuda(q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring, state, state_out, out, pos)
    if q_raw.dtype != torch.bfloat16 or v_raw.dtype != torch.bfloat16:
        raise ValueError("q_raw, k_raw and v_raw must be bf16")
    if pos is not None and pos.dtype != torch.int32:
        raise ValueError("pos must be int32")
    rc = load().gdn_recurrent_step_prologue(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(g_raw),
                                            _ptr(beta_raw), _ptr(conv_w), _ptr(ring), _ptr(pos),
                                            _ptr(state), _ptr(state_out), _ptr(out), B, H, dk, dv,
                                            gate, _act_code(activation), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_recurrent_step_prologue")
    return out


def chunk_fwd_prologue(q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring=None, pos0=None,
                       state_in=None, *, activation: str = "silu", out=None, state_out=None,
                       return_state: bool = True, fused: bool = False, stream=None):
    """The prefill from a layer's raw projections (gdn_chunk_fwd_prologue):
    the prologue of ``prologue``, then the recurrence -- as two passes
    through scratch, or with ``fused`` applied inside the prefill kernel while
    it loads (dk = dv = 128; other shapes take the two passes).  Arguments as
    ``prologue`` and ``chunk_fwd``; the ring (if given) is read and updated.
    Returns (out [B,T,H,dv] fp32, final state or None)."""
    B, T, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    gate = GATE_CHANNEL if g_raw.dim() == 4 else GATE_SCALAR
    dev = v_raw.device
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=torch.float32, device=dev)
    if state_out is None and return_state:
        state_out = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    _check_cuda(q_raw, k_raw, v_raw, g_raw, beta_raw, conv_w, ring, pos0, state_in, out, state_out)
    if q_raw.dtype != torch.bfloat16 or v_raw.dtype != torch.bfloat16:
        raise ValueError("q_raw, k_raw and v_raw must be bf16")
    if pos0 is not None and pos0.dtype != torch.int32:
        raise ValueError("pos0 must be int32")
    rc = load().gdn_chunk_fwd_prologue(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(g_raw),
                                       _ptr(beta_raw), _ptr(conv_w), _ptr(ring), _ptr(pos0),
                                       _ptr(state_in), _ptr(out), _ptr(state_out), B, T, H, dk, dv,
                                       gate, _act_code(activation), int(bool(fused)),
                                       _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_fwd_prologue")
    return out, state_out


def check(stream=None) -> int:
    """Synchronise the stream and report a bounded-wait timeout, if any."""
    return int(load().gdn_check(_stream(stream)))
