"""fp64 CPU oracle for the Gated DeltaNet recurrence -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``gated_delta_rule_77_b200``) never imports, links or calls it,
and the two share no code: the only module both sides use is ``synth`` (seeded
input generation, no recurrence arithmetic).

Contents
  * ``run``        -- the token-by-token recurrence in fp64 (plain C,
                      ``gdn_oracle.c``), parallel over independent (b, h)
                      pairs with OpenMP.
  * ``run_steps``  -- the same recurrence fed one token per step from
                      per-step tensors laid out [steps, B, H, ...] (the decode
                      layout); a pure reshape around ``run``.
  * ``dense``      -- tiny-size fp64 NumPy forms used to pin ``run``: the
                      literal transition-matrix product and the chunk
                      (UT / WY) closed form.

The method: Atomic-GDN2 model card, section 2.1 "Gated DeltaNet-2"
(S_t = (I - b k k^T) Diag(a) S_{t-1} + b k v^T, o_t = S_t^T q_t, a = exp(g)).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "gdn_oracle.c"
_BUILD = _HERE / "_build"
_LIB_PATH = _BUILD / "libgdn_oracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile the C oracle with gcc (fp64, no fast-math, OpenMP)."""
    _BUILD.mkdir(exist_ok=True)
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(f".so.tmp{os.getpid()}")
        subprocess.run(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", str(_SRC), "-o", str(tmp), "-lm"],
            check=True,
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(str(build()))
        dp = ctypes.POINTER(ctypes.c_double)
        lib.gdn_oracle_run.restype = ctypes.c_int
        lib.gdn_oracle_run.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                       ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                       ctypes.c_long, ctypes.c_long, ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_long), ctypes.c_long, ctypes.c_int]
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: take the exact values it holds
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def run(q, k, v, g, beta, s0=None, *, per_channel: bool, heads=None, threads: int | None = None):
    """Token-by-token fp64 recurrence.

    q, k: [B, T, H, dk]; v: [B, T, H, dv]; g: [B, T, H] (scalar gate) or
    [B, T, H, dk] (per-channel gate); beta: [B, T, H]; s0: [B, H, dk, dv] or
    None (zero initial state).  Inputs may be NumPy arrays or torch tensors of
    any float dtype; their exact values are upcast to fp64.

    ``heads``: optional iterable of flat (b * H + h) indices to compute; other
    pairs' outputs are returned as NaN.  Returns (out [B, T, H, dv],
    s_final [B, H, dk, dv]) as fp64 NumPy arrays.
    """
    q, k, v, g, beta, s0 = (_f64(x) for x in (q, k, v, g, beta, s0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != (B, T, H, dk) or v.shape != (B, T, H, dv) or beta.shape != (B, T, H):
        raise ValueError("inconsistent shapes")
    if per_channel:
        if g.shape != (B, T, H, dk):
            raise ValueError("per-channel g must be [B, T, H, dk]")
    elif g.shape != (B, T, H):
        raise ValueError("scalar g must be [B, T, H]")
    if s0 is not None and s0.shape != (B, H, dk, dv):
        raise ValueError("s0 must be [B, H, dk, dv]")
    out = np.full((B, T, H, dv), np.nan)
    sT = np.full((B, H, dk, dv), np.nan)
    sel = None
    n_sel = 0
    if heads is not None:
        sel_arr = np.ascontiguousarray(np.asarray(list(heads), dtype=np.int64))
        sel = sel_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_long))
        n_sel = int(sel_arr.size)
    rc = _load().gdn_oracle_run(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0),
                                _ptr(out), _ptr(sT), B, T, H, dk, dv, int(bool(per_channel)),
                                sel, n_sel, int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError("oracle failed")
    return out, sT


def run_steps(q, k, v, g, beta, s0=None, *, per_channel: bool, heads=None, threads=None):
    """The recurrence fed one token per step from decode-layout inputs.

    q, k: [N, B, H, dk]; v: [N, B, H, dv]; g: [N, B, H] or [N, B, H, dk];
    beta: [N, B, H]; s0: [B, H, dk, dv].  Returns (out [N, B, H, dv],
    s_final [B, H, dk, dv]).  Pure relayout around ``run``.
    """
    q, k, v, g, beta = (np.swapaxes(_f64(x), 0, 1) for x in (q, k, v, g, beta))
    out, sT = run(q, k, v, g, beta, s0, per_channel=per_channel, heads=heads, threads=threads)
    return np.ascontiguousarray(np.swapaxes(out, 0, 1)), sT


def rel_err(got, ref) -> float:
    """max |got - ref| / rms(ref) over all elements (the tolerance rule)."""
    got = _f64(got)
    ref = _f64(ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref)) / rms) if rms > 0 else float(np.max(np.abs(got - ref)))
