"""The no-allocation entry point, gdn_chunk_fwd_segments_noalloc, on the GPU.

It exists for callers that cannot let the library allocate device memory --
their memory belongs to another allocator, or their step must never stall in
an allocator or fail for lack of memory -- and takes its scratch from a fixed
32 MiB array compiled into the library instead.  These tests call it through
the C ABI (ctypes, raw device pointers) and compare it with the allocating
entry point, gdn_chunk_fwd_segments, on the same inputs: two calls in a row,
so that the data the first call leaves in the shared array cannot leak into
the second.  A call too large for the array must be refused without a launch.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import oracle
from synth import prefill_inputs

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call(fn, x, segments, stream):
    B, T, H, dk = x["q"].shape
    dv = x["v"].shape[-1]
    out = torch.full((B, T, H, dv), float("nan"), dtype=torch.float32, device="cuda")
    s_out = torch.full((B, H, dk, dv), float("nan"), dtype=torch.float32, device="cuda")
    gate = 1 if x["g"].dim() == 4 else 0
    rc = fn(_ptr(x["q"]), _ptr(x["k"]), _ptr(x["v"]), _ptr(x["g"]), _ptr(x["beta"]), _ptr(x["s0"]),
            _ptr(out), _ptr(s_out), B, T, H, dk, dv, gate, segments, ctypes.c_void_p(stream))
    return rc, out, s_out


def test_noalloc_matches_allocating_entry_point_on_two_calls(gdn):
    lib = gdn.load()
    stream = torch.cuda.current_stream().cuda_stream
    cases = [(401, "channel", 1, 1000, 2, 4), (402, "scalar", 2, 700, 3, 3)]
    for seed, gate, B, T, H, segments in cases:
        host = prefill_inputs(B, T, H, 128, 128, gate=gate, s0_std=0.1, seed=seed)
        x = {n: (None if t is None else t.cuda()) for n, t in host.items()}
        rc_ref, out_ref, s_ref = _call(lib.gdn_chunk_fwd_segments, x, segments, stream)
        rc_na, out_na, s_na = _call(lib.gdn_chunk_fwd_segments_noalloc, x, segments, stream)
        torch.cuda.synchronize()
        assert rc_ref == gdn.GDN_OK and rc_na == gdn.GDN_OK, (rc_ref, rc_na)
        assert oracle.rel_err(out_na.cpu(), out_ref.cpu().double()) <= TOL / 2
        assert oracle.rel_err(s_na.cpu(), s_ref.cpu().double()) <= TOL / 2
        ref_o, ref_s = oracle.run(host["q"], host["k"], host["v"], host["g"], host["beta"],
                                  host["s0"], per_channel=gate == "channel")
        assert oracle.rel_err(out_na.cpu(), ref_o) <= TOL
        assert oracle.rel_err(s_na.cpu(), ref_s) <= TOL


def test_noalloc_refuses_calls_beyond_its_array(gdn):
    lib = gdn.load()
    stream = torch.cuda.current_stream().cuda_stream
    # 1 x 32 segments x 16 heads = 512 segment states of 64 KiB, twice: > 32 MiB.
    host = prefill_inputs(1, 2048, 16, 128, 128, gate="scalar", seed=403)
    x = {n: (None if t is None else t.cuda()) for n, t in host.items()}
    rc, out, _ = _call(lib.gdn_chunk_fwd_segments_noalloc, x, 32, stream)
    torch.cuda.synchronize()
    assert rc == gdn.GDN_ERR_SCRATCH_LIMIT
    assert bool(torch.isnan(out).all())          # nothing was launched
