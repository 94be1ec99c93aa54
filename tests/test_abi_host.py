"""The C ABI on the host: the library loads, exports every declared symbol,
and rejects invalid calls before launching anything (no GPU needed).

Every call here fails validation on purpose, so no kernel is launched and
no fake pointer is ever dereferenced.
"""
import ctypes
import re
from pathlib import Path

import pytest

import gated_delta_rule_77_b200 as gdn

HEADER = Path(__file__).resolve().parent.parent / "include" / "gdn.h"
A = 0x10000          # 16-byte aligned fake device addresses, spaced apart
MB = 1 << 20


def declared_symbols():
    text = HEADER.read_text()
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_77_b200 import build
    build.build()
    return gdn.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert set(names) == set(gdn.SYMBOLS)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in [(0, "GDN_OK"), (-1, "GDN_ERR_INVALID_ARG"), (-2, "GDN_ERR_UNSUPPORTED"),
                       (-3, "GDN_ERR_MISALIGNED"), (-4, "GDN_ERR_CUDA"), (-5, "GDN_ERR_NOMEM"),
                       (-6, "GDN_ERR_TIMEOUT"), (-7, "GDN_ERR_SCRATCH_LIMIT"), (7, "GDN_ERR_UNKNOWN")]:
        assert gdn.status_string(code) == name


def _prefill(lib, q=A, k=A + 64 * MB, v=A + 128 * MB, g=A + 192 * MB, beta=A + 256 * MB,
             s_in=A + 320 * MB, out=A + 384 * MB, s_out=A + 448 * MB, B=1, T=16, H=1, dk=128, dv=128,
             gate=0, io=0, chunk=0):
    c = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.gdn_chunk_fwd_ex(c(q), c(k), c(v), c(g), c(beta), c(s_in), c(out), c(s_out),
                                B, T, H, dk, dv, gate, io, chunk, None)


def _step(lib, q=A, k=A + 64 * MB, v=A + 128 * MB, g=A + 192 * MB, beta=A + 256 * MB,
          s_in=A + 320 * MB, s_out=A + 320 * MB, out=A + 448 * MB, B=1, H=1, dk=128, dv=128, gate=1,
          io=0):
    c = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.gdn_recurrent_step_ex(c(q), c(k), c(v), c(g), c(beta), c(s_in), c(s_out), c(out),
                                     B, H, dk, dv, gate, io, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(k=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(v=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(g=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(beta=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(out=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(B=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(H=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(T=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(gate=2), gdn.GDN_ERR_INVALID_ARG),
    (dict(io=5), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dv=32), gdn.GDN_ERR_UNSUPPORTED),
    (dict(chunk=48), gdn.GDN_ERR_UNSUPPORTED),
    (dict(io=1, chunk=64), gdn.GDN_ERR_UNSUPPORTED),
    (dict(q=A + 8), gdn.GDN_ERR_MISALIGNED),
    (dict(s_out=A + 448 * MB + 4), gdn.GDN_ERR_MISALIGNED),
    (dict(out=A + 16), gdn.GDN_ERR_INVALID_ARG),                     # out overlaps q
    (dict(out=A + 320 * MB), gdn.GDN_ERR_INVALID_ARG),               # out overlaps state_in
    (dict(s_out=A + 128 * MB), gdn.GDN_ERR_INVALID_ARG),             # state_out overlaps v
    (dict(s_out=A + 320 * MB + 4096), gdn.GDN_ERR_INVALID_ARG),      # partial state overlap
])
def test_prefill_rejects(lib, kw, status):
    assert _prefill(lib, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(s_in=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(s_out=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(out=A + 320 * MB), gdn.GDN_ERR_INVALID_ARG),               # out overlaps state
    (dict(dk=100), gdn.GDN_ERR_UNSUPPORTED),
    (dict(gate=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(v=A + 128 * MB + 2), gdn.GDN_ERR_MISALIGNED),
    (dict(beta=A + 256 * MB + 2), gdn.GDN_ERR_MISALIGNED),
    (dict(g=A + 192 * MB + 4), gdn.GDN_ERR_MISALIGNED),
])
def test_step_rejects(lib, kw, status):
    assert _step(lib, **kw) == status


def test_scalar_gate_and_beta_need_only_4_byte_alignment(lib):
    # A per-step slice of a [steps, B, H] tensor starts at a multiple of 4 bytes.
    # With state_in = None the call is rejected for that reason, not alignment.
    assert _step(lib, gate=0, g=A + 192 * MB + 4, beta=A + 256 * MB + 12, s_in=None) == \
        gdn.GDN_ERR_INVALID_ARG


def test_segments_entry_point_rejects(lib):
    c = ctypes.c_void_p
    call = lambda segs, dk=128, B=1: lib.gdn_chunk_fwd_segments(  # noqa: E731
        c(A), c(A + 64 * MB), c(A + 128 * MB), c(A + 192 * MB), c(A + 256 * MB), None,
        c(A + 384 * MB), c(A + 448 * MB), B, 16, 1, dk, 128, 0, segs, None)
    assert call(-1) == gdn.GDN_ERR_INVALID_ARG
    assert call(4, dk=64) == gdn.GDN_ERR_UNSUPPORTED
    assert call(4, B=0) == gdn.GDN_ERR_INVALID_ARG


def _pro(lib, qr=A, kr=A + 64 * MB, vr=A + 128 * MB, gr=A + 192 * MB, br=A + 256 * MB,
         w=A + 300 * MB, ring=A + 310 * MB, pos=A + 319 * MB, q=A + 320 * MB, k=A + 384 * MB,
         v=A + 448 * MB, g=A + 512 * MB, beta=A + 576 * MB, B=1, T=16, H=1, dk=128, dv=128, gate=0,
         act=1):
    c = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.gdn_prologue(c(qr), c(kr), c(vr), c(gr), c(br), c(w), c(ring), c(pos), c(q), c(k),
                            c(v), c(g), c(beta), B, T, H, dk, dv, gate, act, None)


@pytest.mark.parametrize("kw,status", [
    (dict(qr=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(w=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(beta=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(act=2), gdn.GDN_ERR_INVALID_ARG),
    (dict(gate=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(T=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=32), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dv=256), gdn.GDN_ERR_UNSUPPORTED),
    (dict(w=A + 300 * MB + 8), gdn.GDN_ERR_MISALIGNED),      # conv taps are read as float4
    (dict(ring=A + 310 * MB + 4), gdn.GDN_ERR_MISALIGNED),
    (dict(gate=1, gr=A + 192 * MB + 8), gdn.GDN_ERR_MISALIGNED),
    (dict(pos=A + 319 * MB + 2), gdn.GDN_ERR_MISALIGNED),
    (dict(q=A + 32), gdn.GDN_ERR_INVALID_ARG),               # q overlaps q_raw (no in-place)
    (dict(v=A + 384 * MB + 64), gdn.GDN_ERR_INVALID_ARG),    # v overlaps k
    (dict(ring=A + 128 * MB), gdn.GDN_ERR_INVALID_ARG),      # ring overlaps v_raw
    (dict(beta=A + 310 * MB), gdn.GDN_ERR_INVALID_ARG),      # beta overlaps the ring
])
def test_prologue_rejects(lib, kw, status):
    assert _pro(lib, **kw) == status


def test_prologue_with_no_tokens_launches_nothing(lib):
    # T = 0: every per-token pointer may be null and nothing is launched.
    assert _pro(lib, T=0, qr=None, kr=None, vr=None, gr=None, br=None, q=None, k=None, v=None,
                g=None, beta=None) == gdn.GDN_OK


def _step_pro(lib, qr=A, kr=A + 64 * MB, vr=A + 128 * MB, gr=A + 192 * MB, br=A + 256 * MB,
              w=A + 300 * MB, ring=A + 310 * MB, pos=A + 319 * MB, s_in=A + 320 * MB,
              s_out=A + 320 * MB, out=A + 448 * MB, B=1, H=1, dk=128, dv=128, gate=1, act=1):
    c = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.gdn_recurrent_step_prologue(c(qr), c(kr), c(vr), c(gr), c(br), c(w), c(ring),
                                           c(pos), c(s_in), c(s_out), c(out), B, H, dk, dv, gate,
                                           act, None)


@pytest.mark.parametrize("kw,status", [
    (dict(ring=None), gdn.GDN_ERR_INVALID_ARG),              # the ring is required
    (dict(s_in=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(out=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(B=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(act=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(s_in=A + 320 * MB + 4, s_out=A + 320 * MB + 4), gdn.GDN_ERR_MISALIGNED),
    (dict(out=A + 320 * MB), gdn.GDN_ERR_INVALID_ARG),       # out overlaps the state
    (dict(s_out=A + 320 * MB + 1024), gdn.GDN_ERR_INVALID_ARG),   # partial state overlap
    (dict(s_in=A + 310 * MB, s_out=A + 310 * MB), gdn.GDN_ERR_INVALID_ARG),  # state on the ring
])
def test_step_prologue_rejects(lib, kw, status):
    assert _step_pro(lib, **kw) == status


def _steps(lib, q=A, k=A + 64 * MB, v=A + 128 * MB, g=A + 192 * MB, beta=A + 256 * MB,
           s_in=A + 320 * MB, s_out=A + 320 * MB, snap=A + 512 * MB, out=A + 448 * MB, B=1, T=4, H=1,
           dk=128, dv=128, gate=1):
    c = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.gdn_recurrent_steps(c(q), c(k), c(v), c(g), c(beta), c(s_in), c(s_out), c(snap),
                                   c(out), B, T, H, dk, dv, gate, None)


@pytest.mark.parametrize("kw,status", [
    (dict(s_in=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(s_out=None, snap=None), gdn.GDN_ERR_INVALID_ARG),      # nothing would be kept
    (dict(T=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dv=48), gdn.GDN_ERR_UNSUPPORTED),
    (dict(snap=A + 512 * MB + 4), gdn.GDN_ERR_MISALIGNED),
    (dict(snap=A + 448 * MB), gdn.GDN_ERR_INVALID_ARG),          # snapshots overlap out
    (dict(snap=A + 320 * MB), gdn.GDN_ERR_INVALID_ARG),          # snapshots overlap the state
    (dict(out=A + 320 * MB + 64), gdn.GDN_ERR_INVALID_ARG),      # out overlaps the state
])
def test_recurrent_steps_rejects(lib, kw, status):
    assert _steps(lib, **kw) == status


def _select(lib, snap=A, nacc=A + 300 * MB, state=A + 320 * MB, B=2, T=4, H=2, dk=128, dv=128):
    c = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.gdn_state_select(c(snap), c(nacc), c(state), B, T, H, dk, dv, None)


@pytest.mark.parametrize("kw,status", [
    (dict(snap=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(nacc=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(state=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(T=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=32), gdn.GDN_ERR_UNSUPPORTED),
    (dict(state=A + 320 * MB + 8), gdn.GDN_ERR_MISALIGNED),
    (dict(nacc=A + 300 * MB + 2), gdn.GDN_ERR_MISALIGNED),
    (dict(state=A + 1024), gdn.GDN_ERR_INVALID_ARG),             # state overlaps the snapshots
])
def test_state_select_rejects(lib, kw, status):
    assert _select(lib, **kw) == status


def _bwd(lib, q=A, k=A + 64 * MB, v=A + 128 * MB, g=A + 192 * MB, beta=A + 256 * MB, s_in=None,
         do=A + 320 * MB, ds_out=None, dq=A + 512 * MB, dk=A + 576 * MB, dv=A + 640 * MB,
         dg=A + 704 * MB, dbeta=A + 768 * MB, ds_in=None, B=1, T=16, H=1, Dk=128, Dv=128, gate=1):
    c = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.gdn_chunk_bwd(c(q), c(k), c(v), c(g), c(beta), c(s_in), c(do), c(ds_out), c(dq), c(dk),
                             c(dv), c(dg), c(dbeta), c(ds_in), B, T, H, Dk, Dv, gate, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(do=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dg=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(T=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(gate=7), gdn.GDN_ERR_INVALID_ARG),
    (dict(Dk=48), gdn.GDN_ERR_UNSUPPORTED),
    (dict(H=70000), gdn.GDN_ERR_UNSUPPORTED),
    (dict(do=A + 320 * MB + 4), gdn.GDN_ERR_MISALIGNED),
    (dict(dg=A + 704 * MB + 4), gdn.GDN_ERR_MISALIGNED),          # per-channel dg: 16 bytes
    (dict(dq=A + 64), gdn.GDN_ERR_INVALID_ARG),                   # dq overlaps q
    (dict(dv=A + 576 * MB + 32), gdn.GDN_ERR_INVALID_ARG),        # dv overlaps dk
    (dict(ds_in=A + 320 * MB), gdn.GDN_ERR_INVALID_ARG),          # d_state_in overlaps d_out
])
def test_chunk_bwd_rejects(lib, kw, status):
    assert _bwd(lib, **kw) == status


def test_decoupled_steps_rejects(lib):
    c = ctypes.c_void_p
    call = lambda bw, out=A + 448 * MB, T=4: lib.gdn_recurrent_steps_decoupled(  # noqa: E731
        c(A), c(A + 64 * MB), c(A + 128 * MB), c(A + 192 * MB), c(A + 256 * MB),
        None if bw is None else c(bw), c(A + 320 * MB), c(A + 320 * MB), None, c(out),
        1, T, 1, 128, 128, 1, None)
    assert call(None) == gdn.GDN_ERR_INVALID_ARG                  # the write gate is required
    assert call(A + 300 * MB + 2) == gdn.GDN_ERR_MISALIGNED
    assert call(A + 448 * MB) == gdn.GDN_ERR_INVALID_ARG          # overlaps out
    assert call(A + 300 * MB, T=0) == gdn.GDN_ERR_INVALID_ARG
    assert call(A + 300 * MB, out=A + 16) == gdn.GDN_ERR_INVALID_ARG   # out overlaps q
