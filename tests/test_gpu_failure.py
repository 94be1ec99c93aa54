"""Failure detection on the GPU without a GPU fault: a bounded wait that runs out.

The prep-pool prefill's state chains wait on flags in global memory that prep
CTAs set once a task record is stored.  Two test hooks of the library make
such a wait run out safely: GDN_TEST_WITHHOLD_TASK names one task whose flag
is never set, and GDN_TEST_FLAG_BUDGET_NS shortens the chains' flag-wait
budget (2 s by default) to 2 ms.  Only that flag is withheld: no TMA or
tensor-core completion is held back, and prep CTAs never wait for chains, so
every other wait of the launch ends normally.  The chain whose record never
comes gives up, records the timeout in the device status word, drains its own
copies and returns; ``gdn_check`` then reports GDN_ERR_TIMEOUT, and the next
call on the same context is correct.
"""
import pytest
import torch

import oracle
from synth import prefill_inputs

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _call(gdn, x):
    dev = torch.device("cuda")
    out, s = gdn.chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta")), x["s0"].to(dev))
    return out, s


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("chunk", [0, 2])
def test_withheld_record_times_out_and_the_next_call_is_clean(gdn, gate, chunk, monkeypatch):
    B, T, H = 1, 300, 2                      # 5 chunks per (batch, head); tasks = pair * 5 + chunk
    x = prefill_inputs(B, T, H, 128, 128, gate=gate, s0_std=0.1, seed=500 + chunk)
    assert gdn.check() == gdn.GDN_OK         # nothing pending from earlier tests
    monkeypatch.setenv("GDN_CHUNK_KERNEL", "pool")
    monkeypatch.setenv("GDN_TEST_WITHHOLD_TASK", str(1 * 5 + chunk))   # pair 1
    monkeypatch.setenv("GDN_TEST_FLAG_BUDGET_NS", "2000000")
    out, _ = _call(gdn, x)
    assert gdn.check() == gdn.GDN_ERR_TIMEOUT
    # Pair 0 never waited on the withheld flag: its outputs are complete.
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                              per_channel=gate == "channel")
    assert oracle.rel_err(out[:, :, 0].cpu(), ref_o[:, :, 0]) <= TOL
    assert gdn.check() == gdn.GDN_OK         # the status word was cleared by the read

    monkeypatch.delenv("GDN_TEST_WITHHOLD_TASK")
    monkeypatch.delenv("GDN_TEST_FLAG_BUDGET_NS")
    out, s = _call(gdn, x)
    assert gdn.check() == gdn.GDN_OK
    assert oracle.rel_err(out.cpu(), ref_o) <= TOL
    assert oracle.rel_err(s.cpu(), ref_s) <= TOL


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_pool_without_scratch_falls_back_to_the_cluster_form(gdn, gate, monkeypatch):
    """GDN_TEST_FAIL_WORKSPACE makes the library's scratch allocation fail, as
    on a full device.  The unsegmented prefill then runs the cluster form,
    which needs no scratch, and still returns the right answer; the segment
    path, which cannot run without scratch, reports GDN_ERR_NOMEM."""
    x = prefill_inputs(2, 300, 3, 128, 128, gate=gate, s0_std=0.1, seed=510)
    monkeypatch.setenv("GDN_TEST_FAIL_WORKSPACE", "1")
    out, s = _call(gdn, x)
    assert gdn.check() == gdn.GDN_OK
    ref_o, ref_s = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["s0"],
                              per_channel=gate == "channel")
    assert oracle.rel_err(out.cpu(), ref_o) <= TOL
    assert oracle.rel_err(s.cpu(), ref_s) <= TOL
    dev = torch.device("cuda")
    with pytest.raises(gdn.GdnError) as err:
        gdn.chunk_fwd(*(x[n].to(dev) for n in ("q", "k", "v", "g", "beta")), x["s0"].to(dev),
                      segments=3)
    assert err.value.status == gdn.GDN_ERR_NOMEM
    monkeypatch.delenv("GDN_TEST_FAIL_WORKSPACE")
    out, s = _call(gdn, x)
    assert gdn.check() == gdn.GDN_OK
    assert oracle.rel_err(out.cpu(), ref_o) <= TOL
