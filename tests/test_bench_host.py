"""Host-side logic of bench.py (CPU only): algorithmic byte / flop accounting,
the reference arm's JSON line, and the max-over-ranks timing with two gloo
ranks."""
import dataclasses
import json
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
from synth import CONFIGS


def test_prefill_accounting_matches_hand_count():
    cfg = CONFIGS[2]
    th = 8 * 2048 * 8                       # token-heads
    per = 256 + 256 + 256 + 512 + 4 + 512   # q, k, v bf16; g, beta, out fp32
    assert bench.prefill_bytes(cfg, False) == th * per + 8 * 8 * 128 * 128 * 4
    assert bench.prefill_flops(cfg) == pytest.approx(th * (3 * 64 * 128 + 2 * 64 * 128 + 64 * 64 / 3
                                                            + 6 * 128 * 128))


def test_algorithmic_bytes_match_the_per_token_head_figures():
    # q, k, v 768 B + g 4 B (scalar) + beta 4 B + out 256 B (bf16) per
    # token-head, plus the final state (64 KiB per (b, h)); S0 = 0 is not read.
    assert bench.algorithmic_bytes(CONFIGS[5]) == 262144 * 16 * 1032 + 16 * 65536
    # Per-channel g is 512 B per token-head.
    assert bench.algorithmic_bytes(CONFIGS[2]) == 8 * 2048 * 8 * 1540 + 64 * 65536
    # S0 != 0 is read as well as S_T written.
    assert bench.algorithmic_bytes(CONFIGS[3]) == 4 * 8192 * 12 * 1032 + 2 * 48 * 65536


def test_chunk_path_kernels_follow_the_dispatch_rule():
    assert len(bench.chunk_path_kernels(CONFIGS[5])) == 3            # 16 pairs: 9 segments
    assert bench.chunk_path_kernels(CONFIGS[2]) == ["chunk_pool_kernel"]   # per-channel, n = 2: pool
    assert len(bench.chunk_path_kernels(dataclasses.replace(CONFIGS[2], B=4, H=12))) == 3   # n = 3
    assert len(bench.chunk_path_kernels(CONFIGS[3])) == 3            # scalar, 48 pairs: 3 segments
    scalar = CONFIGS[3]
    # scalar gate, 2 segments: taken with 64 pairs (128 of 148 SMs), not with 50 (100 SMs)
    assert len(bench.chunk_path_kernels(dataclasses.replace(scalar, B=4, H=16, T=2048))) == 3
    assert bench.chunk_path_kernels(dataclasses.replace(scalar, B=5, H=10, T=8192)) == ["chunk_pool_kernel"]
    # too short for segments (31 chunks), and too many pairs for the pool
    assert bench.chunk_path_kernels(dataclasses.replace(scalar, B=4, H=12, T=1984)) == ["chunk_pool_kernel"]
    assert bench.chunk_path_kernels(dataclasses.replace(scalar, B=8, H=12, T=8192)) == ["chunk_fwd_kernel"]


def test_decode_accounting_matches_hand_count():
    # 2 x 64 MiB of state + q,k,v bf16 + per-channel g + beta + fp32 out
    assert bench.decode_bytes(CONFIGS[4]) == 136_056_832


def test_reference_arm_prints_contract_line(capsys, monkeypatch):
    monkeypatch.setattr(bench, "cpu_cores", lambda: 2)
    rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3",
                     "--sample-tokens", "512"])
    assert rc == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["T"] == 262144 and line["config"]["H"] == 16


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, _ = bench.dist_setup(world, backend="gloo")
    try:
        bench.barrier(w)
        q.put((r, bench.max_over_ranks(float(10 + r), w)))
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 11.0), (1, 11.0)]


def test_traffic_figures_follow_the_kernel_and_its_sources(monkeypatch):
    """bench.py reports an ncu traffic figure only for the kernel it was
    captured on and only while the kernel's sources hash as at the capture."""
    entry = json.loads(bench.TRAFFIC_FILE.read_text())["decode"]
    assert bench.ncu_traffic("decode") == float(entry["dram_bytes_per_launch"])
    assert bench.ncu_traffic("no_such_workload") is None
    layer = json.loads(bench.TRAFFIC_FILE.read_text())["gdn2_layer"]
    assert bench.ncu_traffic("gdn2_layer", "chunk_pool_kernel") == float(layer["dram_bytes_per_launch"])
    assert bench.ncu_traffic("gdn2_layer", "chunk_fwd_kernel (zero-start + transition CTAs)") is None
    monkeypatch.setattr(bench, "source_sha1", lambda names: "0" * 40)
    assert bench.ncu_traffic("decode") is None
