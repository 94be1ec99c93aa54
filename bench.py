"""Benchmark of the Gated DeltaNet hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one chunkwise prefill (gdn_chunk_fwd) of the GDN-2 layer workload:
B=8 sequences, H=8 heads, T=2048 tokens, dk=dv=128, bf16 q/k/v, per-channel
gate g in [-5, 0], beta = sigmoid(N(0,1)), zero initial state, fp32 state
and output.  Inputs are synthetic (seeded recipe in synth/), resident in HBM
when the timed region starts; they total 235 MB per step, more than the
126 MB L2, so no L2 flush is needed between steps.

The same run also measures the decode mode (gdn_recurrent_step) on its own
workload -- B=64 sequences, H=16, d=128, per-channel gate, fp32 state
carried in place -- with L2 flushed before every timed step (the 64 MiB
state would otherwise stay in the 126 MB L2), reported under "decode".

Measured beside them, each as its own object of the same JSON line:
  "prologue"            the input prologue: the prefill pass (gdn_prologue) on
                        the GDN-2 layer shape and the decode step with the
                        prologue fused in (gdn_recurrent_step_prologue);
  "multi_token_decode"  4 draft tokens with per-token state snapshots;
  "backward"            the prefill gradients (gdn_chunk_bwd), GDN-2 layer shape;
  "decoupled_decode"    a decode step with separate erase and write gates;
  "long_context"        one sequence of 262,144 tokens over 16 heads through
                        the segment-parallel path.

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
GPU (weak scaling, no collective on the data path); the reported time is
the max over ranks.  Prints one JSON line on rank 0.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the reference arm of this comparison).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))

import numpy as np  # noqa: E402
import torch  # noqa: E402

from synth import CONFIGS, config_inputs, prologue_inputs  # noqa: E402

PREFILL_CFG = CONFIGS[2]
DECODE_CFG = CONFIGS[4]
LONG_CFG = CONFIGS[5]
L2_BYTES = 126 * 1024 * 1024
METRIC = "GDN prefill tokens/s + % tensor roofline; decode state GB/s vs HBM peak"
PROFILE_SUMMARY = ROOT / "profiles" / "chunk_pool_kernel_gdn2_layer_B8H8T2048.md"
# The sources the prefill kernel of this workload is compiled from (a cluster
# of two CTAs per (batch, head): 2 * B * H = 128 <= 148 SMs).
KERNEL_SOURCES = ("chunk_pair_sm100.cu", "chunk_common.cuh", "sm100_util.cuh")


# ---------------------------------------------------------------- accounting --
def prefill_bytes(cfg, with_state_in: bool) -> int:
    """Algorithmic HBM bytes of one prefill call: every input read once,
    every output written once (q,k,v bf16; g, beta fp32; out fp32; states)."""
    th = cfg.B * cfg.T * cfg.H
    per = 2 * cfg.dk + 2 * cfg.dk + 2 * cfg.dv + 4 * (cfg.dk if cfg.per_channel else 1) + 4 + 4 * cfg.dv
    st = cfg.B * cfg.H * cfg.dk * cfg.dv * 4
    return th * per + st * (2 if with_state_in else 1)


def prefill_flops(cfg, C: int = 64) -> float:
    """Algorithmic flops per token-head of the chunk algebra: 3 C dk + 2 C dv
    + C^2 / 3 + 6 dk dv (the triangular halves only; wasted tile work and the
    extra passes of split-precision operands are not counted)."""
    per = 3 * C * cfg.dk + 2 * C * cfg.dv + C * C / 3 + 6 * cfg.dk * cfg.dv
    return per * cfg.B * cfg.T * cfg.H


def decode_bytes(cfg) -> int:
    bh = cfg.B * cfg.H
    state = 2 * bh * cfg.dk * cfg.dv * 4
    qkv = bh * (2 * cfg.dk + cfg.dv) * 2
    g = bh * (cfg.dk if cfg.per_channel else 1) * 4
    return state + qkv + g + bh * 4 + bh * cfg.dv * 4


def measured_peaks() -> dict:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def kernel_source_sha1() -> str:
    """sha1 over the prefill kernel's source files, in KERNEL_SOURCES order."""
    import hashlib
    h = hashlib.sha1()
    for name in KERNEL_SOURCES:
        h.update((ROOT / "gated_delta_rule_77_b200" / "csrc" / name).read_bytes())
    return h.hexdigest()


def ncu_traffic():
    """dram read+write bytes per launch of the chunk kernel from the committed
    ncu summary, or None when the kernel source changed since that capture
    (the summary records the sha1 of the sources it measured)."""
    if not PROFILE_SUMMARY.exists():
        return None
    fields = {}
    for line in PROFILE_SUMMARY.read_text().splitlines():
        if ":" in line and not line.startswith(("|", " ", "#")):
            key, val = line.split(":", 1)
            fields[key.strip()] = val.strip()
    if fields.get("kernel_source_sha1") != kernel_source_sha1():
        return None
    try:
        return float(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- clocks --------
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.index = index
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.error = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:  # pragma: no cover - NVML missing
            self.error = repr(e)
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception as e:  # pragma: no cover
                self.error = repr(e)
                return
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self) -> dict:
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                **({"error": self.error} if self.error else {})}


# ---------------------------------------------------------------- distributed ---
def dist_setup(n_gpus: int, backend: str | None = None):
    """Process-group set-up for torchrun launches; returns (rank, world, local).
    NCCL on GPUs (one process per GPU), gloo otherwise or when asked."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    if world != n_gpus and rank == 0:
        print(f"warning: --gpus {n_gpus} but WORLD_SIZE={world}", file=sys.stderr)
    return rank, world, local


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank scalar (timings are reported as the slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- CPU oracle ----
def oracle_sample(cfg, n_pairs: int, threads: int):
    """Times the fp64 oracle on the first n_pairs (b, h) pairs of the workload;
    returns (seconds, equivalent tokens) where tokens = pairs * T / H."""
    import oracle
    x = config_inputs(cfg, B=max(1, -(-n_pairs // cfg.H)))
    f = {k: (None if v is None else np.ascontiguousarray(v.double().numpy())) for k, v in x.items()}
    heads = list(range(n_pairs))
    t0 = time.perf_counter()
    oracle.run(f["q"], f["k"], f["v"], f["g"], f["beta"], f["s0"], per_channel=cfg.per_channel,
               heads=heads, threads=threads)
    dt = time.perf_counter() - t0
    return dt, n_pairs * cfg.T / cfg.H


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    cfg = PREFILL_CFG
    cores = cpu_cores()
    n_pairs = min(cfg.B * cfg.H, cores)
    for _ in range(args.warmup):
        oracle_sample(cfg, n_pairs, cores)
    total_t = 0.0
    total_tok = 0.0
    for _ in range(args.steps):
        dt, tok = oracle_sample(cfg, n_pairs, cores)
        total_t += dt
        total_tok += tok
    value = total_tok / total_t
    sample = (f"{n_pairs} (b,h) pairs x T={cfg.T} per step of the {cfg.name} workload, fp64, "
              f"one pair per thread")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def workload_config(cfg) -> dict:
    return {"workload": "GDN-2 layer prefill (chunkwise, per-channel gate)", "B": cfg.B,
            "H": cfg.H, "T": cfg.T, "dk": cfg.dk, "dv": cfg.dv, "gate": cfg.gate,
            "inputs": "bf16 q/k/v, fp32 g/beta, zero initial state, fp32 state and output",
            "chunk": 64,
            "l2": f"inputs {prefill_bytes(cfg, False) / 1e6:.0f} MB per step > 126 MB L2 (no flush)"}


# ---------------------------------------------------------------- GPU arm -------
def time_events(fn, steps: int, stream) -> float:
    """Seconds for `steps` calls of fn, CUDA events on the launching stream."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / 1e3


def run_ours(args, rank: int, world: int, local: int):
    import gated_delta_rule_77_b200 as gdn
    gdn.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()
    cfg = PREFILL_CFG

    x = config_inputs(cfg, seed=cfg.index + 1000 * rank)
    q, k, v, g, beta = (x[n].to(dev) for n in ("q", "k", "v", "g", "beta"))
    out = torch.empty(cfg.B, cfg.T, cfg.H, cfg.dv, dtype=torch.float32, device=dev)
    s_out = torch.empty(cfg.B, cfg.H, cfg.dk, cfg.dv, dtype=torch.float32, device=dev)

    def step():
        gdn.chunk_fwd(q, k, v, g, beta, None, out=out, state_out=s_out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        dt = time_events(step, args.steps, stream)
    torch.cuda.synchronize()
    barrier(world)
    dt = max_over_ranks(dt, world)
    if gdn.check(stream) != gdn.GDN_OK:
        raise RuntimeError("the chunk kernel reported an abandoned wait")

    tokens = cfg.B * cfg.T * args.steps * world
    value = tokens / dt
    t_launch = dt / args.steps
    nbytes = prefill_bytes(cfg, False)
    nflops = prefill_flops(cfg)
    achieved_gbs = nbytes / t_launch / 1e9
    traffic = ncu_traffic()
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": traffic,
                "kernel": "chunk_pool_kernel<per-channel>", "bytes_per_launch": nbytes,
                "peak_source": peaks["source"]}
    tflops = nflops / t_launch / 1e12
    tensor = {"achieved_tflops": tflops, "peak_tflops": peaks["bf16_tflops"],
              "frac": tflops / peaks["bf16_tflops"], "flops_per_launch": nflops,
              "attainable_frac": min(1.0, (nbytes / (peaks["hbm_gbs"] * 1e9)) / t_launch)}

    # End to end through the public API with pinned host buffers: every step
    # copies its inputs host -> device, runs the call and copies its output
    # device -> host, all inside the timed region.  Two device buffer sets and
    # separate copy streams let step i + 1's upload and step i's download
    # overlap step i's compute (PCIe is full duplex); the timed region runs
    # from before the first upload to after the last download.
    host = {n: x[n].pin_memory() for n in ("q", "k", "v", "g", "beta")}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size()
    sets = [dict(q=q, k=k, v=v, g=g, beta=beta, out=out, s_out=s_out)]
    sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in sets]      # inputs of a set uploaded
    ev_done = [torch.cuda.Event() for _ in sets]    # call on a set finished
    ev_out = [torch.cuda.Event() for _ in sets]     # output of a set downloaded
    for i in range(2):                              # all events start recorded
        ev_done[i].record(stream)
        ev_out[i].record(stream)

    def e2e_step(i):
        st = sets[i % 2]
        up.wait_event(ev_done[i % 2])               # the set's previous call read its inputs
        with torch.cuda.stream(up):
            for n in ("q", "k", "v", "g", "beta"):
                st[n].copy_(host[n], non_blocking=True)
        ev_in[i % 2].record(up)
        stream.wait_event(ev_in[i % 2])
        stream.wait_event(ev_out[i % 2])            # the set's previous output was downloaded
        gdn.chunk_fwd(st["q"], st["k"], st["v"], st["g"], st["beta"], None, out=st["out"],
                      state_out=st["s_out"], stream=stream)
        ev_done[i % 2].record(stream)
        down.wait_event(ev_done[i % 2])
        with torch.cuda.stream(down):
            out_h.copy_(st["out"], non_blocking=True)
        ev_out[i % 2].record(down)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e2e_steps = max(2, min(args.steps, 10))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(up)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(down)
    e1.synchronize()
    dt_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    e2e = {"value": cfg.B * cfg.T * e2e_steps * world / dt_e2e, "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "overlap": "two buffer sets; uploads, calls and downloads on three streams"}

    decode = run_decode(gdn, dev, stream, peaks, world, rank)
    prologue = run_prologue(gdn, dev, stream, peaks, world, rank)
    multitoken = run_multitoken(gdn, dev, stream, peaks, world, rank)
    backward = run_backward(gdn, dev, stream, peaks, world, rank)
    decoupled = run_decoupled(gdn, dev, stream, peaks, world, rank)
    long_context = run_long_context(gdn, dev, stream, peaks, world, rank)

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cores = cpu_cores()
            n_pairs = cfg.B * cfg.H
            cdt, ctok = oracle_sample(cfg, n_pairs, cores)
            cpu = {"value": ctok / cdt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                   "sample": f"the full workload once ({n_pairs} (b,h) pairs x T={cfg.T}), fp64, "
                             f"{cdt:.1f} s wall on {cores} threads"}
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_launch,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "config": workload_config(cfg), "roofline": roofline,
                "tensor": tensor, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": args.steps, "clocks": clk.summary(), "decode": decode,
                "prologue": prologue, "multi_token_decode": multitoken, "backward": backward,
                "decoupled_decode": decoupled, "long_context": long_context}
        print(json.dumps(line))
    return 0


def prologue_bytes(B, T, H, dk, dv, per_channel: bool) -> int:
    """Algorithmic HBM bytes of one prologue pass: per token-head the raw
    q, k, v (bf16) read and q, k, v written (bf16), g read and written (fp32,
    dk values per channel gate or 1), beta read and written (fp32); per
    (b, h) three ring slots read and min(T, 4) written (fp32); the taps once."""
    C = 2 * dk + dv
    gate = dk if per_channel else 1
    per_tok = 2 * (2 * C) + 2 * 4 * gate + 2 * 4
    return B * T * H * per_tok + B * H * (3 + min(T, 4)) * C * 4 + H * C * 4 * 4


def run_prologue(gdn, dev, stream, peaks, world, rank, steps: int = 20, warmup: int = 3):
    """The prologue's two forms, each timed alone (median of single-launch
    CUDA-event timings).  The prefill pass moves 337 MB, more than L2; the
    decode step's state is evicted from L2 before every timed step."""
    pc = PREFILL_CFG
    x = prologue_inputs(pc.B, pc.T, pc.H, pc.dk, pc.dv, gate=pc.gate, seed=pc.index + 1000 * rank)
    xd = {n: (None if t is None else t.to(dev)) for n, t in x.items()}
    args = [xd[n] for n in ("q_raw", "k_raw", "v_raw", "g_raw", "beta_raw", "conv_w")]
    times = []
    for i in range(warmup + steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gdn.prologue(*args, xd["ring"], xd["pos0"], stream=stream)
        e1.record(stream)
        e1.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1) / 1e3)
    t_pre = max_over_ranks(statistics.median(times), world)
    b_pre = prologue_bytes(pc.B, pc.T, pc.H, pc.dk, pc.dv, pc.per_channel)
    del xd, args

    dc = DECODE_CFG
    y = prologue_inputs(dc.B, 4, dc.H, dc.dk, dc.dv, gate=dc.gate, seed=dc.index + 1000 * rank)
    yd = {n: t.to(dev) for n, t in y.items()}
    state = torch.zeros(dc.B, dc.H, dc.dk, dc.dv, dtype=torch.float32, device=dev)
    out = torch.empty(dc.B, dc.H, dc.dv, dtype=torch.float32, device=dev)
    steps_in = [[yd[n][:, j].contiguous() for n in ("q_raw", "k_raw", "v_raw", "g_raw",
                                                    "beta_raw")] for j in range(4)]
    pos = [yd["pos0"] + j for j in range(warmup + steps)]
    flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    times = []
    for i in range(warmup + steps):
        torch.sum(flush, dim=0, out=sink)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gdn.recurrent_step_prologue(*steps_in[i % 4], yd["conv_w"], yd["ring"], state, pos[i],
                                    out=out, stream=stream)
        e1.record(stream)
        e1.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1) / 1e3)
    t_dec = max_over_ranks(statistics.median(times), world)
    C = 2 * dc.dk + dc.dv
    b_dec = (decode_bytes(dc) + dc.B * dc.H * (3 + 1) * C * 4 + dc.H * C * 16)
    hbm = peaks["hbm_gbs"]
    return {
        "prefill_pass": {"kernel": "prologue_kernel + prologue_ring_kernel",
                         "us": t_pre * 1e6, "bytes": b_pre, "GB/s": b_pre / t_pre / 1e9,
                         "frac": b_pre / t_pre / 1e9 / hbm, "peak": hbm,
                         "config": {"workload": "input prologue of the GDN-2 layer prefill",
                                    "B": pc.B, "T": pc.T, "H": pc.H, "dk": pc.dk, "dv": pc.dv,
                                    "gate": pc.gate, "activation": "silu", "ring": True}},
        "decode_fused": {"kernel": "recurrent_prologue_kernel", "us_per_step": t_dec * 1e6,
                         "bytes": b_dec, "GB/s": b_dec / t_dec / 1e9,
                         "frac": b_dec / t_dec / 1e9 / hbm, "peak": hbm,
                         "config": {"workload": "decode step with the prologue fused in",
                                    "B": dc.B, "H": dc.H, "dk": dc.dk, "dv": dc.dv,
                                    "gate": dc.gate, "l2": "evicted before every timed step"}},
        "timing": f"median of {steps} single-launch CUDA-event timings each"}


def backward_flops(cfg, C: int = 32) -> float:
    """fp32 multiply-adds x 2 of the chunkwise backward per launch, counted
    from its products per 32-token chunk: 10 C dk dv (state-sized products in
    the two chains and the gradient pass) + C^2 (9 dk + 7 dv) (chunk-local
    products), plus the C^3 / 3 solve twice."""
    n_chunks = cfg.B * cfg.H * -(-cfg.T // C)
    macs = 10 * C * cfg.dk * cfg.dv + C * C * (9 * cfg.dk + 7 * cfg.dv) + 2 * C ** 3 / 3
    return 2.0 * macs * n_chunks


def run_backward(gdn, dev, stream, peaks, world, rank, steps: int = 10, warmup: int = 3):
    """gdn_chunk_bwd on the GDN-2 layer shape.  Its products run on the
    tensor cores (mma.sync, bf16 operands split hi + lo, three passes), so
    the roofline is the measured dense bf16 peak, against the algorithmic
    flops of one pass."""
    from synth import grad_inputs, prefill_inputs
    cfg = PREFILL_CFG
    x = prefill_inputs(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, gate=cfg.gate, s0_std=0.1,
                       seed=cfg.index + 1000 * rank)
    do, dsT = grad_inputs(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, seed=cfg.index + 1000 * rank)
    d = {n: x[n].to(dev) for n in ("q", "k", "v", "g", "beta", "s0")}
    do, dsT = do.to(dev), dsT.to(dev)
    times = []
    for i in range(warmup + steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gdn.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["s0"], do, dsT, stream=stream)
        e1.record(stream)
        e1.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1) / 1e3)
    t = max_over_ranks(statistics.median(times), world)
    fl = backward_flops(cfg)
    peak = peaks["bf16_tflops"]
    return {"metric": "prefill backward tokens/s", "value": cfg.B * cfg.T * world / t,
            "unit": "tokens/s", "ms_per_call": t * 1e3,
            "roofline": {"bound": "tensor", "achieved": fl / t / 1e12, "peak": peak,
                         "unit": "TFLOP/s", "frac": fl / t / 1e12 / peak, "flops_per_call": fl,
                         "peak_source": peaks["source"]},
            "config": {"workload": "GDN-2 layer prefill gradients (dq, dk, dv, dg, dbeta, dS0)",
                       "B": cfg.B, "H": cfg.H, "T": cfg.T, "dk": cfg.dk, "dv": cfg.dv,
                       "gate": cfg.gate, "chunk": 32},
            "timing": f"median of {steps} single-call CUDA-event timings"}


def run_multitoken(gdn, dev, stream, peaks, world, rank, T: int = 4, steps: int = 20,
                   warmup: int = 3):
    """Multi-token decode (T draft tokens per sequence, state after every
    token kept) on the decode shape, L2 evicted before every timed call."""
    from synth import prefill_inputs
    cfg = DECODE_CFG
    x = prefill_inputs(cfg.B, T, cfg.H, cfg.dk, cfg.dv, gate=cfg.gate, s0_std=cfg.s0_std,
                       seed=cfg.index + 1000 * rank)
    d = {n: x[n].to(dev) for n in ("q", "k", "v", "g", "beta", "s0")}
    snap = torch.empty(cfg.B, T, cfg.H, cfg.dk, cfg.dv, dtype=torch.float32, device=dev)
    out = torch.empty(cfg.B, T, cfg.H, cfg.dv, dtype=torch.float32, device=dev)
    flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    times = []
    for i in range(warmup + steps):
        torch.sum(flush, dim=0, out=sink)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], d["s0"], snapshots=snap,
                            out=out, stream=stream)
        e1.record(stream)
        e1.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1) / 1e3)
    t = max_over_ranks(statistics.median(times), world)
    bh = cfg.B * cfg.H
    st = cfg.dk * cfg.dv * 4
    per_tok = 2 * (2 * cfg.dk + cfg.dv) + 4 * (cfg.dk if cfg.per_channel else 1) + 4 + 4 * cfg.dv
    nbytes = bh * (st + T * st + T * per_tok)
    gbs = nbytes / t / 1e9
    return {"metric": "multi-token decode GB/s", "value": gbs, "unit": "GB/s",
            "us_per_call": t * 1e6, "frac": gbs / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"],
            "bytes_per_call": nbytes, "tokens_per_s": cfg.B * T * world / t,
            "config": {"workload": "multi-token decode with per-token state snapshots",
                       "B": cfg.B, "H": cfg.H, "T": T, "dk": cfg.dk, "dv": cfg.dv,
                       "gate": cfg.gate, "l2": "evicted before every timed call"},
            "timing": f"median of {steps} single-call CUDA-event timings"}


def run_long_context(gdn, dev, stream, peaks, world, rank, steps: int = 3, warmup: int = 2):
    """The long-context prefill (one sequence of 262,144 tokens, 16 heads,
    scalar gate with 10% g = 0) through the automatic segment-parallel path;
    inputs 3.4 GB, far above L2."""
    cfg = LONG_CFG
    x = config_inputs(cfg, seed=cfg.index + 1000 * rank)
    q, k, v, g, beta = (x[n].to(dev) for n in ("q", "k", "v", "g", "beta"))
    del x
    out = torch.empty(cfg.B, cfg.T, cfg.H, cfg.dv, dtype=torch.float32, device=dev)
    s_out = torch.empty(cfg.B, cfg.H, cfg.dk, cfg.dv, dtype=torch.float32, device=dev)
    times = []
    for i in range(warmup + steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gdn.chunk_fwd(q, k, v, g, beta, None, out=out, state_out=s_out, stream=stream)
        e1.record(stream)
        e1.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1) / 1e3)
    if gdn.check(stream) != gdn.GDN_OK:
        raise RuntimeError("the long-context prefill reported an abandoned wait")
    t = max_over_ranks(statistics.median(times), world)
    nbytes = prefill_bytes(cfg, False)
    return {"metric": "long-context prefill tokens/s", "value": cfg.B * cfg.T * world / t,
            "unit": "tokens/s", "ms_per_call": t * 1e3,
            "roofline": {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": nbytes / t / 1e9 / peaks["hbm_gbs"],
                         "bytes_per_call": nbytes},
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "T": cfg.T, "dk": cfg.dk,
                       "dv": cfg.dv, "gate": cfg.gate, "path": "segment-parallel (automatic)"},
            "timing": f"median of {steps} single-call CUDA-event timings"}


def run_decoupled(gdn, dev, stream, peaks, world, rank, steps: int = 20, warmup: int = 3):
    """One decode step with separate erase and write gates on the decode
    shape (state in place, L2 evicted before every timed step)."""
    from synth import prefill_inputs, write_gate
    cfg = DECODE_CFG
    x = prefill_inputs(cfg.B, 1, cfg.H, cfg.dk, cfg.dv, gate=cfg.gate, s0_std=cfg.s0_std,
                       seed=cfg.index + 1000 * rank)
    d = {n: x[n].to(dev) for n in ("q", "k", "v", "g", "beta", "s0")}
    bw = write_gate(cfg.B, 1, cfg.H, seed=cfg.index + 1000 * rank).to(dev)
    out = torch.empty(cfg.B, 1, cfg.H, cfg.dv, dtype=torch.float32, device=dev)
    state = d["s0"]
    flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    times = []
    for i in range(warmup + steps):
        torch.sum(flush, dim=0, out=sink)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], state, state_out=state,
                            snapshots=None, out=out, beta_write=bw, stream=stream)
        e1.record(stream)
        e1.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1) / 1e3)
    t = max_over_ranks(statistics.median(times), world)
    nbytes = decode_bytes(cfg) + cfg.B * cfg.H * 4
    gbs = nbytes / t / 1e9
    return {"metric": "decoupled-gate decode state GB/s", "value": gbs, "unit": "GB/s",
            "us_per_step": t * 1e6, "frac": gbs / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"],
            "bytes_per_step": nbytes,
            "config": {"workload": "decode step, separate erase and write gates", "B": cfg.B,
                       "H": cfg.H, "dk": cfg.dk, "dv": cfg.dv, "gate": cfg.gate,
                       "l2": "evicted before every timed step"},
            "timing": f"median of {steps} single-step CUDA-event timings"}


def run_decode(gdn, dev, stream, peaks, world, rank, steps: int = 20, warmup: int = 3):
    """Decode-mode step time with L2 flushed before each timed step."""
    cfg = DECODE_CFG
    x = config_inputs(cfg, steps=4, seed=cfg.index + 1000 * rank)
    q, k, v, g, beta = (x[n].to(dev) for n in ("q", "k", "v", "g", "beta"))
    state = x["s0"].to(dev)
    out = torch.empty(cfg.B, cfg.H, cfg.dv, dtype=torch.float32, device=dev)
    # Evict the state from L2 by reading a buffer twice its size: a read
    # leaves L2 clean, so the timed step pays for its own traffic only.
    flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    times = []
    for i in range(warmup + steps):
        torch.sum(flush, dim=0, out=sink)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gdn.recurrent_step(q[i % 4], k[i % 4], v[i % 4], g[i % 4], beta[i % 4], state, out=out,
                           stream=stream)
        e1.record(stream)
        e1.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1) / 1e3)
    t = max_over_ranks(statistics.median(times), world)
    nbytes = decode_bytes(cfg)
    gbs = nbytes / t / 1e9
    return {"metric": "decode state GB/s", "value": gbs, "unit": "GB/s",
            "us_per_step": t * 1e6, "frac": gbs / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"],
            "bytes_per_step": nbytes, "tokens_per_s": cfg.B * world / t,
            "config": {"workload": "recurrent decode step", "B": cfg.B, "H": cfg.H, "dk": cfg.dk,
                       "dv": cfg.dv, "gate": cfg.gate, "state": "fp32 in place",
                       "l2": "evicted before every timed step by reading 2x L2 (state 64 MiB < L2)"},
            "timing": f"median of {steps} single-step CUDA-event timings"}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            return run_reference(args, rank, world)
        return run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
