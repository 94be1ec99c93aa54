"""Benchmark of the Gated DeltaNet hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one chunkwise prefill (gdn_chunk_fwd) of the largest workload that
fits one GPU, the long-context prefill: B=1 sequence of T=262,144 tokens,
H=16 heads, dk=dv=128, bf16 q/k/v, scalar gate per head with 10% of tokens
g=0 and the rest g=-min(softplus(N(0,1)),5), beta=sigmoid(N(0,1)), zero
initial state, fp32 state carried across chunks, fp32 output.  Inputs are
synthetic (seeded recipe in synth/) and resident in HBM when the timed region
starts; at 3.4 GB per step they are far above the 126 MB L2, so no flush is
needed.  The library picks its segment-parallel path for this shape.

The JSON line also carries, as compact objects:
  "prefill"  the two other prefill workloads (GDN-2 layer B8 H8 T2048 with a
             per-channel gate; scalar gate B4 H12 T8192 with S0 != 0), each
             with its HBM roofline fraction and the fp64 oracle's tokens/s;
  "next"     the prologue pass, the prefill backward, 4-token decode with
             snapshots and the decoupled-gate decode step;
  "decode"   the decode mode (gdn_recurrent_step): B=64, H=16, d=128,
             per-channel gate, 1024 successive steps captured in one CUDA
             graph, each step on one of 6 rotating 64 MiB states (384 MiB,
             more than 2x L2), so that every step's state read and the
             write-back of its update cross HBM inside the timed region;
             median per step over 5 graph replays.

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
GPU (weak scaling, no collective on the data path); the reported time is the
max over ranks.  Prints one JSON line on rank 0.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the headline workload (the reference arm of this comparison).
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

HEAD_CFG = CONFIGS[5]          # the headline: the largest single-GPU workload
LAYER_CFG = CONFIGS[2]
TRAIN_CFG = CONFIGS[3]
DECODE_CFG = CONFIGS[4]
L2_BYTES = 126 * 1024 * 1024
METRIC = "GDN prefill tokens/s + % tensor roofline; decode state GB/s vs HBM peak"
TRAFFIC_FILE = ROOT / "profiles" / "traffic.json"


def _r(x, n=4):
    """Round to n significant digits (keeps the JSON line short)."""
    if x is None or not isinstance(x, float) or x == 0 or not np.isfinite(x):
        return x
    return float(f"{x:.{n}g}")


# ---------------------------------------------------------------- accounting --
def prefill_bytes(cfg, with_state_in: bool, out_elem_bytes: int = 4) -> int:
    """HBM bytes of one prefill call with every input read once and every
    output written once: q, k, v bf16; g (dk values per channel gate, else 1)
    and beta fp32; out at out_elem_bytes per element; the final state, and the
    initial state when one is read (64 KiB per (b, h) each)."""
    th = cfg.B * cfg.T * cfg.H
    per = 2 * cfg.dk + 2 * cfg.dk + 2 * cfg.dv + 4 * (cfg.dk if cfg.per_channel else 1) + 4
    per += out_elem_bytes * cfg.dv
    st = cfg.B * cfg.H * cfg.dk * cfg.dv * 4
    return th * per + st * (2 if with_state_in else 1)


def algorithmic_bytes(cfg) -> int:
    """The algorithmic bytes of a prefill workload: the per-token-head figure
    (q, k, v 768 B, g 4 or 512 B, beta 4 B, out 256 B as bf16) times the
    token-heads, plus the states read and written once.  The library writes
    its output in fp32 (512 B per token-head); that extra write is not
    counted, so the roofline fraction is conservative."""
    return prefill_bytes(cfg, cfg.s0_std > 0, out_elem_bytes=2)


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


def source_sha1(names) -> str:
    """sha1 over the named kernel sources (gated_delta_rule_77_b200/csrc), in order."""
    import hashlib
    h = hashlib.sha1()
    for name in names:
        h.update((ROOT / "gated_delta_rule_77_b200" / "csrc" / name).read_bytes())
    return h.hexdigest()


def ncu_traffic(key: str, kernel: str | None = None):
    """DRAM read + write bytes per launch of a workload's dominant kernel, from
    the committed ncu figures (profiles/traffic.json), or None when the kernel
    sources changed since that capture (the entry records their sha1) or the
    workload now runs another kernel than the one captured (`kernel`: the
    dominant kernel's name as chunk_path_kernels gives it)."""
    if not TRAFFIC_FILE.exists():
        return None
    entry = json.loads(TRAFFIC_FILE.read_text()).get(key)
    if not entry:
        return None
    try:
        if kernel is not None and entry["kernel"].split("<")[0].split(" ")[0] != kernel.split(" ")[0]:
            return None
        if source_sha1(entry["sources"]) != entry["sources_sha1"]:
            return None
        return float(entry["dram_bytes_per_launch"])
    except (KeyError, OSError, ValueError):
        return None


def chunk_path_kernels(cfg, sms: int = 148) -> list:
    """The kernels one gdn_chunk_fwd call launches for a workload (bf16 I/O,
    d = 128), following the library's automatic choice: the segment-parallel
    path when it picks n > 1 segments (n = #SMs // (B*H) from 32 chunks, when
    n >= 3, or with a scalar gate n = 2 with 2*B*H >= 0.85 #SMs), else the
    prep pool when 2*B*H <= #SMs, else one CTA per (batch, head)."""
    bh = cfg.B * cfg.H
    nchunks = -(-cfg.T // 64)
    n = sms // bh
    two = n == 2 and not cfg.per_channel and 2 * bh * 100 >= 85 * sms
    if nchunks >= 32 and (n >= 3 or two):
        return ["chunk_fwd_kernel (zero-start + transition CTAs)", "combine_segments_kernel",
                "segment_correction_kernel"]
    if 2 * bh <= sms:
        return ["chunk_pool_kernel"]
    return ["chunk_fwd_kernel"]


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
def oracle_sample(cfg, threads: int, n_pairs: int | None = None, T: int | None = None):
    """Times the fp64 oracle on a sample of a workload: the first n_pairs
    (b, h) pairs over the first T tokens (defaults: all).  Returns
    (seconds, tokens) where tokens = pairs * T / H (sequence tokens)."""
    import oracle
    n_pairs = n_pairs or cfg.B * cfg.H
    T = T or cfg.T
    x = config_inputs(cfg, B=max(1, -(-n_pairs // cfg.H)), T=T)
    f = {k: (None if v is None else np.ascontiguousarray(v.double().numpy())) for k, v in x.items()}
    t0 = time.perf_counter()
    oracle.run(f["q"], f["k"], f["v"], f["g"], f["beta"], f["s0"], per_channel=cfg.per_channel,
               heads=list(range(n_pairs)), threads=threads)
    dt = time.perf_counter() - t0
    return dt, n_pairs * T / cfg.H


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# The oracle's bounded sample of the headline workload: every head over the
# first 16,384 tokens (1/16 of the sequence; the recurrence costs the same per
# token everywhere).
HEAD_SAMPLE_T = 16384


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    cfg = HEAD_CFG
    cores = cpu_cores()
    T = args.sample_tokens or HEAD_SAMPLE_T
    for _ in range(args.warmup):
        oracle_sample(cfg, cores, T=T // 4)
    total_t = 0.0
    total_tok = 0.0
    for _ in range(args.steps):
        dt, tok = oracle_sample(cfg, cores, T=T)
        total_t += dt
        total_tok += tok
    value = total_tok / total_t
    sample = (f"all {cfg.B * cfg.H} (b,h) pairs over the first {T} of {cfg.T} tokens per step, "
              f"fp64, one pair per thread")
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
    return {"workload": "long-context prefill (chunkwise, scalar gate, 10% g=0)", "B": cfg.B,
            "H": cfg.H, "T": cfg.T, "dk": cfg.dk, "dv": cfg.dv, "gate": cfg.gate,
            "inputs": "bf16 q/k/v, fp32 g/beta, zero S0, fp32 state and output",
            "chunk": 64, "l2": "inputs 3.4 GB per step > 126 MB L2 (no flush)"}


# ---------------------------------------------------------------- timing helpers -
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


def median_single(fn, stream, steps: int, warmup: int) -> float:
    """Median seconds of single calls, each bracketed by CUDA events."""
    times = []
    for i in range(warmup + steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        e1.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1) / 1e3)
    return statistics.median(times)


def graph_steps(step, n: int, stream, replays: int = 5) -> tuple[float, str]:
    """Per-step seconds of n successive calls step(i, stream) captured in one
    CUDA graph: the median over `replays` replays of (replay time / n), CUDA
    events on the replay stream.  If capture is refused, the n calls are
    timed as plain back-to-back launches instead (same median rule)."""
    s = torch.cuda.Stream()
    s.wait_stream(stream)
    with torch.cuda.stream(s):
        for i in range(3):                   # warm-up outside the graph
            step(i, s)
    s.synchronize()
    how = f"{n} steps in one CUDA graph, median of {replays} replays"
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            for i in range(n):
                step(i, s)
        run = graph.replay
        graph.replay()
    except Exception as e:   # capture refused: plain launches
        torch.cuda.synchronize()
        graph = None
        how = f"{n} back-to-back launches (graph capture failed: {type(e).__name__}), median of {replays}"

        def run():
            for i in range(n):
                step(i, s)
    s.synchronize()
    times = []
    for _ in range(replays):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        with torch.cuda.stream(s):
            run()
        e1.record(s)
        e1.synchronize()
        times.append(e0.elapsed_time(e1) / 1e3 / n)
    del graph
    return statistics.median(times), how


# ---------------------------------------------------------------- GPU arm -------
def run_only(args, local: int):
    """One workload alone, for profiling under ncu (no JSON line): the
    headline prefill (optionally at a shorter T), a prefill workload, or the
    decode graph."""
    import dataclasses
    import gated_delta_rule_77_b200 as gdn
    gdn.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()
    if args.only == "decode":
        print(json.dumps(run_decode(gdn, dev, stream, peaks, 1, 0, n_steps=64)))
        return 0
    cfg = {"long": HEAD_CFG, "layer": LAYER_CFG, "train": TRAIN_CFG}[args.only]
    if args.T:
        cfg = dataclasses.replace(cfg, T=args.T)
    x = config_inputs(cfg)
    q, k, v, g, beta = (x[n].to(dev) for n in ("q", "k", "v", "g", "beta"))
    s0 = x["s0"].to(dev) if x["s0"] is not None else None
    out = torch.empty(cfg.B, cfg.T, cfg.H, cfg.dv, dtype=torch.float32, device=dev)
    s_out = torch.empty(cfg.B, cfg.H, cfg.dk, cfg.dv, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        gdn.chunk_fwd(q, k, v, g, beta, s0, out=out, state_out=s_out, stream=stream)
    t = time_events(lambda: gdn.chunk_fwd(q, k, v, g, beta, s0, out=out, state_out=s_out,
                                          stream=stream), args.steps, stream) / args.steps
    if gdn.check(stream) != gdn.GDN_OK:
        raise RuntimeError("the prefill reported an abandoned wait")
    print(json.dumps({"only": args.only, "T": cfg.T, "us_per_call": t * 1e6,
                      "frac": algorithmic_bytes(cfg) / t / 1e9 / peaks["hbm_gbs"]}))
    return 0


def run_ours(args, rank: int, world: int, local: int):
    import gated_delta_rule_77_b200 as gdn
    gdn.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()
    cfg = HEAD_CFG

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
        raise RuntimeError("the prefill reported an abandoned wait")

    value = cfg.B * cfg.T * args.steps * world / dt
    t_call = dt / args.steps
    nbytes = algorithmic_bytes(cfg)
    nflops = prefill_flops(cfg)
    gbs = nbytes / t_call / 1e9
    roofline = {"bound": "hbm", "achieved": _r(gbs), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": _r(gbs / peaks["hbm_gbs"]), "traffic": ncu_traffic("long_context", chunk_path_kernels(HEAD_CFG)[0]),
                "bytes_per_call": nbytes, "kernels": chunk_path_kernels(cfg),
                "peak_source": peaks["source"]}
    tflops = nflops / t_call / 1e12
    tensor = {"achieved_tflops": _r(tflops), "frac_burst": _r(tflops / peaks["bf16_tflops"]),
              "attainable_frac": _r(min(1.0, (nbytes / (peaks["hbm_gbs"] * 1e9)) / t_call)),
              "flops_per_call": nflops}
    e2e = run_e2e(gdn, dev, stream, x, out, s_out, world, (q, k, v, g, beta))
    del x

    layer = run_prefill(gdn, LAYER_CFG, dev, stream, peaks, world, rank)
    train = run_prefill(gdn, TRAIN_CFG, dev, stream, peaks, world, rank)
    decode = run_decode(gdn, dev, stream, peaks, world, rank)
    nxt = {"prologue": run_prologue(gdn, dev, stream, peaks, world, rank),
           "backward": run_backward(gdn, dev, stream, peaks, world, rank),
           "multi_token_decode": run_multitoken(gdn, dev, stream, peaks, world, rank),
           "decoupled_decode": run_decoupled(gdn, dev, stream, peaks, world, rank)}

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cores = cpu_cores()
            cdt, ctok = oracle_sample(cfg, cores, T=HEAD_SAMPLE_T)
            cpu = {"value": _r(ctok / cdt), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                   "sample": f"all 16 heads over the first {HEAD_SAMPLE_T} tokens, fp64, "
                             f"{cdt:.1f} s on {min(cores, 16)} threads"}
            for sub, c in ((layer, LAYER_CFG), (train, TRAIN_CFG)):
                cdt, ctok = oracle_sample(c, cores)
                sub["cpu_tok_s"] = _r(ctok / cdt)
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_call,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "config": workload_config(cfg), "roofline": roofline,
                "tensor": tensor, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": len(roofline["kernels"]) * args.steps, "clocks": clk.summary(),
                "next": nxt, "prefill": {"gdn2_layer_B8H8T2048": layer,
                                         "scalar_B4H12T8192": train},
                "decode": decode}
        print(json.dumps(line))
    return 0


def run_e2e(gdn, dev, stream, x, out, s_out, world, dev_inputs, steps: int = 3):
    """The headline metric end to end through the public API: every step
    copies its inputs host -> device from pinned memory, runs the call and
    copies the output and final state device -> host, all inside the timed
    region.  Two device buffer sets and separate copy streams let step i + 1's
    upload and step i's download overlap step i's call."""
    cfg = HEAD_CFG
    names = ("q", "k", "v", "g", "beta")
    host = {n: x[n].pin_memory() for n in names}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    s_h = torch.empty(s_out.shape, dtype=s_out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size() + s_h.numel() * s_h.element_size()
    sets = [dict(zip(names, dev_inputs), out=out, s_out=s_out)]
    sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in sets]
    ev_done = [torch.cuda.Event() for _ in sets]
    ev_out = [torch.cuda.Event() for _ in sets]
    for i in range(2):
        ev_done[i].record(stream)
        ev_out[i].record(stream)

    def e2e_step(i):
        st = sets[i % 2]
        up.wait_event(ev_done[i % 2])
        with torch.cuda.stream(up):
            for n in names:
                st[n].copy_(host[n], non_blocking=True)
        ev_in[i % 2].record(up)
        stream.wait_event(ev_in[i % 2])
        stream.wait_event(ev_out[i % 2])
        gdn.chunk_fwd(st["q"], st["k"], st["v"], st["g"], st["beta"], None, out=st["out"],
                      state_out=st["s_out"], stream=stream)
        ev_done[i % 2].record(stream)
        down.wait_event(ev_done[i % 2])
        with torch.cuda.stream(down):
            out_h.copy_(st["out"], non_blocking=True)
            s_h.copy_(st["s_out"], non_blocking=True)
        ev_out[i % 2].record(down)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(up)
    for i in range(steps):
        e2e_step(i)
    e1.record(down)
    e1.synchronize()
    dt = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    del sets
    return {"value": _r(cfg.B * cfg.T * steps * world / dt), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": _r(1e3 * dt / steps), "overlap": "2 buffer sets, 3 streams"}


def run_prefill(gdn, cfg, dev, stream, peaks, world, rank, steps: int = 20, warmup: int = 3):
    """A prefill workload timed as back-to-back calls (inputs exceed L2)."""
    x = config_inputs(cfg, seed=cfg.index + 1000 * rank)
    q, k, v, g, beta = (x[n].to(dev) for n in ("q", "k", "v", "g", "beta"))
    s0 = x["s0"].to(dev) if x["s0"] is not None else None
    del x
    out = torch.empty(cfg.B, cfg.T, cfg.H, cfg.dv, dtype=torch.float32, device=dev)
    s_out = torch.empty(cfg.B, cfg.H, cfg.dk, cfg.dv, dtype=torch.float32, device=dev)

    def step():
        gdn.chunk_fwd(q, k, v, g, beta, s0, out=out, state_out=s_out, stream=stream)

    for _ in range(warmup):
        step()
    t = max_over_ranks(time_events(step, steps, stream) / steps, world)
    if gdn.check(stream) != gdn.GDN_OK:
        raise RuntimeError("the prefill reported an abandoned wait")
    nbytes = algorithmic_bytes(cfg)
    gbs = nbytes / t / 1e9
    key = "gdn2_layer" if cfg is LAYER_CFG else "scalar_train"
    return {"tok_s": _r(cfg.B * cfg.T * world / t), "us": _r(t * 1e6), "GB/s": _r(gbs),
            "frac": _r(gbs / peaks["hbm_gbs"]),
            "tensor_frac": _r(prefill_flops(cfg) / t / 1e12 / peaks["bf16_tflops"]),
            "traffic": ncu_traffic(key, chunk_path_kernels(cfg)[0]), "kernels": chunk_path_kernels(cfg)}


def run_decode(gdn, dev, stream, peaks, world, rank, n_steps: int = 1024, n_states: int = 6,
               n_inputs: int = 128):
    """1024 successive decode steps on rotating states (see the module
    docstring); inputs cycle over 128 distinct steps (170 MB, above L2)."""
    cfg = DECODE_CFG
    x = config_inputs(cfg, steps=n_inputs, seed=cfg.index + 1000 * rank)
    q, k, v, g, beta = (x[n].to(dev) for n in ("q", "k", "v", "g", "beta"))
    states = [x["s0"].to(dev) for _ in range(n_states)]
    outs = [torch.empty(cfg.B, cfg.H, cfg.dv, dtype=torch.float32, device=dev) for _ in range(2)]

    def step(i, s):
        j = i % n_inputs
        gdn.recurrent_step(q[j], k[j], v[j], g[j], beta[j], states[i % n_states],
                           out=outs[i % 2], stream=s)

    t, how = graph_steps(step, n_steps, stream)
    t = max_over_ranks(t, world)
    nbytes = decode_bytes(cfg)
    gbs = nbytes / t / 1e9
    return {"GB/s": _r(gbs), "frac": _r(gbs / peaks["hbm_gbs"]), "us_per_step": _r(t * 1e6),
            "bytes_per_step": nbytes, "tok_s": _r(cfg.B * world / t),
            "traffic": ncu_traffic("decode"),
            "how": f"{how}; {n_states} rotating 64 MiB states (>2x L2)"}


def prologue_bytes(B, T, H, dk, dv, per_channel: bool) -> int:
    """Algorithmic HBM bytes of one prologue pass: per token-head the raw
    q, k, v (bf16) read and q, k, v written (bf16), g read and written (fp32,
    dk values per channel gate or 1), beta read and written (fp32); per
    (b, h) three ring slots read and min(T, 4) written (fp32); the taps once."""
    C = 2 * dk + dv
    gate = dk if per_channel else 1
    per_tok = 2 * (2 * C) + 2 * 4 * gate + 2 * 4
    return B * T * H * per_tok + B * H * (3 + min(T, 4)) * C * 4 + H * C * 4 * 4


def run_prologue(gdn, dev, stream, peaks, world, rank):
    """The prologue's prefill pass at the GDN-2 layer shape (337 MB, above L2;
    median of single launches) and the decode step with the prologue fused in
    (rotating states in one graph, as the plain decode)."""
    pc = LAYER_CFG
    x = prologue_inputs(pc.B, pc.T, pc.H, pc.dk, pc.dv, gate=pc.gate, seed=pc.index + 1000 * rank)
    xd = {n: (None if t is None else t.to(dev)) for n, t in x.items()}
    args = [xd[n] for n in ("q_raw", "k_raw", "v_raw", "g_raw", "beta_raw", "conv_w")]
    t_pre = max_over_ranks(median_single(
        lambda: gdn.prologue(*args, xd["ring"], xd["pos0"], stream=stream), stream, 20, 3), world)
    b_pre = prologue_bytes(pc.B, pc.T, pc.H, pc.dk, pc.dv, pc.per_channel)
    # The same layer from its raw projections in one call: its default route
    # (the two passes through scratch) and the fused kernel (the prologue
    # inside the prefill), against the two calls timed apart.
    out = torch.empty(pc.B, pc.T, pc.H, pc.dv, dtype=torch.float32, device=dev)
    s_out = torch.empty(pc.B, pc.H, pc.dk, pc.dv, dtype=torch.float32, device=dev)
    t_call = max_over_ranks(median_single(
        lambda: gdn.chunk_fwd_prologue(*args, xd["ring"], xd["pos0"], None, out=out, state_out=s_out,
                                       stream=stream), stream, 20, 3), world)
    t_fused = max_over_ranks(median_single(
        lambda: gdn.chunk_fwd_prologue(*args, xd["ring"], xd["pos0"], None, out=out, state_out=s_out,
                                       fused=True, stream=stream), stream, 20, 3), world)
    q, k, v, g, beta = gdn.prologue(*args, xd["ring"], xd["pos0"], stream=stream)
    t_chunk = max_over_ranks(median_single(
        lambda: gdn.chunk_fwd(q, k, v, g, beta, None, out=out, state_out=s_out, stream=stream),
        stream, 20, 3), world)
    del xd, args, q, k, v, g, beta, out, s_out

    dc = DECODE_CFG
    n_in, n_states = 16, 6
    y = prologue_inputs(dc.B, n_in, dc.H, dc.dk, dc.dv, gate=dc.gate, seed=dc.index + 1000 * rank)
    yd = {n: t.to(dev) for n, t in y.items()}
    steps_in = [[yd[n][:, j].contiguous() for n in ("q_raw", "k_raw", "v_raw", "g_raw",
                                                    "beta_raw")] for j in range(n_in)]
    states = [torch.zeros(dc.B, dc.H, dc.dk, dc.dv, dtype=torch.float32, device=dev)
              for _ in range(n_states)]
    rings = [yd["ring"].clone() for _ in range(n_states)]
    out = torch.empty(dc.B, dc.H, dc.dv, dtype=torch.float32, device=dev)

    def step(i, s):
        gdn.recurrent_step_prologue(*steps_in[i % n_in], yd["conv_w"], rings[i % n_states],
                                    states[i % n_states], yd["pos0"], out=out, stream=s)

    t_dec, how = graph_steps(step, 256, stream)
    t_dec = max_over_ranks(t_dec, world)
    C = 2 * dc.dk + dc.dv
    b_dec = decode_bytes(dc) + dc.B * dc.H * (3 + 1) * C * 4 + dc.H * C * 16
    hbm = peaks["hbm_gbs"]
    return {"prefill_pass_us": _r(t_pre * 1e6), "prefill_pass_frac": _r(b_pre / t_pre / 1e9 / hbm),
            "layer_call_us": _r(t_call * 1e6), "fused_kernel_us": _r(t_fused * 1e6),
            "two_calls_us": _r((t_pre + t_chunk) * 1e6),
            "decode_fused_us": _r(t_dec * 1e6), "decode_fused_frac": _r(b_dec / t_dec / 1e9 / hbm)}


def backward_flops(cfg, C: int = 32) -> float:
    """fp32 multiply-adds x 2 of the chunkwise backward per launch, counted
    from its products per 32-token chunk: 10 C dk dv (state-sized products in
    the two chains and the gradient pass) + C^2 (9 dk + 7 dv) (chunk-local
    products), plus the C^3 / 3 solve twice."""
    n_chunks = cfg.B * cfg.H * -(-cfg.T // C)
    macs = 10 * C * cfg.dk * cfg.dv + C * C * (9 * cfg.dk + 7 * cfg.dv) + 2 * C ** 3 / 3
    return 2.0 * macs * n_chunks


def run_backward(gdn, dev, stream, peaks, world, rank):
    """gdn_chunk_bwd on the GDN-2 layer shape (median of single calls);
    roofline: the measured dense bf16 peak against one pass's flops."""
    from synth import grad_inputs, prefill_inputs
    cfg = LAYER_CFG
    x = prefill_inputs(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, gate=cfg.gate, s0_std=0.1,
                       seed=cfg.index + 1000 * rank)
    do, dsT = grad_inputs(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, seed=cfg.index + 1000 * rank)
    d = {n: x[n].to(dev) for n in ("q", "k", "v", "g", "beta", "s0")}
    do, dsT = do.to(dev), dsT.to(dev)
    t = max_over_ranks(median_single(
        lambda: gdn.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["s0"], do, dsT,
                              stream=stream), stream, 10, 3), world)
    fl = backward_flops(cfg)
    return {"ms": _r(t * 1e3), "tok_s": _r(cfg.B * cfg.T * world / t),
            "tensor_frac": _r(fl / t / 1e12 / peaks["bf16_tflops"])}


def run_multitoken(gdn, dev, stream, peaks, world, rank, T: int = 4, n_sets: int = 3):
    """4 draft tokens with per-token snapshots on the decode shape: 64 calls in
    one graph over 3 rotating (state, snapshot) sets (960 MiB)."""
    from synth import prefill_inputs
    cfg = DECODE_CFG
    x = prefill_inputs(cfg.B, T, cfg.H, cfg.dk, cfg.dv, gate=cfg.gate, s0_std=cfg.s0_std,
                       seed=cfg.index + 1000 * rank)
    d = {n: x[n].to(dev) for n in ("q", "k", "v", "g", "beta")}
    states = [x["s0"].to(dev) for _ in range(n_sets)]
    snaps = [torch.empty(cfg.B, T, cfg.H, cfg.dk, cfg.dv, dtype=torch.float32, device=dev)
             for _ in range(n_sets)]
    out = torch.empty(cfg.B, T, cfg.H, cfg.dv, dtype=torch.float32, device=dev)

    def step(i, s):
        gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], states[i % n_sets],
                            snapshots=snaps[i % n_sets], out=out, stream=s)

    t, _ = graph_steps(step, 64, stream)
    t = max_over_ranks(t, world)
    bh = cfg.B * cfg.H
    st = cfg.dk * cfg.dv * 4
    per_tok = 2 * (2 * cfg.dk + cfg.dv) + 4 * (cfg.dk if cfg.per_channel else 1) + 4 + 4 * cfg.dv
    nbytes = bh * (st + T * st + T * per_tok)
    gbs = nbytes / t / 1e9
    return {"us": _r(t * 1e6), "frac": _r(gbs / peaks["hbm_gbs"])}


def run_decoupled(gdn, dev, stream, peaks, world, rank, n_states: int = 6):
    """The decoupled-gate decode step: 256 steps in one graph over 6 rotating
    states (as the plain decode)."""
    from synth import prefill_inputs, write_gate
    cfg = DECODE_CFG
    x = prefill_inputs(cfg.B, 1, cfg.H, cfg.dk, cfg.dv, gate=cfg.gate, s0_std=cfg.s0_std,
                       seed=cfg.index + 1000 * rank)
    d = {n: x[n].to(dev) for n in ("q", "k", "v", "g", "beta")}
    bw = write_gate(cfg.B, 1, cfg.H, seed=cfg.index + 1000 * rank).to(dev)
    states = [x["s0"].to(dev) for _ in range(n_states)]
    out = torch.empty(cfg.B, 1, cfg.H, cfg.dv, dtype=torch.float32, device=dev)

    def step(i, s):
        st = states[i % n_states]
        gdn.recurrent_steps(d["q"], d["k"], d["v"], d["g"], d["beta"], st, state_out=st,
                            snapshots=None, out=out, beta_write=bw, stream=s)

    t, _ = graph_steps(step, 256, stream)
    t = max_over_ranks(t, world)
    nbytes = decode_bytes(cfg) + cfg.B * cfg.H * 4
    gbs = nbytes / t / 1e9
    return {"us": _r(t * 1e6), "frac": _r(gbs / peaks["hbm_gbs"])}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sample-tokens", type=int, default=None,
                    help="reference arm: tokens per step of the oracle's sample (default 16384)")
    ap.add_argument("--only", choices=["long", "layer", "train", "decode"], default=None,
                    help="profiling: run one workload alone and print its time, no JSON line")
    ap.add_argument("--T", type=int, default=None, help="with --only: a shorter sequence length")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            return run_reference(args, rank, world)
        if args.only:
            return run_only(args, local)
        return run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
