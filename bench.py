"""Throughput of the fused DiT-block per-token hot path on B200.

One step = one pass of the whole path over the workload, five libsol launches on one
stream (AdaLN -> QKV epilogue -> prologue -> SwiGLU -> gated residual; see
dit_block_b200/block.py).  Default workload: the full-resolution 10 s grid, 61x48x84 =
245,952 tokens, d=5120, 40x128 heads, SwiGLU width 13,824, bf16, 0.1% +-50 outliers.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

N > 1 is launched by torchrun, one rank per GPU; every rank processes its own copy of
the workload (weak scaling, no collective on the data path) and the time is the max
over ranks.  With --shard the ranks split one workload's tokens into contiguous ranges
instead (strong scaling, still no collective on the data path).  Rank 0 prints one JSON
line.

value       algorithmic HBM bytes of all ranks' steps / device time (GB/s); every tensor
            element an op must read or write counts once (216,064 B per token per step).
e2e         the same metric through the C ABI's host-buffer call (sol_dit_block_host): per
            step, pinned host -> device copies of every input, the five launches,
            device -> host copies of every output, all inside the timed region, chunked
            and overlapped across three streams by the library.
roofline    the SwiGLU launch (the largest byte mover): achieved GB/s from CUDA events
            around each launch in the timed steps, against the measured HBM copy peak.
cpu_baseline / --impl reference
            the fp64 oracle (C, OpenMP on all host cores) on a bounded token sample.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from dit_block_b200 import workloads  # noqa: E402

METRIC = "fused DiT-op HBM GB/s & tokens/s at 125k/246k tokens; % of B200 HBM peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
SPEC_HBM_GBS = 8000.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_swiglu.json")
PER_CONFIG = ("lowres", "fullres_5s", "fullres_10s", "packed_av")
OPS = ("adaln_modulate", "dit_epilogue", "dit_prologue", "swiglu", "gated_residual")
DOMINANT = "swiglu"


def bytes_per_token(w) -> dict:
    e = 2 if w.dtype == torch.bfloat16 else 4
    return {"adaln_modulate": 2 * w.d * e, "dit_epilogue": 4 * w.hd * e, "dit_prologue": 4 * w.d * e,
            "swiglu": 3 * w.inner * e, "gated_residual": 3 * w.d * e}


def dtype_name(w) -> str:
    return "bf16" if w.dtype == torch.bfloat16 else "f32"


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device: torch.device, period_s: float = 0.01):
        self.period = period_s
        self.samples: list[int] = []
        self.reasons = 0
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that the clocks are unknown
            self.err = str(e)
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self._stop.set()
        self._t.join()
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------------------ helpers

def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_peak():
    """Dense bf16 TFLOP/s of a cuBLAS GEMM timed alone on this machine's B200s (burst)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def measured_bf16_sustained():
    """The same GEMM run back to back for seconds under the power cap (sustained)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def source_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in ("k_stream.cu", "common.cuh"):
        with open(os.path.join(ROOT, "dit_block_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(n_tokens: int):
    """DRAM bytes of one SwiGLU launch over n_tokens tokens: the ncu capture committed in
    profiles/traffic_swiglu.json (dram__bytes_read.sum + dram__bytes_write.sum of one launch
    on a small case), scaled by tokens -- SwiGLU's traffic grows in proportion to the rows
    it streams.  None if the file is absent or was taken on different kernel source."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    try:
        if t["kernel_source_sha256_16"] != source_digest():
            return None
        return (float(t["dram_bytes_read"]) + float(t["dram_bytes_write"])) / float(t["tokens"]) * n_tokens
    except (KeyError, ValueError, ZeroDivisionError):
        return None


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def all_ranks_agree(ok: bool, world: int, device) -> bool:
    """True only if every rank passes `ok`: a decision that changes which collectives a
    rank takes next must be the same on every rank."""
    if world == 1:
        return bool(ok)
    import torch.distributed as dist
    t = torch.tensor([1 if ok else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item())


def max_over_ranks(vals: list[float], world: int, device) -> list[float]:
    if world == 1:
        return vals
    import torch.distributed as dist
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


# -------------------------------------------------------------------------- CPU oracle

def _bits(t):
    c = t.detach().contiguous().cpu()
    if c.dtype == torch.bfloat16:
        return c.view(torch.int16).numpy().view(np.uint16).copy()
    return c.numpy().copy()


class OracleChain:
    """The oracle's pass over a token sample (same five operators, same shapes)."""

    def __init__(self, w, n_tokens: int):
        import oracle
        oracle.build()
        self.o = oracle
        self.w = w
        inp = workloads.block_inputs(w, "cpu", n_tokens=n_tokens)
        self.n = n_tokens
        self.a = {k: _bits(v) for k, v in inp.items() if isinstance(v, torch.Tensor)}
        self.pos = None if inp["pos"] is None else inp["pos"].numpy()

    def step(self):
        o, w, a = self.o, self.w, self.a
        sel = dict(stream_id=a.get("stream_id"), n_streams=w.n_streams,
                   tokens_per_sample=w.tokens_per_sample)
        o.adaln_modulate(a["x"], a["shift_msa"], a["scale_msa"], eps=w.eps, **sel)
        o.dit_epilogue(a["qkv"], a["wq"], a["wk"], n_heads=w.n_heads, head_dim=w.head_dim,
                       pos=self.pos, grid=w.grid, tokens_per_sample=w.tokens_per_sample,
                       dims=w.rope_dims, theta=w.theta, eps=w.eps)
        o.dit_prologue(a["x"], a["y_attn"], a["gate_msa"], a["shift_mlp"], a["scale_mlp"], eps=w.eps,
                       **sel)
        o.swiglu(a["u"], w.inner)
        o.gated_residual(a["x"], a["y_mlp"], a["gate_mlp"], **sel)

    def bytes_per_step(self) -> int:
        return sum(bytes_per_token(self.w).values()) * self.n


def cpu_baseline(w, target_s: float = 10.0, sample_tokens: int = 1024) -> dict:
    chain = OracleChain(w, sample_tokens)
    chain.step()  # warm-up (page faults, thread pool)
    t0 = time.perf_counter()
    reps = 0
    while True:
        chain.step()
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_s or reps >= 1000:
            break
    gbs = chain.bytes_per_step() * reps / el / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": chain.o.num_threads(), "kind": "oracle",
            "sample": f"{reps} passes of the 5-op chain over {sample_tokens} tokens of {w.name} "
                      f"({el:.1f} s, fp64, OpenMP)",
            "tokens_per_s": round(sample_tokens * reps / el, 1)}


# ------------------------------------------------------------------------- arms

def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    chain = OracleChain(w, args.ref_tokens)
    for _ in range(args.warmup):
        chain.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        chain.step()
    el = time.perf_counter() - t0
    gbs = chain.bytes_per_step() * args.steps / el / 1e9
    cores = chain.o.num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "tokens": w.n_tokens, "sample_tokens": args.ref_tokens,
                   "d": w.d, "heads": f"{w.n_heads}x{w.head_dim}", "swiglu_inner": w.inner,
                   "parallelism": "replicas", "l2": "host run"},
        "tokens_per_s": round(args.ref_tokens * args.steps / el, 1),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.ref_tokens} tokens of {w.name} per step"},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, w):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    from dit_block_b200 import block, build, sol
    build.build()
    sol.lib()

    if args.shard:
        # strong scaling: rank r takes its contiguous range of the workload's tokens
        from dit_block_b200 import shard
        n_total = w.n_tokens if args.tokens is None else min(args.tokens, w.n_tokens)
        t0, t1 = shard.token_ranges(n_total, world)[rank]
        bufs = shard.ShardBuffers(w, t0, t1, dev)
    else:
        bufs = block.BlockBuffers.allocate(w, dev, n_tokens=args.tokens)
        n_total = bufs.n_tokens * world
    n = bufs.n_tokens
    bpt = bytes_per_token(w)
    step_bytes = sum(bpt.values()) * n
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local])

    # ---- device-resident timing
    for _ in range(args.warmup):
        bufs.step()
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev)
    clocks.start()
    total_ms, op_times = time_passes(bufs, args.steps, stream)
    barrier()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    per_op_ms = {op: sum(t) / len(t) for op, t in op_times.items()}
    total_ms, = max_over_ranks([total_ms], world, dev)
    ms_step = total_ms / args.steps
    all_bytes = sum(bpt.values()) * n_total  # every rank's tokens of one step
    value = all_bytes * args.steps / (total_ms * 1e-3) / 1e9

    peak, peak_kind = measured_peak()
    headline = config_entry(w, n, total_ms, args.steps, op_times, peak)

    # ---- ops beyond the block pass, each timed alone on the same workload
    extras = not args.shard
    next_ops = {} if (args.no_next or not extras) else time_next_ops(bufs, dev, args)
    linear_ops = {} if (args.no_next or args.linear_tokens <= 0 or not extras) else \
        time_linear_ops(w, dev, args.linear_tokens)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e and extras:
        e2e = run_e2e(args, bufs, dev, world, step_bytes)
    elif args.shard:
        e2e = {"value": None, "unit": "GB/s", "error": "not measured for token shards (run without --shard)"}

    mix_ref = stream_mix_reference(n, w.d, dev)

    dom_ms = per_op_ms[DOMINANT]
    dom_bytes = bpt[DOMINANT] * n
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    traffic = ncu_traffic(n)
    per_op = {op: {"ms": round(per_op_ms[op], 4),
                   "ms_median": round(statistics.median(op_times[op]), 4), "ms_min": round(min(op_times[op]), 4),
                   "GB_s": round(bpt[op] * n / (per_op_ms[op] * 1e-3) / 1e9, 1),
                   "frac_of_measured_peak": round(bpt[op] * n / (per_op_ms[op] * 1e-3) / 1e9 / peak, 4),
                   "frac_of_spec_peak": round(bpt[op] * n / (per_op_ms[op] * 1e-3) / 1e9 / SPEC_HBM_GBS, 4),
                   "bytes_per_token": bpt[op]} for op in OPS}
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "strong" if args.shard else "weak", "vs_baseline": None,
        "dtype": dtype_name(w), "data": "synthetic",
        "config": {"workload": w.name, "tokens": n_total, "tokens_per_rank": n, "grid": list(w.grid),
                   "batch": w.batch,
                   "d": w.d, "heads": f"{w.n_heads}x{w.head_dim}", "swiglu_inner": w.inner,
                   "bytes_per_token": sum(bpt.values()),
                   "parallelism": (f"token shards x{world}" if args.shard else f"replicas x{world}")
                   if world > 1 else "single GPU",
                   "l2": "no flush: every op streams >= 2.5 GB, far above the 126 MB L2"},
        "tokens_per_s": round(n_total * args.steps / (total_ms * 1e-3), 1),
        "frac_of_measured_hbm_peak": round(value / world / peak, 4),
        "frac_of_spec_hbm_peak": round(value / world / SPEC_HBM_GBS, 4),
        "per_op": per_op,
        "roofline": {"bound": "hbm", "kernel": "k_swiglu", "achieved": round(achieved, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": None if traffic is None else int(traffic),
                     "algorithmic_bytes": dom_bytes,
                     "mix_reference": mix_ref,
                     "frac_of_torch_add_2r1w": round(achieved / mix_ref["torch_add_2r1w_GB_s"], 4)},
        "clocks": clk,
        "per_config": None,
        "next_ops": next_ops,
        "linear_ops": linear_ops,
        "gpu_launches": len(OPS) * args.steps,
        "e2e": e2e,
    }
    full_size = args.tokens is None or args.tokens >= w.n_tokens
    bufs.close()
    del bufs
    torch.cuda.empty_cache()
    if not args.no_per_config and full_size and w.dtype == torch.bfloat16 and not args.shard:
        # every bf16 workload, one at a time; each rank times its own copy (the max over
        # ranks is taken for the chain time)
        pc = time_per_config(args, dev, peak, {w.name: headline})
        for name, e in pc.items():
            e["chain_ms"], = max_over_ranks([e["chain_ms"]], world, dev)
        line["per_config"] = pc
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def time_passes(bufs, steps: int, stream):
    """Device time of `steps` back-to-back passes (CUDA events on `stream`) and each
    launch's own duration per pass (events between the launches)."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(OPS) + 1)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(steps):
        ev[s][0].record(stream)
        for j, op in enumerate(OPS):
            bufs.launch(op)
            ev[s][j + 1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    op_times = {op: [ev[s][j].elapsed_time(ev[s][j + 1]) for s in range(steps)] for j, op in enumerate(OPS)}
    return start.elapsed_time(end), op_times


def config_entry(w, n: int, total_ms: float, steps: int, op_times: dict, peak: float) -> dict:
    """Chain and per-op throughput of one workload, as fractions of the measured copy peak
    and of the 8 TB/s spec."""
    bpt = bytes_per_token(w)
    step_bytes = sum(bpt.values()) * n
    ms = total_ms / steps
    gbs = step_bytes / (ms * 1e-3) / 1e9
    ops = {}
    for op in OPS:
        t = sum(op_times[op]) / len(op_times[op])
        g = bpt[op] * n / (t * 1e-3) / 1e9
        ops[op] = {"ms": round(t, 4), "ms_median": round(statistics.median(op_times[op]), 4),
                   "GB_s": round(g, 1), "frac_of_measured_peak": round(g / peak, 4),
                   "frac_of_spec_peak": round(g / SPEC_HBM_GBS, 4)}
    return {"tokens": n, "steps": steps, "chain_ms": round(ms, 4), "GB_s": round(gbs, 1),
            "tokens_per_s": round(n / (ms * 1e-3), 1), "frac_of_measured_peak": round(gbs / peak, 4),
            "frac_of_spec_peak": round(gbs / SPEC_HBM_GBS, 4), "per_op": ops}


def time_per_config(args, dev, peak: float, done: dict) -> dict:
    """Every bf16 workload timed like the headline (one at a time: its buffers are
    allocated, timed over args.config_steps passes and freed before the next)."""
    from dit_block_b200 import block
    stream = torch.cuda.current_stream(dev)
    out = {}
    for name in PER_CONFIG:
        if name in done:
            out[name] = done[name]
            continue
        w = workloads.WORKLOADS[name]
        bufs = block.BlockBuffers.allocate(w, dev)
        for _ in range(args.warmup):
            bufs.step()
        torch.cuda.synchronize(dev)
        total, op_times = time_passes(bufs, args.config_steps, stream)
        out[name] = config_entry(w, bufs.n_tokens, total, args.config_steps, op_times, peak)
        bufs.close()
        del bufs
        torch.cuda.empty_cache()
    return out


def stream_mix_reference(n: int, d: int, dev) -> dict:
    """Context for the HBM denominators: torch's own elementwise kernels on bf16 [n, d]
    (2.5 GB per tensor at the full workload), timed like the ops.  The measured copy peak
    is a 1 read : 1 write stream; the gated residual and SwiGLU read two bytes per byte
    written, a mix this GPU streams faster, so their fraction of the copy peak can pass 1."""
    g = torch.Generator(device=dev).manual_seed(7)
    x = torch.randn(n, d, device=dev, dtype=torch.bfloat16, generator=g)
    y = torch.randn(n, d, device=dev, dtype=torch.bfloat16, generator=g)
    o = torch.empty_like(x)
    stream = torch.cuda.current_stream(dev)
    e = n * d * 2
    ms_add = _time(lambda: torch.add(x, y, out=o), 10, stream)
    ms_copy = _time(lambda: o.copy_(x), 10, stream)
    del x, y, o
    return {"torch_add_2r1w_GB_s": round(3 * e / (ms_add * 1e-3) / 1e9, 1),
            "torch_copy_1r1w_GB_s": round(2 * e / (ms_copy * 1e-3) / 1e9, 1),
            "shape": [n, d], "dtype": "bf16"}


def _time(fn, reps: int, stream) -> float:
    """Median milliseconds of `fn` over `reps` launches (CUDA events on `stream`)."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    for i in range(reps):
        ev[i].record(stream)
        fn()
    ev[reps].record(stream)
    torch.cuda.synchronize()
    return statistics.median(ev[i].elapsed_time(ev[i + 1]) for i in range(reps))


def _time_interleaved(fns, reps: int, stream) -> list[float]:
    """Median milliseconds of each of `fns`, timed in turn within every repetition (CUDA
    events on `stream`)."""
    for fn in fns:
        for _ in range(3):
            fn()
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
          for _ in fns]
    for r in range(reps):
        for i, fn in enumerate(fns):
            ev[i][r][0].record(stream)
            fn()
            ev[i][r][1].record(stream)
    torch.cuda.synchronize()
    return [statistics.median(a.elapsed_time(b) for a, b in ev[i]) for i in range(len(fns))]


def time_next_ops(bufs, dev, args) -> dict:
    """Each op outside the block pass, timed alone at the workload's size (median of
    20 launches), with its algorithmic bytes per token."""
    from dit_block_b200 import sol
    w, i = bufs.w, bufs.inp
    n = bufs.n_tokens
    e = 2 if w.dtype == torch.bfloat16 else 4
    peak, _ = measured_peak()
    stream = torch.cuda.current_stream(dev)
    out = {}
    cache = torch.empty_like(bufs.x2)
    cache.copy_(i["y_attn"])
    sums = torch.empty((w.batch, 2), dtype=torch.float64, device=dev)
    sel = bufs.sel()
    fn = lambda: sol.gated_residual_cache_diff(bufs.x2, bufs.x1, i["y_mlp"], i["gate_mlp"], cache, sums,
                                               refresh=True, **sel)
    ms = _time(fn, 20, stream)
    b = 5 * w.d * e  # read x, y, cache; write out, cache
    out["gated_residual_cache_diff"] = {"ms": round(ms, 4), "bytes_per_token": b,
                                        "GB_s": round(b * n / (ms * 1e-3) / 1e9, 1),
                                        "frac_of_measured_peak": round(b * n / (ms * 1e-3) / 1e9 / peak, 4)}
    del cache
    blk = 64
    nb = sol.subblock_count(n, w.tokens_per_sample, blk)
    pq = torch.empty((nb, w.hd), dtype=w.dtype, device=dev)
    pk = torch.empty((nb, w.hd), dtype=w.dtype, device=dev)
    fn = lambda: sol.dit_epilogue_pool(i["qkv"], pq, pk, bufs.rope, n_heads=w.n_heads, head_dim=w.head_dim,
                                       wq=i["wq"], wk=i["wk"], pos=i["pos"], grid=w.grid,
                                       tokens_per_sample=w.tokens_per_sample, block_tokens=blk, eps=w.eps)
    ms = _time(fn, 20, stream)
    b = 4 * w.hd * e  # read and write q and k
    pooled = 2 * nb * w.hd * e  # the pooled rows
    out["dit_epilogue_pool"] = {"ms": round(ms, 4), "bytes_per_token": b, "pooled_bytes": pooled,
                                "GB_s": round((b * n + pooled) / (ms * 1e-3) / 1e9, 1),
                                "frac_of_measured_peak": round((b * n + pooled) / (ms * 1e-3) / 1e9 / peak, 4)}
    del pq, pk
    # convention variants: q, k of the packed row -> head-major [sample, head, token, dim]
    tps = w.tokens_per_sample
    qh = torch.empty((w.batch, w.n_heads, tps, w.head_dim), dtype=w.dtype, device=dev)
    kh = torch.empty_like(qh)
    q, k = i["qkv"][:, :w.hd], i["qkv"][:, w.hd:2 * w.hd]
    wfull = torch.ones((w.hd,), dtype=w.dtype, device=dev)
    for name, kw in (("qk_ex_head_major_output", dict(wq=i["wq"], wk=i["wk"])),
                     ("qk_ex_across_heads_rotate_half", dict(wq=wfull, wk=wfull, norm_span=sol.NORM_ACROSS_HEADS,
                                                             pairing=sol.ROPE_HALF))):
        fn = lambda: sol.qk_rmsnorm_rope3d_ex(qh, kh, q, k, bufs.rope, n_heads=w.n_heads, head_dim=w.head_dim,
                                              pos=i["pos"], grid=w.grid, tokens_per_sample=tps, eps=w.eps,
                                              out_strides=(w.head_dim, tps * w.head_dim,
                                                           w.n_heads * tps * w.head_dim), **kw)
        ms = _time(fn, 20, stream)
        out[name] = {"ms": round(ms, 4), "bytes_per_token": b,
                     "GB_s": round(b * n / (ms * 1e-3) / 1e9, 1),
                     "frac_of_measured_peak": round(b * n / (ms * 1e-3) / 1e9 / peak, 4)}
    del qh, kh
    return out


def time_linear_ops(w, dev, m: int) -> dict:
    """The block's linear layers with the per-token operators fused in (tcgen05 GEMMs),
    each timed alone on `m` tokens of the workload's first sample (seeded inputs of its
    shapes, weights ~ N(0, 1/in_features); median of 10 launches), beside the same work
    unfused: a cuBLAS GEMM (torch.matmul) plus the libsol per-token kernel, the bare
    cuBLAS GEMM and the bare libsol GEMM."""
    from dit_block_b200 import sol, workloads as wl
    if w.dtype != torch.bfloat16 or w.head_dim != 128:
        return {}
    m = min(int(m), w.tokens_per_sample)
    peak, src = measured_bf16_peak()
    stream = torch.cuda.current_stream(dev)
    i = {"x": wl.activation(w, "x", m, w.d, dev), "y_attn": wl.activation(w, "y_attn", m, w.d, dev),
         "wq": wl.norm_weight(w, "wq", dev), "wk": wl.norm_weight(w, "wk", dev)}
    for k in ("shift_msa", "scale_msa", "gate_msa", "gate_mlp"):
        i[k] = wl.modulation(w, k, dev)
    rope = sol.Rope3D(w.rope_dims, w.theta, w.max_pos)
    x = i["x"]
    hd, d, inner = w.hd, w.d, w.inner
    # ops on one sample's tokens: modulation rows of sample 0, positions from its grid
    sel = dict(n_streams=1, tokens_per_sample=0)
    sus, sus_src = measured_bf16_sustained()
    out = {"tokens": m, "peak_tflops": peak, "peak_source": src + " (burst cuBLAS bf16)",
           "sustained_peak_tflops": sus, "sustained_peak_source": sus_src + " (cuBLAS bf16 under the power cap)",
           "adaln_strategy": "stage"}

    def entry(name, flops, fused, unfused, cublas, plain, saved_bytes):
        # the four arms alternate launch by launch, so clock drift under the power cap
        # affects them alike
        tf, tu, tcb, tp = _time_interleaved([fused, unfused, cublas, plain], 10, stream)
        ach = flops / (tf * 1e-3) / 1e12
        out[name] = {"ms": round(tf, 4), "TFLOP_s": round(ach, 1), "frac_of_bf16_peak": round(ach / peak, 4),
                     "frac_of_sustained_bf16_peak": round(ach / sus, 4),
                     "unfused_ms": round(tu, 4), "cublas_gemm_ms": round(tcb, 4),
                     "libsol_plain_gemm_ms": round(tp, 4), "plain_gemm_vs_cublas": round(tcb / tp, 3),
                     "speedup_vs_unfused": round(tu / tf, 3),
                     "hbm_bytes_saved_per_token": saved_bytes}

    ws = sol.adaln_workspace(m, 3 * hd, d, device=dev)
    Wqkv = wl.linear_weight(w, "w_qkv", 3 * hd, d, dev)
    qkv = torch.empty((m, 3 * hd), dtype=w.dtype, device=dev)
    h = torch.empty_like(x)
    sh, sc = i["shift_msa"][:1], i["scale_msa"][:1]
    fused = lambda: sol.adaln_qkv_rope(qkv, x, Wqkv, rope, sh, sc, workspace=ws, n_heads=w.n_heads,
                                       wq=i["wq"], wk=i["wk"], grid=w.grid, eps=w.eps, **sel)

    def unfused():
        sol.adaln_modulate(h, x, sh, sc, eps=w.eps, **sel)
        torch.matmul(h, Wqkv.t(), out=qkv)
        sol.dit_epilogue(qkv, rope, n_heads=w.n_heads, head_dim=w.head_dim, wq=i["wq"], wk=i["wk"],
                         grid=w.grid, eps=w.eps)
    entry("adaln_qkv_rope", 2.0 * m * d * 3 * hd, fused, unfused, lambda: torch.matmul(x, Wqkv.t(), out=qkv),
          lambda: sol.linear(qkv, x, Wqkv), 2 * d * 2 + 2 * (2 * hd) * 2)
    del Wqkv, qkv, h, ws

    for name, K, wname, gate in (("o_proj_gated_residual", d, "w_o", "gate_msa"),
                                 ("down_proj_gated_residual", inner, "w_down", "gate_mlp")):
        a = i["y_attn"] if K == d else wl.activation(w, "act", m, K, dev)
        W = wl.linear_weight(w, wname, d, K, dev)
        o = torch.empty_like(x)
        y = torch.empty_like(x)
        g = i[gate][:1]
        fused = lambda: sol.linear_gated_residual(o, x, a, W, g, **sel)

        def unfused():
            torch.matmul(a, W.t(), out=y)
            sol.gated_residual(o, x, y, g, **sel)
        entry(name, 2.0 * m * K * d, fused, unfused, lambda: torch.matmul(a, W.t(), out=y),
              lambda: sol.linear(y, a, W), 2 * d * 2)
        del a, W, o, y

    Wup = wl.linear_weight(w, "w_up", 2 * inner, d, dev)
    act = torch.empty((m, inner), dtype=w.dtype, device=dev)
    u = torch.empty((m, 2 * inner), dtype=w.dtype, device=dev)
    fused = lambda: sol.linear_swiglu(act, x, Wup)

    def unfused():
        torch.matmul(x, Wup.t(), out=u)
        sol.swiglu(act, u, inner=inner)
    entry("up_proj_swiglu", 2.0 * m * d * 2 * inner, fused, unfused, lambda: torch.matmul(x, Wup.t(), out=u),
          lambda: sol.linear(u, x, Wup), 2 * (2 * inner) * 2)
    # the MLP input in one pass: AdaLN -> up projection -> SwiGLU
    ws2 = sol.adaln_workspace(m, 2 * inner, d, device=dev)
    fused = lambda: sol.adaln_linear_swiglu(act, x, Wup, i["shift_msa"][:1], i["scale_msa"][:1], workspace=ws2,
                                            eps=w.eps, **sel)
    h2 = torch.empty_like(x)

    def unfused():
        sol.adaln_modulate(h2, x, i["shift_msa"][:1], i["scale_msa"][:1], eps=w.eps, **sel)
        torch.matmul(h2, Wup.t(), out=u)
        sol.swiglu(act, u, inner=inner)
    entry("adaln_up_proj_swiglu", 2.0 * m * d * 2 * inner, fused, unfused, lambda: torch.matmul(x, Wup.t(), out=u),
          lambda: sol.linear(u, x, Wup), 2 * d * 2 + 2 * (2 * inner) * 2)
    del Wup, act, u, ws2, h2
    rope.close()
    return out


def run_linear_only(args, w):
    """--linear-only: the fused linear-layer timings alone, one JSON line."""
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    from dit_block_b200 import sol
    sol.lib()
    res = time_linear_ops(w, dev, args.linear_tokens)
    torch.cuda.synchronize(dev)
    print(json.dumps({"workload": w.name, "linear_ops": res, "device_errors": sol.device_errors()}), flush=True)
    return 0


def run_e2e(args, bufs, dev, world, step_bytes):
    """The pass through the C ABI's host-buffer call (sol_dit_block_host, driven by
    dit_block_b200.pipeline): pinned host inputs in, five launches per chunk, pinned host
    outputs back; every copy is inside the timed region and overlapped with compute across
    three streams by the library."""
    from dit_block_b200 import pipeline
    w, i = bufs.w, bufs.inp
    n = bufs.n_tokens
    pipe = pipeline.HostBlockPipeline(w, dev, chunk_tokens=args.e2e_chunk)
    h2d, d2h = pipe.bytes_per_pass(n)
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = 0
    # every rank of the node pins its own buffers; all ranks take the same decision, since
    # skipping also skips the barrier and the reduction below
    need = (h2d + d2h) * world
    if not all_ranks_agree(need <= 0.4 * avail, world, dev):
        pipe.close()
        return {"value": None, "unit": "GB/s",
                "error": f"skipped: {need / 1e9:.1f} GB of pinned host buffers over {world} rank(s) > 40% "
                         f"of the {avail / 1e9:.1f} GB available host memory (on some rank)"}
    host_in, host_out, host_mod = pipeline.host_buffers(w, n)
    for k in pipeline.IN_NAMES:
        host_in[k].copy_(i[k])
    for k in pipeline.MOD_NAMES:
        host_mod[k].copy_(i[k])
    pipe.set_weights(i["wq"], i["wk"])
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.e2e_warmup):
        pipe.run(host_in, host_out, host_mod)
    torch.cuda.synchronize(dev)
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[dev.index])
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.e2e_steps):
        pipe.run(host_in, host_out, host_mod)
    end.record(stream)
    torch.cuda.synchronize(dev)
    ms = start.elapsed_time(end)
    ms, = max_over_ranks([ms], world, dev)
    val = step_bytes * world * args.e2e_steps / (ms * 1e-3) / 1e9
    pipe.close()
    del host_in, host_out, host_mod
    return {"value": round(val, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": args.e2e_steps, "ms_per_step": round(ms / args.e2e_steps, 2),
            "api": "sol_dit_block_host (C ABI; pinned host buffers, via dit_block_b200.pipeline.HostBlockPipeline)",
            "chunk_tokens": args.e2e_chunk}


def main(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="fullres_10s", choices=sorted(workloads.WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--tokens", type=int, default=None,
                   help="run only the first N tokens of the workload (small profiling cases)")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--e2e-warmup", type=int, default=1)
    p.add_argument("--e2e-chunk", type=int, default=8192, help="tokens per pipelined chunk")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-next", action="store_true", help="skip timing the ops outside the block pass")
    p.add_argument("--linear-tokens", type=int, default=32768,
                   help="tokens of the fused linear-layer timings (0 skips them)")
    p.add_argument("--linear-only", action="store_true",
                   help="time only the fused linear layers (prints their own JSON line)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--shard", action="store_true",
                   help="strong scaling: split the workload's tokens into one contiguous range per rank "
                        "(no collective on the data path) instead of a full replica per rank")
    p.add_argument("--no-per-config", action="store_true",
                   help="skip timing the other bf16 workloads (per_config)")
    p.add_argument("--config-steps", type=int, default=20, help="passes timed per workload in per_config")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--ref-tokens", type=int, default=256, help="oracle token sample per reference step")
    args = p.parse_args(argv)
    if args.warmup < 3:
        p.error("--warmup must be >= 3")
    w = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.linear_only:
        return run_linear_only(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
