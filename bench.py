"""Throughput benchmark of the MoE FFN forward layer on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
python bench.py --all-workloads [--table PATH]   (one line per workload, and a markdown table)

A step is one pass of the whole hot path (route -> dispatch -> expert up/down -> combine)
over one batch of the workload, enqueued through the C ABI with CUDA events between the
kernels (the same kernels moe_forward launches). Inputs are resident in HBM; L2 is flushed
(a 512 MiB write, then a read of it) between timed steps, outside the per-step events. Rank 0 prints one JSON
line. With N>1 (torchrun) every rank runs an independent replica on its own GPU (the layer
has no data-path collective); value = tokens of all ranks / max-over-ranks time.

--impl reference times the CPU oracle on the host cores: K steps after W warm-up steps, each
step the oracle's forward on a bounded token sample of the same workload (the throughput is
extrapolated to the workload's N), and prints the same line with "impl": "reference".

Without --steps, K is chosen after the warm-up so that the timed region lasts about 1.5 s.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE fwd tokens/s; grouped-GEMM TFLOP/s & %bf16 peak; route/combine % HBM BW"
L2_FLUSH_BYTES = 512 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Datasheet figures of one B200 (dense, no sparsity), for the second denominator of every
# fraction: 2.25 PFLOP/s bf16 at the 1965 MHz maximum SM clock, 8 TB/s HBM3e.
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_HBM_GBS = 8000.0
DATASHEET_SM_MHZ = 1965.0
DATASHEET_SMS = 148
TIMED_REGION_TARGET_S = 1.5


# ------------------------------------------------------------------ small host helpers

def load_peaks():
    """The roofline denominators: MEASURED_PEAKS.json's figures, each missing one taken from
    the fallback table. Returns (peaks, source): "measured", "fallback", or "measured
    (fallback: <keys>)" when the file lacks some of them."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if not isinstance(d, dict):
            raise ValueError("not an object")
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"
    peaks, missing = {}, []
    for k, v in FALLBACK_PEAKS.items():
        try:
            peaks[k] = float(d[k])
        except (KeyError, TypeError, ValueError):
            peaks[k] = v
            missing.append(k)
    if len(missing) == len(FALLBACK_PEAKS):
        return peaks, "fallback"
    return peaks, "measured" if not missing else f"measured (fallback: {', '.join(missing)})"


def peak_key_source(peak_src: str, key: str) -> str:
    """Where one denominator came from, given load_peaks()'s source string."""
    if peak_src == "fallback" or (peak_src.startswith("measured (fallback:") and key in peak_src):
        return "fallback"
    return "measured (MEASURED_PEAKS.json)"


def workload_desc(cfg, w8: bool = False, packed: bool = False) -> str:
    act = {0: "SiLU", 1: "GELU(erf)", 2: "GELU(tanh)"}[cfg.activation]
    s = (f"{cfg.name}: N={cfg.N} D={cfg.D} F={cfg.F} E={cfg.E} k={cfg.k} {act} "
         f"{'renormalised' if cfg.renormalize else 'no-renorm'} top-k")
    if cfg.capacity_factor > 0:
        s += f", CF={cfg.capacity_factor}"
    if cfg.min_capacity > 0:
        s += f", min_capacity={cfg.min_capacity}"
    if cfg.capacity_order == 1:
        s += ", token-major slots"
    if cfg.drop_policy == 1:
        s += ", kept gates renormalised on drops"
    if w8:
        s += ", 8-bit expert weights (fp32 scale per expert and output column)"
        if packed:
            s += ", repacked K-contiguous at load time"
    return s


def dtype_name(cfg) -> str:
    from top_routing_expert_fp32_b200 import configs
    return "bf16" if cfg.dtype == configs.DTYPE_BF16 else "f32"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(value: float, device) -> float:
    """Max over ranks (all ranks call it, same order)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and getattr(device, "type", "cpu") == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(tokens_per_rank: int, world: int, max_ms_total: float, steps: int) -> dict:
    """Whole-job throughput from the slowest rank's time."""
    ms_per_step = max_ms_total / steps
    return dict(value=tokens_per_rank * world * steps / (max_ms_total / 1e3),
                ms_per_step=ms_per_step)


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a background thread."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []  # (t, sm_mhz, reasons_mask)
        self.period = period_s
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                if not uuid.startswith("GPU-"):
                    uuid = "GPU-" + uuid
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.time(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self, t0: float, t1: float) -> dict:
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        if len(win) < 3:
            win = self.samples
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = sorted({name for _, _, m in win for name, bit in self.REASONS.items() if m & bit})
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(win)}


def source_hash(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profile(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture, if it matches the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel][workload]
        if e["source_sha"] != source_hash(e["sources"]):
            return None
        return e["bytes_per_launch"]
    except Exception:
        return None


# ------------------------------------------------------------------ CPU oracle timing

class OracleSample:
    """The oracle (as it stands) on token samples of the workload: step(n, first) runs its
    full forward on tokens [first, first + n) (wrapping around N) and returns the seconds it
    took. Without capacity the tokens are independent, so a sample costs per token what the
    whole batch costs; with capacity the sample is its own batch of n tokens (capacity
    recomputed for n)."""

    def __init__(self, cfg, w8: bool = False, inp=None, wq=None):
        """inp / wq: the GPU arm's own input tensors (copied to the host here), else the
        same recipe drawn on the host."""
        import oracle
        from top_routing_expert_fp32_b200 import configs, inputs
        self.cfg, self.w8, self.oracle = cfg, w8, oracle
        self.same_values = inp is not None
        if inp is None:
            inp = inputs.make_inputs(cfg, "cpu", weights=not w8)
        if w8 and wq is None:
            wq = inputs.make_w8_weights(cfg, "cpu")
        self.od = oracle.BF16 if cfg.dtype == configs.DTYPE_BF16 else oracle.F32
        self.X = oracle.torch_to_numpy(inp.X.cpu())
        self.Wr = inp.W_r.cpu().numpy()
        self.b = None if inp.bias is None else inp.bias.cpu().numpy()
        self.opts = dict(k=cfg.k, cf=cfg.capacity_factor, renorm=cfg.renormalize,
                         act=cfg.activation, dtype=self.od, min_capacity=cfg.min_capacity,
                         order=cfg.capacity_order, drop_policy=cfg.drop_policy)
        if w8:
            self.qs = [t.cpu().numpy() for t in (wq.W1q, wq.S1, wq.W2q, wq.S2, wq.W3q, wq.S3)]
        else:
            self.W = [oracle.torch_to_numpy(w.cpu()) for w in (inp.W1, inp.W2, inp.W3)]
        self.cores = oracle.num_threads()

    def routing_check(self, gpu_idx) -> dict:
        """Tokens whose GPU top-k (set or order) differs from the oracle's routing of its fp64
        logits, and the largest top-k margin among them (near ties are below 1e-4)."""
        o = self.oracle
        l64, l32 = o.router_logits(self.X, self.od, self.Wr, self.b)
        ro = o.route(l32, k=self.cfg.k, renorm=self.cfg.renormalize)
        flips = (gpu_idx != ro["idx"]).any(1)
        margin = o.topk_margin(l64, self.cfg.k)
        return {"tokens": int(self.cfg.N), "flips": int(flips.sum()),
                "max_margin_of_flips": float(margin[flips].max()) if flips.any() else None,
                "near_tie_margin": 1e-4}

    def step(self, n: int, first: int = 0) -> float:
        import numpy as np
        N = self.cfg.N
        n = max(1, min(n, N))
        rows = (np.arange(first, first + n) % N) if first + n > N else slice(first, first + n)
        X = np.ascontiguousarray(self.X[rows])
        t = time.perf_counter()
        if self.w8:
            self.oracle.forward_w8(X, self.Wr, self.b, *self.qs, **self.opts)
        else:
            self.oracle.forward(X, self.Wr, self.b, *self.W, **self.opts)
        return time.perf_counter() - t

    def calibrate(self, seconds: float) -> int:
        """Tokens per sample so that one step takes about `seconds` (at least one token per
        host thread's worth of records)."""
        n = max(1, -(-self.cores // self.cfg.k))
        dt = self.step(n)
        while dt < seconds / 4 and n < self.cfg.N:
            n = min(self.cfg.N, n * 2)
            dt = self.step(n)
        return max(1, min(self.cfg.N, int(n * seconds / max(dt, 1e-4))))


def oracle_tokens_per_s(cfg, budget_s: float = 12.0, w8: bool = False, sampler=None):
    """cpu_baseline of the GPU arm: the oracle on one bounded token sample of the workload
    (about budget_s of CPU work), extrapolated to tokens/s."""
    o = sampler or OracleSample(cfg, w8)
    n = o.calibrate(budget_s / 2)
    dt = o.step(n)
    vals = "the GPU arm's input values" if o.same_values else "inputs of the same recipe"
    return dict(value=n / dt, unit="tokens/s", cores=o.cores, kind="oracle",
                sample=f"first {n} of {cfg.N} tokens of the workload ({vals}), full forward "
                       f"in fp64, {dt:.1f} s wall; tokens/s extrapolated from the sample",
                extrapolated=n < cfg.N)


def run_reference(args, cfg, w8: bool, packed: bool) -> dict:
    """The reference arm: the oracle as it stands, W warm-up steps and then exactly K timed
    steps, each its full forward on a bounded sample of the workload's tokens (consecutive
    slices, wrapping around N). The whole run is sized to end within a few minutes."""
    o = OracleSample(cfg, w8)
    per_step = min(6.0, 150.0 / max(1, args.steps + args.warmup))
    n = o.calibrate(per_step)
    first = 0
    for _ in range(args.warmup):
        o.step(n, first)
        first = (first + n) % cfg.N
    total = 0.0
    for _ in range(args.steps):
        total += o.step(n, first)
        first = (first + n) % cfg.N
    value = args.steps * n / total
    sample = (f"{n} of {cfg.N} tokens per step (consecutive slices), full forward in fp64, "
              f"{total:.1f} s wall over {args.steps} steps; tokens/s extrapolated to the "
              f"workload")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * cfg.N / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64",
            "data": "synthetic, seeded: the GPU arm's recipe and shapes, drawn on the host",
            "config": {"workload": workload_desc(cfg, w8, packed),
                       "sample_tokens_per_step": n},
            "extrapolated": n < cfg.N,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": o.cores,
                             "kind": "oracle", "sample": sample, "extrapolated": n < cfg.N},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ GPU arm

def run_gpu(args, cfg, world, rank, device):
    import torch
    from top_routing_expert_fp32_b200 import abi, configs, inputs

    torch.cuda.set_device(device)
    peaks, peak_src = load_peaks()
    w8 = args.weights in ("w8", "w8p")
    packed = args.weights == "w8p"
    inp = inputs.make_inputs(cfg, device, seed=cfg.seed + rank * 0, weights=not w8)
    wq = inputs.make_w8_weights(cfg, device) if w8 else None
    N, E, k, D, F = cfg.N, cfg.E, cfg.k, cfg.D, cfg.F
    p = abi.problem(cfg)
    ws = abi.workspace(p, device)
    if packed:
        # Load-time repacking (outside every timed region): K-contiguous copies, scales shared.
        W1p = torch.empty((E, F, D), dtype=torch.int8, device=device)
        W2p = torch.empty_like(W1p)
        W3p = torch.empty((E, D, F), dtype=torch.int8, device=device)
        abi.pack_w8(p, wq.W1q, wq.W2q, wq.W3q, W1p, W2p, W3p)
        wq = inputs.MoEWeights8(W1p, wq.S1, W2p, wq.S2, W3p, wq.S3)
        torch.cuda.synchronize(device)
    # 8-bit weights: the transposed tensor-memory-operand kernel when packed or when the
    # experts hold few rows (N k <= 64 E), else the shared-memory one.
    w8_kernel = ("grouped_gemm_w8t" if packed or N * k <= 64 * E else "grouped_gemm_w8")
    up_kernel = (f"{w8_kernel}<dual{', K-contiguous' if packed else ''}>" if w8
                 else "grouped_gemm_sm100<dual>")
    tdt = inp.X.dtype
    R = N * k
    logits = None
    idx = torch.empty((N, k), dtype=torch.int32, device=device)
    gate = torch.empty((N, k), dtype=torch.float32, device=device)
    load = torch.empty((E,), dtype=torch.int32, device=device)
    offsets = torch.empty((E + 1,), dtype=torch.int32, device=device)
    pos = torch.empty((N, k), dtype=torch.int32, device=device)
    dropped = torch.empty((N, k), dtype=torch.uint8, device=device)
    row_token = torch.empty((R,), dtype=torch.int32, device=device)
    X_perm = torch.empty((R, D), dtype=tdt, device=device)
    H = torch.empty((R, F), dtype=tdt, device=device)
    Y = torch.empty((R, D), dtype=tdt, device=device)
    out = torch.empty((N, D), dtype=tdt, device=device)
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.int32, device=device)
    flush_sum = torch.empty((), dtype=torch.int64, device=device)

    def flush_l2():
        # Write 512 MiB (evicts X, H, Y), then read it back so that the dirty lines the write
        # leaves in L2 are written back here, not inside the next step's first kernel.
        flush.fill_(1)
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)
    stream = torch.cuda.current_stream(device)

    names = ["route", "dispatch", "up", "down", "combine"]
    # Kernels per step: one router (tensor-core for bf16 X, SIMT for fp32 X; with bf16 X and
    # more than 16 experts a small kernel writes the router's bf16 operand first), one
    # cooperative dispatch (count, slot assignment and gather), one launch each for up, down,
    # combine.
    route_launches = 2 if (cfg.dtype == configs.DTYPE_BF16 and cfg.E > 16) else 1
    launches = {"route": route_launches, "dispatch": 1, "up": 1, "down": 1, "combine": 1}

    def step(ev):
        ev[0].record()
        abi.route(p, inp.X, inp.W_r, inp.bias, logits, idx, gate, None, ws)
        ev[1].record()
        abi.dispatch(p, inp.X, idx, load, offsets, pos, dropped, row_token, X_perm, ws)
        ev[2].record()
        if packed:
            abi.expert_up_w8p(p, X_perm, offsets, wq.W1q, wq.S1, wq.W2q, wq.S2, H, ws)
        elif w8:
            abi.expert_up_w8(p, X_perm, offsets, wq.W1q, wq.S1, wq.W2q, wq.S2, H, ws)
        else:
            abi.expert_up(p, X_perm, offsets, inp.W1, inp.W2, H, ws)
        ev[3].record()
        if packed:
            abi.expert_down_w8p(p, H, offsets, wq.W3q, wq.S3, Y, ws)
        elif w8:
            abi.expert_down_w8(p, H, offsets, wq.W3q, wq.S3, Y, ws)
        else:
            abi.expert_down(p, H, offsets, inp.W3, Y, ws)
        ev[4].record()
        abi.combine(p, Y, idx, gate, offsets, pos, dropped, out)
        ev[5].record()

    def new_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(6)]

    warm = []
    for _ in range(args.warmup):
        ev = new_events()
        step(ev)
        warm.append(ev)
        flush_l2()
    torch.cuda.synchronize(device)
    if abi.device_error(ws) != 0:
        raise RuntimeError("device error during warm-up")
    if args.steps is None:  # enough steps for a timed region of about TIMED_REGION_TARGET_S
        t_step = min(ev[0].elapsed_time(ev[5]) for ev in warm[-2:]) / 1e3
        want = max(20, min(20000, math.ceil(TIMED_REGION_TARGET_S / max(t_step, 1e-6))))
        args.steps = int(reduce_max(float(want), device))

    # With --graph the step (its five stages and the events between them) is captured once
    # into a CUDA graph and each timed step is one replay; the stage times are read after each
    # replay (a host wait between steps, outside the events).
    graph, graph_note = None, None
    if args.graph:
        try:
            # external: recorded as event nodes of the graph, readable after each replay
            gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)]
            graph = torch.cuda.CUDAGraph()
            torch.cuda.synchronize(device)
            with torch.cuda.graph(graph):
                step(gev)
            for _ in range(2):
                graph.replay()
                flush_l2()
            torch.cuda.synchronize(device)
            if abi.device_error(ws) != 0:
                raise RuntimeError("device error in the captured step")
        except Exception as ex:  # capture unsupported here: time the steps as launched
            graph, graph_note = None, f"capture failed: {ex}"[:200]
            torch.cuda.synchronize(device)

    sampler = ClockSampler(device.index).start()
    barrier(device)
    torch.cuda.synchronize(device)
    t_wall0 = time.time()
    evs = []
    if graph is not None:
        for _ in range(args.steps):
            graph.replay()
            gev[5].synchronize()
            evs.append([gev[i].elapsed_time(gev[i + 1]) for i in range(5)])
            flush_l2()   # outside the step's events
    else:
        for _ in range(args.steps):
            ev = new_events()
            step(ev)
            evs.append(ev)
            flush_l2()   # outside the step's events
    torch.cuda.synchronize(device)
    barrier(device)
    t_wall1 = time.time()
    sampler.stop()
    if graph is None:  # stage times from the events of each step
        evs = [[ev[i].elapsed_time(ev[i + 1]) for i in range(5)] for ev in evs]
    if abi.device_error(ws) != 0:
        raise RuntimeError("device error during the timed steps")
    clocks = sampler.summary(t_wall0, t_wall1)
    clocks["timed_region_s"] = t_wall1 - t_wall0
    # The tensor-core denominator: the sustained cuBLAS figure for kernels timed inside a long
    # run (a timed region of a second or more, or the power cap active), the burst figure for
    # a short one; the other is reported beside it.
    sustained = clocks["timed_region_s"] >= 1.0 or "sw_power_cap" in clocks.get("reasons", [])

    per = {n: [ev[i] for ev in evs] for i, n in enumerate(names)}
    total_ms = sum(sum(ev) for ev in evs)
    max_total = reduce_max(total_ms, device)
    agg = aggregate(N, world, max_total, args.steps)
    mean = {n: sum(v) / len(v) for n, v in per.items()}

    kept = int(offsets[E].item())
    tokens_with_kept = int((dropped == 0).any(1).sum().item())
    es = 2 if cfg.dtype == configs.DTYPE_BF16 else 4
    flops_up = 4.0 * kept * D * F
    flops_down = 2.0 * kept * D * F
    bytes_route = N * D * es + D * E * 4 + N * k * 8
    bytes_gather = (tokens_with_kept + kept) * D * es
    bytes_combine = kept * D * es + N * D * es + N * k * 13
    hbm = peaks["hbm_gbs"]
    tc_burst = peaks["bf16_tflops"]
    tc = peaks["bf16_tflops_sustained"] if sustained else tc_burst
    tc_kind = "bf16 sustained" if sustained else "bf16 burst"
    kern = {
        "route": {"ms": mean["route"], "GB/s": bytes_route / mean["route"] / 1e6},
        "dispatch": {"ms": mean["dispatch"], "gather_GB/s_lower_bound":
                     bytes_gather / mean["dispatch"] / 1e6},
        "up": {"ms": mean["up"], "TFLOP/s": flops_up / mean["up"] / 1e9},
        "down": {"ms": mean["down"], "TFLOP/s": flops_down / mean["down"] / 1e9},
        "combine": {"ms": mean["combine"], "GB/s": bytes_combine / mean["combine"] / 1e6},
    }
    for n in ("route", "combine"):
        kern[n]["frac_hbm"] = kern[n]["GB/s"] / hbm
        kern[n]["frac_8TBs"] = kern[n]["GB/s"] / DATASHEET_HBM_GBS
    # The router's other ceiling: the 2 N D E multiply-adds of fp32 logits on the fp32 FMA
    # units (148 SMs x 128 lanes x 2 FLOP per clock at the datasheet clock). At E = 64 it is
    # longer than the HBM time, so no fp32 SIMT router reaches the HBM target there; this
    # router runs the contraction on the tensor cores (three bf16 terms of W_r).
    ffma_floor_s = 2.0 * N * D * E / (DATASHEET_SMS * 128 * 2 * DATASHEET_SM_MHZ * 1e6)
    kern["route"]["fp32_ffma_floor_us"] = ffma_floor_s * 1e6
    kern["route"]["hbm_floor_us"] = bytes_route / (hbm * 1e9) * 1e6
    kern["route"]["time_over_larger_floor"] = (max(ffma_floor_s, bytes_route / (hbm * 1e9))
                                               / (mean["route"] / 1e3))
    for n in ("up", "down"):
        kern[n]["frac_bf16_peak"] = kern[n]["TFLOP/s"] / tc
        kern[n]["frac_bf16_burst"] = kern[n]["TFLOP/s"] / tc_burst
        kern[n]["frac_bf16_datasheet"] = kern[n]["TFLOP/s"] / DATASHEET_BF16_TFLOPS
    ffn_ms = mean["up"] + mean["down"]
    gemm_tflops = 6.0 * kept * D * F / ffn_ms / 1e9

    # Roofline of the up-projection kernel: the larger of its FLOPs at the bf16 peak and its
    # algorithmic bytes at the HBM peak (A rows read once, the weights of every expert that
    # keeps a row read once, H written once).
    used = int((offsets[1:] - offsets[:-1] > 0).sum().item())
    # 8-bit weights: one byte per weight plus the fp32 column scales.
    ew = 1 if w8 else es
    bytes_up = kept * D * es + used * 2.0 * (D * F * ew + (F * 4 if w8 else 0)) + kept * F * es
    t_tensor = flops_up / (tc * 1e12) if cfg.dtype == configs.DTYPE_BF16 else 0.0
    t_hbm = bytes_up / (hbm * 1e9)
    dom = "up"
    psrc = peak_key_source(peak_src, "bf16_tflops_sustained" if sustained else "bf16_tflops")
    if t_tensor < t_hbm:
        psrc = peak_key_source(peak_src, "hbm_gbs")
    if t_tensor >= t_hbm:
        roof = {"kernel": up_kernel + " (expert up-projection + gating)",
                "bound": "tensor", "achieved": kern["up"]["TFLOP/s"], "peak": tc,
                "unit": "TFLOP/s", "frac": kern["up"]["TFLOP/s"] / tc,
                "peak_source": f"{psrc}, {tc_kind}", "frac_burst": kern["up"]["TFLOP/s"] / tc_burst,
                "flops_per_launch": flops_up}
    else:
        gbs = bytes_up / mean["up"] / 1e6
        roof = {"kernel": up_kernel
                + " (expert up-projection; bound by streaming the used experts' weights)",
                "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                "frac": gbs / hbm, "peak_source": psrc, "bytes_per_launch": bytes_up}
    roof["min_us"] = {"tensor": t_tensor * 1e6, "hbm": t_hbm * 1e6}
    roof["denominator"] = ("peak = the " + (f"cuBLAS {tc_kind} GEMM figure" if
                           roof["bound"] == "tensor" else "HBM copy bandwidth") +
                           f" ({psrc}); frac_datasheet uses the B200 datasheet figure")
    roof["peak_datasheet"] = (DATASHEET_BF16_TFLOPS if roof["bound"] == "tensor"
                              else DATASHEET_HBM_GBS)
    roof["frac_datasheet"] = roof["achieved"] / roof["peak_datasheet"]
    roof["experts_used"] = used
    # Same two-sided bound for both GEMMs: frac_roofline = bound time / measured time.
    bytes_down = kept * F * es + used * (D * F * ew + (D * 4 if w8 else 0)) + kept * D * es
    for n, fl, by in (("up", flops_up, bytes_up), ("down", flops_down, bytes_down)):
        t_min = max(fl / (tc * 1e12) if cfg.dtype == configs.DTYPE_BF16 else 0.0,
                    by / (hbm * 1e9))
        kern[n]["frac_roofline"] = t_min * 1e3 / mean[n]
    roof["traffic"] = traffic_from_profile(
        ("up_w8p" if packed else "up_w8" if w8 else "up"), cfg.name)

    # end-to-end through the public entry points, host X in and host out inside the timed
    # region: moe_forward_host (bf16 weights; it copies and synchronises itself) or, for 8-bit
    # weights, pinned-host copies around moe_forward_w8. For bf16 weights the reported value is
    # the streamed form, moe_forward_host_many over the timed steps (calls of up to 8 batches:
    # each batch's input and output copies overlap the neighbouring batches' layers), and the
    # one-call-per-step figure is kept beside it.
    ws_h = abi.workspace(p, device, host=True)
    xh = inp.X.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    xd = torch.empty_like(inp.X)
    od = torch.empty_like(inp.X)

    def e2e_call():
        if w8:
            xd.copy_(xh, non_blocking=True)
            abi.forward_w8(p, xd, inp.W_r, inp.bias, wq, od, ws, packed=packed)
            oh.copy_(od, non_blocking=True)
        else:
            abi.forward_host(p, xh, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, oh, ws_h)

    for _ in range(2):
        e2e_call()
    torch.cuda.synchronize(device)
    barrier(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e_total = 0.0
    for _ in range(args.steps):
        flush_l2()
        e0.record(stream)
        e2e_call()
        e1.record(stream)
        e1.synchronize()
        e_total += e0.elapsed_time(e1)
    e_max = reduce_max(e_total, device)
    e2e_value = N * world * args.steps / (e_max / 1e3)
    e2e_single = None
    if not w8:
        e2e_single = e2e_value
        nb = min(args.steps, 8)
        xh_many = xh.unsqueeze(0).expand(nb, -1, -1).contiguous().pin_memory()
        oh_many = torch.empty_like(xh_many).pin_memory()
        abi.forward_host_many(p, xh_many, inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3, oh_many,
                              ws_h)
        torch.cuda.synchronize(device)
        barrier(device)
        e_total = 0.0
        done = 0
        while done < args.steps:
            n = min(nb, args.steps - done)
            flush_l2()
            e0.record(stream)
            abi.forward_host_many(p, xh_many[:n], inp.W_r, inp.bias, inp.W1, inp.W2, inp.W3,
                                  oh_many[:n], ws_h)
            e1.record(stream)
            e1.synchronize()
            e_total += e0.elapsed_time(e1)
            done += n
        e_max = reduce_max(e_total, device)
        e2e_value = N * world * args.steps / (e_max / 1e3)
        del xh_many, oh_many
    h2d = N * D * es
    d2h = N * D * es
    # The layer's diagnostics (an extra, untimed route call that also writes prob_colsum).
    colsum = torch.empty((E,), dtype=torch.float32, device=device)
    abi.route(p, inp.X, inp.W_r, inp.bias, None, idx, gate, colsum, ws)
    abi.dispatch(p, inp.X, idx, load, offsets, pos, dropped, row_token, X_perm, ws)
    torch.cuda.synchronize(device)
    load_h = load.cpu().double()
    diagnostics = {"balance_loss": abi.balance_loss(p, load, colsum),
                   "drop_rate": abi.drop_rate(p, dropped),
                   "load_max_over_mean": float(load_h.max() / load_h.mean())}
    barrier(device)

    line = {
        "metric": METRIC, "value": agg["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": agg["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype_name(cfg),
        "data": "synthetic, seeded: X~N(0,1), W_r/W1/W2~N(0,1/D), W3~N(0,1/F)"
                + (", bias~N(0,2)" if cfg.router_bias_var > 0 else ""),
        "config": {"workload": workload_desc(cfg, w8, packed), "tokens_per_gpu": N,
                   "expert_weights": "int8 + fp32 scale per expert and output column" if w8
                   else dtype_name(cfg),
                   "parallelism": f"replicas x{world} (no data-path collective)",
                   "l2": "flushed between steps (512 MiB write + read-back, outside the step events)",
                   "launch": ("CUDA graph of the step, one replay per step" if graph is not None
                              else "stream launches" + (f" ({graph_note})" if graph_note else "")),
                   "kept_records": kept,
                   "diagnostics": diagnostics,
                   "grouped_gemm_TFLOP/s": gemm_tflops,
                   "grouped_gemm_frac_bf16_peak": gemm_tflops / tc,
                   "kernels": kern},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "api": (f"moe_forward_w8{'p' if packed else ''} between pinned-host copies of"
                        " X and out" if w8 else
                        "moe_forward_host_many (pinned host batches in and out, up to 8 per "
                        "call; each batch's copies overlap the neighbouring batches' layers)")
                       + "; copies in the timed region",
                "single_call_value": e2e_single,
                "single_call_api": None if w8 else "moe_forward_host, one call per step"},
        "gpu_launches": sum(launches.values()) * args.steps,
        "clocks": clocks,
    }
    mhz = line["clocks"].get("sm_mhz")
    if roof["bound"] == "tensor" and mhz:
        # Tensor throughput scales with the SM clock: the achieved rate against the datasheet
        # peak scaled to the median clock of the timed region.
        roof["frac_datasheet_at_run_clock"] = roof["achieved"] / (
            DATASHEET_BF16_TFLOPS * float(mhz) / DATASHEET_SM_MHZ)
    # For the oracle leg (not printed): the routing of the benched inputs, and the inputs.
    line["_gpu_idx"] = idx.cpu().numpy()
    line["_inp"], line["_wq"] = inp, wq
    return line


def run_gpu_ep(args, cfg, world, rank, device):
    """Expert-parallel layer (ep.forward): experts in contiguous blocks over the ranks, each
    rank routing its own cfg.N tokens (weak scaling). Every step: route + dispatch, count and
    row exchanges (NCCL all_to_all_single), expert-major reorder, the rank's grouped GEMMs,
    reorder back, return exchange, combine. Device time per step, max over ranks."""
    import torch
    from top_routing_expert_fp32_b200 import configs, ep, inputs

    torch.cuda.set_device(device)
    peaks, peak_src = load_peaks()
    full = inputs.make_inputs(cfg, device)
    e0, e1 = ep.expert_ranges(cfg.E, world)[rank]
    W1, W2, W3 = (w[e0:e1].clone() for w in (full.W1, full.W2, full.W3))
    X = full.X if rank == 0 else inputs.randn((cfg.N, cfg.D), 1.0, full.X.dtype, device,
                                              cfg.seed + 1 + rank, inputs.TID_X)
    W_r, bias = full.W_r, full.bias
    del full
    torch.cuda.empty_cache()
    comp = ep.CudaCompute(cfg, W_r, bias, W1, W2, W3, device)
    N, D, F, k = cfg.N, cfg.D, cfg.F, cfg.k
    es = X.element_size()
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.int32, device=device)
    flush_sum = torch.empty((), dtype=torch.int64, device=device)

    def flush_l2():
        flush.fill_(1)
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)
    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        ep.forward(comp, X, cfg.E)
    torch.cuda.synchronize(device)
    assert comp.device_error() == 0
    barrier(device)
    sampler = ClockSampler(device.index)
    sampler.start()
    t_wall0 = time.time()
    e0v = torch.cuda.Event(enable_timing=True)
    e1v = torch.cuda.Event(enable_timing=True)
    total = 0.0
    kept = 0
    off_rank = 0
    for _ in range(args.steps):
        flush_l2()
        e0v.record(stream)
        _, info = ep.forward(comp, X, cfg.E)
        e1v.record(stream)
        e1v.synchronize()
        total += e0v.elapsed_time(e1v)
        plan = info["plan"]
        kept = sum(plan.send_rows)
        # rows leaving this rank: its records for other ranks' experts, then the outputs it
        # returns to other ranks
        off_rank = ((kept - plan.send_rows[rank]) +
                    (sum(plan.recv_rows) - plan.recv_rows[rank])) * D * es
    t_wall1 = time.time()
    sampler.stop()
    mx = reduce_max(total, device)
    agg = aggregate(N, world, mx, args.steps)
    tc, hbm = peaks["bf16_tflops"], peaks["hbm_gbs"]
    # Step bound: the expert GEMM FLOPs of this rank's received rows at the bf16 peak, or the
    # rows this rank sends off-rank (both exchanges) at the measured 770 GB/s peer copy rate.
    recv = sum(plan.recv_rows)
    flops = 6.0 * recv * D * F
    t_tc = flops / (tc * 1e12)
    t_link = off_rank / 770e9
    step_s = agg["ms_per_step"] / 1e3
    roof = {"kernel": "whole expert-parallel step (expert GEMMs of the received rows; "
                      "off-rank rows over NVLink)",
            "bound": "tensor" if t_tc >= t_link else "nvlink",
            "achieved": (flops / step_s / 1e12) if t_tc >= t_link else off_rank / step_s / 1e9,
            "peak": tc if t_tc >= t_link else 770.0,
            "unit": "TFLOP/s" if t_tc >= t_link else "GB/s",
            "peak_source": (peak_key_source(peak_src, "bf16_tflops") + ", bf16 burst"
                            if t_tc >= t_link
                            else "measured 8-GPU peer copy per direction (pool figure)"),
            "traffic": None}
    roof["frac"] = roof["achieved"] / roof["peak"]

    xh = X.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    xd = torch.empty_like(X)

    def e2e_call():
        xd.copy_(xh, non_blocking=True)
        out, _ = ep.forward(comp, xd, cfg.E)
        oh.copy_(out, non_blocking=True)

    e2e_call()
    torch.cuda.synchronize(device)
    barrier(device)
    et = 0.0
    for _ in range(args.steps):
        flush_l2()
        e0v.record(stream)
        e2e_call()
        e1v.record(stream)
        e1v.synchronize()
        et += e0v.elapsed_time(e1v)
    e_max = reduce_max(et, device)
    barrier(device)
    # route (plus the router operand with bf16 X and more than 16 experts), dispatch,
    # 2 reorders, up + down, combine
    launches = (2 if (cfg.dtype == configs.DTYPE_BF16 and cfg.E > 16) else 1) + 1 + 2 + 2 + 1
    return {
        "metric": METRIC, "value": agg["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": agg["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype_name(cfg),
        "data": "synthetic, seeded: X~N(0,1) per rank, W_r/W1/W2~N(0,1/D), W3~N(0,1/F)",
        "config": {"workload": workload_desc(cfg), "tokens_per_gpu": N,
                   "parallelism": f"ep{world}: experts in contiguous blocks, rank {rank} holds "
                                  f"{e0}..{e1 - 1}; NCCL all_to_all_single exchanges",
                   "l2": "flushed between steps (512 MiB write + read-back, outside the step events)",
                   "kept_records_per_rank": kept,
                   "a2a_bytes_model_per_step": ep.a2a_bytes(N * world, D, k, es),
                   "off_rank_bytes_per_step_rank0": off_rank},
        "roofline": roof,
        "e2e": {"value": N * world * args.steps / (e_max / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": N * D * es, "d2h_bytes_per_step": N * D * es,
                "api": "ep.forward between pinned-host copies of X and out; copies in the "
                       "timed region"},
        "gpu_launches": launches * args.steps,
        "clocks": sampler.summary(t_wall0, t_wall1),
    }


# ------------------------------------------------------------------ main

ALL_WORKLOADS = ["tiny_f32", "mixtral", "grok1", "capacity", "capacity_k1", "capacity_gshard",
                 "decode"]


def oracle_leg(line, cfg, w8: bool, budget_s: float = 12.0):
    """Rank 0 at N=1 only, after the GPU work: the oracle timed on a sample of the GPU arm's own
    inputs (cpu_baseline), and the GPU routing compared with the oracle's (near-tie flips)."""
    o = OracleSample(cfg, w8, inp=line["_inp"], wq=line["_wq"])
    line["cpu_baseline"] = oracle_tokens_per_s(cfg, budget_s=budget_s, w8=w8, sampler=o)
    line["config"]["routing_vs_oracle"] = o.routing_check(line["_gpu_idx"])


def strip_private(line):
    for key in [k for k in line if k.startswith("_")]:
        del line[key]
    return line


def table_row(line) -> str:
    c = line["config"]
    k = c["kernels"]
    d = c.get("diagnostics", {})
    rv = c.get("routing_vs_oracle", {})
    cb = line.get("cpu_baseline") or {}
    clk = line.get("clocks", {})
    r = line["roofline"]
    return ("| {w} | {v:.4g} | {ms:.3f} | {up:.0f} ({upf:.2f}) | {dn:.0f} ({dnf:.2f}) | "
            "{rt:.1f} ({rtf:.2f}) | {cb:.1f} ({cbf:.2f}) | {roof:.2f} {bound} | {e2e:.4g} | "
            "{bl:.4f} | {dr:.4f} | {lm:.3f} | {fl} | {cpu} | {mhz} / {rs} |").format(
        w=c["workload"].split(":")[0], v=line["value"], ms=line["ms_per_step"],
        up=k["up"]["TFLOP/s"], upf=k["up"]["frac_roofline"], dn=k["down"]["TFLOP/s"],
        dnf=k["down"]["frac_roofline"], rt=k["route"]["ms"] * 1e3,
        rtf=k["route"]["frac_hbm"], cb=k["combine"]["ms"] * 1e3, cbf=k["combine"]["frac_hbm"],
        roof=r["frac"], bound=r["bound"], e2e=line["e2e"]["value"],
        bl=d.get("balance_loss", float("nan")), dr=d.get("drop_rate", float("nan")),
        lm=d.get("load_max_over_mean", float("nan")), fl=rv.get("flips", "-"),
        cpu=f"{cb['value']:.3g} ({cb.get('cores')} thr)" if cb else "-",
        mhz=clk.get("sm_mhz"), rs=",".join(clk.get("reasons", [])) or "-")


TABLE_HEAD = ("| workload | tokens/s | ms/step | up TF/s (roof) | down TF/s (roof) | route us "
              "(frac HBM) | combine us (frac HBM) | roofline frac | e2e tokens/s | balance loss "
              "| drop rate | load max/mean | near-tie flips | CPU oracle tokens/s | SM MHz / "
              "reasons |\n|" + "---|" * 15)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for a timed region of about 1.5 s)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--tokens", type=int, default=None,
                    help="override N (smaller cases for profiling)")
    ap.add_argument("--ffn", type=int, default=None,
                    help="override F (smaller weight footprint for profiling)")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "w8", "w8p"],
                    help="expert weights: bf16, or int8 with per-column fp32 scales")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "ep"],
                    help="replicas: one independent layer per GPU; ep: experts split over the "
                         "GPUs, rows exchanged by all-to-all (bf16 weights)")
    ap.add_argument("--graph", action="store_true",
                    help="capture the step into a CUDA graph and time its replays")
    ap.add_argument("--all-workloads", action="store_true",
                    help="one line per workload (1 GPU), each with diagnostics, near-tie flips "
                         "against the oracle's routing and the oracle's CPU throughput")
    ap.add_argument("--table", default=None,
                    help="with --all-workloads: also write a markdown table to this path")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from top_routing_expert_fp32_b200 import configs
    cfg = configs.CONFIGS[args.workload or configs.BENCH_WORKLOAD]
    if args.tokens is not None:
        cfg = cfg.with_(N=args.tokens, name=f"{cfg.name}_n{args.tokens}")
    if args.ffn is not None:
        cfg = cfg.with_(F=args.ffn, name=f"{cfg.name}_f{args.ffn}")
    world, rank, local = dist_env()
    w8 = args.weights != "bf16"

    if args.impl == "reference":
        if rank != 0:
            return 0
        if args.steps is None:
            args.steps = 20
        line = run_reference(args, cfg, w8, args.weights == "w8p")
        line["n_gpus"] = world
        print(json.dumps(line))
        return 0

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    if args.all_workloads:
        if world != 1:
            raise SystemExit("--all-workloads runs on one GPU")
        device = torch.device("cuda", local)
        rows = []
        steps = args.steps
        for name in ALL_WORKLOADS:
            c = configs.CONFIGS[name]
            args.steps = steps if steps is not None else 10
            line = run_gpu(args, c, 1, 0, device)
            if not args.no_cpu_baseline:
                oracle_leg(line, c, w8, budget_s=8.0)
            strip_private(line)
            print(json.dumps(line), flush=True)
            rows.append(table_row(line))
            del line
            torch.cuda.empty_cache()
        if args.table:
            with open(args.table, "w") as f:
                f.write(TABLE_HEAD + "\n" + "\n".join(rows) + "\n")
        return 0

    ep_mode = args.parallel == "ep"
    if ep_mode and w8:
        raise SystemExit("--parallel ep runs bf16 expert weights")
    launched = "MASTER_ADDR" in os.environ  # under torchrun: its env:// rendezvous and store
    if world > 1 or (ep_mode and launched):
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif ep_mode:  # the exchanges need a process group, even of one rank
        import socket
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
        sk.close()
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    if ep_mode and args.steps is None:
        args.steps = 20
    line = (run_gpu_ep if ep_mode else run_gpu)(args, cfg, world, rank, device)
    if rank == 0:
        if not args.no_cpu_baseline and world == 1 and not ep_mode:
            oracle_leg(line, cfg, w8)
        else:
            line["cpu_baseline"] = None
        print(json.dumps(strip_private(line)))
    else:
        strip_private(line)
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
