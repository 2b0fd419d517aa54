#!/usr/bin/env python
"""Benchmark of the MoE layer hot path (route -> dispatch -> grouped FFN ->
combine) on B200, printing one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode]
  python bench.py --impl reference ...   # the CPU oracle, timed on host cores

One step = one whole layer over one batch of the workload (default: the
decode layer, T=128, H=7168, E=256, top-8, I=2048, FP8 block-scaled weights).
Under torchrun every rank runs its own replica on its own GPU (the layer has no
data-path collective); value = tokens of all ranks / max over ranks of the
device time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer µs & tokens/s (decode T=128, prefill T=8192); % of HBM/FP8 roofline"
PROFILES = os.path.join(ROOT, "profiles")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--config", default="decode")
    p.add_argument("--T", type=int, default=None, help="override the token count")
    p.add_argument("--E", type=int, default=None, help="override the expert count (small profiling cases)")
    p.add_argument("--shared-expert", action="store_true",
                   help="add one shared expert every token also goes through (weight 1)")
    p.add_argument("--compact", action="store_true",
                   help="compact expert windows: a counting pass, then windows packed back to back")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="wall-clock budget of the CPU oracle sample")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the prefill and MX FP4 objects of the default bench line")
    p.add_argument("--record-traffic", default=None, metavar="NCU_CSV",
                   help="write the DRAM bytes per launch found in an ncu --csv metrics log to "
                        "profiles/traffic.json (with --tag and --kernel) and exit")
    p.add_argument("--tag", default="grouped_ffn/decode")
    p.add_argument("--kernel", default="ffn_tc_kernel")
    p.add_argument("--how", default="")
    p.add_argument("--overlap-sweep", action="store_true",
                   help="print one JSON line per workload (decode, prefill on compact windows) timing "
                        "the layer with dispatch beside the grouped FFN over a sweep of partition sizes")
    p.add_argument("--fp8-gemm-peak", action="store_true",
                   help="print one JSON line: cuBLAS e4m3 GEMM throughput on this GPU (8192^3, "
                        "tensor-wise scales), best of 10 and back to back for 4 s with clocks, for "
                        "context beside the 2 x bf16 roof")
    p.add_argument("--report", action="store_true",
                   help="instead of the single bench line: one JSON line per workload "
                        "(tiny, decode, prefill, skew, dispatch+combine sweep) with per-stage "
                        "times and roofline fractions")
    return p.parse_args()


def overrides(args) -> dict:
    o = {}
    if args.T:
        o["T"] = args.T
    if args.E:
        o["E"] = args.E
    if getattr(args, "shared_expert", False):
        o["shared"] = 1
    if getattr(args, "compact", False):
        o["compact"] = 1
    return o


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), \
        int(os.environ.get("WORLD_SIZE", 1))


def max_over_ranks(value: float, device=None) -> float:
    """The largest of every rank's value (one all-reduce); the value itself
    when there is no process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: the tokens of all ranks over the slowest rank's time."""
    return tokens_per_rank * world / (max_ms / 1000.0)


# ------------------------------------------------------------ GPU clocks --

class ClockSampler:
    """Samples the SM clock, its maximum, board power and the active clock
    event (throttle) reasons of one GPU every few milliseconds through NVML,
    in a background thread, while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device_index: int, period_s: float = 0.002):
        self.idx = torch_device_index
        self.period = period_s
        self.rows = []
        self.thread = None
        self.stop_flag = False
        self.nvml = None
        self.handle = None

    def _open(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        self.nvml = pynvml
        try:
            props = torch.cuda.get_device_properties(self.idx)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def _run(self):
        nv, h = self.nvml, self.handle
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.rows.append((sm, mx, pw, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        import threading
        try:
            self._open()
        except Exception:
            self.nvml = None
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.rows and time.time() - t0 < 1.0:
            time.sleep(0.001)

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=2)
        if not self.rows:
            return None
        reasons = set()
        for r in self.rows:
            for bit, name in self.REASONS.items():
                if r[3] & bit:
                    reasons.add(name)
        loaded = [r[0] for r in self.rows if r[2] > 200.0] or [r[0] for r in self.rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in self.rows),
                "reasons": sorted(reasons), "samples": len(self.rows),
                "power_w_max": max(r[2] for r in self.rows), "source": "NVML, 2 ms period"}


# ------------------------------------------------------------ CPU oracle --

def oracle_sample(spec, inp, seconds: float, max_tokens: int | None = None, threads: int | None = None):
    """Time the CPU oracle on the first tokens of the workload until `seconds`
    of wall time are spent, on all host cores or on `threads` of them.
    Returns (tokens, elapsed_s, cores)."""
    import numpy as np
    import torch
    import oracle

    all_cores = len(os.sched_getaffinity(0))
    cores = oracle.set_threads(threads if threads else all_cores)
    odt = {"f32": oracle.F32, "bf16": oracle.BF16, "e4m3": oracle.E4M3, "e2m1": oracle.E2M1}

    def host(t):
        t = t.detach().cpu().contiguous()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    logits = host(inp["logits"])
    x = host(inp["x"])
    idx, _ = oracle.route(logits, spec.k, spec.renorm)
    if spec.shared:   # every token also goes through the shared expert E
        idx = np.concatenate([idx, np.full((idx.shape[0], 1), spec.E, idx.dtype)], axis=1)
    limit = spec.T if max_tokens is None else min(spec.T, max_tokens)
    chunk = max(1, min(cores, limit))
    done = 0
    elapsed = 0.0
    while done < limit and elapsed < seconds:
        t1 = min(limit, done + chunk)
        kw = {}
        if not spec.identity:
            experts = sorted(set(idx[done:t1].ravel().tolist()))
            for n in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
                # 4-bit weights: the oracle reads per-row scales, the library scale atoms
                m = n + "_rows" if (spec.weight == "e2m1" and n[0] == "s") else n
                if inp.get(m) is not None:
                    kw[n] = {e: host(inp[m][e]) for e in experts}
        p = oracle.Problem(spec.T, spec.H, spec.E, spec.k, spec.I, shared=spec.shared, x_dtype=odt[spec.act],
                           xq_dtype=odt[spec.xq], w_dtype=odt[spec.weight], h_dtype=odt[spec.h],
                           y_dtype=odt[spec.y], out_dtype=odt[spec.out], renorm=spec.renorm,
                           identity=spec.identity, **kw)
        t_start = time.perf_counter()
        oracle.moe_layer(p, x, logits, done, t1)
        elapsed += time.perf_counter() - t_start
        done = t1
    oracle.set_threads(all_cores)
    return done, elapsed, cores


# ------------------------------------------------------------ roofline --

def ffn_algorithmic_bytes(spec, counts):
    """Bytes the grouped FFN must move at least once: the weights of every
    touched expert (matrices + scales), the dispatched rows read, h written
    and read back, y written."""
    from combine_softmax_top_b200 import workloads as W
    el = {"f32": 4, "bf16": 2, "e4m3": 1}
    touched = int((counts > 0).sum())
    rows = int(counts.sum())
    w = touched * W.bytes_per_expert(spec)
    xs = spec.H // 128 * 4 if spec.xq == "e4m3" else 0
    hs = spec.I // 128 * 4 if spec.h == "e4m3" else 0
    act = rows * (spec.H * el[spec.xq] + xs) + 2 * rows * (spec.I * el[spec.h] + hs) \
        + rows * spec.H * el[spec.y]
    return w + act, touched


def ffn_flops(spec, rows):
    return 6.0 * spec.H * spec.I * rows


TRAFFIC_JSON = os.path.join(PROFILES, "traffic.json")


def recorded_traffic(kernel_tag: str, algorithmic_bytes: int):
    """DRAM bytes per launch of the FFN kernel for one workload: the ratio of
    DRAM bytes to algorithmic bytes that `python bench.py --record-traffic`
    took from an ncu capture of a smaller case of the same kernel variant,
    applied to this launch's algorithmic bytes; None unless the capture was
    taken on the current source of the kernel."""
    if not os.path.exists(TRAFFIC_JSON):
        return None
    rec = json.load(open(TRAFFIC_JSON)).get(kernel_tag)
    if not rec or rec.get("source_sha") != kernel_source_sha() or "traffic_ratio" not in rec:
        return None
    return int(round(rec["traffic_ratio"] * algorithmic_bytes))


def ncu_dram_bytes(csv_path: str, kernel_regex: str):
    """Mean dram__bytes_read.sum + dram__bytes_write.sum per launch of the
    kernels matching `kernel_regex` in an ncu `--csv` metrics log, and the
    number of launches it covers."""
    import csv
    import re as _re
    per = {}
    with open(csv_path, newline="") as f:
        rows = [r for r in csv.reader(f) if r]
    head = next(i for i, r in enumerate(rows) if "Metric Name" in r)
    cols = rows[head]
    ki, mi, vi, ui, ii = (cols.index(c) for c in ("Kernel Name", "Metric Name", "Metric Value", "Metric Unit", "ID"))
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    for r in rows[head + 1:]:
        if len(r) <= vi or not _re.search(kernel_regex, r[ki]):
            continue
        if r[mi] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            v = float(r[vi].replace(",", "")) * scale.get(r[ui], 1)
            per[r[ii]] = per.get(r[ii], 0.0) + v
    if not per:
        raise ValueError(f"no DRAM byte metrics for {kernel_regex!r} in {csv_path}")
    return sum(per.values()) / len(per), len(per)


def record_traffic(args):
    """Write one profiles/traffic.json entry from an ncu capture of the
    workload named by --config/--T/--E/--compact: its DRAM bytes per launch
    over the launch's algorithmic bytes (routing recomputed on the host from
    the same seeded logits, top-k on the logits)."""
    import numpy as np
    import torch
    from combine_softmax_top_b200 import workloads as W
    mean, n = ncu_dram_bytes(args.record_traffic, args.kernel)
    spec = W.spec(args.config, **overrides(args))
    inp = W.make_inputs(spec, seed=args.seed, device="cpu", with_weights=False)
    idx = torch.topk(inp["logits"], spec.k, dim=1).indices
    counts = torch.bincount(idx.flatten(), minlength=spec.E).numpy()
    if spec.shared:
        counts = np.concatenate([counts, [spec.T]])
    algo, touched = ffn_algorithmic_bytes(spec, counts)
    rec = json.load(open(TRAFFIC_JSON)) if os.path.exists(TRAFFIC_JSON) else {}
    rec[args.tag] = {"source_sha": kernel_source_sha(), "traffic_ratio": mean / algo,
                     "captured": {"workload": workload_config(spec, 1)["workload"], "dram_bytes_per_launch": int(round(mean)),
                                  "algorithmic_bytes_per_launch": int(algo), "touched_experts": touched, "launches": n},
                     "kernel": args.kernel, "how": args.how}
    with open(TRAFFIC_JSON, "w") as f:
        json.dump(rec, f, indent=1, sort_keys=True)
        f.write("\n")
    print(json.dumps({args.tag: rec[args.tag]}))


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "combine_softmax_top_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.startswith("ffn_") or name.endswith(".cuh"):
            h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------ reference --

def workload_config(spec, world: int) -> dict:
    """The `config` object of both arms' lines (one definition, so that the
    two describe the same workload)."""
    from combine_softmax_top_b200 import workloads as W
    wgb = 0.0 if spec.identity else W.bytes_per_expert(spec) * spec.ne / 1e9
    return {"workload": f"{spec.name} MoE layer T={spec.T} H={spec.H} E={spec.E} "
                        f"top-{spec.k}{' + 1 shared expert' if spec.shared else ''} I={spec.I} "
                        f"{WEIGHT_DESC.get(spec.weight, spec.weight)}",
            "T": spec.T, "H": spec.H, "E": spec.E, "topk": spec.k, "I": spec.I, "shared_experts": spec.shared,
            "compact_windows": spec.compact,
            "act_dtype": spec.act, "xq_dtype": spec.xq, "weight_dtype": spec.weight, "h_dtype": spec.h,
            "y_dtype": spec.y, "out_dtype": spec.out,
            "parallelism": f"replicas x{world}",
            "l2": "flushed (256 MB write) before every timed step" +
                  (f"; weights {wgb:.1f} GB > 126 MB L2" if wgb > 0.126 else "")}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on the host cores, on
    the same inputs as the GPU arm (drawn with the same generator, on the GPU
    when there is one, then copied to the host once). One step is a bounded
    sample of the workload: the oracle runs the layer on the first tokens
    until the step's time budget is spent; ms_per_step is the measured wall
    time of those steps."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    from combine_softmax_top_b200 import workloads as W
    import torch
    spec = W.spec(args.config, **overrides(args))
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    inp = W.make_inputs(spec, seed=args.seed, device=dev)
    inp = {k: (v.cpu() if v is not None else None) for k, v in inp.items()}
    if dev.type == "cuda":
        torch.cuda.empty_cache()
    per_step = max(1.0, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(spec, inp, per_step / 4)
    tok = el = 0.0
    cores = 1
    walls = []
    for _ in range(args.steps):
        w0 = time.perf_counter()
        n, e, cores = oracle_sample(spec, inp, per_step)
        walls.append(time.perf_counter() - w0)
        tok += n
        el += e
    value = tok / el
    per = tok / max(1, args.steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * float(statistics.mean(walls)), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64",
        "data": f"synthetic (seeded; the GPU arm's inputs, drawn on {dev.type} and copied to the host)",
        "config": workload_config(spec, world),
        "step": f"a bounded sample: the layer on the first {per:.0f} of {spec.T} tokens "
                f"(up to {per_step:.1f}s of oracle time per step)",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {per:.0f} of {spec.T} tokens per step, {args.steps} steps"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


EL = {"f32": 4, "bf16": 2, "e4m3": 1}
# Weight formats in the workload line. Both block-scaled tensor-core paths
# (e4m3 tokens against e4m3 or MX FP4 weights) are rated at the 8-bit peak,
# twice the measured bf16 one.
WEIGHT_DESC = {"e4m3": "e4m3 128x128-block weights, bf16 tokens",
               "e2m1": "MX FP4 weights (e2m1, UE8M0 per 32), e4m3 tokens, bf16 x"}


def route_bytes(spec):
    return spec.T * (4 * spec.E + 8 * spec.ks)


def dispatch_bytes(spec):
    """x read once, k rows (+ scales and scale atoms) written, pos/row_src
    (k + 1 slots with a shared expert)."""
    per_pair = spec.H * EL[spec.xq] + 8
    if spec.xq == "e4m3":
        per_pair += 2 * (spec.H // 128) * 4
    return spec.T * (spec.H * EL[spec.act] + 4 * spec.ks + spec.ks * per_pair)


def combine_bytes(spec):
    """k rows gathered (identity: e4m3 rows + scales), pos and weights, out written."""
    if spec.identity:
        row = spec.H * EL[spec.xq] + ((spec.H // 128) * 4 if spec.xq == "e4m3" else 0)
    else:
        row = spec.H * EL[spec.y]
    return spec.T * (spec.ks * (row + 8) + spec.H * EL[spec.out])


def time_layer(spec, inp, b, steps, warmup, stream, flush):
    """Per-stage device times (ms, one row per step) through the per-stage
    C-ABI calls, with L2 flushed before every step (flush=None: warm L2, the
    previous step's data left in it)."""
    import numpy as np
    import torch
    from combine_softmax_top_b200 import moe

    w = moe.weights_struct(inp) if not spec.identity else moe.moe_weights()
    bufs = b.dispatch_bufs()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        moe.moe_route(b.shape, inp["logits"], b.topk_idx, b.topk_w, b.ws, stream)
        if ev:
            ev[1].record(stream)
        moe.moe_dispatch(b.shape, inp["x"], b.topk_idx, b.ws, bufs, stream)
        if ev:
            ev[2].record(stream)
        if not spec.identity:
            moe.moe_grouped_ffn(b.shape, bufs, w, b.ws, b.y, stream)
        if ev:
            ev[3].record(stream)
        moe.moe_combine(b.shape, bufs, b.y, b.topk_w, b.ws, b.out, stream)
        if ev:
            ev[4].record(stream)

    for _ in range(max(3, warmup)):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        step(evs[i])
    torch.cuda.synchronize()
    rc = moe.moe_poll_status(b.ws, stream)
    if rc != 0:
        raise RuntimeError(f"layer reported {moe.moe_status_string(rc)}")
    return np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in range(steps)])


def time_e2e_pipelined(spec, inp, b, w, bufs, stream, flush, steps, dev):
    """Steps of H2D (x, logits) -> moe_layer -> D2H (out), copies overlapped
    with the neighbouring steps' layers on two copy streams (one per
    direction, so the two directions of the host link overlap too); returns
    ms per step from the first copy to the last. The layer is the public
    moe_layer call with its intermediates in its own workspace."""
    import torch
    from combine_softmax_top_b200 import moe
    from combine_softmax_top_b200 import workloads as W
    lw = moe.alloc_layer(spec, device=dev)
    hx = inp["x"].cpu().pin_memory()
    hl = inp["logits"].cpu().pin_memory()
    ho = [torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory() for _ in range(2)]
    dx = [torch.empty_like(inp["x"]) for _ in range(2)]
    dl = [torch.empty_like(inp["logits"]) for _ in range(2)]
    dout = [lw.out, torch.empty_like(lw.out)]
    cs = torch.cuda.Stream(device=dev)        # host -> device
    co = torch.cuda.Stream(device=dev)        # device -> host
    weight_bytes = 0 if spec.identity else W.bytes_per_expert(spec) * spec.ne
    flush_each = weight_bytes < 4 * 126 * (1 << 20)    # weights not well above the 126 MB L2
    n = steps                                      # pipeline fill and drain included (conservative)
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_done = [torch.cuda.Event() for _ in range(n)]
    ev_out = [torch.cuda.Event() for _ in range(n)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def h2d(i):
        with torch.cuda.stream(cs):
            if i >= 2:
                cs.wait_event(ev_done[i - 2])      # step i - 2 no longer reads buffer i % 2
            dx[i % 2].copy_(hx, non_blocking=True)
            dl[i % 2].copy_(hl, non_blocking=True)
            ev_in[i].record(cs)

    t0.record(cs)
    h2d(0)
    for i in range(n):
        if i + 1 < n:
            h2d(i + 1)
        stream.wait_event(ev_in[i])
        if i >= 2:
            stream.wait_event(ev_out[i - 2])       # out buffer i % 2 was read back
        if flush_each:
            flush.zero_()
        moe.moe_layer(lw.shape, dx[i % 2], dl[i % 2], w, lw.ws, dout[i % 2], stream)
        ev_done[i].record(stream)
        with torch.cuda.stream(co):
            co.wait_event(ev_done[i])
            ho[i % 2].copy_(dout[i % 2], non_blocking=True)
            ev_out[i].record(co)
    cs.wait_event(ev_out[n - 1])
    t1.record(cs)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return {"ms": ms, "unit": "tokens/s",
            "h2d_bytes_per_step": hx.numel() * hx.element_size() + hl.numel() * hl.element_size(),
            "d2h_bytes_per_step": ho[0].numel() * ho[0].element_size(),
            "how": "H2D of step i+1 and D2H of step i on two copy streams beside step i's layer, "
                   "first H2D to last D2H over all steps; "
                   + ("L2 flushed before each layer" if flush_each else "weights larger than L2, no flush")}


def time_whole_layer(spec, inp, b, steps, warmup, flush):
    """Whole-layer device time (ms per step) through the public moe_layer call:
    stream-launched, and as the replay of a CUDA graph holding one call. L2 is
    flushed before every timed step; the workspace's epoch protocol needs no
    host work between replays."""
    import numpy as np
    import torch
    from combine_softmax_top_b200 import moe

    for _ in range(max(3, warmup)):
        flush.zero_()
        moe.run_layer(b, inp)
    torch.cuda.synchronize()

    def timed(fn):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        return float(np.median([e0.elapsed_time(e1) for e0, e1 in evs]))

    stream_ms = timed(lambda: moe.run_layer(b, inp))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        moe.run_layer(b, inp)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        moe.run_layer(b, inp)
    for _ in range(3):
        flush.zero_()
        g.replay()
    graph_ms = timed(g.replay)
    rc = moe.moe_poll_status(b.ws)
    del g
    if rc != 0:
        raise RuntimeError(f"layer reported {moe.moe_status_string(rc)}")
    return stream_ms, graph_ms


def time_overlap(spec, inp, dev, flush, steps, warmup, splits=(8, 20, 32), green=(20,)):
    """The whole layer with dispatch beside the grouped FFN (moe_layer_overlap)
    against the same layer run stage after stage (moe_layer), both with their
    intermediates in a layer workspace, L2 flushed before every timed step,
    median device time on the launching stream (the join makes that stream
    wait for the dispatch stream, so the interval covers both). Each split
    gives dispatch P SMs' worth of CTAs and the FFN's persistent grid the
    other SMs; it is timed stream-launched and as the replay of a CUDA graph
    of one call (route and the counting pass, then dispatch and the FFN as
    two concurrent branches, then combine). `green` splits enforce the
    partition with two green contexts (P SMs for dispatch, the rest for the
    layer's other kernels), stream-launched only."""
    import numpy as np
    import torch
    from combine_softmax_top_b200 import moe

    lw = moe.alloc_layer(spec, device=dev)
    w = moe.weights_struct(inp)

    def timed(fn):
        for _ in range(max(3, warmup)):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e0, e1 in evs:
            flush.zero_()
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        rc = moe.moe_poll_status(lw.ws)
        if rc != 0:
            raise RuntimeError(f"layer reported {moe.moe_status_string(rc)}")
        return float(np.median([e0.elapsed_time(e1) for e0, e1 in evs]))

    def graphed(fn):
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            fn()
        ms = timed(g.replay)
        del g
        return ms

    def serial():
        moe.moe_layer(lw.shape, inp["x"], inp["logits"], w, lw.ws, lw.out)

    res = {"serial_us": timed(serial) * 1e3, "serial_graph_us": graphed(serial) * 1e3, "splits": {}}
    ref = lw.out.clone()
    for P, is_green in [(P, False) for P in splits] + [(P, True) for P in green]:
        key = f"{P}" + ("_green" if is_green else "")
        try:
            ov = moe.Overlap(P, green=is_green, device=dev)
        except Exception as exc:   # torch without green contexts, or the driver refuses one
            res["splits"][key] = {"unavailable": str(exc)[:200]}
            continue

        def over(ov=ov):
            moe.overlap_layer(lw.shape, inp["x"], inp["logits"], w, lw.ws, lw.out, ov)

        try:
            r = {"us": timed(over) * 1e3}
            if is_green:
                r["dispatch_sms"], r["main_sms"] = ov.ov.dispatch_sms, ov.ov.ffn_sms
            else:
                r["graph_us"] = graphed(over) * 1e3
        except Exception as exc:
            r = {"unavailable": str(exc)[:200]}
        else:
            r["same_bits"] = bool(torch.equal(lw.out, ref))
        ov.close()
        res["splits"][key] = r
    best = min((v["us"], k) for k, v in res["splits"].items() if "us" in v)
    res["best"] = {"split": best[1], "us": best[0], "gain_vs_serial": res["serial_us"] / best[0]}
    res["how"] = ("moe_layer vs moe_layer_overlap on a layer workspace; median of the timed steps, "
                  "L2 flushed before each; split = SMs sized for dispatch, the FFN grid the rest")
    del lw
    return res


def run_fp8_gemm_peak(args):
    """A library e4m3 GEMM (torch._scaled_mm, i.e. cuBLAS) on this GPU: the
    dense FP8 rate a plain GEMM reaches here, burst (best of 10 launches) and
    under the power cap (back to back for 4 s, clocks sampled meanwhile).
    Context for the prefill FFN's tensor fraction, not a roof of its own."""
    import torch
    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(args.seed)
    n = 8192
    a = (torch.randn(n, n, device="cuda", generator=g) * 0.5).to(torch.float8_e4m3fn)
    b = (torch.randn(n, n, device="cuda", generator=g) * 0.5).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device="cuda")

    def mm():
        return torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

    for _ in range(5):
        mm()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    clocks = ClockSampler(0)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    calls, t0 = 0, time.time()
    e0.record()
    while time.time() - t0 < 4.0:
        for _ in range(20):
            mm()
        calls += 20
        torch.cuda.synchronize()
    e1.record()
    torch.cuda.synchronize()
    flop = 2.0 * n ** 3
    print(json.dumps({"metric": "cuBLAS e4m3 GEMM 8192^3", "burst_tflops": flop / (best * 1e-3) / 1e12,
                      "sustained_tflops": flop * calls / (e0.elapsed_time(e1) * 1e-3) / 1e12,
                      "clocks": clocks.stop(), "how": "torch._scaled_mm e4m3 x e4m3 -> bf16, tensor-wise scales"}))


def run_overlap_sweep(args):
    import torch
    from combine_softmax_top_b200 import workloads as W
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for spec in (W.spec("decode"), W.spec("prefill", compact=1), W.spec("decode_fp4")):
        inp = W.make_inputs(spec, seed=args.seed, device=dev)
        clocks = ClockSampler(0)
        clocks.start()
        r = time_overlap(spec, inp, dev, flush, args.steps, args.warmup,
                         splits=(2, 4, 8, 12, 16, 20, 24, 32, 48), green=(8, 20))
        r["clocks"] = clocks.stop()
        r["workload"] = workload_config(spec, 1)["workload"] + (", compact windows" if spec.compact else "")
        print(json.dumps(r), flush=True)
        del inp
        torch.cuda.empty_cache()


def run_report(args):
    import numpy as np
    import torch
    from combine_softmax_top_b200 import moe
    from combine_softmax_top_b200 import workloads as W

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    peaks, kind = load_peaks()
    hbm = peaks["hbm_gbs"]
    cases = [W.spec("tiny"), W.spec("decode"), W.spec("prefill"), W.spec("skew"),
             W.spec("decode", shared=1), W.spec("prefill", shared=1),
             W.spec("prefill", compact=1), W.spec("skew", compact=1),
             W.spec("decode_fp4"), W.spec("prefill_fp4"), W.spec("decode_fp4", shared=1)] + \
        [W.spec("decode", T=t) for t in (1, 8, 32, 512)] + \
        [W.spec("sweep", T=t) for t in W.SWEEP_T]
    for spec in cases:
        inp = W.make_inputs(spec, seed=args.seed, device=dev)
        b = moe.alloc_buffers(spec, device=dev)
        clocks = ClockSampler(0)
        clocks.start()
        st = time_layer(spec, inp, b, args.steps, args.warmup, stream, flush).mean(0)
        clk = clocks.stop()
        counts = b.counts.cpu().numpy()
        layer_ms = float(st.sum())
        line = {"report": spec.name + ("+shared" if spec.shared else "") + ("+compact" if spec.compact else ""),
                "T": spec.T, "H": spec.H, "E": spec.E,
                "topk": spec.k, "shared_experts": spec.shared, "compact_windows": spec.compact,
                "expert_buffer_rows": spec.rows(),
                "I": None if spec.identity else spec.I, "dtype": spec.weight if not spec.identity else spec.xq,
                "layer_us": layer_ms * 1e3, "tokens_per_s": spec.T / (layer_ms / 1e3),
                "stage_us": {k: float(v * 1e3) for k, v in zip(["route", "dispatch", "grouped_ffn", "combine"], st)},
                "peak_source": kind, "clocks": clk}
        rb, db, cb = route_bytes(spec), dispatch_bytes(spec), combine_bytes(spec)
        warm = time_layer(spec, inp, b, args.steps, args.warmup, stream, None).mean(0)
        line["stage_us_warm_l2"] = {k: float(v * 1e3) for k, v in
                                    zip(["route", "dispatch", "grouped_ffn", "combine"], warm)}
        whole_ms, graph_ms = time_whole_layer(spec, inp, b, args.steps, args.warmup, flush)
        line["layer_call_us"] = whole_ms * 1e3         # one moe_layer call, stream-launched
        line["layer_graph_us"] = graph_ms * 1e3        # the same call replayed from a CUDA graph
        line["graph_tokens_per_s"] = spec.T / (graph_ms / 1e3)
        line["route_GBps"] = rb / (st[0] / 1e3) / 1e9
        line["dispatch_GBps"] = db / (st[1] / 1e3) / 1e9
        line["combine_GBps"] = cb / (st[3] / 1e3) / 1e9
        line["dispatch_frac_hbm"] = line["dispatch_GBps"] / hbm
        line["combine_frac_hbm"] = line["combine_GBps"] / hbm
        if spec.identity:
            line["permutation_GBps"] = (db + cb) / ((st[1] + st[3]) / 1e3) / 1e9
            line["permutation_frac_hbm"] = line["permutation_GBps"] / hbm
        else:
            abytes, touched = ffn_algorithmic_bytes(spec, counts)
            flops = ffn_flops(spec, int(counts.sum()))
            tc_peak = peaks["bf16_tflops"] * (2.0 if spec.weight in ("e4m3", "e2m1") else 1.0)
            line["ffn_GBps"] = abytes / (st[2] / 1e3) / 1e9
            line["ffn_TFLOPs"] = flops / (st[2] / 1e3) / 1e12
            line["ffn_frac_hbm"] = line["ffn_GBps"] / hbm
            line["ffn_frac_tensor"] = line["ffn_TFLOPs"] / tc_peak
            line["ffn_bound"] = "hbm" if abytes / (hbm * 1e9) >= flops / (tc_peak * 1e12) else "tensor"
            line["touched_experts"] = touched
        print(json.dumps(line), flush=True)
        del inp, b
        torch.cuda.empty_cache()


# ------------------------------------------------------------ ours --

def ffn_roofline(spec, counts, ffn_ms, peaks, peak_kind, burst=True):
    """The grouped FFN launch against both of its roofs: its algorithmic
    bytes at the measured HBM copy rate and its FLOPs at the tensor peak of
    its operand type (block-scaled 8-bit and 4-bit paths: twice the measured
    bf16 GEMM rate, the nominal ratio). `bound` names the roof that is higher
    (the slower of the two ideal times)."""
    abytes, touched = ffn_algorithmic_bytes(spec, counts)
    flops = ffn_flops(spec, int(counts.sum()))
    bf16 = peaks["bf16_tflops"] if burst else peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    tc_peak = bf16 * (2.0 if spec.weight in ("e4m3", "e2m1") else 1.0)
    gbs = abytes / (ffn_ms / 1000.0) / 1e9
    tfs = flops / (ffn_ms / 1000.0) / 1e12
    t_hbm = abytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    src = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback"
    # the same roof at the power-capped rate: the FFN is timed inside a loop
    # of back-to-back layers, where the part runs at its power cap
    sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * (tc_peak / bf16)
    return {"bound": "hbm" if t_hbm >= t_tc else "tensor",
            "tensor": {"achieved": tfs, "peak": tc_peak, "unit": "TFLOP/s", "frac": tfs / tc_peak,
                       "peak_how": ("2 x " if tc_peak != bf16 else "") +
                                   ("burst" if burst else "sustained") + " bf16 GEMM, " + src,
                       "peak_sustained": sus, "frac_sustained": tfs / sus},
            "hbm": {"achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                    "peak_how": "copy bandwidth, " + src},
            "algorithmic_bytes_per_launch": abytes, "flops_per_launch": flops, "touched_experts": touched,
            "launch_ms": ffn_ms}


def measure_extras(args, dec_inp, dev, stream, flush, world):
    """The other half of the metric and the 4-bit weight format, in the same
    run as the headline decode line: the prefill layer (T = 8192, e4m3
    weights, compact windows so the expert buffers hold 98 k rows instead of
    2.1 M), and the decode and prefill layers with MX FP4 weights. Each is
    timed like the headline (per-stage CUDA events on the launching stream,
    L2 flushed before every step, clocks sampled during the timed steps).
    The e4m3 prefill layer reuses the decode layer's weights: both draw them
    from the same seeded streams at the same shapes."""
    import torch
    from combine_softmax_top_b200 import moe
    from combine_softmax_top_b200 import workloads as W
    peaks, peak_kind = load_peaks()
    rank, local_rank, _ = dist_env()
    out = {}
    wkeys = ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")
    fp4_w = None
    for key, name in (("prefill", "prefill"), ("decode_fp4", "decode_fp4"), ("prefill_fp4", "prefill_fp4")):
        spec = W.spec(name, compact=1) if name.startswith("prefill") else W.spec(name)
        inp = W.make_inputs(spec, seed=args.seed + rank, device=dev, with_weights=False)
        if spec.weight == "e4m3":
            inp.update({k: dec_inp[k] for k in wkeys})
        else:
            if fp4_w is None:
                full = W.make_inputs(spec, seed=args.seed + rank, device=dev)
                fp4_w = {k: v for k, v in full.items() if k in wkeys}
                del full
            inp.update(fp4_w)
        b = moe.alloc_buffers(spec, device=dev)
        clocks = ClockSampler(local_rank)
        clocks.start()
        st = time_layer(spec, inp, b, args.steps, args.warmup, stream, flush)
        clk = clocks.stop()
        mean = st.mean(0)
        ms = max_over_ranks(float(st.sum(1).mean()), dev)
        ffn_ms = max_over_ranks(float(mean[2]), dev)
        counts = b.counts.cpu().numpy()
        out[key] = {
            "workload": workload_config(spec, world)["workload"] +
                        (", compact windows" if spec.compact else ""),
            "T": spec.T, "value": job_throughput(spec.T, world, ms), "unit": "tokens/s",
            "us_per_layer": ms * 1000.0, "steps": args.steps,
            "stage_us": {k: float(v * 1000.0) for k, v in zip(["route", "dispatch", "grouped_ffn", "combine"], mean)},
            "roofline": ffn_roofline(spec, counts, ffn_ms, peaks, peak_kind),
            "expert_buffer_rows": spec.rows(),
            "l2": "flushed (256 MB write) before every timed step",
            "clocks": clk,
        }
        out[key]["roofline"]["traffic"] = recorded_traffic(f"grouped_ffn/{spec.name}",
                                                           out[key]["roofline"]["algorithmic_bytes_per_launch"])
        if key == "prefill":
            out[key]["overlap"] = time_overlap(spec, inp, dev, flush, args.steps, args.warmup)
        del inp, b
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from combine_softmax_top_b200 import moe
    from combine_softmax_top_b200 import workloads as W

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    spec = W.spec(args.config, **overrides(args))
    inp = W.make_inputs(spec, seed=args.seed + rank, device=dev)
    b = moe.alloc_buffers(spec, device=dev)
    w = moe.weights_struct(inp) if not spec.identity else moe.moe_weights()
    bufs = b.dispatch_bufs()
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        moe.moe_route(b.shape, inp["logits"], b.topk_idx, b.topk_w, b.ws, stream)
        if ev:
            ev[1].record(stream)
        moe.moe_dispatch(b.shape, inp["x"], b.topk_idx, b.ws, bufs, stream)
        if ev:
            ev[2].record(stream)
        if not spec.identity:
            moe.moe_grouped_ffn(b.shape, bufs, w, b.ws, b.y, stream)
        if ev:
            ev[3].record(stream)
        moe.moe_combine(b.shape, bufs, b.y, b.topk_w, b.ws, b.out, stream)
        if ev:
            ev[4].record(stream)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    rc = moe.moe_poll_status(b.ws, stream)
    if rc != 0:
        raise RuntimeError(f"layer reported {moe.moe_status_string(rc)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    t_all0.record(stream)
    for i in range(args.steps):
        flush.zero_()                      # L2 flushed between timed steps
        step(evs[i])
    t_all1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    rc = moe.moe_poll_status(b.ws, stream)
    if rc != 0:
        raise RuntimeError(f"layer reported {moe.moe_status_string(rc)}")

    stage = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)]
                      for i in range(args.steps)])          # ms
    step_ms = stage.sum(1)
    ms = max_over_ranks(float(step_ms.mean()), dev)
    tokens_all = spec.T * world
    value = job_throughput(spec.T, world, ms)

    # end to end through the C ABI with host buffers: every step copies its x
    # and logits from pinned host memory, runs the layer and reads its output
    # back. The copies of step i + 1 (H2D) and step i (D2H) run on a copy
    # stream beside step i's layer (double-buffered device inputs and
    # outputs), as a serving loop would; the timed region runs from the first
    # H2D to the last D2H. Weights above L2 size stream from HBM every step;
    # smaller layers get the L2 flush before each layer, inside the region.
    e2e = None
    if not args.no_e2e:
        e2e = time_e2e_pipelined(spec, inp, b, w, bufs, stream, flush, args.steps, dev)
        e2e["value"] = job_throughput(spec.T, world, max_over_ranks(e2e.pop("ms"), dev))

    # the whole layer through one moe_layer call, stream-launched and replayed
    # from a CUDA graph (outside the timed region above; reported beside it)
    call_ms, graph_ms = time_whole_layer(spec, inp, b, args.steps, args.warmup, flush)
    call_ms = max_over_ranks(call_ms, dev)
    graph_ms = max_over_ranks(graph_ms, dev)
    graph = {"us_per_layer": graph_ms * 1000.0, "value": job_throughput(spec.T, world, graph_ms),
             "unit": "tokens/s", "stream_launched_us_per_layer": call_ms * 1000.0,
             "how": "one moe_layer call captured in a CUDA graph; median replay, L2 flushed before each"}

    counts = b.counts.cpu().numpy()
    peaks, peak_kind = load_peaks()
    ffn_ms = float(stage[:, 2].mean())
    roofline = None
    if not spec.identity:
        # decode-size GEMMs stream weights (HBM bound); big-batch GEMMs are
        # bound by the tensor pipe: the headline keys name the higher roof
        both = ffn_roofline(spec, counts, ffn_ms, peaks, peak_kind)
        top = both[both["bound"]]
        roofline = {"bound": both["bound"], "achieved": top["achieved"], "peak": top["peak"],
                    "unit": top["unit"], "frac": top["frac"], "kernel": "grouped_ffn",
                    "algorithmic_bytes_per_launch": both["algorithmic_bytes_per_launch"],
                    "flops_per_launch": both["flops_per_launch"], "touched_experts": both["touched_experts"],
                    "launch_ms": ffn_ms, "peak_source": top["peak_how"],
                    "traffic": recorded_traffic(f"grouped_ffn/{spec.name}",
                                                both["algorithmic_bytes_per_launch"])}

    extras = {}
    if args.config == "decode" and not overrides(args) and not args.no_extra:
        # dispatch beside the grouped FFN on an SM partition (before the
        # extras free the decode buffers' neighbours)
        extras["overlap"] = time_overlap(spec, inp, dev, flush, args.steps, args.warmup)
        extras.update(measure_extras(args, inp, dev, stream, flush, world))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, el, cores = oracle_sample(spec, inp, args.cpu_seconds)
        cpu = {"value": n / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"first {n} of {spec.T} tokens of the same workload ({el:.1f}s)"}
        if spec.name in ("tiny", "decode"):   # the same on one core
            n1, el1, _ = oracle_sample(spec, inp, min(args.cpu_seconds, 10.0), threads=1)
            cpu["one_core"] = {"value": n1 / el1, "unit": "tokens/s", "cores": 1,
                               "sample": f"first {n1} of {spec.T} tokens ({el1:.1f}s)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
            "us_per_layer": ms * 1000.0, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if spec.weight == "e4m3" else spec.weight,
            "data": "synthetic (seeded; random-init weights, no checkpoint)",
            "config": workload_config(spec, world),
            "stage_us": {k: float(stage[:, j].mean() * 1000.0)
                         for j, k in enumerate(["route", "dispatch", "grouped_ffn", "combine"])},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "graph_replay": graph,
            "gpu_launches": args.steps * moe.kernels_per_layer(spec),
            "clocks": clk,
        }
        line.update(extras)
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.record_traffic:
        record_traffic(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.report:
        run_report(args)
    elif args.overlap_sweep:
        run_overlap_sweep(args)
    elif args.fp8_gemm_peak:
        run_fp8_gemm_peak(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
