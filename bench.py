#!/usr/bin/env python
"""Throughput benchmark of the TTT layer on B200.

One step = one TTT-Linear full-batch layer forward (Gram pass, update, apply -- the whole
path, one kernel) over one batch at the high-resolution stage-1 shape: B=32 images, a 56x56
token grid (N=3136), one head of d=64, bf16 Q/K/V, fp32 W0, eta=1.  Inputs are seeded
synthetic N(0,1)/sqrt(d) values.

Timing: W warm-up steps, then EXACTLY K steps captured in one CUDA graph and timed with CUDA
events on the launching stream, bracketed by a barrier and device synchronisation, max over
ranks.  The steps cycle through R input/output sets whose total size exceeds four times the
126 MB L2, so every step reads its inputs from HBM.  With --gpus N (torchrun) every rank runs
its own batch (units are independent: weak scaling, no data-path collective).

Extra keys: `roofline` (algorithmic bytes per launch / average launch time vs the measured
HBM copy peak), `e2e` (same metric through the public API with pinned host buffers, copies
inside the timed region), `cpu_baseline` (the fp64 oracle on the host cores, bounded
sample), `clocks` (NVML samples during the timed region), `gpu_launches`, `other_paths`
(device time of the conv, MLP and chunked paths at their shapes).

`--impl reference` times the CPU oracle instead (the reference arm: there is no reference
code to install; the oracle restates the method).
"""
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
sys.path.insert(0, ROOT)

METRIC = "TTT-layer fwd tokens/s and achieved HBM GB/s (% of B200 peak) at N=3136"
WL = dict(workload="ttt_linear_fullbatch", grid="56x56", B=32, H=1, N=3136, d=64, eta=1.0)
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="skip e2e, cpu baseline, other paths")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--only", choices=["dwconv", "mlp", "chunked", "backward", "oneway", "minibatch", "convscan",
                                       "block"],
                    default=None,
                    help="time one other path alone (used for per-kernel ncu captures)")
    return ap.parse_args()


def peaks():
    """(HBM copy GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]),
                float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured")
    except Exception:
        return FALLBACK_HBM_GBS, 1590.0, 1400.0, "fallback"


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# ------------------------------------------------------------------ device timing ------
SLEEP_CYCLES = 4_000_000  # ~2 ms at 1.9 GHz: covers the host's graph submission


LEAD_STEPS = 2  # untimed steps at the head of the timed graph, before the start event


def graph_timed(stream, dev, step, steps, pg=None, sampler=None, counter=None):
    """Capture LEAD_STEPS + `steps` calls of step(i) in one CUDA graph and time the last `steps`
    with CUDA events recorded as nodes of the graph.  The start event sits on a side branch
    that depends on the last lead-in step alone, so it records when that step completes
    without holding back the first timed step (which, launched as a dependent launch, overlaps
    the lead-in's tail as every step overlaps its predecessor's); the stop event records when
    the last timed step completes.  The window is thus `steps` consecutive steps, completion to
    completion, with the host's submission and the graph's start outside it.  A device-side
    sleep still precedes the replay, so the host has submitted it before the GPU starts.
    Returns (ms of the timed steps, ms of one replay of the whole graph with events outside it
    and no sleep, launches counted by `counter` while the timed steps were captured)."""
    import torch
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device=dev)
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    fork, join = torch.cuda.Event(), torch.cuda.Event()
    n_launched = None
    with torch.cuda.stream(stream):
        graph.capture_begin()
        for i in range(LEAD_STEPS):
            step(i)
        fork.record(stream)
        side.wait_event(fork)
        e0.record(side)
        c0 = counter() if counter else None
        for i in range(LEAD_STEPS, LEAD_STEPS + steps):
            step(i)
        if counter:
            n_launched = counter() - c0
        join.record(side)
        stream.wait_event(join)
        e1.record(stream)
        graph.capture_end()
        graph.replay()  # upload and one warm replay (untimed)
    torch.cuda.synchronize(dev)
    # the whole replay with the host submission inside the window (reported separately)
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    with torch.cuda.stream(stream):
        graph.replay()
    w1.record(stream)
    torch.cuda.synchronize(dev)
    ms_whole = w0.elapsed_time(w1)
    barrier(pg, dev)
    torch.cuda.synchronize(dev)
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        with torch.cuda.stream(stream):
            torch.cuda._sleep(SLEEP_CYCLES)
            graph.replay()
        torch.cuda.synchronize(dev)
    barrier(pg, dev)
    ms = e0.elapsed_time(e1)
    del graph
    return ms, ms_whole, n_launched


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


# ------------------------------------------------------------------ rank plumbing ------
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def barrier(pg, device):
    if pg is not None:
        import torch
        if device.type == "cuda":
            pg.barrier(device_ids=[device.index])
        else:
            pg.barrier()


def max_over_ranks(pg, x, device):
    if pg is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank):
    """Seed of a rank's synthetic inputs: every rank draws its own batch (weak scaling)."""
    return 1000 + rank


def job_tokens_per_s(world, tokens_per_step, steps, ms_max):
    """Whole-job throughput: the tokens all ranks processed over the slowest rank's time."""
    return world * tokens_per_step * steps / (ms_max / 1e3)


# ------------------------------------------------------------------ clocks -------------
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML every `period` s while active."""

    def __init__(self, index, period=0.002):
        self.samples = []
        self.ok = False
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = statistics.median(s[0] for s in self.samples)
        bits = 0
        for _, r in self.samples:
            bits |= r
        names = [n for b, n in REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ traffic record -----
def kernel_traffic(kernel_files, summary_name):
    """dram bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    h = hashlib.sha256()
    for f in kernel_files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    sha = h.hexdigest()[:16]
    path = os.path.join(ROOT, "profiles", summary_name)
    try:
        with open(path) as fh:
            text = fh.read()
    except OSError:
        return None, sha
    rec = {}
    for line in text.splitlines():
        if line.startswith("traffic_bytes_per_launch:"):
            rec["traffic"] = float(line.split(":", 1)[1])
        if line.startswith("kernel_source_sha:"):
            rec["sha"] = line.split(":", 1)[1].strip()
    if rec.get("sha") == sha and "traffic" in rec:
        return rec["traffic"], sha
    return None, sha


# ------------------------------------------------------------------ CPU oracle ---------
def cpu_oracle_rate(seconds, B, H, N, d, seed=0):
    """Tokens/s of the fp64 oracle on the host cores for the bench workload (bounded)."""
    import oracle
    from linear_attention_split_b200 import inputs
    inp = inputs.linear_inputs(B, H, N, d, dtype="bf16", seed=seed)
    q, k, v, w0 = (oracle._f64(inp[x]) for x in ("q", "k", "v", "w0"))
    threads = oracle.default_threads()
    # one unit per thread per pass keeps every core busy; passes repeat until `seconds`
    per = min(B, threads)
    t0 = time.perf_counter()
    tokens = 0
    passes = 0
    while True:
        b0 = (passes * per) % B
        sl = slice(b0, b0 + per)
        oracle.linear_fullbatch(q[sl], k[sl], v[sl], w0, threads=threads)
        tokens += q[sl].shape[0] * N
        passes += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": min(threads, per), "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{passes} passes of {per} units (b, h) x N={N} tokens each of the "
                      f"B={B} batch, {dt:.1f} s wall, fp64 per-token loops, one unit per thread"}


def cpu_config_rates(target_s=1.5):
    """The oracle's rate on each of the layer's workloads, on a bounded sample: whole images
    (all heads or channels of one batch entry), doubled until a sample takes `target_s`, then
    scaled to tokens/s.  Plus one single-thread time of the fp32 14x14 layer."""
    import oracle
    from linear_attention_split_b200 import inputs
    threads = oracle.default_threads()
    res = {"cpu_model": cpu_model(), "threads": threads}

    def run(kind, B, kw, call):
        n = 1
        while True:
            inp = inputs.make(kind, seed=0, B=n, **kw)
            t0 = time.perf_counter()
            call(inp)
            dt = time.perf_counter() - t0
            if dt >= target_s or n >= B:
                break
            n = min(B, n * 2)
        N = kw.get("N", kw.get("Hg", 1) * kw.get("Wg", 1))
        return {"tokens_per_s": n * N / dt, "sample": f"{n} of B={B} images, {dt:.2f} s",
                "est_full_config_s": dt * B / n}

    lin = lambda i: oracle.linear_fullbatch(i["q"], i["k"], i["v"], i["w0"], threads=threads)
    res["linear_f32_14x14"] = run("linear", 1, dict(H=1, N=196, d=64, dtype="f32"), lin)
    inp = inputs.linear_inputs(1, 1, 196, 64, dtype="f32")
    t0 = time.perf_counter()
    oracle.linear_fullbatch(inp["q"], inp["k"], inp["v"], inp["w0"], threads=1)
    res["linear_f32_14x14"]["single_thread_s"] = time.perf_counter() - t0
    res["linear_vits_bf16"] = run("linear", 64, dict(H=6, N=196, d=64, dtype="bf16"), lin)
    res["linear_56x56_bf16"] = run("linear", 32, dict(H=1, N=3136, d=64, dtype="bf16"), lin)
    res["dwconv_56x56_bf16"] = run("dwconv", 32, dict(Hg=56, Wg=56, C=64, dtype="bf16"),
                                   lambda i: oracle.dwconv_fullbatch(i["q"], i["k"], i["v"], i["w0"],
                                                                     threads=threads))
    res["mlp_64x64_bf16"] = run("mlp", 16, dict(H=12, N=4096, d=64, dtype="bf16"),
                                lambda i: oracle.mlp_fullbatch(i["q"], i["k"], i["v"], i["w1"], i["w2"],
                                                               threads=threads))
    res["chunked_80x80_bf16"] = run("chunked", 8, dict(H=3, N=6400, d=64, dtype="bf16"),
                                    lambda i: oracle.linear_chunked(i["q"], i["k"], i["v"], i["w0"], 64,
                                                                    threads=threads))
    return res


def reference_sample(B, N, threads, unit_s, budget):
    """Per-step sample of the reference arm: (units, tokens per unit, threads used).
    Whole units (b, h) in passes of min(B, threads) parallel units while one pass fits the
    per-step budget; otherwise min(B, threads) units, each cut to its first n tokens, n sized
    so that the pass fits.  The oracle runs one unit per thread, so the threads used are
    min(threads, units)."""
    par = max(1, min(B, threads))
    if budget >= unit_s:
        units = max(1, min(B, int(budget / max(unit_s, 1e-9)) * par))
        n = N
    else:
        units = par
        n = max(16, min(N, int(N * budget / max(unit_s, 1e-9))))
    return units, n, min(threads, units)


# ------------------------------------------------------------------ our arm ------------
def run_ours(args):
    import torch
    from linear_attention_split_b200 import ttt

    world, rank, local, pg = dist_setup(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hbm_peak, tf_burst, tf_sust, peak_src = peaks()
    B, H, N, d, eta = WL["B"], WL["H"], WL["N"], WL["d"], WL["eta"]
    per_set = 4 * B * H * N * d * 2
    R = max(2, math.ceil(4 * L2_BYTES / per_set))
    g = torch.Generator(device=dev)
    g.manual_seed(rank_seed(rank))
    sets = []
    for _ in range(R):
        q, k, v = (torch.randn((B, H, N, d), generator=g, device=dev) / math.sqrt(d) for _ in range(3))
        sets.append(dict(q=q.bfloat16(), k=k.bfloat16(), v=v.bfloat16(),
                         out=torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)))
    w0 = torch.randn((H, d, d), generator=g, device=dev) / math.sqrt(d)
    stream = torch.cuda.Stream(device=dev)

    def step(i):
        s = sets[i % R]
        ttt.ttt_linear_fullbatch(s["q"], s["k"], s["v"], w0, s["out"], None, eta, None, stream)

    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            step(i)
    torch.cuda.synchronize(dev)
    assert ttt.device_error() == 0
    # the K timed steps in one graph (launch overhead out of the measurement)
    sampler = ClockSampler(dev.index)
    ms, ms_whole, n_launched = graph_timed(stream, dev, step, args.steps, pg=pg, sampler=sampler,
                                           counter=ttt.kernel_launch_count)
    ms = max_over_ranks(pg, ms, dev)
    assert ttt.device_error() == 0
    kernels_per_step = 1  # the tensor-core TTT-Linear path is a single kernel per call
    gpu_launches = args.steps * kernels_per_step
    ms_step = ms / args.steps
    tokens_step = B * N
    value = job_tokens_per_s(world, tokens_step, args.steps, ms)
    alg_bytes = 8 * B * H * N * d
    alg_flops = 6 * B * H * N * d * d
    achieved = alg_bytes / (ms_step / 1e3) / 1e9
    traffic, sha = kernel_traffic(["linear_attention_split_b200/csrc/linear_tc5.cuh",
                                   "linear_attention_split_b200/csrc/common.cuh"],
                                  "linear_tc5_56x56.md")

    rec = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "TTT-Linear full-batch step, B=32 x 56x56 tokens (N=3136), 1 head, d=64, "
                               "bf16 Q/K/V, fp32 W0, eta=1",
                   "global_batch": B * world, "seq_len": N, "heads": H, "head_dim": d,
                   "parallelism": f"independent batches per rank (dp{world}), no collective",
                   "l2": f"{R} rotating input/output sets of {per_set / 1e6:.1f} MB "
                         f"({R * per_set / 1e6:.0f} MB > 4x L2)",
                   "timing": f"{LEAD_STEPS} untimed lead-in steps and the K timed steps in one "
                             "CUDA graph; CUDA events recorded as graph nodes: the start when the "
                             "last lead-in step completes (on a side branch, so the first timed "
                             "step still overlaps it), the stop when the K-th step completes",
                   "whole_replay_ms_events_outside_graph": ms_whole,
                   "fixed_cost_ms_outside_window": max(0.0, ms_whole - ms * (args.steps + LEAD_STEPS)
                                                       / args.steps)},
        "hbm_gbs": achieved, "pct_of_8tbs": 100 * achieved / NOMINAL_HBM_GBS,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic,
                     "peak_source": ("measured copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                                     if peak_src == "measured" else
                                     f"fallback: {FALLBACK_HBM_GBS:.0f} GB/s, an earlier B200 copy "
                                     "measurement (MEASURED_PEAKS.json absent)"),
                     "kernel": "lin5::linear_tc5_kernel", "kernel_source_sha": sha,
                     "algorithmic_bytes_per_launch": alg_bytes,
                     "tensor_tflops": alg_flops / (ms_step / 1e3) / 1e12},
        "gpu_launches": gpu_launches,
        "library_launch_counter_delta": n_launched,  # launches captured for the K timed steps
    }
    rec["clocks"] = sampler.summary()

    if not args.no_extras:
        rec["e2e"] = e2e_leg(ttt, dev, stream, w0, B, H, N, d, eta, min(args.steps, 200), world, pg)
        rec["other_paths"] = other_paths(ttt, dev, stream, hbm_peak, tf_burst, tf_sust, peak_src=peak_src)
        if rank == 0 and world == 1:
            rec["cpu_baseline"] = cpu_oracle_rate(args.cpu_seconds, B, H, N, d)
            rec["cpu_baseline"]["configs"] = cpu_config_rates()
        elif rank == 0:
            rec["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(rec), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def e2e_leg(ttt, dev, stream, w0, B, H, N, d, eta, steps, world, pg):
    """Same metric through the public API with pinned host buffers: every step copies Q, K, V
    host->device, runs the layer and reads O back to the host.  Steps are pipelined as a
    stream of batches would be: two device buffer sets, the copies in on one stream, the layer
    on another and the copy out on a third, so that step i+1's inputs cross PCIe while step
    i-1's output comes back (the link carries both directions at once)."""
    import torch
    g = torch.Generator()
    g.manual_seed(7)
    hq, hk, hv = (((torch.randn((B, H, N, d), generator=g) / math.sqrt(d)).bfloat16()).pin_memory()
                  for _ in range(3))
    ho = [torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    sets = [{x: torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev) for x in "qkvo"} for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in, ev_cmp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def one(i):
        b, st = i % 2, sets[i % 2]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_cmp[b])  # step i-2's layer has read this set's inputs
            st["q"].copy_(hq, non_blocking=True)
            st["k"].copy_(hk, non_blocking=True)
            st["v"].copy_(hv, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # step i-2's output has left this set
            ttt.ttt_linear_fullbatch(st["q"], st["k"], st["v"], w0, st["o"], None, eta, None, stream)
            ev_cmp[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            ho[b].copy_(st["o"], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(3):
        one(i)
    torch.cuda.synchronize(dev)
    barrier(pg, dev)
    e0.record(s_in)
    for i in range(steps):
        one(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(pg, e0.elapsed_time(e1), dev)
    nbytes = B * H * N * d * 2
    return {"value": job_tokens_per_s(world, B * N, steps, ms), "unit": "tokens/s",
            "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
            "ms_per_step": ms / steps, "steps": steps,
            "note": "pinned host buffers, the C-ABI call, eager launches; steps pipelined over two device "
                    "buffer sets with copy-in, compute and copy-out streams (both PCIe directions busy)"}


def other_paths(ttt, dev, stream, hbm_peak, tf_burst, tf_sust, only=None, iters=None, peak_src=None):
    """Device time per call of the other paths at their workload shapes.  Each path cycles
    through rotating input/output sets whose total exceeds four times the L2 (so inputs come
    from HBM), K calls in one CUDA graph, timed like the headline.  `only` restricts the run
    to one path; `iters` overrides the timed call count."""
    import torch
    from linear_attention_split_b200 import inputs
    res = {}

    def sets_for(per_set_bytes):
        return max(2, math.ceil(4 * L2_BYTES / per_set_bytes))

    def rotating(make, R):
        out = []
        for r in range(R):
            inp = {k: v.to(dev) for k, v in make(r).items()}
            inp["out"] = torch.empty_like(inp["q"])
            out.append(inp)
        return out

    def workspace(nbytes):
        return torch.empty(max(1, nbytes), dtype=torch.uint8, device=dev)

    def timed(fn, R, n):
        n = iters if iters is not None else n
        with torch.cuda.stream(stream):
            for i in range(3):
                fn(i % R)
        torch.cuda.synchronize(dev)
        ms, _, _ = graph_timed(stream, dev, lambda i: fn(i % R), n)
        return ms / n

    if only in (None, "dwconv"):  # 3x3 depthwise conv, B=32, 56x56, C=64
        nb = 8 * 32 * 3136 * 64
        R = sets_for(nb)
        S = rotating(lambda r: inputs.dwconv_inputs(32, 56, 56, 64, seed=100 + r), R)
        ws = workspace(ttt.ttt_dwconv_fullbatch_workspace_bytes(32, 56, 56, 64, 1))
        ms = timed(lambda i: ttt.ttt_dwconv_fullbatch(S[i]["q"], S[i]["k"], S[i]["v"], S[i]["w0"], S[i]["out"],
                                                      None, 1.0, ws, stream), R, 200)
        res["dwconv_56x56_c64"] = {"ms": ms, "tokens_per_s": 32 * 3136 / (ms / 1e3),
                                   "hbm_gbs": nb / (ms / 1e3) / 1e9,
                                   "frac_of_hbm_peak": nb / (ms / 1e3) / 1e9 / hbm_peak,
                                   "l2": f"{R} rotating sets of {nb / 1e6:.1f} MB (> 4x L2)"}
        del S, ws
    if only in (None, "mlp"):  # TTT-MLP, B=16, H=12, N=4096, d=64, h=256 (403 MB per set)
        R = 2
        S = rotating(lambda r: inputs.mlp_inputs(16, 12, 4096, 64, seed=200 + r), R)
        ws = workspace(ttt.ttt_mlp_fullbatch_workspace_bytes(16, 12, 4096, 64, 256, 1))
        ms = timed(lambda i: ttt.ttt_mlp_fullbatch(S[i]["q"], S[i]["k"], S[i]["v"], S[i]["w1"], S[i]["w2"],
                                                   S[i]["out"], None, None, 1.0, ws, stream), R, 10)
        fl = 14 * 16 * 12 * 4096 * 64 * 256
        tf = fl / (ms / 1e3) / 1e12
        res["mlp_64x64_d64_h256"] = {"ms": ms, "tokens_per_s": 16 * 4096 / (ms / 1e3), "tflops": tf,
                                     "frac_of_tensor_peak": tf / tf_burst,
                                     "frac_of_sustained_peak": tf / tf_sust,
                                     "peak": "burst bf16 (MEASURED_PEAKS.json bf16_tflops, else the "
                                             "fallback in res['peaks']): 10 calls, a few ms in all"}
        del S, ws
    if only in (None, "chunked"):  # chunked bidirectional, B=8, H=3, N=6400, d=64, chunk 64
        nb = 8 * 8 * 3 * 6400 * 64
        R = sets_for(nb)
        S = rotating(lambda r: inputs.chunked_inputs(8, 3, 6400, 64, seed=300 + r), R)
        ws = workspace(ttt.ttt_linear_chunked_bidir_workspace_bytes(8, 3, 6400, 64, 64, 1))
        ms = timed(lambda i: ttt.ttt_linear_chunked_bidir(S[i]["q"], S[i]["k"], S[i]["v"], S[i]["w0"],
                                                          S[i]["out"], 64, 1.0, ws, stream), R, 50)
        res["chunked_80x80_b64"] = {"ms": ms, "tokens_per_s": 8 * 6400 / (ms / 1e3),
                                    "us_per_chunk_step": ms * 1e3 / 100,
                                    "hbm_gbs_min_traffic": nb / (ms / 1e3) / 1e9,
                                    "l2": f"{R} rotating sets of {nb / 1e6:.1f} MB (> 4x L2)"}
        del S, ws
    if only in (None, "backward"):  # TTT-Linear backward at the forward's shape, B=32, 56x56, d=64
        nb = 7 * 32 * 3136 * 64 * 2  # read Q, K, V, dO; write dQ, dK, dV
        R = sets_for(nb)

        def mk(r):
            x = inputs.linear_bwd_inputs(32, 1, 3136, 64, seed=400 + r)
            return {"q": x["q"], "k": x["k"], "v": x["v"], "w0": x["w0"], "dout": x["dout"]}
        S = rotating(mk, R)
        for x in S:
            x["dk"], x["dv"], x["dw0"] = torch.empty_like(x["q"]), torch.empty_like(x["q"]), torch.empty_like(x["w0"])
        ws = workspace(ttt.ttt_linear_fullbatch_bwd_workspace_bytes(32, 1, 3136, 64, 1))
        ms = timed(lambda i: ttt.ttt_linear_fullbatch_bwd(S[i]["q"], S[i]["k"], S[i]["v"], S[i]["w0"], S[i]["dout"],
                                                          S[i]["out"], S[i]["dk"], S[i]["dv"], S[i]["dw0"], 1.0, ws,
                                                          stream), R, 200)
        res["linear_bwd_56x56_d64"] = {"ms": ms, "tokens_per_s": 32 * 3136 / (ms / 1e3),
                                       "hbm_gbs": nb / (ms / 1e3) / 1e9,
                                       "frac_of_hbm_peak": nb / (ms / 1e3) / 1e9 / hbm_peak,
                                       "bytes": "read Q, K, V, dO and write dQ, dK, dV once (the kernels "
                                                "read dO, K, V twice)", "kernels_per_call": 4,
                                       "l2": f"{R} rotating sets of {nb / 1e6:.1f} MB (> 4x L2)"}
        del S, ws
    if only in (None, "oneway"):  # one-way (raster) chunked scan, 80x80, chunk 64
        nb = 8 * 8 * 3 * 6400 * 64
        R = sets_for(nb)
        S = rotating(lambda r: inputs.chunked_inputs(8, 3, 6400, 64, seed=500 + r), R)
        ms = timed(lambda i: ttt.ttt_linear_chunked(S[i]["q"], S[i]["k"], S[i]["v"], S[i]["w0"], S[i]["out"], 64,
                                                    1.0, 1, None, stream), R, 50)
        res["chunked_one_way_80x80_b64"] = {"ms": ms, "tokens_per_s": 8 * 6400 / (ms / 1e3),
                                            "us_per_chunk_step": ms * 1e3 / 100,
                                            "hbm_gbs_min_traffic": nb / (ms / 1e3) / 1e9}
        del S
    if only in (None, "convscan"):  # Conv2d-preprocessed bidirectional scan, 80x80, chunk 64
        nb = 8 * 8 * 3 * 6400 * 64
        R = sets_for(nb)
        S = rotating(lambda r: inputs.chunked_conv_inputs(8, 3, 80, 80, 64, seed=600 + r), R)
        ws = workspace(ttt.ttt_linear_chunked_conv_workspace_bytes(8, 3, 80, 80, 64, 64, 0, 1))
        ms = timed(lambda i: ttt.ttt_linear_chunked_conv(S[i]["q"], S[i]["k"], S[i]["v"], S[i]["w0"], S[i]["wk"],
                                                         S[i]["wv"], S[i]["out"], 80, 80, 64, 1.0, 0, ws, stream), R, 50)
        res["chunked_conv_80x80_b64"] = {"ms": ms, "tokens_per_s": 8 * 6400 / (ms / 1e3),
                                         "hbm_gbs_min_traffic": nb / (ms / 1e3) / 1e9, "kernels_per_call": 3}
        del S, ws
    if only in (None, "minibatch"):  # mini-batch training, chunks of 64, 2 epochs, B=32, 56x56
        nb = 8 * 32 * 3136 * 64
        R = sets_for(nb)
        S = rotating(lambda r: inputs.linear_inputs(32, 1, 3136, 64, seed=700 + r), R)
        ws = workspace(ttt.ttt_linear_minibatch_workspace_bytes(32, 1, 3136, 64, 64, 2, 1))
        ms = timed(lambda i: ttt.ttt_linear_minibatch(S[i]["q"], S[i]["k"], S[i]["v"], S[i]["w0"], S[i]["out"], 64,
                                                      2, None, 1.0, ws, stream), R, 5)
        res["minibatch_56x56_b64_e2"] = {"ms": ms, "tokens_per_s": 32 * 3136 / (ms / 1e3),
                                         "hbm_gbs_min_traffic": nb / (ms / 1e3) / 1e9, "kernels_per_call": 2,
                                         "note": "the scan's tensor-core recurrence in training mode (98 dependent "
                                                 "steps), then the apply O = Q W_final"}
        del S, ws
    if only in (None, "block"):  # the ViT^3 block at the stage-1 width: B=32, 56x56, C=64, 2 heads of 32
        nb = 32 * 3136 * 64 * 2 * 2  # x in, y out
        R = sets_for(nb * 4)

        def mk(r):
            x = inputs.block_inputs(32, 56, 56, 64, 2, seed=800 + r)
            x["q"] = x["x"]  # rotating() sizes "out" after "q"
            return x
        S = rotating(mk, R)
        ws = workspace(ttt.ttt_vit3_block_workspace_bytes(32, 56, 56, 64, 2, 1))
        ms = timed(lambda i: ttt.ttt_vit3_block(S[i]["x"], S[i]["wqkvg"], S[i]["w0"], S[i]["wc"], S[i]["wo"],
                                                S[i]["out"], 56, 56, 2, 1.0, ws, stream), R, 100)
        inter = 32 * 3136 * 64 * 2 * (1 + 5 + 3 + 1 + 1 + 1)  # x, QKVG+O writes, QKV+O+G reads, x again, y
        res["vit3_block_56x56_c64_h2"] = {"ms": ms, "tokens_per_s": 32 * 3136 / (ms / 1e3),
                                          "hbm_gbs_in_out": nb / (ms / 1e3) / 1e9,
                                          "hbm_gbs_with_intermediates": inter / (ms / 1e3) / 1e9,
                                          "frac_of_hbm_peak_with_intermediates": inter / (ms / 1e3) / 1e9 / hbm_peak,
                                          "kernels_per_call": 3}
        del S, ws
    assert ttt.device_error() == 0
    res["peaks"] = {"hbm_gbs": hbm_peak, "bf16_tflops_burst": tf_burst,
                    "bf16_tflops_sustained": tf_sust, "source": peak_src}
    return res


def run_only(args):
    """One of the other paths alone (a small, self-contained command for ncu captures)."""
    import torch
    from linear_attention_split_b200 import ttt
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm_peak, tf_burst, tf_sust, peak_src = peaks()
    stream = torch.cuda.Stream(device=dev)
    res = other_paths(ttt, dev, stream, hbm_peak, tf_burst, tf_sust, only=args.only, iters=args.steps,
                      peak_src=peak_src)
    print(json.dumps({"only": args.only, "steps": args.steps, "result": res}), flush=True)


# ------------------------------------------------------------------ reference arm ------
def run_reference(args):
    """The oracle as it stands, on the host cores, on this workload (bounded per-step sample)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from linear_attention_split_b200 import inputs
    B, H, N, d, eta = WL["B"], WL["H"], WL["N"], WL["d"], WL["eta"]
    threads = oracle.default_threads()
    inp = inputs.linear_inputs(B, H, N, d, dtype="bf16", seed=0)
    q, k, v, w0 = (oracle._f64(inp[x]) for x in ("q", "k", "v", "w0"))
    # size each step so that warm-up + K steps stay within about two minutes
    t0 = time.perf_counter()
    oracle.linear_fullbatch(q[:1], k[:1], v[:1], w0, threads=1)
    unit_s = time.perf_counter() - t0
    budget = 120.0 / max(1, args.steps + args.warmup)
    units, n, cores = reference_sample(B, N, threads, unit_s, budget)
    sl = slice(0, units)
    qs, ks, vs = (oracle._f64(x[sl, :, :n]) for x in (q, k, v))  # contiguous, copied once
    for _ in range(args.warmup):
        oracle.linear_fullbatch(qs, ks, vs, w0, eta, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.linear_fullbatch(qs, ks, vs, w0, eta, threads=threads)
    dt = time.perf_counter() - t0
    value = units * n * args.steps / dt
    sample = (f"each step: {units} of the B={B} units (b, h), {n} of their N={N} tokens, d={d}, "
              f"fp64 oracle, one unit per thread, {cores} threads")
    rec = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": "TTT-Linear full-batch step, B=32 x 56x56 tokens (N=3136), 1 head, d=64, "
                                  "bf16 Q/K/V, fp32 W0, eta=1", "global_batch": B, "seq_len": N,
                      "parallelism": "host threads"},
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": sample, "cpu_model": cpu_model()},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(rec), flush=True)


def main():
    args = parse()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.only:
        run_only(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
