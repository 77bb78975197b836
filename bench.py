"""Throughput of the expert-choice MoE FFN layer on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--intermediate split|bf16]

A step is one pass of the whole layer (router + softmax, per-expert top-C select, token
lists, gathered GEMM1 + SwiGLU, GEMM2 + combine weight, fixed-order combine) over one
batch of seeded synthetic tokens. The default workload is a 1024 px CFG pair: two images
of 64 x 64 = 4096 patch tokens, T = 8192, d = 2048, 64 experts, F = 1024, C = 128,
tokens scaled by LogNormal(0, 0.5).

Multi-GPU: expert-choice selection over the flat token axis couples every token, so the
layer does not shard without changing its result; N GPUs run N independent replicas
(one batch each, seed = rank), and value = all ranks' tokens / the slowest rank's time.

`--impl reference` times the CPU oracle (fp64 numpy) on this host's cores instead, on
the same workload and metric (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "expert-choice MoE layer tokens/s & TFLOP/s vs B200 bf16 peak; select/combine GB/s"
L2_FLUSH_BYTES = 256 << 20  # twice the 126 MB L2


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="1024px_cfg")
    ap.add_argument("--intermediate", choices=("split", "bf16"), default="split")
    ap.add_argument("--tma-gather", action="store_true",
                    help="gather the gate/up GEMM's token rows with TMA tile::gather4")
    ap.add_argument("--l2-flush", choices=("write+read", "write"), default="write+read",
                    help="before every timed step write a buffer twice the size of L2; "
                         "with +read, then read a second one, so that the written lines "
                         "are written back to HBM before the step's first event instead "
                         "of inside the step")
    ap.add_argument("--e2e-streams", type=int, default=3,
                    help="streams the end-to-end steps rotate over (each with its own "
                         "workspace and pinned output)")
    ap.add_argument("--tensor-workload", default="batch4_1024px_cfg",
                    help="a tensor-bound workload timed in the same run (its own key of "
                         "the JSON line); empty to skip")
    ap.add_argument("--tensor-intermediate", choices=("split", "bf16"), default="bf16",
                    help="storage of H and Y for the tensor-bound workload: its tokens are "
                         "N(0, 1), so plain bf16 intermediates meet every tolerance (the "
                         "full-row parity test checks it) and the down GEMM runs one MMA "
                         "per k-step instead of the split pair's two")
    ap.add_argument("--min-timed-s", type=float, default=1.0,
                    help="repeat the timed region (each repeat exactly --steps steps between "
                         "a barrier + synchronize) until the repeats cover at least this "
                         "many seconds of step time, so the clock record spans a long load")
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="only run this many layer calls of the workload, untimed, and exit "
                         "(a short, fixed launch sequence for ncu captures)")
    ap.add_argument("--shared-f", type=int, default=0,
                    help="add a shared SwiGLU expert of this width and the block's gated "
                         "residual (out = x + tanh(clamp(gate2)) * ffn_out)")
    return ap.parse_args()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        # the SM clock the sustained figure was taken at, where the file records one
        mhz = next((v for k, v in d.items() if isinstance(v, (int, float))
                    and "sustained" in k and "mhz" in k.lower()), None)
        return dict(hbm=d["hbm_gbs"], tensor=d["bf16_tflops"],
                    tensor_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    sustained_mhz=mhz, source="measured")
    # fallback: the sustained bf16 figure was taken at about 1.3 GHz under the power cap
    return dict(hbm=6650.0, tensor=1590.0, tensor_sustained=1400.0, sustained_mhz=1300.0,
                source="fallback")


L2_NOTE = {
    "write+read": ("GPU arm: L2 flushed before every timed step (a 256 MiB write, then a "
                   "256 MiB read that evicts the written lines; both outside the step's "
                   "events); the CPU reference arm has no L2 flush"),
    "write": ("GPU arm: L2 flushed before every timed step (a 256 MiB write, outside the "
              "step's events); the CPU reference arm has no L2 flush"),
}


def _workload_config(w, l2_flush="write+read"):
    """The `config` object of the JSON line: the same for both arms on one workload."""
    return {
        "workload": f"{w.name}: T={w.T} tokens, d={w.d}, E={w.E} experts, SwiGLU F={w.F}, "
                    f"capacity_factor={w.capacity_factor:g} (C={w.C}"
                    + (f" per segment of {w.T // w.segments} tokens)" if w.segments > 1 else ")"),
        "T": w.T, "d": w.d, "E": w.E, "F": w.F, "C": w.C, "segments": w.segments,
        "l2": L2_NOTE[l2_flush],
    }


# ---- algorithmic bytes / flops of each stage ----------------------------------------------
#
# Algorithmic bytes are the minimum each stage must move with every intermediate in the
# layer's own type (bf16 H and Y for bf16 layers): router x + W_r in, scores + scores_t
# out; gate/up GEMM W1|W3, the gathered rows and H; down GEMM W2, H and Y; combine Y and
# out. These are the roofline numerators. Design bytes are what this implementation
# moves on purpose beyond them: with split intermediates H is a bf16 hi/lo pair and Y is
# fp32 (4 bytes each), plus the small index arrays the kernels read.

def stage_bytes(w, shared_f=0):
    """Algorithmic bytes per stage and layer call (with a shared expert of width
    shared_f: its weights, its gathered rows, H and Y, and the residual read)."""
    T, d, E, F, Ce, Fs = w.T, w.d, w.E, w.F, w.Ce, shared_f
    b = {
        "router": 2 * T * d + 2 * d * E + 2 * 4 * T * E,
        "select": 4 * T * E + 8 * E * Ce,
        "csr": 4 * E * Ce + 4 * (T + 1) + 4 * E * Ce,
        "gemm1_swiglu": 2 * 2 * E * d * F + 2 * E * Ce * d + 2 * E * Ce * F,
        "gemm2_scale": 2 * E * F * d + 2 * E * Ce * F + 2 * E * Ce * d,
        "combine": 2 * E * Ce * d + 2 * T * d,
    }
    if Fs:
        b["gemm1_swiglu"] += 2 * 2 * d * Fs + 2 * T * d + 2 * T * Fs
        b["gemm2_scale"] += 2 * Fs * d + 2 * T * Fs + 2 * T * d
        b["combine"] += 2 * T * d + 2 * T * d
    return b


def gather_bytes(w):
    """The standalone gather (each expert's chosen rows of x copied into one contiguous
    block): E*Ce bf16 rows read and written. The layer does not run it; its gate/up GEMM
    reads the same rows into its A tiles (those bytes are in gemm1_swiglu above)."""
    return 2 * 2 * w.E * w.Ce * w.d


def stage_design_bytes(w, intermediate="split", shared_f=0):
    """Bytes each stage moves as built: split intermediates keep H as a bf16 hi/lo pair
    and Y in fp32; the down GEMM also reads the combine weights and the rows' token-major
    positions, the combine the token lists."""
    T, d, E, F, Ce, Fs = w.T, w.d, w.E, w.F, w.Ce, shared_f
    hb = yb = 4 if intermediate == "split" else 2
    b = dict(stage_bytes(w, shared_f))
    b["gemm1_swiglu"] += (hb - 2) * E * Ce * F + 4 * E * Ce
    b["gemm2_scale"] += (hb - 2) * E * Ce * F + (yb - 2) * E * Ce * d + 8 * E * Ce
    b["combine"] += (yb - 2) * E * Ce * d + 4 * (T + 1)
    if Fs:
        b["gemm1_swiglu"] += (hb - 2) * T * Fs
        b["gemm2_scale"] += (hb - 2) * T * Fs + (yb - 2) * T * d
        b["combine"] += (yb - 2) * T * d
    return b


def stage_flops(w, shared_f=0):
    """Algorithmic FLOPs of the contractions (the split intermediates' second set of
    down-projection MMAs is executed work, not counted here)."""
    T, d, E, F, Ce, Fs = w.T, w.d, w.E, w.F, w.Ce, shared_f
    return {"router": 2 * T * d * E, "gemm1_swiglu": 4 * E * Ce * d * F + 4 * T * d * Fs,
            "gemm2_scale": 2 * E * Ce * F * d + 2 * T * Fs * d}


def _traffic(kernel_stage, workload):
    """dram read+write bytes per launch from the committed ncu summary of this kernel and
    workload, or None when there is none or the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", f"{kernel_stage}_{workload}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    if not m or not h:
        return None
    src = os.path.join(ROOT, "diffusion_transformer_moe_b200", "csrc",
                       STAGE_SOURCE.get(kernel_stage, "experts_sm100.cu"))
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != h.group(1):
        return None
    return float(m.group(1))


# the source file of each stage's kernel (a summary is stale once its file changes)
STAGE_SOURCE = {"router": "router_sm100.cu", "select": "select.cu", "csr": "select.cu",
                "gemm1_swiglu": "experts_sm100.cu", "gemm2_scale": "experts_sm100.cu",
                "combine": "combine.cu"}


# ---- clocks during the timed region ----------------------------------------------------

class ClockSampler:
    """Samples SM clocks and clock-event reasons through NVML (read only) from a thread
    that starts before the warm-up, every half millisecond, each sample stamped with the
    host time; the record keeps the samples taken inside the timed region (mark()
    brackets it), so that even a region of a few milliseconds holds several."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []        # (host time, SM MHz, reason mask)
        self.window = None
        self.mx = None
        self.err = None
        self._stop = threading.Event()
        self._switch = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = self.gpu
            if vis:
                first = vis.split(",")[self.gpu].strip()
                idx = int(first) if first.isdigit() else self.gpu
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.mx = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nv = pynvml
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = f"nvml unavailable: {type(e).__name__}"
            return
        # let the sampling thread run between the launching thread's calls
        self._switch = sys.getswitchinterval()
        sys.setswitchinterval(1e-4)
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _sample(self):
        nv = self.nv
        mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            mask = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((time.perf_counter(), mhz, mask))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception as e:
                self.err = f"nvml sample failed: {type(e).__name__}"
                return
            self._stop.wait(0.0005)

    def mark(self, which):
        """mark("begin") / mark("end") around the timed region."""
        t = time.perf_counter()
        self.window = (t, t) if which == "begin" else (self.window[0], t)

    def stop(self):
        if self.err and not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err]}
        self._stop.set()
        self.t.join(timeout=2)
        if self._switch is not None:
            sys.setswitchinterval(self._switch)
        inside = self.samples
        if self.window is not None:
            lo, hi = self.window
            inside = [x for x in self.samples if lo <= x[0] <= hi]
            if not inside:  # none landed inside: the ones nearest each end
                inside = sorted(self.samples, key=lambda x: min(abs(x[0] - lo),
                                                                 abs(x[0] - hi)))[:2]
        if not inside:
            self._sample()
            inside = self.samples[-1:]
        reasons = sorted(name for name, bit in self.REASONS.items()
                         if any(m & bit for _, _, m in inside))
        return {"sm_mhz": statistics.median(m for _, m, _ in inside), "sm_max_mhz": self.mx,
                "reasons": reasons, "samples": len(inside)}


# ---- the CPU oracle (reference arm and cpu_baseline) --------------------------------------

def _oracle_inputs(w, seed):
    from diffusion_transformer_moe_b200 import inputs as I
    a = I.make_inputs(w, seed=seed)
    return (I.to_numpy_f64(a["x"]), I.to_numpy_f64(a["W_r"]), a["W1"].float().numpy(),
            a["W3"].float().numpy(), a["W2"].float().numpy())


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()
             if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _oracle_step(w, data, experts=None):
    """One oracle pass: router, scores and selection over all tokens, then the SwiGLU
    experts and combine for `experts` (all experts if None). Returns (seconds spent,
    seconds the whole layer would take: the expert part scaled to all E experts)."""
    from oracle import nmoe_oracle as O
    import numpy as np
    x, W_r, W1, W3, W2 = data
    t0 = time.perf_counter()
    p = O.scores_from_logits(O.router_logits(x, W_r))
    idx = O.select(O.round_f32(p), w.C, w.segments)
    wts = O.combine_weights(p, idx)
    t1 = time.perf_counter()
    ex = range(w.E) if experts is None else experts
    out = np.zeros_like(x)
    for e in ex:
        out[idx[e]] += wts[e][:, None] * O.swiglu_ffn(x[idx[e]], W1[e], W3[e], W2[e])
    t2 = time.perf_counter()
    scale = w.E / max(1, len(ex))
    return t2 - t0, (t1 - t0) + scale * (t2 - t1)


def _sample_plan(w, data, budget_s):
    """Experts per step so that one step stays within budget_s (whole layer if it fits)."""
    _, full = _oracle_step(w, data)
    if full <= budget_s:
        return None, f"the whole {w.name} layer (all {w.T} tokens, all {w.E} experts)"
    k = max(1, int(w.E * budget_s / full))
    return k, (f"router, scores and selection over all {w.T} tokens of {w.name}, plus the "
               f"SwiGLU experts and combine of {k} of the {w.E} experts (rotating), the "
               f"expert time scaled to all {w.E} experts")


def cpu_baseline(w, seed=0, budget_s=12.0):
    data = _oracle_inputs(w, seed)
    k, what = _sample_plan(w, data, budget_s)
    spent, est, n = 0.0, 0.0, 0
    while spent < budget_s:
        ex = None if k is None else [(n * k + j) % w.E for j in range(k)]
        s_, e_ = _oracle_step(w, data, ex)
        spent += s_
        est += e_
        n += 1
    return {"value": w.T * n / est, "unit": "tokens/s", "cores": _oracle_threads(),
            "kind": "oracle", "sample": f"{what}; fp64 numpy oracle, {n} steps after one "
                                        f"untimed, {spent:.1f} s of CPU time"}


def run_reference(args, w, rank):
    if rank != 0:
        return
    data = _oracle_inputs(w, 0)
    budget = 150.0 / max(1, args.steps + args.warmup)
    k, what = _sample_plan(w, data, budget)
    step = 0

    def one():
        nonlocal step
        ex = None if k is None else [(step * k + j) % w.E for j in range(k)]
        step += 1
        return _oracle_step(w, data, ex)[1]

    for _ in range(args.warmup):
        one()
    tot = sum(one() for _ in range(args.steps))
    value = w.T * args.steps / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _workload_config(w, args.l2_flush),
        "impl_options": {"arithmetic": "fp64 numpy oracle on the host cores"},
        "parallelism": "one host process (rank 0)",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": _oracle_threads(),
                         "kind": "oracle", "sample": f"each step: {what}"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---- multi-rank plumbing (replicas) ---------------------------------------------------------

def max_over_ranks(vals, dist, device):
    """Element-wise maximum of per-rank timings. Every rank calls it, in the same order."""
    if dist is None:
        return [float(v) for v in vals]
    import torch
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def replica_throughput(T, world, K, ms):
    """Whole-job tokens/s: every rank ran K batches of T tokens; ms is the slowest rank's
    total time for them."""
    return T * world * K / (ms / 1e3)


# ---- our CUDA path ---------------------------------------------------------------------

def _device_inputs(w, seed, dev, shared_f):
    import torch
    from diffusion_transformer_moe_b200 import inputs as I
    a = I.make_inputs(w, seed=seed)
    d = {k: v.to(dev) for k, v in a.items()}
    block = {}
    if shared_f:
        g = torch.Generator().manual_seed(1000 + seed)
        block = dict(shared=tuple((torch.randn(*sh, generator=g) / sh[0] ** 0.5)
                                  .to(d["x"].dtype).to(dev)
                                  for sh in ((w.d, shared_f), (w.d, shared_f),
                                             (shared_f, w.d))),
                     residual=d["x"],
                     gate2=torch.randn(w.segments, w.d, generator=g).to(dev))
    return a, d, block


class Flush:
    """Before every timed step: write a buffer twice the size of L2; with "write+read",
    then read a second one, so that the written lines are written back here and the step
    starts from an L2 that holds nothing of its own and owes no write-back (the state
    ncu's cache control gives each kernel)."""

    def __init__(self, mode, dev):
        import torch
        self.buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.clean = (torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
                      if mode == "write+read" else None)

    def __call__(self):
        self.buf.zero_()
        if self.clean is not None:
            self.clean.amax()


def _timed_steps(step, K, flush, stream, barrier, clocks=None, mark=("begin", "end")):
    """Exactly K steps between a barrier + synchronize on both sides; the L2 flush runs
    before each step, outside its CUDA events (recorded on the launching stream).
    Returns the summed milliseconds of the K steps."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    if clocks is not None and mark[0]:
        clocks.mark(mark[0])
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if clocks is not None and mark[1]:
        clocks.mark(mark[1])
    barrier()
    return sum(s_.elapsed_time(e_) for s_, e_ in ev)


def _repeated_regions(run_region, clocks, min_s, dist, dev):
    """The timed region, repeated: run_region(marks) times one region of exactly K steps
    (marking the clock window's begin / end as told) and returns its milliseconds. The
    first region fixes how many repeats cover min_s seconds of step time (the largest
    count over the ranks, so that every rank runs the same collective sequence); the clock
    record spans all of them. Returns the per-region milliseconds."""
    import math
    first = run_region(("begin", None))
    want = max(1, math.ceil(min_s * 1e3 / max(first, 1e-6))) if min_s > 0 else 1
    reps = int(max_over_ranks([float(want)], dist, dev)[0])
    regions = [first]
    for _ in range(1, reps):
        regions.append(run_region((None, None)))
    clocks.mark("end")
    return regions


def measure(args, w, seed, dev, dist, K, W, inter, shared_f=0, extras=True):
    """Times the layer on workload w: K steps back to back (the headline), K traced steps
    (per-stage events), and with `extras` a replayed CUDA graph and the end-to-end
    steps through host buffers. Returns the per-rank measurements."""
    import torch
    import diffusion_transformer_moe_b200 as nm

    a, d, block = _device_inputs(w, seed, dev, shared_f)
    x, W_r, W1, W3, W2 = d["x"], d["W_r"], d["W1"], d["W3"], d["W2"]
    ws = torch.empty(nm.workspace_size(w.T, w.d, w.E, w.F, w.C, intermediate=inter,
                                       n_segments=w.segments, host_io=True,
                                       shared_f=shared_f or None),
                     dtype=torch.uint8, device=dev)
    out = torch.empty_like(x)
    flush = Flush(args.l2_flush, dev)
    stream = torch.cuda.current_stream()
    trace = nm.Trace(K)

    def step(tr=None):
        nm.forward(x, W_r, W1, W3, W2, w.C, out=out, workspace=ws, intermediate=inter,
                   n_segments=w.segments, trace=tr, tma_gather=args.tma_gather, **block)

    def barrier():
        if dist is not None:
            dist.barrier()

    clocks = ClockSampler(dev.index)
    clocks.start()
    for _ in range(W):
        flush()
        step()
    torch.cuda.synchronize()
    if nm.get_last_error() != 0:
        raise RuntimeError("device-side check failed during warm-up")

    # the timed region: K whole-layer steps, launched back to back as a user would,
    # repeated until the repeats cover --min-timed-s, with the SM clocks sampled throughout
    regions = _repeated_regions(
        lambda mk: _timed_steps(step, K, flush, stream, barrier, clocks, mark=mk), clocks,
        args.min_timed_s, dist, dev)
    ms = sum(regions) / len(regions)   # mean milliseconds of one K-step region
    clk = clocks.stop()
    # per-stage times: K more steps with CUDA events between the stages (the events keep
    # the stages from overlapping their launches, so this pass is not the headline)
    traced_ms = _timed_steps(lambda: step(trace), K, flush, stream, barrier)
    stage_ms, ncalls = trace.read()
    trace.close()
    r = dict(ms=ms, regions=len(regions), region_ms=regions, traced_ms=traced_ms, clocks=clk,
             stage_ms={k: v / max(ncalls, 1) for k, v in stage_ms.items()},
             launches=nm.kernels_per_call(w.T, w.d, w.E, w.F, w.C, intermediate=inter,
                                          n_segments=w.segments, shared_f=shared_f or None))
    if extras:
        # the same step replayed from a CUDA graph (one captured layer call; the flush
        # stays outside the graph and the events)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize()
        r["graph_ms"] = _timed_steps(graph.replay, K, flush, stream, barrier)
        del graph
        r.update(_e2e(args, w, a, d, block, ws, inter, K, W, dev, barrier))
        # the standalone gather of the chosen rows (not part of the layer's step)
        _, scores_t = nm.router(x, W_r, n_segments=w.segments)
        idx = nm.select(scores_t, w.C, n_segments=w.segments, csr=False)[0]
        packed = torch.empty(idx.numel(), w.d, dtype=x.dtype, device=dev)
        nm.gather_rows(x, idx, out=packed)
        r["gather_ms"] = _timed_steps(lambda: nm.gather_rows(x, idx, out=packed), K, flush,
                                      stream, barrier) / K
        del packed
    if nm.get_last_error() != 0:
        raise RuntimeError("device-side check failed during the timed steps")
    return r


def _e2e(args, w, a, d, block, ws, inter, K, W, dev, barrier):
    """End to end through the C ABI with host buffers: every step copies its x in from
    pinned host memory and its out back to pinned host memory inside the call. Steps
    rotate over --e2e-streams streams (each with its own workspace and host output);
    with three, a step's copy in never waits behind an earlier step's copy back on its
    own stream, so the copies in run back to back while the layer and the copies back of
    earlier steps overlap them (PCIe carries both directions at once). The weights, read
    every step, are larger than L2, so no flush."""
    import torch
    import diffusion_transformer_moe_b200 as nm
    n_streams = max(1, args.e2e_streams)
    stream = torch.cuda.current_stream()
    x_host = a["x"].pin_memory()
    streams = [stream] + [torch.cuda.Stream(device=dev) for _ in range(n_streams - 1)]
    wss = [ws] + [torch.empty_like(ws) for _ in range(n_streams - 1)]
    outs = [torch.empty_like(x_host).pin_memory() for _ in range(n_streams)]

    def e2e_step(i):
        j = i % n_streams
        nm.forward(x_host, d["W_r"], d["W1"], d["W3"], d["W2"], w.C, out=outs[j],
                   workspace=wss[j], n_segments=w.segments, intermediate=inter,
                   host_io=True, tma_gather=args.tma_gather, stream=streams[j], **block)

    for i in range(max(n_streams, W // 2)):
        e2e_step(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t0.record(streams[0])
    for s_ in streams[1:]:
        s_.wait_event(t0)
    for i in range(K):
        e2e_step(i)
    for s_ in streams[1:]:
        streams[0].wait_stream(s_)
    t1.record(streams[0])
    torch.cuda.synchronize()
    barrier()
    e2e_ms = t0.elapsed_time(t1)
    # the same steps' copies alone (x in, out back, the same streams and buffers): the
    # end-to-end step's PCIe ceiling
    xd = [torch.empty_like(d["x"]) for _ in range(n_streams)]
    od = [torch.empty(outs[0].shape, dtype=outs[0].dtype, device=dev) for _ in range(n_streams)]

    def copy_step(i):
        j = i % n_streams
        with torch.cuda.stream(streams[j]):
            xd[j].copy_(x_host, non_blocking=True)
            outs[j].copy_(od[j], non_blocking=True)

    for i in range(n_streams):
        copy_step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t0.record(streams[0])
    for s_ in streams[1:]:
        s_.wait_event(t0)
    for i in range(K):
        copy_step(i)
    for s_ in streams[1:]:
        streams[0].wait_stream(s_)
    t1.record(streams[0])
    torch.cuda.synchronize()
    barrier()
    return dict(e2e_ms=e2e_ms, copy_ms=t0.elapsed_time(t1), e2e_streams=n_streams,
                h2d=x_host.numel() * x_host.element_size(),
                d2h=outs[0].numel() * outs[0].element_size())


def _stage_report(w, stage_ms, peaks, inter, shared_f):
    """Per-stage µs, algorithmic GB/s and fraction of HBM, FLOP rate and fraction of the
    sustained bf16 peak, and the bytes as built."""
    sb = stage_bytes(w, shared_f)
    db = stage_design_bytes(w, inter, shared_f)
    sf = stage_flops(w, shared_f)
    out = {}
    for name, ms_ in stage_ms.items():
        s_ = ms_ / 1e3
        st = {"us": s_ * 1e6, "GB/s": sb[name] / s_ / 1e9,
              "hbm_frac": sb[name] / s_ / 1e9 / peaks["hbm"],
              "design_GB/s": db[name] / s_ / 1e9}
        if name in sf:
            st["TFLOP/s"] = sf[name] / s_ / 1e12
            st["tensor_frac"] = st["TFLOP/s"] / peaks["tensor_sustained"]
            if name == "gemm2_scale" and inter == "split":
                # the hi and lo halves of H each run their own MMAs into one accumulator
                st["executed_TFLOP/s"] = 2 * st["TFLOP/s"]
        out[name] = st
    return out


def _gather_report(w, ms, peaks):
    """The standalone gather's HBM figure (timed alone, K launches, L2 flushed before
    each)."""
    b = gather_bytes(w)
    return {"us": ms * 1e3, "GB/s": b / (ms / 1e3) / 1e9,
            "hbm_frac": b / (ms / 1e3) / 1e9 / peaks["hbm"], "bytes_per_launch": b,
            "how": "nmoe_rows_gather of the layer's own idx [E, Ce] from x into one block "
                   "per expert, timed alone; the layer fuses this copy into the gate/up "
                   "GEMM's A-tile loads, so it is not part of the step"}


def _roofline(w, stage_ms, peaks, inter, shared_f):
    """The dominant kernel's roofline: the larger of its algorithmic byte time and its
    FLOP time at the measured peaks (the sustained tensor figure: the kernel runs inside
    a long step)."""
    sb = stage_bytes(w, shared_f)
    db = stage_design_bytes(w, inter, shared_f)
    sf = stage_flops(w, shared_f)
    dom = max(stage_ms, key=lambda k: stage_ms[k])
    dom_s = stage_ms[dom] / 1e3
    src = "MEASURED_PEAKS.json" if peaks["source"] == "measured" else "fallback"
    if sf.get(dom, 0) / (peaks["tensor_sustained"] * 1e12) > sb[dom] / (peaks["hbm"] * 1e9):
        achieved = sf[dom] / dom_s / 1e12
        return {"kernel": dom, "bound": "tensor", "achieved": achieved,
                "peak": peaks["tensor_sustained"], "unit": "TFLOP/s",
                "frac": achieved / peaks["tensor_sustained"],
                "algorithmic_flops_per_launch": sf[dom],
                "peak_source": f"{src} bf16_tflops_sustained", "traffic": None}
    achieved = sb[dom] / dom_s / 1e9
    return {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm"],
            "unit": "GB/s", "frac": achieved / peaks["hbm"],
            "algorithmic_bytes_per_launch": sb[dom],
            "design_bytes_per_launch": db[dom],
            "design_frac": db[dom] / dom_s / 1e9 / peaks["hbm"],
            "peak_source": f"{src} hbm_gbs", "traffic": _traffic(dom, w.name)}


def profile_calls(args, w, dev):
    """args.profile_calls layer calls, nothing timed: the launch sequence an ncu capture
    selects its kernels from (five kernels per call on the tensor-core path)."""
    import torch
    import diffusion_transformer_moe_b200 as nm
    _, d, block = _device_inputs(w, 0, dev, args.shared_f)
    ws = torch.empty(nm.workspace_size(w.T, w.d, w.E, w.F, w.C, intermediate=args.intermediate,
                                       n_segments=w.segments, shared_f=args.shared_f or None),
                     dtype=torch.uint8, device=dev)
    out = torch.empty_like(d["x"])
    for _ in range(args.profile_calls):
        nm.forward(d["x"], d["W_r"], d["W1"], d["W3"], d["W2"], w.C, out=out, workspace=ws,
                   intermediate=args.intermediate, n_segments=w.segments,
                   tma_gather=args.tma_gather, **block)
    torch.cuda.synchronize()
    if nm.get_last_error() != 0:
        raise RuntimeError("device-side check failed")


def run_ours(args, w, rank, world, local_rank, dist):
    import torch
    from diffusion_transformer_moe_b200 import inputs as I

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.profile_calls:
        profile_calls(args, w, dev)
        return
    inter = args.intermediate
    K, W = args.steps, args.warmup
    m = measure(args, w, rank, dev, dist, K, W, inter, args.shared_f)
    tb = None
    if args.tensor_workload and args.tensor_workload != w.name:
        torch.cuda.empty_cache()
        wt = I.WORKLOADS[args.tensor_workload]
        tb = measure(args, wt, rank, dev, dist, K, W, args.tensor_intermediate, 0,
                     extras=False)
    keys = (["ms", "traced_ms", "graph_ms", "e2e_ms", "copy_ms", "gather_ms"]
            + (["tb_ms"] if tb else []))
    vals = ([m["ms"], m["traced_ms"], m["graph_ms"], m["e2e_ms"], m["copy_ms"], m["gather_ms"]]
            + ([tb["ms"]] if tb else []))
    mx = dict(zip(keys, max_over_ranks(vals, dist, dev)))
    if rank != 0:
        return

    peaks = _peaks()
    per_step_s = mx["ms"] / 1e3 / K
    flops = w.expert_flops() + w.router_flops() + 6.0 * w.T * w.d * args.shared_f
    line = {
        "metric": METRIC, "value": replica_throughput(w.T, world, K, mx["ms"]),
        "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": mx["ms"] / K, "higher_is_better": True, "scaling": "weak",
        "timed_regions": {"count": m["regions"], "steps_each": K,
                          "ms_per_step_each": [round(x / K, 5) for x in m["region_ms"]],
                          "how": "the K-step timed region repeated until the repeats cover "
                                 f"{args.min_timed_s:g} s of step time; value and ms_per_step "
                                 "are their mean (the slowest rank's)"},
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _workload_config(w, args.l2_flush),
        "parallelism": f"replicas x{world} (one independent layer per GPU, no exchange)",
        "impl_options": {"intermediates": inter,
                         "gather": "tma gather4" if args.tma_gather else "cp.async",
                         **({"shared_f": args.shared_f,
                             "block": "x + tanh(clamp(gate2, -2, 2)) * (shared + routed)"}
                            if args.shared_f else {})},
        "tflops": flops / per_step_s / 1e12,
        "tensor_frac_of_layer": flops / per_step_s / 1e12 / peaks["tensor_sustained"],
        "roofline": _roofline(w, m["stage_ms"], peaks, inter, args.shared_f),
        "stages": _stage_report(w, m["stage_ms"], peaks, inter, args.shared_f),
        "gather": _gather_report(w, mx["gather_ms"], peaks),
        "traced_ms_per_step": mx["traced_ms"] / K,
        "graph_replay": {"ms_per_step": mx["graph_ms"] / K,
                         "value": replica_throughput(w.T, world, K, mx["graph_ms"]),
                         "how": "one captured layer call, replayed K times"},
        "gpu_launches": K * m["launches"],
        "e2e": {"value": replica_throughput(w.T, world, K, mx["e2e_ms"]), "unit": "tokens/s",
                "h2d_bytes_per_step": m["h2d"], "d2h_bytes_per_step": m["d2h"],
                "ms_per_step": mx["e2e_ms"] / K,
                "how": "nmoe_forward_ex with host_io (x copied in, out copied back to pinned "
                       "host memory inside each call), steps rotating over "
                       f"{m['e2e_streams']} streams",
                "copies_only_ms_per_step": mx["copy_ms"] / K,
                "frac_of_copies_only": mx["copy_ms"] / mx["e2e_ms"],
                "pcie_GBps_per_direction": m["h2d"] * K / (mx["copy_ms"] / 1e3) / 1e9},
        "clocks": m["clocks"],
    }
    if tb is not None:
        wt = I.WORKLOADS[args.tensor_workload]
        t_s = mx["tb_ms"] / 1e3 / K
        tflops = wt.expert_flops() + wt.router_flops()
        ti = args.tensor_intermediate
        st = _stage_report(wt, tb["stage_ms"], peaks, ti, 0)
        line["tensor_bound"] = {
            "config": _workload_config(wt, args.l2_flush), "intermediates": ti,
            "steps": K, "warmup": W, "ms_per_step": mx["tb_ms"] / K,
            "timed_regions": tb["regions"],
            "value": replica_throughput(wt.T, world, K, mx["tb_ms"]), "unit": "tokens/s",
            "tflops": tflops / t_s / 1e12,
            "tensor_frac_of_layer": tflops / t_s / 1e12 / peaks["tensor_sustained"],
            "peak": peaks["tensor_sustained"],
            "peak_source": ("MEASURED_PEAKS.json" if peaks["source"] == "measured"
                            else "fallback") + " bf16_tflops_sustained",
            "gemms": {k: st[k] for k in ("gemm1_swiglu", "gemm2_scale")},
            "stages": st, "gpu_launches": K * tb["launches"],
            "clocks": tb["clocks"],
        }
        mhz, ref = tb["clocks"].get("sm_mhz"), peaks.get("sustained_mhz")
        if mhz and ref:
            # tensor throughput scales with the SM clock: the sustained peak at the median
            # clock this run held under the power cap
            pk = peaks["tensor_sustained"] * mhz / ref
            line["tensor_bound"]["clock_normalized"] = {
                "sm_mhz": mhz, "peak_reference_mhz": ref, "peak_at_sm_mhz": pk,
                "tensor_frac_of_layer": tflops / t_s / 1e12 / pk,
                "gemms": {k: st[k]["TFLOP/s"] / pk for k in ("gemm1_swiglu", "gemm2_scale")},
            }
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)


def main():
    args = _args()
    from diffusion_transformer_moe_b200 import inputs as I
    w = I.WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
        dist = tdist
    try:
        run_ours(args, w, rank, world, local_rank, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
