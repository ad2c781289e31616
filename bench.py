"""Benchmark of the MoE dispatch / combine path on B200.

One step = one pass of the whole path over one batch: routing metadata
(moe_prepare), dispatch (moe_dispatch_rows, or moe_dispatch_rows_fp8 for the
fp8 workload) and combine (moe_combine), on seeded synthetic inputs already
resident in HBM.  Prints ONE JSON line (rank 0).

By default every workload runs: the headline is the largest single-GPU one
(T=131072, H=2048, E=64, top-6, fp16 -> fp32 combine) and the other four
are reported under "per_workload" with the same fields.  ``--workload NAME``
runs one workload alone as the headline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|all]
    python bench.py --impl reference ...   # the CPU oracle on the host cores

Multi-GPU runs (torchrun, one process per GPU) are independent replicas:
the path has no exchange step, so every rank runs the same workload on its
own GPU and the value is the total over ranks ("scaling": "weak"), timed as
the maximum over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import glob
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import CONFIGS, make_workload  # noqa: E402

HEADLINE_WORKLOAD = "zipf_fp16_t131072_h2048_e64_k6"
METRIC = "dispatch+combine tokens/s and effective HBM GB/s (% of B200 peak), 1 GPU"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
DTYPE_BYTES = {"bf16": 2, "fp16": 2, "fp32": 4, "fp8_e4m3": 1}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(w):
    """Minimal HBM bytes of each step: every input read once, every output
    written once (the x row is read once though written k times)."""
    S, T, H, E = w.S, w.T, w.H, w.E
    bx = DTYPE_BYTES[w.x_dtype]
    bd = DTYPE_BYTES[w.dispatch_dtype]
    by = DTYPE_BYTES[w.y_dtype]
    bo = DTYPE_BYTES[w.out_dtype]
    fp8 = w.dispatch_dtype == "fp8_e4m3"
    prepare = 4 * S + 4 * E + 4 * (E + 1) + 8 * S + (4 * (E + 1) if fp8 else 0)
    dispatch = T * H * bx + S * H * bd + 4 * S
    if fp8:
        dispatch += 4 * S * (H // 128) + 8 * (E + 1)  # scales, expert and scale offsets
    combine = S * H * by + 4 * S + 4 * S + T * H * bo
    return {"prepare": prepare, "dispatch": dispatch, "combine": combine}


# Sources each timed kernel is built from: its own file and the shared headers.
KERNEL_SOURCES = {
    "dispatch": ["dispatch.cu", "kernels.h", "launch.h", "moe_device.cuh"],
    "dispatch_nvfp4": ["dispatch.cu", "kernels.h", "launch.h", "moe_device.cuh"],
    "combine": ["combine.cu", "kernels.h", "launch.h", "moe_device.cuh"],
}


def src_hash(step):
    """sha256 (16 hex digits) of the sources the kernel of `step` is built from."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[step]:
        with open(os.path.join(ROOT, "combine_permute_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel_key):
    """dram read+write bytes per launch from the committed ncu summary, if it
    was taken on the kernel's current sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d["kernels"][kernel_key]
        step = kernel_key.split("@")[0]
        return e["dram_bytes_per_launch"] if e.get("src_hash") == src_hash(step) else None
    except Exception:
        return None


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML during the timed
    region (read-only)."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _sample(self):
        mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
        bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        self.samples.append(mhz)
        for b, name in self.REASONS.items():
            if bits & b:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(0.002)

    def __enter__(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return None
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "source": "nvml"}


def percentiles(ms):
    a = np.asarray(ms)
    return {"p50": float(np.percentile(a, 50)), "p90": float(np.percentile(a, 90)),
            "p99": float(np.percentile(a, 99)), "mean": float(a.mean())}


# ---------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline leg)
# ---------------------------------------------------------------------------

def _oracle_step(oracle, w, ids, wt, xb, yb):
    A = w.block_align if w.dispatch_dtype == "fp8_e4m3" else 1
    m = oracle.prepare(ids, w.E, A)
    if w.dispatch_dtype == "fp8_e4m3":
        oracle.dispatch_fp8(xb, w.x_dtype, ids, m)
    else:
        oracle.dispatch(xb, w.k, m["input_perm"])
    oracle.combine(yb, w.y_dtype, m["output_perm"], wt, w.out_dtype)


def _host_inputs(w, T_sample):
    import torch
    ws = w.scaled(T_sample, name=w.name)
    ids, wt, x, y = make_workload(ws)
    xb = x.view(torch.int16).numpy().view(np.uint16) if x.dtype != torch.float32 else x.numpy()
    yb = y.view(torch.int16).numpy().view(np.uint16) if y.dtype != torch.float32 else y.numpy()
    return ws, ids, wt, xb, yb


def oracle_sample_plan(w, step_budget_s, openmp=False):
    """A bounded sample of workload ``w`` for the oracle: the same routing,
    shapes and dtypes on the first T_s tokens, T_s sized from a 256-token
    calibration step so that one oracle step takes about ``step_budget_s``.
    Returns T_s and a function that runs one oracle step on it."""
    import oracle
    oracle.lib()
    ctx = oracle.openmp() if openmp else _null_ctx()
    cal_T = max(1, min(w.T, 256))
    ws, ids, wt, xb, yb = _host_inputs(w, cal_T)
    with ctx:
        _oracle_step(oracle, ws, ids, wt, xb, yb)  # first call pays the loader
        t0 = time.perf_counter()
        _oracle_step(oracle, ws, ids, wt, xb, yb)
        per_tok = (time.perf_counter() - t0) / cal_T
    T_s = int(max(1, min(w.T, step_budget_s / max(per_tok, 1e-9))))
    ws, ids, wt, xb, yb = _host_inputs(w, T_s)

    def run():
        with (oracle.openmp() if openmp else _null_ctx()):
            _oracle_step(oracle, ws, ids, wt, xb, yb)
    return T_s, run


class _null_ctx:
    def __enter__(self):
        return None

    def __exit__(self, *a):
        return False


def time_oracle(w, budget_s=12.0, openmp=False):
    """The oracle's whole step (prepare, dispatch, combine) on a bounded token
    sample of ``w``, repeated until ``budget_s`` has passed (at least twice):
    tokens per second, the threads it used and what the sample was."""
    import oracle
    T_s, run = oracle_sample_plan(w, budget_s / 4, openmp)
    n, t0 = 0, time.perf_counter()
    while True:
        run()
        n += 1
        if n >= 2 and time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    cores = oracle.threads(openmp)
    build = ("the same C source built with OpenMP over the dispatch and combine rows "
             "(prepare one thread)" if openmp else "plain single-threaded build")
    return {"value": T_s * n / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} oracle steps on the first {T_s} of {w.T} tokens of {w.name}",
            "build": build}


def cpu_baseline(w, budget_s):
    """The oracle timed on the host cores: the OpenMP build on every core
    (the line's value and core count) and the plain build on one core."""
    multi = time_oracle(w, budget_s * 0.4, openmp=True)
    single = time_oracle(w, budget_s * 0.6, openmp=False)
    out = dict(multi)
    out["single_core"] = {k: single[k] for k in ("value", "cores", "sample", "build")}
    return out


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    K, W = args.steps, args.warmup
    T_s, run = oracle_sample_plan(w, args.ref_budget / (K + W))
    for _ in range(W):
        run()
    t0 = time.perf_counter()
    for _ in range(K):
        run()
    dt = time.perf_counter() - t0
    value = T_s * K / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": K, "warmup": W, "ms_per_step": dt / K * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": _dtype_tag(w),
        "data": "synthetic",
        "config": _config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads(),
                         "kind": "oracle",
                         "sample": f"first {T_s} of {w.T} tokens of {w.name} per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _dtype_tag(w):
    return w.x_dtype if w.dispatch_dtype != "fp8_e4m3" else "bf16->fp8_e4m3"


def _config(w, n):
    return {"workload": w.name, "T": w.T, "H": w.H, "E": w.E, "k": w.k,
            "routing": w.routing.mode, "x_dtype": w.x_dtype, "dispatch_dtype": w.dispatch_dtype,
            "y_dtype": w.y_dtype, "out_dtype": w.out_dtype, "seed": w.seed,
            "l2": ("no flush: per-step working set > 126 MB L2" if _step_bytes(w) > L2_BYTES
                   else "flushed: a buffer of twice the L2 size written before every timed step"),
            "parallelism": "replicas" if n > 1 else "single GPU"}


def net_of_events(call_us, step_us):
    """What the timing events between the calls add to a step (the calls
    timed with events, summed, against the event-free step), and each call's
    share of the event-free step: its evented time less an equal share of
    that overhead, so that the shares sum to the step's time."""
    overhead = sum(call_us.values()) - step_us
    return overhead, {c: t - overhead / len(call_us) for c, t in call_us.items()}


def _step_bytes(w):
    return sum(algorithmic_bytes(w).values())


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

class Step:
    """Device buffers and the three calls of one step."""

    def __init__(self, w, dev):
        import torch
        import combine_permute_b200 as moe
        self.moe, self.w, self.dev = moe, w, dev
        ids_np, wt_np, x, y = make_workload(w, device=dev)
        self.ids_np, self.wt_np = ids_np, wt_np
        self.ids = torch.from_numpy(ids_np).to(dev)
        self.wt = torch.from_numpy(wt_np).to(dev)
        self.x, self.y = x, y
        self.fp8 = w.dispatch_dtype == "fp8_e4m3"
        self.A = w.block_align if self.fp8 else None
        i32 = dict(dtype=torch.int32, device=dev)
        S, E = w.S, w.E
        self.meta_bufs = dict(expert_counts=torch.empty(E, **i32),
                              expert_offsets=torch.empty(E + 1, **i32),
                              blockscale_offsets=torch.empty(E + 1, **i32) if self.fp8 else None,
                              input_permutation=torch.empty(S, **i32),
                              output_permutation=torch.empty(S, **i32),
                              diag=torch.empty(2, **i32))
        nws = moe.moe_prepare_workspace_bytes(w.T, w.k, E)
        self.ws = torch.zeros(max(nws, 1), dtype=torch.uint8, device=dev)
        # tiny batches take the one-launch prepare + dispatch path
        self.fused = (not self.fp8) and S <= moe._lib.FUSED_MAX_SLOTS
        if self.fp8:
            self.xq = torch.empty((S, w.H), dtype=torch.uint8, device=dev)
            self.scales = torch.empty((S + E * (w.block_align - 1), w.H // 128),
                                      dtype=torch.float32, device=dev)
        else:
            self.xd = torch.empty((S, w.H), dtype=x.dtype, device=dev)
        from workloads.routing import torch_dtype
        self.out = torch.empty((w.T, w.H), dtype=torch_dtype(w.out_dtype), device=dev)
        # prepare: one launch, or two when its tiles do not all fit on the GPU
        # at once (the graph's kernel nodes give the exact count)
        self.launches_per_step = 2 if self.fused else (2 if nws > 0 and S > 300_000 else 1) + 2

    def prepare(self):
        return self.moe.moe_prepare(self.ids, self.w.E, blockscale_align=self.A, workspace=self.ws,
                                    **self.meta_bufs)

    def dispatch(self, meta):
        if self.fp8:
            self.moe.moe_dispatch_rows_fp8(self.x, self.w.k, meta.output_permutation,
                                           meta.expert_offsets, meta.blockscale_offsets,
                                           blockscale_align=self.A, out_q=self.xq,
                                           out_scales=self.scales)
        else:
            self.moe.moe_dispatch_rows(self.x, self.w.k, meta.input_permutation,
                                       meta.output_permutation, out=self.xd)

    def combine(self, meta):
        self.moe.moe_combine(self.y, meta.output_permutation, self.wt, out=self.out)

    def prepare_dispatch(self):
        """One launch for tiny batches; otherwise prepare then dispatch."""
        if self.fused:
            meta, _ = self.moe.moe_prepare_dispatch(self.ids, self.w.E, self.x, out=self.xd,
                                                    **self.meta_bufs)
            return meta
        meta = self.prepare()
        self.dispatch(meta)
        return meta

    def run(self):
        meta = self.prepare_dispatch()
        self.combine(meta)


class Ranks:
    """One process per GPU: rank bookkeeping, barrier and max-over-ranks.

    The path has no exchange step, so the only collectives are these timing
    helpers (NCCL on GPUs; gloo works the same way on CPU).
    """

    def __init__(self, backend="nccl", device=None, timeout_s=120):
        import datetime
        import torch.distributed as dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        self.dist = dist if self.world > 1 else None
        if self.dist is not None:
            kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
            if backend == "nccl" and device is not None:
                kw["device_id"] = device
            dist.init_process_group(backend, **kw)

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max_over_ranks(self, v: float) -> float:
        if self.dist is None:
            return v
        import torch
        t = torch.tensor([float(v)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()


def graph_kernel_nodes(g):
    """Kernel nodes of a captured CUDA graph (kept with keep_graph=True): the
    kernels one replay launches.  None when the graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as rt
        graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kinds = [rt.cudaGraphNodeGetType(node)[1] for node in nodes[:n]]
        return sum(1 for kind in kinds if kind == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:
        return None


def steps_per_graph(K: int, most: int = 10) -> int:
    """Steps captured in one CUDA graph: the largest divisor of K up to
    `most`, so that exactly K steps run in the timed region."""
    return max(n for n in range(1, most + 1) if K % n == 0)


def whole_job_tokens_per_s(T: int, steps: int, world: int, max_elapsed_ms: float) -> float:
    """Tokens every rank processed, over the slowest rank's time."""
    return T * steps * world / (max_elapsed_ms * 1e-3)


def bench_workload(args, w, dev, ranks, cpu_budget_s):
    """Times one workload: the eager per-call breakdown, the graph-replayed
    headline steps, the end-to-end figure from host buffers and the steps
    beside the path; returns the fields of its JSON entry (rank 0)."""
    import torch

    world, rank, local = ranks.world, ranks.rank, ranks.local
    barrier, max_over_ranks = ranks.barrier, ranks.max_over_ranks
    step = Step(w, dev)
    K, W = args.steps, args.warmup
    stream = torch.cuda.current_stream(dev)
    for _ in range(W):
        step.run()
    torch.cuda.synchronize(dev)

    # ---- timed region 1 (eager launches): K steps with CUDA events around
    #      every call, for the per-call breakdown and the roofline
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    marks = [[ev() for _ in range(4)] for _ in range(K)]
    start, end = ev(), ev()
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks_eager:
        start.record(stream)
        for i in range(K):
            m = marks[i]
            m[0].record(stream)
            if step.fused:  # one launch: prepare and dispatch timed together
                meta = step.prepare_dispatch()
                m[1].record(stream)
            else:
                meta = step.prepare()
                m[1].record(stream)
                step.dispatch(meta)
            m[2].record(stream)
            step.combine(meta)
            m[3].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    eager_ms = max_over_ranks(start.elapsed_time(end))
    per = {"prepare": [], "dispatch": [], "combine": [], "step": []}
    for m in marks:
        per["prepare"].append(m[0].elapsed_time(m[1]))
        per["dispatch"].append(m[1].elapsed_time(m[2]))
        per["combine"].append(m[2].elapsed_time(m[3]))
        per["step"].append(m[0].elapsed_time(m[3]))

    # ---- timed region 2 (the headline): n consecutive steps captured once as
    #      a CUDA graph, the way a serving loop captures a forward pass with
    #      its MoE layers, and replayed K / n times (n = steps_per_graph(K))
    graph_ms, clocks = None, clocks_eager
    kernels_per_step = None
    n_graph = steps_per_graph(K)
    try:
        g = torch.cuda.CUDAGraph(keep_graph=True)
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step.run()
            with torch.cuda.graph(g, stream=side):
                for _ in range(n_graph):
                    step.run()
        nodes = graph_kernel_nodes(g)
        kernels_per_step = nodes // n_graph if nodes else None
        g.instantiate()
        torch.cuda.synchronize(dev)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(dev)
        gs, ge = ev(), ev()
        barrier()
        torch.cuda.synchronize(dev)
        with ClockSampler(local) as clocks_graph:
            gs.record(stream)
            for _ in range(K // n_graph):
                g.replay()
            ge.record(stream)
            torch.cuda.synchronize(dev)
        barrier()
        graph_ms = max_over_ranks(gs.elapsed_time(ge))
        clocks = clocks_graph
        del g
    except Exception as exc:  # a capture failure falls back to the eager number
        print(f"cuda graph timing unavailable: {exc}", file=sys.stderr)
        graph_ms = None

    # ---- timed region 3: the per-call breakdown inside the graph.  The same
    #      n steps captured in a second graph with timing events recorded
    #      between the calls (event nodes of the graph, on the kernels'
    #      stream); replayed K / n times, so every call is timed K times
    #      without the host launch gaps of the eager region.
    per_graph = None
    try:
        per_graph = time_calls_in_graph(step, dev, K, n_graph)
    except Exception as exc:
        print(f"in-graph call timing unavailable: {exc}", file=sys.stderr)
    # ---- timed region 4: every call alone, as its average launch time over
    #      a graph of n back-to-back launches with events only around the
    #      graph (no event between launches, so nothing separates them)
    alone = None
    try:
        alone = time_calls_alone(step, dev, K, n_graph)
    except Exception as exc:
        print(f"back-to-back call timing unavailable: {exc}", file=sys.stderr)

    # ---- timed region 5, only for a step whose working set fits in L2: K
    #      eager steps, each after an L2 flush (a buffer of twice the L2
    #      size written outside the step's events), so that no step finds
    #      its inputs left in L2 by the one before; their sum is the value
    flushed_ms, clocks_flushed = None, None
    if _step_bytes(w) <= L2_BYTES:
        flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        fmarks = [(ev(), ev()) for _ in range(K)]
        barrier()
        torch.cuda.synchronize(dev)
        with ClockSampler(local) as clocks_flushed:
            for i in range(K):
                flush_buf.fill_(i & 0xff)
                fmarks[i][0].record(stream)
                step.run()
                fmarks[i][1].record(stream)
            torch.cuda.synchronize(dev)
        barrier()
        flushed_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in fmarks))
        del flush_buf

    counts = step.meta_bufs["expert_counts"].cpu().numpy()
    diag = step.meta_bufs["diag"].cpu().numpy().tolist()

    # ---- end to end through the public API from pinned host buffers
    e2e = run_e2e(step, w, dev, K, W, barrier, max_over_ranks)
    next_rows = time_next_rows(step, w, dev)
    fused, launches_per_step = step.fused, step.launches_per_step
    del step
    torch.cuda.empty_cache()

    cpu = cpu_baseline(w, cpu_budget_s) if (cpu_budget_s > 0 and rank == 0 and world == 1) else None
    if rank != 0:
        return None

    peak, peak_kind = measured_peak()
    alg = algorithmic_bytes(w)
    if fused:  # prepare and dispatch are one launch, timed together
        alg = {"prepare_dispatch": alg["prepare"] + alg["dispatch"], "combine": alg["combine"]}
        per = {"prepare_dispatch": per["prepare"], "combine": per["combine"], "step": per["step"]}
        if per_graph is not None:
            per_graph = {"prepare_dispatch": per_graph["prepare"],
                         "combine": per_graph["combine"], "step": per_graph["step"]}
        if alone is not None:
            alone = {"prepare_dispatch": alone["prepare"], "combine": alone["combine"]}
    calls = [c for c in ("prepare", "dispatch", "prepare_dispatch", "combine") if c in alg]
    # the breakdown and the roofline use the in-graph times (the calls as the
    # headline's graph runs them); the eager ones add each launch's host and
    # event gap (several microseconds a call) and are kept beside them
    timed = per_graph if per_graph is not None else per
    kern = {c: statistics.mean(timed[c]) for c in calls}
    eager_kern = {c: statistics.mean(per[c]) for c in calls}
    dominant = max((c for c in calls if c != "prepare"), key=lambda c: kern[c])
    kernel_key = f"{dominant}@{w.name}"
    achieved = alg[dominant] / (kern[dominant] * 1e-3) / 1e9
    elapsed_ms = graph_ms if graph_ms is not None else eager_ms
    breakdown = {}
    for k in calls:
        gbs = alg[k] / (kern[k] * 1e-3) / 1e9
        breakdown[k] = {"us_mean": kern[k] * 1e3, "latency_ms": percentiles(timed[k]),
                        "timed": "in graph" if per_graph is not None else "eager",
                        "tokens_per_s": w.T / (kern[k] * 1e-3), "algorithmic_bytes": alg[k],
                        "effective_gbs": gbs, "frac_of_measured_peak": gbs / peak,
                        "frac_of_8tbs_spec": gbs / SPEC_HBM_GBS,
                        "eager_us_mean": eager_kern[k] * 1e3,
                        "eager_latency_ms": percentiles(per[k])}
        if alone is not None:
            a_gbs = alg[k] / (alone[k] * 1e-3) / 1e9
            breakdown[k].update({"alone_us_mean": alone[k] * 1e3, "alone_effective_gbs": a_gbs,
                                 "alone_frac_of_measured_peak": a_gbs / peak,
                                 "alone_frac_of_8tbs_spec": a_gbs / SPEC_HBM_GBS})
    step_alg = sum(alg.values())
    breakdown["end_to_end"] = {
        "latency_ms": percentiles(timed["step"]),
        "eager_latency_ms": percentiles(per["step"]),
        "eager_ms_per_step": eager_ms / K,
        "graph_ms_per_step": None if graph_ms is None else graph_ms / K,
        "effective_gbs": step_alg / (elapsed_ms / K * 1e-3) / 1e9,
        "frac_of_measured_peak": step_alg / (elapsed_ms / K * 1e-3) / 1e9 / peak}
    if per_graph is not None and graph_ms is not None:
        overhead, net = net_of_events({c: kern[c] * 1e3 for c in calls}, graph_ms / K * 1e3)
        breakdown["end_to_end"]["event_overhead_us_per_step"] = overhead
        for c in calls:
            breakdown[c]["us_net_of_events"] = net[c]
            breakdown[c]["net_frac_of_8tbs_spec"] = (
                alg[c] / (net[c] * 1e-6) / 1e9 / SPEC_HBM_GBS if net[c] > 0 else None)
    launch = (f"cuda_graph of {n_graph} steps, replayed {K // n_graph} times"
              if graph_ms is not None else "eager")
    l2_resident = None
    if flushed_ms is not None:
        # the flushed steps are the value; the graph's steps, whose inputs
        # the step before left in L2, are kept beside them
        l2_resident = {"value": whole_job_tokens_per_s(w.T, K, world, elapsed_ms),
                       "ms_per_step": elapsed_ms / K, "launch": launch}
        elapsed_ms, launch = flushed_ms, ("eager steps, each after an L2 flush, CUDA events "
                                          "around each step")
        clocks = clocks_flushed
    return {
        "value": whole_job_tokens_per_s(w.T, K, world, elapsed_ms),
        "ms_per_step": elapsed_ms / K,
        "launch": launch,
        "l2_resident": l2_resident,
        "eager_value": whole_job_tokens_per_s(w.T, K, world, eager_ms),
        "roofline": {"bound": "hbm", "kernel": kernel_key, "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": committed_traffic(kernel_key),
                     "algorithmic_bytes_per_launch": alg[dominant]},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": (kernels_per_step or launches_per_step) * K,
        "gpu_launches_counted_from": ("kernel nodes of the captured step"
                                      if kernels_per_step else "launches per step of each call"),
        "clocks": clocks.summary(),
        "breakdown": breakdown,
        "next_rows": next_rows,
        "expert_load": {"max_tokens_per_expert": int(counts.max()),
                        "min_tokens_per_expert": int(counts.min()),
                        "mean_tokens_per_expert": float(counts.mean()),
                        "imbalance_ratio": float(counts.max() / max(counts.mean(), 1e-9))},
        "diag": diag,
    }


def profile_run(args, workloads, next_rows=False):
    """W warm-up and K eager steps of each workload, nothing else: the
    program the ncu captures run.  With next_rows, one prepare and then W + K
    eager launches of each call beside the path (next_row_calls) instead."""
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    for w in workloads:
        step = Step(w, dev)
        if next_rows:
            for fn in next_row_calls(step, w, dev).values():
                for _ in range(args.warmup + args.steps):
                    fn()
        else:
            for _ in range(args.warmup + args.steps):
                step.run()
        torch.cuda.synchronize(dev)
        del step
        torch.cuda.empty_cache()
    print("profile run done", flush=True)


def run_gpu(args, names, workloads=None):
    """Every workload in ``names`` on this rank's GPU; the first is the
    headline, the others go under "per_workload"."""
    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    if ranks.world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={ranks.world}")
    results = {}
    workloads = workloads or {n: CONFIGS[n] for n in names}
    for i, name in enumerate(names):
        budget = 0.0 if args.no_cpu_baseline else args.cpu_budget * (1.0 if i == 0 else 0.5)
        results[name] = bench_workload(args, workloads[name], dev, ranks, budget)
    world = ranks.world
    ranks.close()
    if ranks.rank != 0:
        return
    head_name = names[0]
    w = workloads[head_name]
    r = results[head_name]
    line = {
        "metric": METRIC, "value": r["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": _dtype_tag(w),
        "data": "synthetic",
        "config": _config(w, world),
    }
    line.update({k: v for k, v in r.items() if k not in ("value", "ms_per_step")})
    if len(names) > 1:
        line["per_workload"] = {
            n: dict(results[n], config=_config(workloads[n], world), dtype=_dtype_tag(workloads[n]))
            for n in names[1:]}
    print(json.dumps(line), flush=True)


def time_calls_in_graph(step, dev, K, n_graph):
    """Per-call durations (ms) of n_graph consecutive steps captured as one
    CUDA graph with timing events recorded between the calls, the graph
    replayed K / n_graph times: K samples per call."""
    import torch
    ev = lambda: torch.cuda.Event(enable_timing=True, external=True)  # noqa: E731
    marks = [[ev() for _ in range(4)] for _ in range(n_graph)]
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for m in marks:
                m[0].record(side)
                if step.fused:
                    meta = step.prepare_dispatch()
                    m[1].record(side)
                else:
                    meta = step.prepare()
                    m[1].record(side)
                    step.dispatch(meta)
                m[2].record(side)
                step.combine(meta)
                m[3].record(side)
    torch.cuda.synchronize(dev)
    g.replay()
    torch.cuda.synchronize(dev)
    per = {"prepare": [], "dispatch": [], "combine": [], "step": []}
    for _ in range(K // n_graph):
        g.replay()
        torch.cuda.synchronize(dev)
        for m in marks:
            per["prepare"].append(m[0].elapsed_time(m[1]))
            per["dispatch"].append(m[1].elapsed_time(m[2]))
            per["combine"].append(m[2].elapsed_time(m[3]))
            per["step"].append(m[0].elapsed_time(m[3]))
    del g
    return per


def time_calls_alone(step, dev, K, n):
    """Average launch time (ms) of each call of the step, alone: a CUDA graph
    of n back-to-back launches of that call on the step's buffers (the
    metadata of one prepare), events only around the graph, replayed K / n
    times."""
    import torch
    meta = step.prepare_dispatch() if step.fused else step.prepare()
    torch.cuda.synchronize(dev)
    calls = {"combine": lambda: step.combine(meta)}
    if step.fused:
        calls["prepare"] = step.prepare_dispatch
    else:
        calls["prepare"] = step.prepare
        calls["dispatch"] = lambda: step.dispatch(meta)
    out = {}
    for name, fn in calls.items():
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            fn()
            with torch.cuda.graph(g, stream=side):
                for _ in range(n):
                    fn()
        torch.cuda.synchronize(dev)
        g.replay()
        torch.cuda.synchronize(dev)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(max(1, K // n)):
            g.replay()
        e.record()
        torch.cuda.synchronize(dev)
        out[name] = s.elapsed_time(e) / (max(1, K // n) * n)
        del g
    return out


NEXT_TILE = 128  # rows per tile of the grouped-GEMM layout timed beside the path
EP_RANKS = 2     # ranks of the exchange between GPUs, emulated on this GPU


def next_row_bytes(w):
    """Algorithmic bytes of the calls beside the timed path (next_row_calls)."""
    S, E = w.S, w.E
    max_tiles = max(1, -(-S // NEXT_TILE) + min(E, S))
    x_b = 4 if w.x_dtype == "fp32" else 2
    return {
        "tile_layout_t128": (8 * S + 8 * E + 4 * (E + 1) + 8 * max_tiles + 4 * S
                             + 4 * max_tiles * NEXT_TILE + 8),
        "problem_sizes": 4 * E + 24 * E,
        "dispatch_nvfp4": w.T * w.H * x_b + S * (w.H // 2 + w.H // 16) + 4 * S + 8 * (E + 1),
        # the exchange's own kernels, both owners' buffers on this GPU
        "ep_peer_layout_r2": (4 * EP_RANKS * E + 4 * S + 4 * (E + 1) + 4 * S + 8 * S
                              + 4 * EP_RANKS + 4 * (E // EP_RANKS + 1)),
        "ep_dispatch_peer_r2": w.T * w.H * x_b + S * w.H * x_b + 8 * S,
        "ep_combine_peer_r2": S * w.H * x_b + 8 * S + 4 * S + w.T * w.H * _out_bytes(w),
    }


def _out_bytes(w):
    return {"fp32": 4, "bf16": 2, "fp16": 2}[w.out_dtype]


def next_row_calls(step, w, dev):
    """The calls beside the timed path, on the step's buffers after one
    prepare: the grouped-GEMM metadata that follows prepare (tile-padded
    layout with 128-row tiles, per-expert problem sizes), the NVFP4 dispatch
    of this workload's activations, and the exchange between GPUs in its
    fused form with EP_RANKS ranks emulated on this GPU (both owners'
    buffers here; every rank routes this step's tokens, and rank 0's layout,
    dispatch and combine are timed).  Returns name -> call."""
    import torch
    moe = step.moe
    meta = step.prepare()
    S, E = w.S, w.E
    max_tiles = max(1, -(-S // NEXT_TILE) + min(E, S))
    calls = {
        "tile_layout_t128": lambda: moe.moe_tile_layout(meta, w.k, NEXT_TILE, max_tiles),
        "problem_sizes": lambda: moe.moe_problem_sizes(meta.expert_counts, 2 * w.H, w.H, w.H, w.H),
    }
    if step.x.dtype in (torch.bfloat16, torch.float16) and w.H % 16 == 0:
        bso = (meta.blockscale_offsets if meta.blockscale_offsets is not None
               else meta.expert_offsets)
        A = step.A or 1
        q = torch.empty((S, w.H // 2), dtype=torch.uint8, device=dev)
        sc = torch.empty((S + E * (A - 1), w.H // 16), dtype=torch.uint8, device=dev)
        calls["dispatch_nvfp4"] = lambda: moe.moe_dispatch_rows_nvfp4(
            step.x, w.k, meta.output_permutation, meta.expert_offsets, bso, out_q=q,
            out_scales=sc)
    if step.x.dtype in (torch.bfloat16, torch.float16) and E % EP_RANKS == 0:
        counts = torch.stack([meta.expert_counts] * EP_RANKS).contiguous()
        lay = moe.moe_ep_peer_layout(counts, 0, step.ids, meta)
        rows = lay.recv_rows.tolist()
        bufs = [torch.empty((max(n, 1), w.H), dtype=step.x.dtype, device=dev) for n in rows]
        step.ep_buffers = bufs  # alive as long as the step (the table refers to them too)
        table = moe.moe_ep_buffer_table(bufs, dev)
        calls["ep_peer_layout_r2"] = lambda: moe.moe_ep_peer_layout(counts, 0, step.ids, meta)
        calls["ep_dispatch_peer_r2"] = lambda: moe.moe_ep_dispatch_peer(step.x, w.k, lay, table)
        calls["ep_combine_peer_r2"] = lambda: moe.moe_ep_combine_peer(
            table, step.x.dtype, w.H, lay, step.wt, out=step.out)
    return calls


def time_next_rows(step, w, dev, reps=20):
    """Each call of next_row_calls timed as a CUDA graph of `reps` calls."""
    import torch

    def timed(fn):
        fn()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for _ in range(reps):
                    fn()
        torch.cuda.synchronize(dev)
        g.replay()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        g.replay()
        e.record()
        torch.cuda.synchronize(dev)
        return s.elapsed_time(e) / reps * 1e3

    nbytes = next_row_bytes(w)
    out = {}
    for name, fn in next_row_calls(step, w, dev).items():
        us = timed(fn)
        out[name] = {"us": us, "algorithmic_bytes": nbytes[name]}
        if name not in ("problem_sizes", "ep_peer_layout_r2"):
            out[name]["effective_gbs"] = nbytes[name] / us / 1e3
    return out


def run_e2e(step, w, dev, K, W, barrier, max_over_ranks):
    """Same step through the public API with inputs copied in from pinned
    host memory and the combined output read back, every step, all inside
    the timed region.  Two forms:

    * pipelined (the value): the copies run on their own streams with two
      sets of device buffers and two pinned outputs, so that step i+1's
      inputs cross the host link while step i computes and step i-1's output
      is read back (the way a serving loop streams batches);
    * serialized: one stream, copy in, compute, copy out, step after step.

    After the timed region one read-back output of each form is checked
    against the device result of the same inputs."""
    import copy as _copy
    import torch
    h_ids = torch.from_numpy(step.ids_np).pin_memory()
    h_wt = torch.from_numpy(step.wt_np).pin_memory()
    h_x = step.x.cpu().pin_memory()
    h_y = step.y.cpu().pin_memory()
    h_out = [torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in (h_ids, h_wt, h_x, h_y))
    d2h = h_out[0].numel() * h_out[0].element_size()
    comp = torch.cuda.current_stream(dev)
    n = max(1, min(K, 20))

    # a second set of input / output buffers; the metadata, workspace and
    # dispatched rows are shared, since the computes run in order on one stream
    other = _copy.copy(step)
    for name in ("ids", "wt", "x", "y", "out"):
        setattr(other, name, torch.empty_like(getattr(step, name)))
    bufs = (step, other)
    copy_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h2d_done = [torch.cuda.Event(), torch.cuda.Event()]
    comp_done = [torch.cuda.Event(), torch.cuda.Event()]
    d2h_done = [torch.cuda.Event(), torch.cuda.Event()]

    def load(st, s):
        with torch.cuda.stream(s):
            st.ids.copy_(h_ids, non_blocking=True)
            st.wt.copy_(h_wt, non_blocking=True)
            st.x.copy_(h_x, non_blocking=True)
            st.y.copy_(h_y, non_blocking=True)

    def pipelined(count):
        for i in range(count):
            b = i % 2
            st = bufs[b]
            with torch.cuda.stream(copy_s):
                if i >= 2:
                    copy_s.wait_event(comp_done[b])  # step i-2 has read these inputs
            load(st, copy_s)
            h2d_done[b].record(copy_s)
            comp.wait_event(h2d_done[b])
            if i >= 2:
                comp.wait_event(d2h_done[b])  # step i-2's output has been read back
            st.run()
            comp_done[b].record(comp)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(comp_done[b])
                h_out[b].copy_(st.out, non_blocking=True)
                d2h_done[b].record(d2h_s)

    def serialized(count):
        for _ in range(count):
            load(step, comp)
            step.run()
            h_out[0].copy_(step.out, non_blocking=True)

    def timed(fn, first, last):
        fn(min(W, 3))
        torch.cuda.synchronize(dev)
        barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(first)
        fn(n)
        e.record(last)
        torch.cuda.synchronize(dev)
        barrier()
        return max_over_ranks(s.elapsed_time(e))

    ms_pipe = timed(pipelined, copy_s, d2h_s)
    ok_pipe = bool(torch.equal(h_out[(n - 1) % 2], bufs[(n - 1) % 2].out.cpu()))
    ms_ser = timed(serialized, comp, comp)
    ok_ser = bool(torch.equal(h_out[0], step.out.cpu()))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    return {"value": w.T * n * world / (ms_pipe * 1e-3), "unit": "tokens/s", "steps": n,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "copies": "own streams, double-buffered, overlapping the compute",
            "serialized": {"value": w.T * n * world / (ms_ser * 1e-3), "unit": "tokens/s",
                           "copies": "one stream: copy in, compute, copy out"},
            "read_back_matches_device": ok_pipe and ok_ser}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="all", choices=["all"] + sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of oracle time per workload (headline); half that for the others")
    ap.add_argument("--ref-budget", type=float, default=90.0,
                    help="seconds of oracle time for the whole reference run")
    ap.add_argument("--tokens", type=int, default=None,
                    help="run the workload's routing, shapes and dtypes at this many tokens "
                         "(smaller cases for profiling)")
    ap.add_argument("--profile-run", action="store_true",
                    help="only the warm-up and K eager steps of each workload, no JSON line "
                         "(a short program for ncu)")
    ap.add_argument("--profile-next", action="store_true",
                    help="like --profile-run, for the calls timed beside the path (tile layout, "
                         "problem sizes, NVFP4 dispatch)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.workload == "all":
        names = [HEADLINE_WORKLOAD] + [n for n in CONFIGS if n != HEADLINE_WORKLOAD]
    else:
        names = [args.workload]
    workloads = {n: CONFIGS[n] if args.tokens is None else CONFIGS[n].scaled(args.tokens)
                 for n in names}
    if args.impl == "reference":
        run_reference(args, workloads[names[0]])
    elif args.profile_run or args.profile_next:
        profile_run(args, [workloads[n] for n in names], next_rows=args.profile_next)
    else:
        run_gpu(args, names, workloads)


if __name__ == "__main__":
    main()
