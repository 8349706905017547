"""Benchmark of the DSA decode layer (lightning indexer -> top-k + page map -> MLA
sparse decode) on one B200, or N independent replicas under torchrun.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload cfg2] [--impl ours|reference]
    python bench.py --workload cfg3 --token-shards R [--gpus R]

Prints one JSON line (rank 0). A step is one dsa_decode_layer call over the whole
batch of the workload, with inputs resident in HBM. Workloads larger than L2 are timed
as back-to-back steps; smaller ones, and the stages timed alone, get an L2 flush before
every call, outside the timed intervals. --token-shards R times the token-sharded step
instead: every row's tokens over R ranks, with two all-gathers (strong scaling); on one
GPU the R ranks run in lockstep in one process.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import dsa_inputs  # noqa: E402

METRIC = "DSA decode layer-calls/s and achieved HBM TB/s (indexer+top-k+MLA)"
UNIT = "layer-calls/s"
L2_BYTES = 126 * 1024 * 1024


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default="cfg2", choices=sorted(dsa_inputs.CONFIGS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying a CUDA graph")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=200)
    p.add_argument("--token-shards", type=int, default=0,
                   help="R > 0: the token-sharded step, every row's tokens over R ranks (under torchrun R must "
                        "equal the number of ranks; on one GPU the R ranks run in lockstep in this process)")
    return p.parse_args()


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(args, backend=None):
    """One process per GPU (torchrun env). By default the path shards by rows with no
    data-path collective: every rank runs its own replica of the workload, and the process
    group only carries the barriers and the max-over-ranks timing. With --token-shards the
    group also carries the token-sharded step's two all-gathers. NCCL on GPUs; gloo when
    asked for (the CPU tests) or when no GPU is present."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, steps: int, ms_max: float) -> float:
    """Layer-calls per second over all replicas, timed by the slowest rank."""
    return world * steps / (ms_max / 1e3)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ our arm

def file_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "indexer": ["deepseek_sparse_attention_head_b200/csrc/indexer.cu",
                "deepseek_sparse_attention_head_b200/csrc/common.cuh"],
    "mla": ["deepseek_sparse_attention_head_b200/csrc/mla.cu",
            "deepseek_sparse_attention_head_b200/csrc/common.cuh"],
}


def measured_peaks():
    """(HBM GB/s, bf16 dense TFLOP/s burst, 'measured' | 'fallback')."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


FP8_OVER_BF16 = 2.0     # nominal dense tensor-core ratio on B200 (4.5 vs 2.25 PFLOP/s)


def measure_fp8_peak(stream, n=8192, reps=30):
    """Dense e4m3 tensor-core throughput of this GPU, measured like the bf16 entry of
    MEASURED_PEAKS.json: a large library GEMM (torch._scaled_mm, e4m3 x e4m3 -> bf16,
    n x n x n, per-tensor scales) timed as a burst of back-to-back calls with CUDA events.
    Returns (TFLOP/s, description) or (None, reason)."""
    try:
        a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
        one = torch.ones((), device="cuda")
        with torch.cuda.stream(stream):
            for _ in range(5):
                torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record(stream)
        e1.synchronize()
        ms = e0.elapsed_time(e1) / reps
        del a, b
        return 2.0 * n ** 3 / (ms / 1e3) / 1e12, f"torch._scaled_mm e4m3 {n}^3 -> bf16, burst of {reps}, CUDA events"
    except Exception as exc:  # noqa: BLE001 - reported in the JSON line, not fatal
        return None, f"fp8 GEMM unavailable: {type(exc).__name__}"


def committed_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from its committed ncu summary, or None when the
    summary is absent, was taken on different kernel sources, or on another workload."""
    try:
        with open(os.path.join(ROOT, "profiles", f"{kernel}_traffic.json")) as f:
            d = json.load(f)
        if d.get("sources_sha") != file_hash(KERNEL_SOURCES[kernel]):
            return None
        if not d.get("workload", "").startswith(workload + ":"):
            return None
        return d
    except (OSError, ValueError):
        return None


def timed_back_to_back(call, reps, stream):
    """Device time in ms of `reps` back-to-back calls of `call` on `stream`."""
    with torch.cuda.stream(stream):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            call()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1)


def timed_flushed(call, reps, stream, flush):
    """Device time in ms of `reps` calls of `call` on `stream`, each timed alone after an L2
    flush (`flush.zero_()`, a buffer larger than L2, outside the timed intervals)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            call()
            b.record(stream)
    evs[-1][1].synchronize()
    return sum(a.elapsed_time(b) for a, b in evs)


def time_stage(call, reps, nbytes, stream, flush):
    """Mean device ms of one `call` after 5 warm-up calls, and how it was timed: back to
    back when one call reads more than L2 holds, else each call alone after an L2 flush."""
    with torch.cuda.stream(stream):
        for _ in range(5):
            call()
    if nbytes > L2_BYTES:
        return (timed_back_to_back(call, reps, stream) / reps,
                f"the call alone, back to back (it reads {nbytes / 1e6:.0f} MB > L2), mean of {reps}")
    return (timed_flushed(call, reps, stream, flush) / reps,
            f"the call alone, L2 flushed before each ({nbytes / 1e6:.1f} MB < L2), mean of {reps}")


def e2e_serial(dsa, case, t, in_keys, pin, out, lse, ws, stream, flush, n, use_graph, world):
    """Device ms of n steps, each copy-in, layer call and copy-out in turn on one stream and
    timed alone after an L2 flush (for workloads that fit in L2). Inputs and outputs cross
    the host link as one packed copy each way (see Packed)."""
    hin = Packed({k: t[k] for k in in_keys}, pinned=True)
    for k in in_keys:
        hin.views[k].copy_(pin[k])
    hout = Packed({"out": out, "lse": lse}, pinned=True)
    din = Packed({k: t[k] for k in in_keys}, device="cuda")
    dout = Packed({"out": out, "lse": lse}, device="cuda")
    dev = din.views
    pg = dsa.Paging(dev["seq_lens"], dev["block_table"], case["num_pages"], case["n_q"], t["q_pos"])

    def body():
        din.buf.copy_(hin.buf, non_blocking=True)
        dsa.dsa_decode_layer(pg, dev["q_idx"], dev.get("q_idx_scale"), dev["head_w"], t["k_cache"], t["k_scale"],
                             dev["q_mla"], t["kv_cache"], t["kv_scale"], case["top_k"], case["softmax_scale"],
                             dout.views["out"], ws, lse=dout.views["lse"], stream=stream)
        hout.buf.copy_(dout.buf, non_blocking=True)

    g = None
    if use_graph:
        with torch.cuda.stream(stream):
            body()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            body()
        stream.synchronize()
    call = g.replay if g is not None else body
    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
    barrier(world)
    torch.cuda.synchronize()
    ms = timed_flushed(call, n, stream, flush)
    torch.cuda.synchronize()
    del g
    how = ("serial steps from one CUDA graph each (one packed copy each way included), L2 flushed before each"
           if use_graph else "serial eager steps (one packed copy each way included), L2 flushed before each")
    return ms, how


class Packed:
    """Tensors laid out back to back (each at a 256-byte boundary) in one buffer, so that a
    step's inputs, or its outputs, cross the host link as one copy: a few-MB copy reaches
    the link's rate where several smaller ones each pay a fixed cost. `views[k]` is a
    contiguous tensor of tensor k's dtype and shape inside the buffer."""

    def __init__(self, like: dict, device=None, pinned=False):
        spans, off = {}, 0
        for k, v in like.items():
            nb = v.numel() * v.element_size()
            spans[k] = (off, nb)
            off += (nb + 255) // 256 * 256
        self.buf = torch.empty(off, dtype=torch.uint8, device=device, pin_memory=pinned)
        self.views = {k: self.buf[o:o + nb].view(like[k].dtype).view(like[k].shape) for k, (o, nb) in spans.items()}
        self.nbytes = off


def e2e_pipelined(dsa, case, t, in_keys, pin, out, lse, ws, stream, n, use_graph, world):
    """Device ms from the first copy-in to the last copy-out of n steps over two buffer sets,
    as a serving loop overlaps them: while step k computes on set k % 2, step k+1's inputs
    are copied into the other set (its own stream) and step k-1's output and lse are copied
    out of it (a third stream). One pipeline stage (copy-in, layer, copy-out, forked and
    joined) is one CUDA graph per set parity. The first stage's copy-out and the last
    stage's copy-in move bytes no step uses: n + 1 copies each way for n steps."""
    K = case["top_k"]
    # one pinned host buffer holds a step's inputs and one its outputs; every set of device
    # buffers is packed the same way, so each direction is one copy per step
    hin = Packed({k: t[k] for k in in_keys}, pinned=True)
    for k in in_keys:
        hin.views[k].copy_(pin[k])
    hout = Packed({"out": out, "lse": lse}, pinned=True)
    sets, packs = [], []
    for si in range(2):
        din = Packed({k: t[k] for k in in_keys}, device="cuda")
        din.buf.copy_(hin.buf)
        dout = Packed({"out": out, "lse": lse}, device="cuda")
        dev = din.views
        pg = dsa.Paging(dev["seq_lens"], dev["block_table"], case["num_pages"], case["n_q"], t["q_pos"])
        sets.append((dev, pg, dout.views["out"], dout.views["lse"]))
        packs.append((din, dout))
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()

    def copy_in(si):
        with torch.cuda.stream(cin):
            packs[si][0].buf.copy_(hin.buf, non_blocking=True)

    def copy_out(si):
        with torch.cuda.stream(cout):
            hout.buf.copy_(packs[si][1].buf, non_blocking=True)

    def stage(si):
        """Step on set si; the other set's inputs in and outputs out meanwhile."""
        other = 1 - si
        fork = torch.cuda.Event()
        fork.record(stream)
        cin.wait_event(fork)
        cout.wait_event(fork)
        copy_in(other)
        copy_out(other)
        dev, pg, o, l = sets[si]
        with torch.cuda.stream(stream):
            dsa.dsa_decode_layer(pg, dev["q_idx"], dev.get("q_idx_scale"), dev["head_w"], t["k_cache"], t["k_scale"],
                                 dev["q_mla"], t["kv_cache"], t["kv_scale"], K, case["softmax_scale"], o, ws, lse=l,
                                 stream=stream)
        j_in, j_out = torch.cuda.Event(), torch.cuda.Event()
        j_in.record(cin)
        j_out.record(cout)
        stream.wait_event(j_in)
        stream.wait_event(j_out)

    graphs = [None, None]
    if use_graph:
        for si in range(2):
            stage(si)
            torch.cuda.synchronize()
            graphs[si] = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graphs[si], stream=stream):
                stage(si)
            torch.cuda.synchronize()

    def run(count):
        copy_in(0)
        ready = torch.cuda.Event()
        ready.record(cin)
        stream.wait_event(ready)
        for k in range(count):
            with torch.cuda.stream(stream):
                if graphs[k % 2] is not None:
                    graphs[k % 2].replay()
                else:
                    stage(k % 2)
        last = torch.cuda.Event()
        last.record(stream)
        cout.wait_event(last)
        copy_out((count - 1) % 2)

    run(4)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cin)
    run(n)
    e1.record(cout)
    e1.synchronize()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del graphs
    how = ("pipelined over two buffer sets: copy-in of the next step and copy-out of the previous one overlap "
           "each step, one packed copy each way per step, " +
           ("one CUDA graph per stage" if use_graph else "eager launches"))
    return ms, how


def run_ours(args, world, rank, local):
    import deepseek_sparse_attention_head_b200 as dsa

    case = dsa_inputs.generate(dsa_inputs.spec(args.workload))
    nbytes = dsa_inputs.algorithmic_bytes(case)
    t = dsa_inputs.to_torch(case, "cuda")
    paging = dsa.Paging(t["seq_lens"], t["block_table"], case["num_pages"], case["n_q"], t["q_pos"])
    Bq, K = case["Bq"], case["top_k"]
    out_dt = torch.float32 if case["out_dtype"] == "fp32" else torch.bfloat16
    out = torch.empty(Bq, 64, 512, dtype=out_dt, device="cuda")
    lse = torch.empty(Bq, 64, dtype=torch.float32, device="cuda")
    ws = dsa.alloc_workspace(dsa.dsa_workspace_size(paging, 0, K, dsa.DSA_OP_LAYER))
    stream = torch.cuda.Stream()

    def step():
        dsa.dsa_decode_layer(paging, t["q_idx"], t["q_idx_scale"], t["head_w"], t["k_cache"], t["k_scale"],
                             t["q_mla"], t["kv_cache"], t["kv_scale"], K, case["softmax_scale"], out, ws, lse=lse,
                             stream=stream)

    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    launches_per_step = dsa.dsa_last_launch_count()
    err = dsa.dsa_get_error(ws, stream)
    if err != 0:
        raise RuntimeError(f"device error {err} in the warm-up call")

    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        stream.synchronize()

    def run(n):
        for _ in range(n):
            if graph is not None:
                graph.replay()
            else:
                step()

    with torch.cuda.stream(stream):
        run(max(3, args.warmup))
    stream.synchronize()

    # Inputs larger than L2 are timed as back-to-back steps; smaller ones get an L2 flush
    # (a 256 MiB write) before every step, outside the timed intervals.
    inputs_exceed_l2 = nbytes["total"] > L2_BYTES
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    if inputs_exceed_l2:
        ms = timed_back_to_back(lambda: run(1), args.steps, stream)
    else:
        ms = timed_flushed(lambda: run(1), args.steps, stream, flush)
    clk = clocks.stop()
    torch.cuda.synchronize()
    barrier(world)
    ms_max = max_over_ranks(ms, world)
    err = dsa.dsa_get_error(ws, stream)
    if err != 0:
        raise RuntimeError(f"device error {err} during the timed region")

    # ---- dominant kernel (indexer stage) timed alone, same stream, same inputs
    scores = torch.empty(Bq, paging.L_layer, dtype=torch.float32, device="cuda")
    ws_i = dsa.alloc_workspace(dsa.dsa_workspace_size(paging, paging.L_layer, 0, dsa.DSA_OP_INDEXER))
    reps = max(20, min(2000, args.steps // 5))

    def idx_call():
        dsa.dsa_indexer_scores(paging, t["q_idx"], t["q_idx_scale"], t["head_w"], t["k_cache"], t["k_scale"],
                               scores, ws_i, stream=stream)

    idx_ms, idx_how = time_stage(idx_call, reps, nbytes["indexer"], stream, flush)

    # ---- MLA stage timed alone on the selection a layer call made (decode + combine kernels)
    phys = torch.empty(Bq, K, dtype=torch.int32, device="cuda")
    with torch.cuda.stream(stream):
        dsa.dsa_decode_layer(paging, t["q_idx"], t["q_idx_scale"], t["head_w"], t["k_cache"], t["k_scale"],
                             t["q_mla"], t["kv_cache"], t["kv_scale"], K, case["softmax_scale"], out, ws, lse=lse,
                             physical_out=phys, stream=stream)
    ws_m = dsa.alloc_workspace(dsa.mla_workspace_size(Bq, K))

    def mla_call():
        dsa.mla_sparse_decode(t["q_mla"], t["kv_cache"], t["kv_scale"], phys, case["softmax_scale"], out, lse, ws_m,
                              stream=stream)

    # the MLA call's bytes: selected latent rows, bf16 queries and the output
    out_b = 4 if case["out_dtype"] == "fp32" else 2
    mla_bytes = nbytes["mla"] + Bq * (2 * 64 * 576 + out_b * 64 * 512)
    mla_ms, mla_how = time_stage(mla_call, reps, mla_bytes, stream, flush)
    if dsa.dsa_get_error(ws_m, stream) != 0:
        raise RuntimeError("device error in the MLA timing calls")

    # ---- end to end through the public API with host buffers: every step copies its
    # query-side inputs in from pinned host memory and its output and lse back out
    in_keys = [k for k in ("q_idx", "q_idx_scale", "head_w", "q_mla", "seq_lens", "block_table") if t[k] is not None]
    pin = {k: t[k].cpu().pin_memory() for k in in_keys}
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
    n_e2e = max(10, args.e2e_steps)
    if inputs_exceed_l2:
        e2e_local, e2e_how = e2e_pipelined(dsa, case, t, in_keys, pin, out, lse, ws, stream, n_e2e,
                                           graph is not None, world)
    else:
        e2e_local, e2e_how = e2e_serial(dsa, case, t, in_keys, pin, out, lse, ws, stream, flush, n_e2e,
                                        graph is not None, world)
    e2e_ms = max_over_ranks(e2e_local, world)

    hbm_peak, bf16_peak, peak_kind = measured_peaks()
    calls_per_s = whole_job_rate(world, args.steps, ms_max)

    def roofline_of(name, call, ms, nb, flops, flop_peak, flop_kind, how):
        """Bound = whichever of HBM bytes and tensor FLOPs gives the longer ideal time."""
        t_hbm = nb / (hbm_peak * 1e9)
        t_tc = flops / (flop_peak * 1e12)
        if t_tc > t_hbm:
            ach = flops / (ms / 1e3) / 1e12
            r = {"bound": "tensor", "achieved": ach, "peak": flop_peak, "peak_kind": flop_kind, "unit": "TFLOP/s",
                 "frac": ach / flop_peak, "traffic": None, "algorithmic_flops": flops}
        else:
            ach = nb / (ms / 1e3) / 1e9
            tr = committed_traffic(name, args.workload)
            r = {"bound": "hbm", "achieved": ach, "peak": hbm_peak,
                 "peak_kind": f"{peak_kind} hbm_gbs (burst copy)", "unit": "GB/s", "frac": ach / hbm_peak,
                 "traffic": None if tr is None else tr["bytes_per_launch"], "algorithmic_bytes": nb}
        r["kernel"] = call
        r["duration_us"] = ms * 1e3
        r["timing"] = how
        return r

    # indexer: keys (+ scales, block table) and queries; fp8 x fp8 contraction
    idx_flops = dsa_inputs.indexer_flops(case)
    fp8 = case["idx_dtype"] != "bf16"
    fp8_peak, fp8_how = (None, "not measured (the indexer is HBM-bound here)")
    if fp8 and idx_flops / (bf16_peak * FP8_OVER_BF16 * 1e12) > nbytes["indexer"] / (hbm_peak * 1e9):
        fp8_peak, fp8_how = measure_fp8_peak(stream)    # tensor-bound (chunked prefill): measure it
    if fp8 and fp8_peak is not None:
        idx_peak, idx_kind = fp8_peak, f"measured fp8 peak ({fp8_how})"
    else:
        idx_peak = bf16_peak * (FP8_OVER_BF16 if fp8 else 1.0)
        idx_kind = (f"{peak_kind} bf16_tflops (burst) x {FP8_OVER_BF16:g} nominal fp8/bf16 ratio" if fp8
                    else f"{peak_kind} bf16_tflops (burst)")
    rf_idx = roofline_of("indexer", "indexer (dsa_indexer_scores call: plan + tcgen05 indexer)", idx_ms,
                         nbytes["indexer"], idx_flops, idx_peak, idx_kind, idx_how)
    # MLA: selected latent rows, bf16 queries and the output; QK (576) + PV (512) per selected row
    sel = int(np.minimum(dsa_inputs.vis_lengths(case), K).sum())
    mla_flops = 2 * sel * 64 * (576 + 512)
    rf_mla = roofline_of("mla", "mla (mla_sparse_decode call: tcgen05 MLA decode + split combine)", mla_ms,
                         mla_bytes, mla_flops, bf16_peak, f"{peak_kind} bf16_tflops (burst)", mla_how)
    # the dominant kernel is the one that takes longer
    roofline, other = (rf_mla, rf_idx) if mla_ms > idx_ms else (rf_idx, rf_mla)
    result = {
        "metric": METRIC,
        "value": calls_per_s,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": (f"{'bf16' if case['idx_dtype'] == 'bf16' else 'e4m3'} indexer + "
                  f"{'bf16' if case['kv_dtype'] == 'bf16' else 'f16 (e4m3 codes times fp16 row multipliers)'} MLA "
                  f"operands, fp32 accumulate"),
        "data": "synthetic (seeded; dsa_inputs)",
        "config": {
            "workload": f"{args.workload}: {dsa_inputs.WORKLOAD_NAMES[args.workload]}",
            "B": case["B"], "n_q": case["n_q"], "sum_L": int(case["seq_lens"].sum()), "top_k": K,
            "algorithmic_bytes_per_step": nbytes["total"],
            "l2": (f"inputs larger than L2 ({nbytes['total'] / 1e6:.0f} MB read per step > 126 MB)"
                   if inputs_exceed_l2 else
                   f"L2 flushed before every step ({nbytes['total'] / 1e6:.1f} MB read per step; 256 MiB "
                   f"write outside the timed intervals)"),
            "launch": "cuda_graph" if graph is not None else "eager",
            "parallelism": f"replicas x{world}",
        },
        "achieved_hbm_tbs": nbytes["total"] / (ms_max / args.steps / 1e3) / 1e12,
        "roofline": roofline,
        "roofline_other_kernel": other,
        "e2e": {"value": world * n_e2e / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": n_e2e, "launch": e2e_how},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if fp8_peak is not None:
        result["fp8_tensor_peak"] = {"tflops": fp8_peak, "how": fp8_how}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(case, budget_s=20.0)
    if graph is not None:
        del graph
    return result


def run_token_sharded(args, world, rank, local):
    """Token-sharded step: every row's tokens spread over R ranks, one exchange step.

    Under torchrun (world == R) each rank runs its share and the exchanges are NCCL
    all-gathers (eager launches). On one GPU the R ranks run in lockstep in this process,
    the exchanges become device copies into one gathered buffer, and the whole step is
    captured in a CUDA graph; each rank's phases are also timed alone, so that the
    critical path of R GPUs (slowest rank's local phase + slowest rank's select and
    attention + the merge, exchanges excluded) can be read beside the one-GPU rate.
    Strong scaling: the total work of a step is fixed."""
    import deepseek_sparse_attention_head_b200 as dsa
    from deepseek_sparse_attention_head_b200.sharded import TokenShardedDecode, shard_bounds

    R = args.token_shards
    if world > 1 and R != world:
        raise SystemExit("--token-shards must equal the number of ranks under torchrun")
    case = dsa_inputs.generate(dsa_inputs.spec(args.workload))
    if case["q_pos"] is not None:
        raise SystemExit("the token-sharded step takes workloads without causal positions")
    nbytes = dsa_inputs.algorithmic_bytes(case)
    t = dsa_inputs.to_torch(case, "cuda")
    B, Bq, K = case["B"], case["Bq"], case["top_k"]
    bounds = np.array([shard_bounds(int(L), R) for L in case["seq_lens"]], dtype=np.int64)
    mine = list(range(R)) if world == 1 else [rank]
    decs = {}
    for r in mine:
        lo, hi = bounds[:, r], bounds[:, r + 1]
        lens = (hi - lo).astype(np.int32)
        npg = (lens + 63) // 64
        lbt = np.full((B, max(1, int(npg.max()))), -1, dtype=np.int32)
        for b in range(B):
            lbt[b, :npg[b]] = case["block_table"][b, lo[b] // 64:lo[b] // 64 + npg[b]]
        paging = dsa.Paging(torch.from_numpy(lens).cuda(), torch.from_numpy(lbt).cuda(), case["num_pages"],
                            case["n_q"])
        decs[r] = TokenShardedDecode(paging, torch.from_numpy(lo.astype(np.int32)).cuda(), K, case["softmax_scale"],
                                     r, R)
    if world == 1:   # one gathered buffer shared by the emulated ranks
        for name in ("all_score", "all_token", "all_out", "all_lse"):
            buf = getattr(decs[0], name)
            for d in decs.values():
                setattr(d, name, buf)
    out_dt = torch.float32 if case["out_dtype"] == "fp32" else torch.bfloat16
    out = torch.empty(Bq, 64, 512, dtype=out_dt, device="cuda")
    lse = torch.empty(Bq, 64, dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()
    idx_in = (t["q_idx"], t["q_idx_scale"], t["head_w"], t["k_cache"], t["k_scale"])
    mla_in = (t["q_mla"], t["kv_cache"], t["kv_scale"])

    def step():
        if world > 1:
            decs[rank].step(*idx_in, *mla_in, out, lse)
            return
        for d in decs.values():
            d.local_phase(*idx_in)
        for r, d in decs.items():
            d.all_score[r].copy_(d.cand_score)
            d.all_token[r].copy_(d.cand_token)
        for d in decs.values():
            d.select_phase()
            d.attend_phase(*mla_in)
        for r, d in decs.items():
            d.all_out[r].copy_(d.state_out)
            d.all_lse[r].copy_(d.state_lse)
        decs[mine[0]].merge_phase(out, lse)   # every rank's merge is the same call

    # warm-up step, eager, counting this process's kernel launches per call
    launches = 0
    with torch.cuda.stream(stream):
        for d in decs.values():
            dsa.dsa_indexer_scores(d.paging, *idx_in, d.scores, d.ws_index)
            launches += dsa.dsa_last_launch_count()
            dsa.dsa_shard_local_topk(d.paging, d.scores, K, d.token_offset, d.cand_score, d.cand_token, d.ws_local)
            launches += dsa.dsa_last_launch_count()
        step()
        for d in decs.values():
            d.select_phase()
            launches += dsa.dsa_last_launch_count()
            d.attend_phase(*mla_in)
            launches += dsa.dsa_last_launch_count()
        decs[mine[0]].merge_phase(out, lse)
        launches += dsa.dsa_last_launch_count()
    stream.synchronize()
    for d in decs.values():
        for w in (d.ws_index, d.ws_local, d.ws_select, d.ws_mla):
            if dsa.dsa_get_error(w, stream) != 0:
                raise RuntimeError("device error in the warm-up step")

    graph = None
    if world == 1 and not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        stream.synchronize()

    def run(n):
        for _ in range(n):
            if graph is not None:
                graph.replay()
            else:
                step()

    with torch.cuda.stream(stream):
        run(max(3, args.warmup))
    stream.synchronize()
    inputs_exceed_l2 = nbytes["total"] > L2_BYTES
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    if inputs_exceed_l2:
        ms = timed_back_to_back(lambda: run(1), args.steps, stream)
    else:
        ms = timed_flushed(lambda: run(1), args.steps, stream, flush)
    clk = clocks.stop()
    torch.cuda.synchronize()
    barrier(world)
    ms_max = max_over_ranks(ms, world)

    per_rank = None
    if world == 1:
        # each emulated rank's phases timed alone: 20 calls of the phase captured in one CUDA
        # graph, replayed a few times on the same stream (device time: a graph per call would
        # time the host's replay rate for phases of a few microseconds)
        per_graph, reps = 20, 5

        def graph_ms(fn):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(per_graph):
                    fn()
            stream.synchronize()
            with torch.cuda.stream(stream):
                g.replay()
            ms_ = timed_back_to_back(g.replay, reps, stream) / (reps * per_graph)
            del g
            return ms_

        per_rank = []
        for d in decs.values():
            t_idx = graph_ms(lambda: dsa.dsa_indexer_scores(d.paging, *idx_in, d.scores, d.ws_index))
            t_topk = graph_ms(lambda: dsa.dsa_shard_local_topk(d.paging, d.scores, K, d.token_offset, d.cand_score,
                                                               d.cand_token, d.ws_local))
            t_sel = graph_ms(d.select_phase)
            t_att = graph_ms(lambda: d.attend_phase(*mla_in))
            per_rank.append({"rank": d.rank, "indexer_ms": t_idx, "local_topk_ms": t_topk, "select_ms": t_sel,
                             "attend_ms": t_att, "local_ms": t_idx + t_topk, "select_attend_ms": t_sel + t_att})
        t_merge = graph_ms(lambda: decs[mine[0]].merge_phase(out, lse))
        crit = (max(p["local_ms"] for p in per_rank) + max(p["select_attend_ms"] for p in per_rank) + t_merge)
    result = {
        "metric": METRIC,
        "value": 1e3 * args.steps / ms_max,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "e4m3 indexer + f16 MLA operands, fp32 accumulate" if case["idx_dtype"] != "bf16" else "bf16",
        "data": "synthetic (seeded; dsa_inputs)",
        "config": {
            "workload": f"{args.workload}: {dsa_inputs.WORKLOAD_NAMES[args.workload]}, token-sharded over {R} ranks",
            "B": B, "n_q": case["n_q"], "sum_L": int(case["seq_lens"].sum()), "top_k": K,
            "parallelism": (f"token shards x{R} (NCCL all-gathers)" if world > 1 else
                            f"token shards x{R} emulated on one GPU (exchanges as device copies)"),
            "launch": "cuda_graph" if graph is not None else "eager",
            "l2": "inputs larger than L2" if inputs_exceed_l2 else "L2 flushed before every step",
            "shard_bounds": bounds.tolist(),
        },
        "exchange_bytes_per_rank": {"candidates": Bq * K * 8, "states": Bq * 64 * (512 + 1) * 4},
        "gpu_launches": launches * args.steps,
        "clocks": clk,
        "roofline": None,
        "e2e": None,
    }
    if per_rank is not None:
        result["per_rank"] = per_rank
        result["merge_ms"] = t_merge
        result["critical_path_ms_excluding_exchanges"] = crit
    if graph is not None:
        del graph
    return result


# ------------------------------------------------------------------ oracle (CPU baseline / reference arm)

def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [int(i.get("num_threads", 1)) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def time_oracle_rows(case, rows, deadline=None):
    import oracle
    t0 = time.perf_counter()
    done = 0
    for r in rows:
        oracle.decode_layer(case, queries=[r])
        done += 1
        if deadline is not None and time.perf_counter() - t0 > deadline:
            break
    return time.perf_counter() - t0, done


def cpu_baseline(case, budget_s=20.0):
    """The oracle as it stands on this host's cores, on whole query rows of the workload
    until about budget_s of CPU work; scaled to layer-calls/s by the row count. A second,
    shorter sample runs the same oracle on one core (BLAS limited to one thread)."""
    rows = list(range(case["Bq"]))
    dt, done = time_oracle_rows(case, rows, deadline=budget_s)
    per_row = dt / done
    res = {"value": 1.0 / (per_row * case["Bq"]), "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
           "sample": f"{done} of {case['Bq']} query rows (full indexer+top-k+MLA per row), {dt:.1f} s"}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            dt1, done1 = time_oracle_rows(case, rows[:max(1, done // 4)], deadline=budget_s / 2)
        res["single_core"] = {"value": 1.0 / (dt1 / done1 * case["Bq"]), "unit": UNIT, "cores": 1,
                              "sample": f"{done1} query rows, {dt1:.1f} s"}
    except ImportError:
        pass
    return res


def run_reference(args, world, rank):
    """Reference arm: the fp64 oracle on the host cores, same workload and unit. Each step
    processes one whole query row (rows cycle through the batch); at most ~150 s in total."""
    case = dsa_inputs.generate(dsa_inputs.spec(args.workload))
    Bq = case["Bq"]
    per_row, _ = time_oracle_rows(case, [0])
    budget = 150.0
    steps = args.steps
    warm = min(args.warmup, 3)
    n_fit = max(1, int(budget / max(per_row, 1e-3)) - warm)
    timed = min(steps, n_fit)
    time_oracle_rows(case, [i % Bq for i in range(warm)])
    dt, done = time_oracle_rows(case, [i % Bq for i in range(timed)])
    value = done / Bq / dt
    return {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": dt / done * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded; dsa_inputs)",
        "config": {"workload": f"{args.workload}: {dsa_inputs.WORKLOAD_NAMES[args.workload]}",
                   "B": case["B"], "n_q": case["n_q"], "top_k": case["top_k"]},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"{done} whole query rows timed (of {steps} requested steps; one row per step, "
                                   f"rows cycle through the {Bq}-row batch)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, world, rank)), flush=True)
        return 0
    world, rank, local = dist_setup(args)
    res = run_token_sharded(args, world, rank, local) if args.token_shards > 0 else run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
