"""Benchmark of the SGA hot path on B200: decode at 128K context (batch 32).

One step = one pass of the whole path over one batch of queries: the indexer
over every cached position, top-2048 selection, sparse latent attention and the
head gate, as one sga_forward call (three kernel launches).  The timed region
is K such steps between CUDA events on the launching stream.  Each kernel is
then timed alone in its own event-timed loop of the matching C-ABI call
(sga_index_scores, sga_topk_select, sga_sparse_mla_attend) for the roofline of
the dominant kernel; an end-to-end region repeats the step with the query-side
inputs copied from pinned host memory and the results copied back; the E4M3
index-key variant is timed like the main region.

Under torchrun every rank is an independent replica with its own batch (weak
scaling); each timed region starts after a barrier and its time is the maximum
over ranks.  Prints one JSON line (rank 0).  `--impl reference` times the fp64
CPU oracle on the host cores instead (a bounded sample of the same workload).
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SGA decode queries/s at 128K ctx; achieved HBM GB/s vs 8 TB/s roofline"
UNIT = "queries/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, help="workload name (default: decode_b32_ctx128k)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", dest="prefill", action="store_false",
                    help="skip the chunked-prefill variant (4096 queries over a 128K cache)")
    ap.add_argument("--no-decode-variants", dest="decode_variants", action="store_false",
                    help="skip the other decode workloads (8K x 4, 32K x 64, 256K x 8 with ties)")
    ap.add_argument("--no-warmup-objective", dest="warmup_objective", action="store_false",
                    help="skip the indexer's sparse warm-up objective (a training-time variant)")
    ap.add_argument("--no-layer", dest="layer", action="store_false",
                    help="skip the whole-layer variant (the projections either side of the path)")
    ap.add_argument("--layer-only", action="store_true",
                    help="run only the whole-layer variant and print it (a profiling case)")
    ap.add_argument("--warmup-only", action="store_true",
                    help="run only the indexer's warm-up objective over the workload's own selection and print it "
                         "(a profiling case)")
    ap.add_argument("--fused-only", action="store_true",
                    help="run only the fused-selection variant (sga_forward_fused, bf16 and E4M3) and print it "
                         "(a profiling case)")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the chunked-prefill variant and print it (a profiling case)")
    ap.add_argument("--prefill-queries", type=int, default=0, help="prefill variant: new queries (default 4096)")
    ap.add_argument("--prefill-ctx", type=int, default=0, help="prefill variant: cache rows (default 131072)")
    ap.add_argument("--cpu-sample-queries", type=int, default=0, help="oracle sample size (0 = auto)")
    ap.add_argument("--batch", type=int, default=0, help="custom decode workload: sequences (with --ctx)")
    ap.add_argument("--ctx", type=int, default=0, help="custom decode workload: context length (with --batch)")
    return ap.parse_args()


def algorithmic_bytes_per_query(ctx: int, top_k: int = 2048, key_bytes: int = 2) -> dict:
    """Bytes the method must move per decode query (intermediate scores excluded).

    k_idx: every causal key once (ctx * 128 * key_bytes: 2 for bf16, 1 for E4M3),
    q_idx 64*128*key_bytes, w 64*2, gathered latent rows top_k * 576 * 2,
    q 64*576*2, gate 64*2, out 64*512*4, idx top_k * 4.
    """
    parts = dict(k_idx=ctx * 128 * key_bytes, q_idx=8192 * key_bytes, w=128, kv_rows=top_k * 1152, q=73728,
                 gate=128, out=131072, idx=top_k * 4)
    parts["total"] = sum(parts.values())
    parts["indexer"] = parts["k_idx"] + parts["q_idx"] + parts["w"]
    return parts


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s measured on this machine (burst: a kernel timed in isolation)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def causal_index_flops(positions) -> float:
    """Multiply-adds of the indexer over every causal key of each query, 2 flops each:
    2 * 64 heads * 128 dims * (t + 1) per query."""
    return float(2 * 64 * 128 * sum(int(t) + 1 for t in positions))


def kernel_counters(kernel_file: str):
    """ncu DRAM traffic per launch for the dominant kernel, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", "counters.json")
    src = os.path.join(ROOT, "sparse_gated_attention_b200", "csrc", kernel_file)
    try:
        with open(path) as f:
            d = json.load(f)
        entry = d[kernel_file]
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
        if entry.get("source_sha256") != sha:
            return None
        return entry
    except Exception:
        return None


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        if not getattr(self, "lines", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


_SAMPLE_CACHE = {}


def cpu_baseline(wl, n_queries: int = 0, min_seconds: float = 10.0, max_queries: int = 400):
    """The oracle, as it stands, on a bounded sample of the workload (host cores).

    n_queries > 0 runs exactly that many queries; otherwise queries are run
    until min_seconds of CPU time have passed (at most max_queries)."""
    import oracle
    from sparse_gated_attention_b200 import synth

    key = (wl.name, wl.ctx, wl.k_range)
    if key not in _SAMPLE_CACHE:
        sample = synth.custom(batch=1, n_q=1, ctx=wl.ctx, first_pos=wl.first_pos if wl.n_q == 1 else wl.ctx - 1,
                              k_range=wl.k_range, name=wl.name + "_sample")
        _SAMPLE_CACHE[key] = synth.make_inputs(sample, device="cpu", seed=0)
    x = _SAMPLE_CACHE[key]
    oracle.build()
    threads = oracle.hardware_threads()
    t0 = time.perf_counter()
    done = 0
    while True:
        oracle.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], n_threads=threads)
        done += 1
        dt = time.perf_counter() - t0
        if (n_queries > 0 and done >= n_queries) or (n_queries <= 0 and (dt >= min_seconds or done >= max_queries)):
            break
    n_queries = done
    return {"value": n_queries / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n_queries} decode queries of {wl.name} (1 sequence, ctx {wl.ctx}, full path, fp64)",
            "seconds": dt}


def run_reference(args, wl, rank):
    if rank != 0:
        return
    steps, warm = args.steps, args.warmup
    nq = args.cpu_sample_queries or 1
    for _ in range(warm):
        cpu_baseline(wl, nq)
    times = []
    vals = []
    for _ in range(steps):
        r = cpu_baseline(wl, nq)
        times.append(r["seconds"])
        vals.append(r)
    total = sum(times)
    value = steps * nq / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": steps,
        "warmup": warm, "ms_per_step": 1000.0 * total / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": vals[0]["cores"], "kind": "oracle",
                         "sample": vals[0]["sample"] + " per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def max_over_ranks(dist, device, ms: float) -> float:
    """The slowest rank's time for a timed region (every rank calls this in the same order)."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(rows_per_rank: int, steps: int, world: int, elapsed_ms: float) -> float:
    """Queries per second over all replicas: every rank decodes its own batch of rows_per_rank
    queries per step (weak scaling), timed by the slowest rank."""
    return rows_per_rank * steps * world / (elapsed_ms / 1e3)


class E2ESlot:
    """One of the two buffer sets of the pipelined end-to-end loop: device inputs
    and outputs, pinned host outputs, and the events that order their reuse."""

    def __init__(self, new_event, **buffers):
        self.__dict__.update(buffers)
        self.inputs_landed = new_event()   # host->device copy of this slot's inputs done
        self.computed = new_event()        # the path has read the inputs and written the outputs
        self.results_home = new_event()    # device->host copy of this slot's outputs done


def e2e_pipelined_step(i, slots, compute, h2d, d2h, issue):
    """Step i of a serving loop on slot i % 2.  Three streams overlap step i+1's
    input copy and step i-1's result copy with step i's kernels:
      h2d:     waits until the slot's previous step has computed (its inputs were read),
               then copies this step's inputs in;
      compute: waits for those inputs and for the slot's previous results to reach
               the host (its outputs are about to be overwritten), then runs the path;
      d2h:     waits for the path, then copies the results out.
    issue(kind, slot, stream) enqueues the work of one kind on a stream."""
    sl = slots[i % 2]
    h2d.wait_event(sl.computed)
    issue("h2d", sl, h2d)
    sl.inputs_landed.record(h2d)
    compute.wait_event(sl.inputs_landed)
    compute.wait_event(sl.results_home)
    issue("compute", sl, compute)
    sl.computed.record(compute)
    d2h.wait_event(sl.computed)
    issue("d2h", sl, d2h)
    sl.results_home.record(d2h)


def config_of(wl):
    return {"workload": wl.name, "batch": wl.batch, "queries_per_seq": wl.n_q, "ctx": wl.ctx, "top_k": wl.top_k,
            "heads": 64, "latent": 576, "index_heads": 64, "index_dim": 128,
            "l2": "inputs larger than L2 (k_idx+kv rows ~1.16 GB/step vs 126 MB L2), no flush",
            "parallelism": "replicas"}


def per_iteration_ms(fn, n, flush, warmup, dev, stream, dist):
    """CUDA-event times of n calls of fn on `stream`, each after an L2 flush (a
    memset of `flush`, outside its events), after `warmup` untimed calls."""
    for _ in range(max(warmup, 3)):
        fn()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
    torch.cuda.synchronize(dev)
    return [a.elapsed_time(b) for a, b in evs]


def decode_variant(sga, synth, name, args, dev, stream, dist, rank, peak) -> dict:
    """One sga_forward step of another decode workload, timed per iteration with
    L2 flushed (256 MB memset) before each; the median is reported."""
    wl = synth.WORKLOADS[name]
    x = synth.make_inputs(wl, device=dev, seed=rank)
    B, T, L, K = wl.batch, wl.n_q, wl.ctx, wl.top_k
    dims = sga.make_dims(B, T, L, K)
    ws = sga.alloc_workspace(dims, sga.OP_FORWARD, dev)
    idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    out = torch.empty((B, T, 64, 512), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def forward():
        sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], top_k=K, idx_out=idx,
                    out=out, ws=ws, stream=stream)

    n = max(5, min(args.steps, 20))
    ms = max_over_ranks(dist, dev, statistics.median(per_iteration_ms(forward, n, flush, args.warmup, dev, stream,
                                                                      dist)))
    if sga.device_status(ws) != 0:
        raise RuntimeError(f"device status set during the {name} variant")
    rows = B * T
    world = dist.get_world_size() if dist is not None else 1
    ab = algorithmic_bytes_per_query(L, K)
    gbs = ab["total"] * rows / (ms * 1e-3) / 1e9
    return {"value": rows * world / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
            "config": f"{name}: {B} sequences x {T} query at position {L - 1}, top_k {K}; median of {n} "
                      f"iterations, L2 flushed (256 MB memset) before each",
            "path_roofline": {"achieved_gbs": gbs, "frac_of_8tbs": gbs / NOMINAL_HBM_GBS,
                              "frac_of_measured": gbs / peak, "bytes_per_query": ab["total"]},
            "gpu_launches": 3}


def prefill_variant(sga, synth, args, dev, stream, dist, rank) -> dict:
    """Times sga_forward and the indexer alone on the chunked-prefill workload
    (4096 queries over a 128K cache unless --prefill-queries / --prefill-ctx say
    otherwise: the last queries of the context, one sequence)."""
    wl = synth.WORKLOADS["prefill_t4096_ctx128k"]
    if args.prefill_queries or args.prefill_ctx:
        T = args.prefill_queries or wl.n_q
        L = args.prefill_ctx or wl.ctx
        wl = synth.custom(batch=1, n_q=T, ctx=L, first_pos=L - T, name=f"prefill_t{T}_ctx{L // 1024}k")
    x = synth.make_inputs(wl, device=dev, seed=rank)
    B, T, L, K = wl.batch, wl.n_q, wl.ctx, wl.top_k
    dims = sga.make_dims(B, T, L, K)
    ws = sga.alloc_workspace(dims, sga.OP_FORWARD, dev)
    ws_i = sga.alloc_workspace(dims, sga.OP_INDEX_SCORES, dev)
    scores = torch.empty((B, T, L), dtype=torch.float32, device=dev)
    idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    out = torch.empty((B, T, 64, 512), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def forward():
        sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], top_k=K, idx_out=idx,
                    out=out, ws=ws, stream=stream)

    def indexer():
        sga.index_scores(x["q_idx"], x["w"], x["k_idx"], x["q_pos"], scores=scores, ws=ws_i, stream=stream)

    n = max(5, min(args.steps, 20))
    chunk_ms = max_over_ranks(dist, dev, statistics.median(per_iteration_ms(forward, n, flush, args.warmup, dev,
                                                                            stream, dist)))
    k1_ms = max_over_ranks(dist, dev, statistics.median(per_iteration_ms(indexer, n, flush, args.warmup, dev,
                                                                         stream, dist)))
    if sga.device_status(ws) != 0 or sga.device_status(ws_i) != 0:
        raise RuntimeError("device status set during the prefill variant")
    positions = x["q_pos"].flatten().tolist()
    flops = causal_index_flops(positions)
    peak_tf, peak_kind = measured_tensor_peak()
    world = dist.get_world_size() if dist is not None else 1
    k1_tf = flops / (k1_ms * 1e-3) / 1e12
    return {"name": wl.name, "value": B * T * world / (chunk_ms * 1e-3), "unit": "queries/s", "ms_per_chunk": chunk_ms,
            "config": f"{wl.name}: {T} new queries at positions {positions[0]}..{positions[-1]} over a "
                      f"{L}-row cache, top_k {K}; median of {n} iterations, L2 flushed (256 MB memset) before each",
            "indexer": {"ms": k1_ms, "tflops": k1_tf, "flops_per_launch": flops, "peak_tflops": peak_tf,
                        "peak_kind": peak_kind, "frac": k1_tf / peak_tf, "bound": "tensor"},
            "gpu_launches": 3}


def graph_replay_ms(make_step, args, dev, dist) -> float:
    """`args.steps` calls of a step captured in one CUDA graph and replayed, as a
    serving loop launches its decode steps.  make_step(stream) returns the step
    bound to a stream; its one-time set-up must have run before (outside the
    capture).  Untimed replays cover at least 3 warm-up steps, then one replay
    is timed between CUDA events on the capture stream (max over ranks)."""
    gs = torch.cuda.Stream(dev)
    gs.wait_stream(torch.cuda.current_stream(dev))
    step = make_step(gs)
    graph = torch.cuda.CUDAGraph()
    # thread-local capture: other threads' CUDA calls (a process group's watchdog) stay legal meanwhile
    with torch.cuda.graph(graph, stream=gs, capture_error_mode="thread_local"):
        for _ in range(args.steps):
            step()
    with torch.cuda.stream(gs):
        for _ in range(max(1, -(-3 // args.steps))):
            graph.replay()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(gs):
        a.record(gs)
        graph.replay()
        b.record(gs)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(dist, dev, a.elapsed_time(b))
    del graph
    return ms


def layer_variant(sga, synth, args, dev, stream, dist, rank, x, dims, idx) -> dict:
    """One whole SGA layer (a separate configuration): h -> projections -> the path
    -> W_UV, o_proj, on the workload's caches (the new tokens' rows are rewritten
    at their positions every step), timed over K steps like the main region."""
    B, T = x["q_pos"].shape
    K = dims.top_k
    lw_t = synth.make_layer_weights(device=dev, seed=rank)
    gl = torch.Generator(device=dev).manual_seed(rank + 99)
    h = torch.randn((B, T, synth.D_MODEL), generator=gl, device=dev).to(torch.bfloat16)
    ws_layer = sga.alloc_layer_workspace(dims, sga.layer_weights(lw_t), sga.LAYER_FORWARD, dev)
    y = torch.empty((B, T, synth.D_MODEL), dtype=torch.float32, device=dev)

    def layer_step(st=stream):
        sga.layer_forward(lw_t, h, x["q_pos"], x["kv"], x["k_idx"], top_k=K, idx_out=idx, y=y, ws=ws_layer,
                          stream=st)

    for _ in range(max(args.warmup, 3)):
        layer_step()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    s4, e4 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s4.record(stream)
    for _ in range(args.steps):
        layer_step()
    e4.record(stream)
    torch.cuda.synchronize(dev)
    layer_ms = max_over_ranks(dist, dev, s4.elapsed_time(e4))
    if sga.device_status(ws_layer) != 0:
        raise RuntimeError("device status set during the layer variant run")
    try:
        graph_ms = graph_replay_ms(lambda st: (lambda: layer_step(st)), args, dev, dist)
        if sga.device_status(ws_layer) != 0:
            raise RuntimeError("device status set during the layer's graph replay")
    except (RuntimeError, TypeError, ValueError) as exc:
        torch.cuda.synchronize(dev)
        graph_ms = f"{type(exc).__name__}: {exc}"
    weight_bytes = sum(t.numel() * t.element_size() for t in lw_t.values())
    return {"ms": layer_ms, "graph_ms": graph_ms, "weight_bytes": weight_bytes,
            "act_bytes": h.numel() * 2 + y.numel() * 4}


def fused_variant(sga, synth, args, wl, x, dev, stream, dist, xf=None, idx=None, out=None) -> dict:
    """The whole path through sga_forward_fused and sga_forward_fused_fp8 on `wl`, each timed like
    the main region (warm-up, then `args.steps` calls as one region, max over ranks); total ms."""
    B, T, L, K = wl.batch, wl.n_q, wl.ctx, wl.top_k
    dims = sga.make_dims(B, T, L, K)
    if xf is None:
        xf = {"q_idx": synth.to_e4m3(x["q_idx"]), "k_idx": synth.to_e4m3(x["k_idx"])}
    if idx is None:
        idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((B, T, 64, 512), dtype=torch.float32, device=dev)
    ws = sga.alloc_workspace(dims, sga.OP_FORWARD_FUSED, dev)
    steps = {
        "bf16": lambda: sga.forward_fused(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"],
                                          top_k=K, idx_out=idx, out=out, ws=ws, stream=stream),
        "fp8": lambda: sga.forward_fused_fp8(xf["q_idx"], x["w"], xf["k_idx"], x["q"], x["kv"], x["gate"],
                                             x["q_pos"], top_k=K, idx_out=idx, out=out, ws=ws, stream=stream),
    }
    res = {}
    for name, step in steps.items():
        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = max_over_ranks(dist, dev, a.elapsed_time(b))
        if sga.device_status(ws) != 0:
            raise RuntimeError(f"device status set during the fused-selection {name} run")
    del ws
    return res


def warmup_objective_variant(sga, args, dev, stream, dist, rank, x, dims, idx, peak) -> dict:
    """The indexer's sparse warm-up objective and its gradients (a training-time
    variant; sga_indexer_warmup) over the headline step's own selection, timed
    over K steps like the main region.  The key gradient is added to one
    [B][L][128] fp32 buffer every step, as an optimiser step would read it."""
    B, T = x["q_pos"].shape
    L, K = dims.kv_stride, dims.top_k
    ws = torch.zeros(sga.indexer_warmup_workspace_size(dims), dtype=torch.uint8, device=dev)
    gk = torch.zeros((B, L, 128), dtype=torch.float32, device=dev)

    def step():
        sga.indexer_warmup(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], idx, grad_k_idx=gk, ws=ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(args.steps):
        step()
    e0.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(dist, dev, s0.elapsed_time(e0))
    if sga.device_status(ws) != 0:
        raise RuntimeError("device status set during the warm-up objective variant")
    rows = B * T
    world = dist.get_world_size() if dist is not None else 1
    # per query: the selected latent and key rows, q, q_idx, w, idx, the q_idx / w
    # gradients and loss written, the key gradient rows read and written (the
    # workspace's per-slot logits and dots are intermediates, not counted)
    per_query = K * 1152 + K * 256 + 73728 + 16384 + 128 + K * 4 + 32768 + 256 + 4 + K * 128 * 4 * 2
    step_ms = ms / args.steps
    gbs = per_query * rows / (step_ms * 1e-3) / 1e9
    return {"value": whole_job_rate(rows, args.steps, world, ms), "unit": UNIT, "ms_per_step": step_ms,
            "config": f"{rows} queries of the headline workload: KL(attention target || indexer softmax) over each "
                      f"query's 2048 selected positions and the gradients of q_idx, w and k_idx (logits, indexer dots "
                      f"and gradient contractions on tcgen05, bf16 operands, fp32 accumulation)",
            "path_roofline": {"achieved_gbs": gbs, "frac_of_8tbs": gbs / NOMINAL_HBM_GBS, "frac_of_measured": gbs / peak,
                              "bytes_per_query": per_query},
            "gpu_launches": 4 * args.steps}


def main():
    args = parse_args()
    from sparse_gated_attention_b200 import synth

    if args.batch and args.ctx:
        wl = synth.custom(batch=args.batch, n_q=1, ctx=args.ctx, first_pos=args.ctx - 1,
                          name=f"decode_b{args.batch}_ctx{args.ctx // 1024}k")
    else:
        wl = synth.WORKLOADS[args.workload or synth.HEADLINE]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, wl, rank)
        return

    import sparse_gated_attention_b200 as sga

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    sga.load_library()
    if args.layer_only:
        wl_l = synth.WORKLOADS[args.workload or synth.HEADLINE]
        xl = synth.make_inputs(wl_l, device=dev, seed=rank)
        dl = sga.make_dims(wl_l.batch, wl_l.n_q, wl_l.ctx, wl_l.top_k)
        il = torch.empty((wl_l.batch, wl_l.n_q, wl_l.top_k), dtype=torch.int32, device=dev)
        res = layer_variant(sga, synth, args, dev, torch.cuda.current_stream(dev), dist, rank, xl, dl, il)
        if rank == 0:
            g = res["graph_ms"]
            print(json.dumps({"variant": "sga_layer", "ms_per_step": res["ms"] / args.steps,
                              "graph_replay_ms_per_step": g / args.steps if isinstance(g, float) else g,
                              "weight_bytes": res["weight_bytes"]}), flush=True)
        return
    if args.warmup_only:
        xo = synth.make_inputs(wl, device=dev, seed=rank)
        do = sga.make_dims(wl.batch, wl.n_q, wl.ctx, wl.top_k)
        io, _ = sga.forward(xo["q_idx"], xo["w"], xo["k_idx"], xo["q"], xo["kv"], xo["gate"], xo["q_pos"],
                            top_k=wl.top_k)
        res = warmup_objective_variant(sga, args, dev, torch.cuda.current_stream(dev), dist, rank, xo, do, io,
                                       measured_peaks()[0])
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"variant": "indexer_warmup", "workload": wl.name, "ms_per_step": res["ms_per_step"]}),
                  flush=True)
        return
    if args.fused_only:
        xo = synth.make_inputs(wl, device=dev, seed=rank)
        res = fused_variant(sga, synth, args, wl, xo, dev, torch.cuda.current_stream(dev), dist)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"variant": "fused_selection", "workload": wl.name,
                              "ms_per_step": {k: v / args.steps for k, v in res.items()}}), flush=True)
        return
    if args.prefill_only:
        res = prefill_variant(sga, synth, args, dev, torch.cuda.current_stream(dev), dist, rank)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"variant": res.pop("name"), **res}), flush=True)
        return

    x = synth.make_inputs(wl, device=dev, seed=rank)
    B, T, L, K = wl.batch, wl.n_q, wl.ctx, wl.top_k
    rows = B * T
    dims = sga.make_dims(B, T, L, K)
    ws_all = sga.alloc_workspace(dims, sga.OP_FORWARD, dev)
    ws_idx = sga.alloc_workspace(dims, sga.OP_INDEX_SCORES, dev)
    ws_topk = sga.alloc_workspace(dims, sga.OP_TOPK_SELECT, dev)
    ws_att = sga.alloc_workspace(dims, sga.OP_SPARSE_MLA_ATTEND, dev)
    scores = torch.empty((B, T, L), dtype=torch.float32, device=dev)
    idx = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    out = torch.empty((B, T, 64, 512), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 3  # indexer, top-k, attention (the attention's split merge needs no combine kernel)
    fused_ok = T < 8 and L <= 262144  # the rows sga_forward_fused selects from candidates

    def fwd_step():
        sga.forward(x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], top_k=K, idx_out=idx,
                    out=out, ws=ws_all, stream=stream)

    def timed(fn, n):
        """CUDA-event time of each of n calls of fn on the stream, after a synchronize."""
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        torch.cuda.synchronize(dev)
        for a, b in evs:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize(dev)
        return [a.elapsed_time(b) for a, b in evs]

    for _ in range(max(args.warmup, 3)):
        fwd_step()
    torch.cuda.synchronize(dev)
    if sga.device_status(ws_all) != 0:
        raise RuntimeError(f"device status {sga.device_status(ws_all)} after warm-up")

    # ---- the timed region: K whole-path steps through sga_forward
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        time.sleep(0.3)
        start.record(stream)
        for _ in range(args.steps):
            fwd_step()
        stop.record(stream)
        torch.cuda.synchronize(dev)
    elapsed_ms = max_over_ranks(dist, dev, start.elapsed_time(stop))
    if sga.device_status(ws_all) != 0:
        raise RuntimeError("device status set during the timed region")

    # ---- per-kernel launch durations (same kernels, one C-ABI call per launch)
    k1 = timed(lambda: sga.index_scores(x["q_idx"], x["w"], x["k_idx"], x["q_pos"], scores=scores, ws=ws_idx,
                                        stream=stream), args.steps)
    k2 = timed(lambda: sga.topk_select(scores, x["q_pos"], top_k=K, idx=idx, ws=ws_topk, stream=stream), args.steps)
    k3 = timed(lambda: sga.sparse_mla_attend(x["q"], x["kv"], idx, x["gate"], out=out, ws=ws_att, stream=stream),
               args.steps)

    # ---- end to end through sga_forward with host buffers (cache resident on the device): every
    # step copies its query-side inputs from pinned host memory and its results back to pinned
    # host memory inside the timed region.  Measured twice: as a serving loop that overlaps the
    # copies of neighbouring steps with the kernels (two buffer slots, a copy stream each way;
    # the reported value), and with all of a step's work in order on one stream.
    host = {k: x[k].cpu().pin_memory() for k in ("q_idx", "w", "q", "gate", "q_pos")}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out.numel() * 4 + idx.numel() * 4

    def new_slot():
        return E2ESlot(lambda: torch.cuda.Event(), inp={k: torch.empty_like(x[k]) for k in host},
                       out=torch.empty_like(out), idx=torch.empty_like(idx),
                       out_h=torch.empty(out.shape, dtype=torch.float32).pin_memory(),
                       idx_h=torch.empty(idx.shape, dtype=torch.int32).pin_memory())

    slots = [new_slot(), new_slot()]
    h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def issue(kind, sl, st):
        with torch.cuda.stream(st):
            if kind == "h2d":
                for k in host:
                    sl.inp[k].copy_(host[k], non_blocking=True)
            elif kind == "compute":
                sga.forward(sl.inp["q_idx"], sl.inp["w"], x["k_idx"], sl.inp["q"], x["kv"], sl.inp["gate"],
                            sl.inp["q_pos"], top_k=K, idx_out=sl.idx, out=sl.out, ws=ws_all, stream=st)
            else:
                sl.out_h.copy_(sl.out, non_blocking=True)
                sl.idx_h.copy_(sl.idx, non_blocking=True)

    def e2e_region(step_fn):
        for i in range(3):
            step_fn(i)
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        h2d_stream.wait_event(t0)  # no copy starts before the timed region
        d2h_stream.wait_event(t0)
        for i in range(args.steps):
            step_fn(i)
        for sl in slots:  # the region ends when the last results are on the host
            stream.wait_event(sl.results_home)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        return max_over_ranks(dist, dev, t0.elapsed_time(t1))

    def serial_step(i):
        sl = slots[0]
        for kind in ("h2d", "compute", "d2h"):
            issue(kind, sl, stream)
        sl.results_home.record(stream)

    e2e_serial_ms = e2e_region(serial_step)
    e2e_mode = "serving loop: step i+1's input copy and step i-1's result copy overlap step i's kernels"
    try:
        e2e_ms = e2e_region(lambda i: e2e_pipelined_step(i, slots, stream, h2d_stream, d2h_stream, issue))
    except (RuntimeError, TypeError, AttributeError, ValueError) as exc:  # keep the in-order number
        torch.cuda.synchronize(dev)
        e2e_ms = e2e_serial_ms
        e2e_mode = f"in order on one stream (the overlapped loop failed: {type(exc).__name__}: {exc})"
    if sga.device_status(ws_all) != 0:
        raise RuntimeError("device status set during the end-to-end run")

    # ---- the E4M3 indexer-key variant (a separate configuration, reported beside
    # the headline): the same workload with q_idx and k_idx stored as E4M3
    # (exact for the integer-valued inputs), timed like the main region.
    xf = {"q_idx": synth.to_e4m3(x["q_idx"]), "k_idx": synth.to_e4m3(x["k_idx"])}

    def fp8_step():
        sga.forward_fp8(xf["q_idx"], x["w"], xf["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], top_k=K,
                        idx_out=idx, out=out, ws=ws_all, stream=stream)

    def region_ms(step, ws, what):
        """Warm-up, then `args.steps` calls timed as one region like the main one (max over ranks)."""
        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        s3, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s3.record(stream)
        for _ in range(args.steps):
            step()
        e3.record(stream)
        torch.cuda.synchronize(dev)
        ms = max_over_ranks(dist, dev, s3.elapsed_time(e3))
        if sga.device_status(ws) != 0:
            raise RuntimeError(f"device status set during the {what} run")
        return ms

    fp8_ms = region_ms(fp8_step, ws_all, "E4M3 variant")

    # ---- the headline step replayed from a CUDA graph (the same sga_forward calls,
    # captured once): what a serving loop that launches through graphs sees
    try:
        graph_ms = graph_replay_ms(lambda st: (lambda: sga.forward(
            x["q_idx"], x["w"], x["k_idx"], x["q"], x["kv"], x["gate"], x["q_pos"], top_k=K, idx_out=idx, out=out,
            ws=ws_all, stream=st)), args, dev, dist)
        if sga.device_status(ws_all) != 0:
            raise RuntimeError("device status set during the graph replay")
    except (RuntimeError, TypeError, ValueError) as exc:
        torch.cuda.synchronize(dev)
        graph_ms = f"{type(exc).__name__}: {exc}"

    # ---- the fused selection (sga_forward_fused, an opt-in entry point with the
    # same results): the indexer appends candidates instead of writing scores
    fused_ms = fused8_ms = None
    if fused_ok:
        fr = fused_variant(sga, synth, args, wl, x, dev, stream, dist, xf=xf, idx=idx, out=out)
        fused_ms, fused8_ms = fr["bf16"], fr["fp8"]
    del xf

    # ---- one whole SGA layer (a separate configuration): h -> projections ->
    # the path -> W_UV, o_proj, on the same caches (the new tokens' rows are
    # rewritten at their positions every step), timed like the main region.
    layer = layer_variant(sga, synth, args, dev, stream, dist, rank, x, dims, idx) if args.layer else None

    # ---- the indexer's sparse warm-up objective (a training-time variant) over this step's selection
    warm = None
    if args.warmup_objective:
        try:
            fwd_step()  # idx of the current inputs
            warm = warmup_objective_variant(sga, args, dev, stream, dist, rank, x, dims, idx, measured_peaks()[0])
        except (RuntimeError, TypeError, ValueError) as exc:
            torch.cuda.synchronize(dev)
            warm = {"error": f"{type(exc).__name__}: {exc}"}
        torch.cuda.empty_cache()

    # ---- the other decode workloads (separate configurations, one line each in `variants`)
    decode_lines = {}
    if args.decode_variants and args.workload is None and not (args.batch and args.ctx):
        peak_gbs, _ = measured_peaks()
        for name in ("decode_b4_ctx8k", "decode_b64_ctx32k", "decode_b8_ctx256k_ties"):
            try:
                decode_lines[name] = decode_variant(sga, synth, name, args, dev, stream, dist, rank, peak_gbs)
            except (RuntimeError, TypeError, ValueError) as exc:
                torch.cuda.synchronize(dev)
                decode_lines[name] = {"error": f"{type(exc).__name__}: {exc}"}
            torch.cuda.empty_cache()

    # ---- chunked prefill (a separate configuration): 4096 new queries over a 128K cache.
    # The indexer is a dense causal contraction here, so it is reported in TFLOP/s against
    # the bf16 tensor peak, with the whole chunk's time.  L2 is flushed (256 MB memset)
    # before every timed iteration, outside its events.
    prefill = None
    if args.prefill:
        try:
            prefill = prefill_variant(sga, synth, args, dev, stream, dist, rank)
        except (RuntimeError, TypeError, ValueError) as exc:
            torch.cuda.synchronize(dev)
            prefill = {"error": f"{type(exc).__name__}: {exc}"}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    ms_per_step = elapsed_ms / args.steps
    value = whole_job_rate(rows, args.steps, world, elapsed_ms)
    ab = algorithmic_bytes_per_query(L, K)
    peak, peak_kind = measured_peaks()
    k1_ms = statistics.mean(k1)
    k1_bytes = ab["indexer"] * rows
    k1_gbs = k1_bytes / (k1_ms * 1e-3) / 1e9
    counters = kernel_counters("sga_index.cu")
    traffic = None
    if counters and counters.get("workload") == wl.name:
        traffic = counters.get("dram_bytes_per_launch")
    path_gbs = ab["total"] * rows / (ms_per_step * 1e-3) / 1e9

    ab8 = algorithmic_bytes_per_query(L, K, key_bytes=1)
    fp8_step_ms = fp8_ms / args.steps
    fp8_gbs = ab8["total"] * rows / (fp8_step_ms * 1e-3) / 1e9
    variants = {"fp8_index_keys": {
        "value": whole_job_rate(rows, args.steps, world, fp8_ms), "unit": UNIT, "ms_per_step": fp8_step_ms,
        "config": f"{wl.name} with q_idx and k_idx stored as E4M3 (exact for the integer-valued inputs)",
        "path_roofline": {"achieved_gbs": fp8_gbs, "frac_of_8tbs": fp8_gbs / NOMINAL_HBM_GBS,
                          "frac_of_measured": fp8_gbs / peak, "bytes_per_query": ab8["total"]},
        "gpu_launches": launches_per_step * args.steps}}
    if isinstance(graph_ms, float):
        g_step_ms = graph_ms / args.steps
        g_gbs = ab["total"] * rows / (g_step_ms * 1e-3) / 1e9
        variants["graph_replay"] = {
            "value": whole_job_rate(rows, args.steps, world, graph_ms), "unit": UNIT, "ms_per_step": g_step_ms,
            "config": f"{wl.name}: the headline's {args.steps} sga_forward calls captured in one CUDA graph and "
                      f"replayed (the launches become graph kernel nodes with their programmatic dependencies)",
            "path_roofline": {"achieved_gbs": g_gbs, "frac_of_8tbs": g_gbs / NOMINAL_HBM_GBS,
                              "frac_of_measured": g_gbs / peak, "bytes_per_query": ab["total"]},
            "gpu_launches": launches_per_step * args.steps}
    else:
        variants["graph_replay"] = {"error": graph_ms}
    if fused_ms is not None:
        for key, ms, bpq, cfg in (("fused_selection", fused_ms, ab["total"], wl.name),
                                  ("fused_selection_fp8_index_keys", fused8_ms, ab8["total"],
                                   f"{wl.name} with q_idx and k_idx stored as E4M3")):
            step_ms = ms / args.steps
            gbs = bpq * rows / (step_ms * 1e-3) / 1e9
            variants[key] = {
                "value": whole_job_rate(rows, args.steps, world, ms), "unit": UNIT, "ms_per_step": step_ms,
                "config": f"{cfg} through sga_forward_fused: the indexer appends the keys at or above a running "
                          f"per-query threshold instead of writing scores; the same indices and outputs",
                "path_roofline": {"achieved_gbs": gbs, "frac_of_8tbs": gbs / NOMINAL_HBM_GBS,
                                  "frac_of_measured": gbs / peak, "bytes_per_query": bpq},
                "gpu_launches": launches_per_step * args.steps}
    variants.update(decode_lines)
    if warm is not None:
        variants["indexer_warmup"] = warm
    if prefill is not None:
        variants[prefill.pop("name", "prefill_t4096_ctx128k")] = prefill
    if layer is not None:
        layer_step_ms = layer["ms"] / args.steps
        layer_bytes = ab["total"] * rows + layer["weight_bytes"] + layer["act_bytes"]
        layer_gbs = layer_bytes / (layer_step_ms * 1e-3) / 1e9
        variants["sga_layer"] = {
            "value": whole_job_rate(rows, args.steps, world, layer["ms"]), "unit": UNIT, "ms_per_step": layer_step_ms,
            "config": f"{wl.name} as one whole SGA layer: d_model 7168, q rank 1536, projections in the library's "
                      f"weight-streaming tcgen05 GEMM (bf16, fp32 accumulation), bf16 activations between contractions",
            "path_roofline": {"achieved_gbs": layer_gbs, "frac_of_8tbs": layer_gbs / NOMINAL_HBM_GBS,
                              "frac_of_measured": layer_gbs / peak, "bytes_per_step": layer_bytes,
                              "weight_bytes": layer["weight_bytes"]},
            # own kernels per step: five GEMMs, two projection preps, the G5 partial sum, the
            # path's three (the attention also writes the bf16 copy of its output for W_UV)
            "gpu_launches": 11 * args.steps}
        if isinstance(layer["graph_ms"], float):
            variants["sga_layer"]["graph_replay_ms_per_step"] = layer["graph_ms"] / args.steps
        else:
            variants["sga_layer"]["graph_replay_error"] = layer["graph_ms"]

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline(wl, args.cpu_sample_queries)
        cpu.pop("seconds", None)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config_of(wl),
        "roofline": {"bound": "hbm", "kernel": "sga_index_kernel", "achieved": k1_gbs, "peak": peak, "unit": "GB/s",
                     "frac": k1_gbs / peak, "peak_kind": peak_kind, "traffic": traffic,
                     "algorithmic_bytes_per_launch": k1_bytes},
        "path_roofline": {"achieved_gbs": path_gbs, "frac_of_8tbs": path_gbs / NOMINAL_HBM_GBS,
                          "frac_of_measured": path_gbs / peak, "bytes_per_query": ab["total"]},
        "stages_ms": {"index": k1_ms, "topk_standalone": statistics.mean(k2), "attend": statistics.mean(k3),
                      "note": "each call timed alone; inside sga_forward the indexer also builds the top-k "
                              "first-level histogram and the top-k skips its histogram pass"},
        "cpu_baseline": cpu,
        "e2e": {"value": whole_job_rate(rows, args.steps, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps,
                "mode": e2e_mode,
                "serial_value": whole_job_rate(rows, args.steps, world, e2e_serial_ms)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "variants": variants,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
