#!/usr/bin/env python
"""Benchmark: activation-sparse FFN decode, tokens/s per layer on B200.

The headline step is one pass of the workload's decode sequence through the hot path
at batch 1: predictor, threshold and compaction, gathered up/gate projection,
gathered down projection and the final sum, one token at a time.  The default
workload is the largest single-GPU one, the 70B-shaped ReGLU layer (d=8192
n=28672 r=1024, fp16, 43% of the neurons carry 80% of the activations; 128
tokens per step).  The tokens are captured once into a CUDA graph; a step is one
replay.  Consecutive tokens use different replicas of the layer's weights so that
no token finds the previous visit's lines in L2 (the bytes touched between two
visits of one replica exceed twice the L2 size), as in a model where the other
layers stream through between two visits of a layer.

The same run then measures every other workload the same way (``per_config`` in
the JSON line): the tiny fp32 and OPT-6.7B-shaped layers at batch 1, the 4-layer
LLaMA-7B-shaped residual stack (own-layer and one-layer-ahead predictor), the
OPT-30B-shaped layer at batch 1, 2, 4, 8 and the 70B-shaped layer at batch
2 ... 32 (16 batches per step over rotating replicas).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sfnn|reference]

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on the
host cores instead, on the same workload and metric.  With N > 1 (torchrun)
each rank runs an independent replica on its own GPU (no data exchange); the
time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workload as W  # noqa: E402

WORKLOAD = "70b_reglu"
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "activation_sparse_ffn_threshold_b200", "csrc")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["sfnn", "reference"], default="sfnn")
    ap.add_argument("--workload", default=WORKLOAD, choices=list(W.CONFIGS))
    ap.add_argument("--replicas", type=int, default=0, help="weight replicas (0: from the L2 size)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="time the headline workload only")
    ap.add_argument("--order", choices=["dealt", "packed", "identity"], default="dealt",
                    help="storage order of the neurons: hotness ranks dealt round-robin to the SM tiles (default), "
                         "hot-packed-first, or the original order (no hotness profile)")
    ap.add_argument("--fused-quota", type=int, default=-1,
                    help="the single-token kernel's rebalancing quota (-1: the hotness profile's default)")
    ap.add_argument("--fused-depths", default="",
                    help="the single-token kernel's request depths 'bstages,c2pre,c1depth' (-1 keeps one)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--rows", choices=["native", "int8", "int4"], default="native",
                    help="storage of the FFN rows for the single-token line: the layer's dtype, or int8 / int4 "
                         "codes with per-row scales")
    ap.add_argument("--stack", action="store_true",
                    help="time the residual stack of the workload's layers (default workload: the "
                         "4-layer LLaMA-7B-shaped ReGLU stack), one token at a time")
    ap.add_argument("--lookahead", action="store_true",
                    help="with --stack: predict each layer's set from the previous layer's input, "
                         "one layer ahead (one fused launch per layer and token, plus one)")
    ap.add_argument("--batch", type=int, default=1,
                    help="tokens per forward call: 1 is the single-token decode (the headline); b > 1 "
                         "times the batched union path on b tokens at a time")
    ap.add_argument("--batch-path", choices=["auto", "cuda_core", "tensor_core", "fused"], default="auto",
                    help="with --batch > 1: the batched path; auto measures, for 4 < b <= 8, two few-token "
                         "launches against tensor cores before timing (a profiler slows the launches and "
                         "skews that measurement: name the path there)")
    ap.add_argument("--tc-shape", default="",
                    help="with --batch > 1: the tensor-core kernels' shape, "
                         "'up_ctas_per_sm,up_chunks_per_step,down_tiles_per_cta'")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="CPU budget of the reference arm (warm-up and timed steps together)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- distributed plumbing
class Dist:
    def __init__(self, gpus: int):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime

            import torch
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local_rank)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = dist
        if gpus != self.world and self.world > 1:
            log(f"note: --gpus {gpus} but WORLD_SIZE {self.world}; using WORLD_SIZE")

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, v: float) -> float:
        return self._reduce(v, "max")

    def sum(self, v: float) -> float:
        return self._reduce(v, "sum")

    def _reduce(self, v, op):
        if self.pg is None:
            return v
        import torch
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([float(v)], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX if op == "max" else self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------- clocks
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except Exception as e:  # pragma: no cover
            log(f"clock sampling unavailable: {e}")
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), power=float(f[3]), hw=f[5], hwt=f[6], swt=f[7],
                                 pcap=f[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        smax = max(r["smax"] for r in rows)
        load = [r for r in rows if r["power"] > 250.0] or rows
        reasons = set()
        for r in load:
            if r["hw"] == "Active":
                reasons.add("hw_slowdown")
            if r["hwt"] == "Active":
                reasons.add("hw_thermal_slowdown")
            if r["swt"] == "Active":
                reasons.add("sw_thermal_slowdown")
            if r["pcap"] == "Active":
                reasons.add("sw_power_cap")
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": max(r["power"] for r in rows)}


# ---------------------------------------------------------------- helpers
def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the sources k_decode1 is built from: a profile of it stays valid while they are unchanged
# The sources each measured path is built from: a committed ncu summary of a path stays
# valid (its DRAM traffic is reported) while they are unchanged.
PATH_SOURCES = {
    "k_decode1": ("async.cuh", "common.cuh", "decode1.cu", "decode1.cuh", "decode_dev.cuh"),
    "multi": ("async.cuh", "common.cuh", "decode_multi.cu", "decode1.cuh", "decode_dev.cuh"),
    "tcgen05": ("async.cuh", "common.cuh", "context.cuh", "tc_batch.cu", "predict.cu", "ffn.cu", "launch.cuh"),
    "lookahead": ("async.cuh", "common.cuh", "decode_ahead.cu", "decode1.cuh", "decode_dev.cuh"),
}


def source_digest(path: str = "k_decode1") -> str:
    h = hashlib.sha256()
    for name in PATH_SOURCES[path]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, summary: str | None = None, path: str = "k_decode1",
                     key: str = "dram_bytes_per_token"):
    """DRAM bytes per unit (token, batch or layer-token) from the committed ncu summary
    profiles/<summary>.md, if it was taken on the current sources of `path`."""
    summary = summary or f"k_decode1_{workload}"
    try:
        text = open(os.path.join(ROOT, "profiles", f"{summary}.md")).read()
    except OSError:
        return None, None
    sha = traffic = None
    for line in text.splitlines():
        if line.startswith("source_sha256_16:"):
            sha = line.split(":", 1)[1].strip()
        if line.startswith(f"{key}:"):
            traffic = float(line.split(":", 1)[1].strip())
    if sha != source_digest(path):
        return None, "stale"
    return traffic, "ncu"


def expected_tokens_active(cfg):
    return cfg.mean_p * cfg.n


def cpu_baseline(cfg, lay, X, seconds: float):
    """The oracle as it stands, on this host's cores, over a bounded sample of tokens."""
    import oracle
    nthreads = oracle.max_threads()
    t0 = time.perf_counter()
    oracle.forward(lay, X[0], nthreads)
    t_one = max(1e-4, time.perf_counter() - t0)
    count = int(max(1, min(X.shape[0] - 1, seconds / t_one)))
    t0 = time.perf_counter()
    active = 0
    for t in range(1, 1 + count):
        active += int(oracle.forward(lay, X[t], nthreads).mask.sum())
    dt = time.perf_counter() - t0
    tok_s = count / dt
    gbs = W.touched_bytes(cfg, active / count) * tok_s / 1e9
    return {"value": tok_s, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
            "sample": f"{count} tokens of {cfg.name} (predictor + sparse FFN, batch 1), fp64 C oracle",
            "effective_gbs": gbs}


# ---------------------------------------------------------------- reference arm (the CPU oracle)
def run_reference(args, dist):
    if dist.rank != 0:
        return 0
    import oracle
    cfg = W.CONFIGS[args.workload]
    lay = W.make_layer(cfg, seed=args.seed)
    X = W.make_tokens(cfg, 64, seed=args.seed)
    nthreads = oracle.max_threads()
    t0 = time.perf_counter()
    oracle.forward(lay, X[0], nthreads)
    t_one = max(1e-4, time.perf_counter() - t0)
    budget = args.ref_seconds  # seconds for warm-up + timed steps together
    per_step = max(1, min(cfg.tokens, int(budget / max(1, args.steps + args.warmup) / t_one)))
    k = 0
    for _ in range(args.warmup):
        for _ in range(per_step):
            oracle.forward(lay, X[k % X.shape[0]], nthreads)
            k += 1
    t0 = time.perf_counter()
    active = 0
    for _ in range(args.steps):
        for _ in range(per_step):
            active += int(oracle.forward(lay, X[k % X.shape[0]], nthreads).mask.sum())
            k += 1
    dt = time.perf_counter() - t0
    tokens = args.steps * per_step
    tok_s = tokens / dt
    line = {
        "impl": "reference", "metric": "sparse-FFN decode tokens/s per layer", "value": tok_s,
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.description, "batch": 1, "tokens_per_step": per_step},
        "effective_gbs": W.touched_bytes(cfg, active / tokens) * tok_s / 1e9,
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"{per_step} token(s) of {cfg.name} per step, fp64 C oracle"},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- the CUDA path
def _device(dist):
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    dev = torch.device("cuda", dist.local_rank if dist.world > 1 else 0)
    torch.cuda.set_device(dev)
    return dev


def _gpu_id(dev) -> str:
    import torch
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    return uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"


def _launches(handles) -> int:
    return sum(h.info()["launches"] for h in handles)


def capture(s, fn, handles):
    """Run ``fn`` once eagerly on stream ``s``, then capture it into a CUDA graph.
    Returns (graph, kernels one replay launches)."""
    import torch
    with torch.cuda.stream(s):
        fn()
    torch.cuda.synchronize()
    l0 = _launches(handles)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    return g, _launches(handles) - l0


def time_graph(g, s, steps, warmup, dist, gpu_id):
    """Warm-up replays, then ``steps`` replays between CUDA events on ``s``, bracketed by
    a barrier and a device synchronisation; SM clocks sampled meanwhile.  Returns
    (this rank's ms, max over ranks of ms, clocks)."""
    import torch
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id) as clk:
        dist.barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            start.record(s)
            for _ in range(steps):
                g.replay()
            stop.record(s)
        torch.cuda.synchronize()
        dist.barrier()
    ms = start.elapsed_time(stop)
    return ms, dist.max(ms), clk.summary()


def time_eager(fn, s, steps, dist):
    """The same, for an eager loop of API calls (end to end): (max over ranks of ms)."""
    import torch
    with torch.cuda.stream(s):
        fn()  # warm-up
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    with torch.cuda.stream(s):
        a.record(s)
        for _ in range(steps):
            fn()
        b.record(s)
    torch.cuda.synchronize()
    return dist.max(a.elapsed_time(b))


def roofline(alg_bytes, unit_us, kernel, traffic=None, traffic_source=None):
    peak, kind = measured_peak()
    achieved = alg_bytes / (unit_us / 1e6) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": traffic, "kernel": kernel, "algorithmic_bytes_per_launch": alg_bytes, "avg_launch_us": unit_us,
            "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)" if kind == "measured" else "fallback 6.65 TB/s",
            "traffic_source": traffic_source}


def _check_errors(handles):
    err = max(h.get_error() for h in handles)
    if err:
        raise SystemExit(f"device-side error latched: {err}")


def _free(*objs):
    import gc

    import torch
    for o in objs:
        for h in (o if isinstance(o, (list, tuple)) else [o]):
            if hasattr(h, "close"):
                h.close()
    gc.collect()
    torch.cuda.empty_cache()


def _order_kw(args):
    order = getattr(args, "order", "dealt")
    return {"use_hotness": order != "identity", "order": "packed" if order == "packed" else "dealt"}


def measure_single(cfg, args, dist, dev, rows=None, headline=False):
    """Batch-1 decode: the workload's tokens, one forward call each, over rotating weight
    replicas, captured in one CUDA graph; one step = one replay."""
    import torch

    import activation_sparse_ffn_threshold_b200 as sf
    T = cfg.tokens
    lay = W.make_layer(cfg, seed=args.seed)
    Xh = W.make_tokens(cfg, T, seed=args.seed + dist.rank)
    e = cfg.esize
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per_token = W.touched_bytes(cfg, expected_tokens_active(cfg))
    if rows:  # rows of one byte (int8) or half a byte (int4) per weight and a scale per row
        qbytes = 1.0 if rows == "int8" else 0.5
        per_token -= expected_tokens_active(cfg) * cfg.nproj * (cfg.d * (e - qbytes) - 4)
    # replicas: bytes touched between two visits of a replica >= 2 x L2 (at most one per
    # token: a layer too small for that, the tiny fp32 one, stays L2-resident anyway)
    R = args.replicas or min(T, max(2, 1 + math.ceil(2 * l2 / per_token)))
    handles = [sf.SparseFFN.from_layer(lay, device=dev, rows=rows, **_order_kw(args)) for _ in range(R)]
    if args.fused_quota != -1:
        for h in handles:
            h.set_fused_quota(args.fused_quota)
    if args.fused_depths:
        for h in handles:
            h.set_fused_depths(*[int(v) for v in args.fused_depths.split(",")])
    info = handles[0].info()
    torch.cuda.synchronize()
    X = torch.from_numpy(Xh).to(dev)
    Y = torch.empty((T, cfg.d), dtype=torch.float32, device=dev)
    # the sets the fused kernel uses for the captured tokens (for the algorithmic byte count)
    counts = np.empty(T, np.int64)
    for t in range(T):
        _, _, c = handles[0].forward_batch(X[t:t + 1], return_sets=True)
        counts[t] = int(c.item())
    bytes_tok = info["predictor_bytes"] + counts * info["row_bytes_per_neuron"] + cfg.d * e + cfg.d * 4
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())

    def step():
        for t in range(T):
            handles[t % R].forward(X[t], Y[t], stream=s)
    g, launches = capture(s, step, handles)
    # one fused launch per token, nothing else: the region's time / launches is the
    # kernel's average launch duration
    assert launches == T, launches
    ms, t_max, clocks = time_graph(g, s, args.steps, args.warmup, dist, _gpu_id(dev))
    _check_errors(handles)
    unit_us = ms * 1e3 / (args.steps * T)
    out = {"value": dist.sum(args.steps * T) / (t_max / 1e3), "unit": "tokens/s", "ms_per_step": t_max / args.steps,
           "avg_us": unit_us, "avg_of": "one token (one k_decode1 launch)", "replicas": R,
           "mean_active_neurons": float(counts.mean()), "gpu_launches": int(launches * args.steps),
           "clocks": clocks, "bytes_per_step": float(bytes_tok.sum())}
    if args.fused_quota != -1:
        out["fused_quota"] = args.fused_quota
    if args.fused_depths:
        out["fused_depths"] = args.fused_depths
    traffic, tsrc = (profiled_traffic(cfg.name) if rows is None else (None, None))
    out["roofline"] = roofline(float(bytes_tok.mean()), unit_us,
                               "k_decode1 (fused single-token decode), the only kernel the timed region launches; "
                               "average launch duration = CUDA-event time of the region / its launches",
                               traffic, tsrc)
    out["effective_gbs"] = float(bytes_tok.sum()) * args.steps / (ms / 1e3) / 1e9
    if headline and not args.no_e2e:
        # end to end through the public API, eager: per step, the step's inputs from pinned
        # host memory in one copy, one forward call per token, the step's outputs back in one
        xin = torch.from_numpy(Xh).pin_memory()
        yout = torch.empty((T, cfg.d), dtype=torch.float32).pin_memory()
        xd = torch.empty((T, cfg.d), dtype=X.dtype, device=dev)
        yd = torch.empty((T, cfg.d), dtype=torch.float32, device=dev)
        e2e_steps = max(1, min(args.steps, 20))

        def one_step():
            xd.copy_(xin, non_blocking=True)
            for t in range(T):
                handles[t % R].forward(xd[t], yd[t], stream=s)
            yout.copy_(yd, non_blocking=True)
        e_max = time_eager(one_step, s, e2e_steps, dist)
        _check_errors(handles)
        out["e2e"] = {"value": dist.sum(e2e_steps * T) / (e_max / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": T * cfg.d * e, "d2h_bytes_per_step": T * cfg.d * 4, "steps": e2e_steps,
                      "timing": "CUDA events around the eager loop (per step: one host-to-device copy of the step's "
                                "inputs, one forward call per token, one device-to-host copy of the outputs), "
                                "max over ranks"}
    out["_lay"] = lay
    del g
    _free(handles)
    return out


def measure_batch(cfg, b, args, dist, dev):
    """b tokens per forward_batch call: predictor of the batch, union of its sets, the
    union's rows once for all b tokens.  A step is BATCHES_PER_STEP such calls over
    rotating weight replicas, captured in one CUDA graph."""
    import torch

    import activation_sparse_ffn_threshold_b200 as sf
    lay = W.make_layer(cfg, seed=args.seed)
    Xh = W.make_tokens(cfg, BATCHES_PER_STEP * b, seed=args.seed + dist.rank, stream_key=b).reshape(
        BATCHES_PER_STEP, b, cfg.d)
    e = cfg.esize
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per_batch = W.touched_bytes(cfg, W.expected_union_density(lay.p, b) * cfg.n, b)
    R = args.replicas or max(2, 1 + math.ceil(2 * l2 / per_batch))
    handles = [sf.SparseFFN.from_layer(lay, device=dev, max_batch=b, **_order_kw(args)) for _ in range(R)]
    tuned = None
    bpath = {"auto": sf.BATCH_AUTO, "cuda_core": sf.BATCH_CUDA_CORE, "tensor_core": sf.BATCH_TENSOR_CORE,
             "fused": sf.BATCH_FUSED}[args.batch_path]
    for h in handles:
        h.set_batch_path(bpath)
        if args.tc_shape:
            h.set_batch_tc_shape(*[int(v) for v in args.tc_shape.split(",")])
    if bpath == sf.BATCH_AUTO and 4 < b <= 8:  # AUTO's measured choice: two few-token launches or tensor cores
        for h in handles:
            t = h.tune_batch_paths()
            tuned = tuned or t
    info = handles[0].info()
    torch.cuda.synchronize()
    X = torch.from_numpy(Xh).to(dev)
    Y = torch.empty((BATCHES_PER_STEP, b, cfg.d), dtype=torch.float32, device=dev)
    unions = np.empty(BATCHES_PER_STEP, np.int64)
    for i in range(BATCHES_PER_STEP):  # union sizes, for the algorithmic byte count
        _, idx, cnt = handles[0].forward_batch(X[i], return_sets=True)
        m = torch.zeros(cfg.n, dtype=torch.bool, device=dev)
        for t in range(b):
            m[idx[t, :int(cnt[t])].long()] = True
        unions[i] = int(m.sum())
    bytes_batch = info["predictor_bytes"] + unions * info["row_bytes_per_neuron"] + b * cfg.d * (e + 4)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())

    def step():
        for i in range(BATCHES_PER_STEP):
            handles[i % R].forward_batch(X[i], Y[i], stream=s)
    g, launches = capture(s, step, handles)
    ms, t_max, clocks = time_graph(g, s, args.steps, args.warmup, dist, _gpu_id(dev))
    _check_errors(handles)
    unit_us = ms * 1e3 / (args.steps * BATCHES_PER_STEP)
    path = batch_path_name(handles[0], b, launches // BATCHES_PER_STEP)
    out = {"value": dist.sum(args.steps * BATCHES_PER_STEP * b) / (t_max / 1e3), "unit": "tokens/s",
           "ms_per_step": t_max / args.steps, "avg_us": unit_us, "avg_of": f"one batch of {b} tokens",
           "replicas": R, "path": path, "kernels_per_batch": launches // BATCHES_PER_STEP,
           "mean_union_rows": float(unions.mean()), "gpu_launches": int(launches * args.steps), "clocks": clocks,
           "bytes_per_step": float(bytes_batch.sum())}
    if tuned:  # ms per call of (two few-token launches, tensor cores), synthetic tokens
        out["tuned_ms"] = {str(k): [round(v[0], 4), round(v[1], 4)] for k, v in tuned.items()}
    two = b > 4 and launches // BATCHES_PER_STEP == 2
    tpath = "multi" if (b <= 4 and handles[0].info()["wdtype"] == 1) or two else "tcgen05"
    summary = f"batch_{cfg.name}_b{b}" + ("_two_launches" if two else "")
    traffic, tsrc = profiled_traffic(cfg.name, summary, tpath, "dram_bytes_per_batch")
    out["roofline"] = roofline(float(bytes_batch.mean()), unit_us,
                               f"one batch of {b} tokens ({launches // BATCHES_PER_STEP} kernels, {path}); "
                               "duration = CUDA-event time of the timed region / batches", traffic, tsrc)
    out["effective_gbs"] = float(bytes_batch.sum()) * args.steps / (ms / 1e3) / 1e9
    del g
    _free(handles)
    return out


def batch_path_name(h, b, kernels_per_batch) -> str:
    """The kernels AUTO (or the chosen path) runs for b tokens on this layer."""
    inf = h.info()
    fused = inf["wdtype"] == 1 and 2 <= b <= 4  # fp16 layers: the few-token fused kernel
    two = inf["wdtype"] == 1 and b > 4 and kernels_per_batch == 2  # two few-token launches
    tc = inf["wdtype"] == 1 and inf["d"] % 128 == 0
    auto = ("fused few-token kernel (CUDA cores)" if fused else
            "two fused few-token launches (measured faster)" if two else ("tcgen05" if tc else "cuda-core"))
    return {0: f"auto: {auto}", 1: "cuda-core", 2: "tcgen05", 3: f"fused: {auto}"}.get(inf["batch_path"], "?")


def measure_stack(cfg, args, dist, dev, lookahead=False, rows=None):
    """x_{l+1} = x_l + FFN_l(x_l) through the workload's layers, one token per
    forward_stack call; a step is the workload's tokens, captured in one CUDA graph."""
    import torch

    import activation_sparse_ffn_threshold_b200 as sf
    T, NL = cfg.tokens, cfg.layers
    layers = W.make_stack(cfg, seed=args.seed)
    Xh = W.make_tokens(cfg, T, seed=args.seed + dist.rank).astype(np.float32)
    handles = [sf.SparseFFN.from_layer(lay, device=dev, rows=rows) for lay in layers]
    info = handles[0].info()
    e = cfg.esize
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    X = torch.from_numpy(Xh).to(dev)
    Y = torch.empty_like(X)
    active = np.zeros(NL)
    for t in range(T):  # the sets the stack's own launches use, for the byte count
        _, _, cnt = sf.forward_stack(handles, X[t], return_sets=True, lookahead=lookahead)
        active += cnt.cpu().numpy().reshape(NL)
    active /= T
    bytes_layer_tok = info["predictor_bytes"] + active * info["row_bytes_per_neuron"] + cfg.d * (e + 4)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())

    def step():
        for t in range(T):
            sf.forward_stack(handles, X[t], Y[t], stream=s, lookahead=lookahead)
    g, launches = capture(s, step, handles)
    ms, t_max, clocks = time_graph(g, s, args.steps, args.warmup, dist, _gpu_id(dev))
    _check_errors(handles)
    layer_us = ms * 1e3 / (args.steps * T * NL)
    out = {"value": dist.sum(args.steps * T * NL) / (t_max / 1e3), "unit": "layer-tokens/s",
           "ms_per_step": t_max / args.steps, "avg_us": layer_us, "avg_of": "one layer of one token",
           "layers": NL, "launches_per_token": launches // T, "gpu_launches": int(launches * args.steps),
           "mean_active_neurons_per_layer": [float(v) for v in active], "clocks": clocks,
           "bytes_per_step": float(bytes_layer_tok.sum()) * T,
           "l2": f"inputs larger than L2: {NL} distinct layers per token, "
                 f"{float(bytes_layer_tok.sum()) / 1e6:.1f} MB touched per token, L2 {l2 / 1e6:.0f} MB"}
    kern = (f"k_decode_ahead (look-ahead stack), {launches // T} launches per token: the input rounding, layer 0's "
            "predictor, one per layer" if lookahead else
            f"k_decode1, one launch per layer and token ({launches // T} launches per token with the input rounding)")
    traffic, tsrc = profiled_traffic(cfg.name, f"stack_{cfg.name}{'_lookahead' if lookahead else ''}",
                                     "lookahead" if lookahead else "k_decode1", "dram_bytes_per_layer_token")
    out["roofline"] = roofline(float(bytes_layer_tok.mean()), layer_us,
                               kern + "; duration = CUDA-event time of the region / layer-tokens", traffic, tsrc)
    out["effective_gbs"] = float(bytes_layer_tok.sum()) * T * args.steps / (ms / 1e3) / 1e9
    if not args.no_e2e:
        xin = torch.from_numpy(Xh).pin_memory()
        yout = torch.empty((T, cfg.d), dtype=torch.float32).pin_memory()
        xd = torch.empty((T, cfg.d), dtype=torch.float32, device=dev)
        yd = torch.empty((T, cfg.d), dtype=torch.float32, device=dev)
        e2e_steps = max(1, min(args.steps, 10))

        def one_step():  # the step's inputs in one copy, one stack call per token, the outputs in one copy
            xd.copy_(xin, non_blocking=True)
            for t in range(T):
                sf.forward_stack(handles, xd[t], yd[t], stream=s, lookahead=lookahead)
            yout.copy_(yd, non_blocking=True)
        e_max = time_eager(one_step, s, e2e_steps, dist)
        out["e2e"] = {"value": dist.sum(e2e_steps * T * NL) / (e_max / 1e3), "unit": "layer-tokens/s",
                      "h2d_bytes_per_step": T * cfg.d * 4, "d2h_bytes_per_step": T * cfg.d * 4,
                      "steps": e2e_steps}
    del g
    _free(handles)
    return out


BATCHES_PER_STEP = 16

# The other workloads, each measured the same way as the headline inside the default run:
# (workload, what, batch)
PER_CONFIG = [
    ("tiny_relu_f32", "single", 1),
    ("opt6.7b_relu", "single", 1),
    ("llama7b_reglu_stack", "stack", 1),
    ("llama7b_reglu_stack", "stack_lookahead", 1),
    ("opt30b_relu", "single", 1),
    ("opt30b_relu", "batch", 2),
    ("opt30b_relu", "batch", 4),
    ("opt30b_relu", "batch", 8),
    ("70b_reglu", "batch", 2),
    ("70b_reglu", "batch", 4),
    ("70b_reglu", "batch", 8),
    ("70b_reglu", "batch", 16),
    ("70b_reglu", "batch", 32),
]


def _summary(cfg, what, b, m):
    """One per_config record: the numbers a reader compares across workloads."""
    r = m["roofline"]
    return {"workload": cfg.description, "what": what, "batch": b, "value": m["value"], "unit": m["unit"],
            "avg_us": m["avg_us"], "avg_of": m["avg_of"], "achieved_gbs": r["achieved"], "frac": r["frac"],
            "algorithmic_bytes": r["algorithmic_bytes_per_launch"], "traffic": r["traffic"],
            **({"path": m["path"], "mean_union_rows": m["mean_union_rows"], "kernels_per_batch":
                m["kernels_per_batch"]} if "path" in m else {}),
            **({"tuned_ms": m["tuned_ms"]} if "tuned_ms" in m else {}),
            **({"mean_active_neurons": m["mean_active_neurons"]} if "mean_active_neurons" in m else {}),
            **({"mean_active_neurons_per_layer": m["mean_active_neurons_per_layer"],
                "launches_per_token": m["launches_per_token"]} if "layers" in m else {}),
            **({"e2e": m["e2e"]["value"]} if m.get("e2e") else {}),
            "clocks": {"sm_mhz": m["clocks"].get("sm_mhz"), "reasons": m["clocks"].get("reasons")}}


def run_sfnn(args, dist):
    """The headline: batch-1 decode of the workload (default: the 70B-shaped ReGLU
    layer, the largest single-GPU configuration), then every other configuration."""
    dev = _device(dist)
    cfg = W.CONFIGS[args.workload]
    rows = None if args.rows == "native" else args.rows
    m = measure_single(cfg, args, dist, dev, rows=rows, headline=True)
    lay = m.pop("_lay")
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        Xc = W.make_tokens(cfg, 64, seed=args.seed + 99)
        cpu = cpu_baseline(cfg, lay, Xc, args.cpu_seconds)
    del lay
    per = None
    if not args.no_per_config:
        per = {}
        steps = args.steps
        for name, what, b in PER_CONFIG:
            if name == args.workload and what == "single":
                continue
            c = W.CONFIGS[name]
            key = f"{name}:{what}:b{b}"
            if what == "single":
                r = measure_single(c, args, dist, dev)
                r.pop("_lay", None)
            elif what == "batch":
                r = measure_batch(c, b, args, dist, dev)
            else:
                r = measure_stack(c, args, dist, dev, lookahead=(what == "stack_lookahead"))
            per[key] = _summary(c, what, b, r)
            log(f"{key}: {r['value']:.1f} {r['unit']}, {r['avg_us']:.2f} us, frac {r['roofline']['frac']:.3f}")
        args.steps = steps
    T = cfg.tokens
    line = {
        "metric": "sparse-FFN decode tokens/s per layer", "value": m["value"], "unit": "tokens/s",
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16" if cfg.esize == 2 else "f32", "data": "synthetic",
        "config": {"workload": cfg.description + (f", {rows} rows (per-row fp32 scales)" if rows else ""),
                   "batch": 1, "tokens_per_step": T, "replicas": m["replicas"], "order": args.order,
                   "l2": f"inputs larger than L2: {m['replicas']} weight replicas rotated per token, "
                         f"{m['bytes_per_step'] / T / 1e6:.1f} MB touched per token",
                   "parallelism": f"replicas x{dist.world} (no exchange)",
                   "mean_active_neurons": m["mean_active_neurons"]},
        "effective_gbs": m["effective_gbs"],
        "roofline": m["roofline"],
        "cpu_baseline": cpu,
        "e2e": m.get("e2e"),
        "gpu_launches": m["gpu_launches"],
        "clocks": m["clocks"],
        "per_config": per,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_batch(args, dist):
    dev = _device(dist)
    cfg = W.CONFIGS[args.workload]
    b = args.batch
    m = measure_batch(cfg, b, args, dist, dev)
    line = {
        "metric": "sparse-FFN batched decode tokens/s per layer", "value": m["value"], "unit": "tokens/s",
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": m["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16" if cfg.esize == 2 else "f32", "data": "synthetic",
        "config": {"workload": cfg.description, "batch": b, "batches_per_step": BATCHES_PER_STEP,
                   "path": m["path"], "replicas": m["replicas"], "order": args.order,
                   "l2": f"inputs larger than L2: {m['replicas']} weight replicas rotated per batch, "
                         f"{m['bytes_per_step'] / BATCHES_PER_STEP / 1e6:.1f} MB touched per batch",
                   "parallelism": f"replicas x{dist.world} (no exchange)", "mean_union_rows": m["mean_union_rows"],
                   **({"tuned_ms": m["tuned_ms"]} if "tuned_ms" in m else {})},
        "effective_gbs": m["effective_gbs"], "roofline": m["roofline"], "cpu_baseline": None, "e2e": None,
        "gpu_launches": m["gpu_launches"], "clocks": m["clocks"],
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_stack(args, dist):
    dev = _device(dist)
    cfg = W.CONFIGS[args.workload]
    la = bool(args.lookahead)
    rows = None if args.rows == "native" else args.rows
    m = measure_stack(cfg, args, dist, dev, lookahead=la, rows=rows)
    line = {
        "metric": f"sparse-FFN decode layer-tokens/s ({cfg.layers}-layer residual stack"
                  f"{', sets predicted one layer ahead' if la else ''})", "value": m["value"],
        "unit": "layer-tokens/s", "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": cfg.description, "batch": 1, "layers": cfg.layers, "tokens_per_step": cfg.tokens,
                   "predictor": "one layer ahead" if la else "own layer", "rows": args.rows, "l2": m["l2"],
                   "parallelism": f"replicas x{dist.world} (no exchange)",
                   "mean_active_neurons_per_layer": m["mean_active_neurons_per_layer"]},
        "effective_gbs": m["effective_gbs"], "roofline": m["roofline"], "cpu_baseline": None, "e2e": m.get("e2e"),
        "gpu_launches": m["gpu_launches"], "clocks": m["clocks"],
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    dist = Dist(args.gpus)
    try:
        if args.impl == "reference":
            return run_reference(args, dist)
        if args.stack:
            if args.workload == WORKLOAD:
                args.workload = "llama7b_reglu_stack"
            return run_stack(args, dist)
        if args.batch > 1:
            return run_batch(args, dist)
        return run_sfnn(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    sys.exit(main())
