"""Benchmark: Spark FFN tokens/s per layer on a Gemma-2-2B-shaped layer (B200).

Headline workload: decode, T = 1 token per step, d_model 2304, r 1152, d_ff 9216,
k 737 (8%), bf16 weights ~N(0, 1/fan_in), q ~N(0, 1) (synthetic: trained
Gemma-2 weights are not available).  A step is one full Spark FFN layer forward
(predictor, statistics, threshold, GELU, compaction, K2/V gather) through the
library's C ABI.  The step cycles over 16 copies of the layer's weights
(1.36 GB, far above the 126 MB L2), so every step reads its weights from HBM.

Also reported in the same JSON line (key "also"): the batched prefill at
T = 16, 64, 256, 1024 and 4096 tokens, the decode variants, the 26-layer
decode stack, Spark Attention for one decoding position and the standalone
statistical top-k on 32768 x 4096 fp32 score rows (k = 256), all timed the
same way.

``--impl reference`` times the fp64 CPU oracle (the only reference this method
has: the pages publish no code) on the host cores, on the same workload.

Launch: ``python bench.py --gpus N --steps K --warmup W``; for N > 1 under
torchrun, every rank runs an independent replica (the path has no exchange
step) and the line reports the aggregate over ranks (weak scaling).
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

D_MODEL, R, D_FF, K = 2304, 1152, 9216, 737
N_COPIES = 16
METRIC = "Spark-FFN tokens/s per layer (T=1, 256) and achieved HBM GB/s vs ~8 TB/s"
DECODE_WORKLOAD = "Gemma-2-2B-shaped Spark FFN layer, decode T=1 (one token per step)"
WEIGHTS_RECIPE = "bf16 ~N(0,1/fan_in), q ~N(0,1), seed 1234"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle CPU baseline")
    ap.add_argument("--no-extra", action="store_true", help="skip the prefill / stat-topk extra lines")
    ap.add_argument("--case", default=None, choices=["decode", "noalloc", "prefill", "predictor", "topk", "topk_causal",
                                                     "huber_bwd", "attention"],
                    help="profiling mode: run only this workload, plain launches (no graph), print per-call time")
    ap.add_argument("--tokens", type=int, default=256, help="--case prefill: tokens per call")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def profile_traffic(name: str, sources):
    """DRAM bytes per launch from a committed ncu summary, or None if absent or the kernel changed since."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    h = hashlib.sha256()
    for s in sources:
        h.update(open(os.path.join(ROOT, s), "rb").read())
    if vals.get("source_sha256") != h.hexdigest()[:16]:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def source_hash(sources):
    h = hashlib.sha256()
    for s in sources:
        h.update(open(os.path.join(ROOT, s), "rb").read())
    return h.hexdigest()[:16]


DECODE_SOURCES = ["activation_sparse_transformer_predictor_b200/csrc/ffn_decode_pg.cu",
                  "activation_sparse_transformer_predictor_b200/csrc/spark_device.cuh"]
TOPK_SOURCES = ["activation_sparse_transformer_predictor_b200/csrc/stat_topk.cu",
                "activation_sparse_transformer_predictor_b200/csrc/spark_device.cuh"]
PRED_SOURCES = ["activation_sparse_transformer_predictor_b200/csrc/umma_gemm.cu",
                "activation_sparse_transformer_predictor_b200/csrc/spark_device.cuh"]


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus, backend="nccl"):
    """One process per GPU (RANK / WORLD_SIZE / LOCAL_RANK / MASTER_* from the launcher); every rank
    runs an independent replica and the group only carries the barrier and the max over ranks."""
    import torch
    if n_gpus <= 1 or "RANK" not in os.environ:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    if backend == "nccl":
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier_sync(world, cuda=True):
    import torch
    if cuda:
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        if cuda:
            torch.cuda.synchronize()


def max_over_ranks(v: float, world: int, device="cuda") -> float:
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_call: float, ms_per_call_max: float, world: int) -> float:
    """Units per second of the whole job: every rank processes units_per_call per call, and the
    slowest rank's time per call (the max over ranks) paces them all."""
    return units_per_call * world * 1e3 / ms_per_call_max


def time_graph(fn_list, steps, warmup, world):
    """Capture one CUDA graph that runs every callable of fn_list once (in order), replay it so
    that `steps` calls run in total, and return device milliseconds (CUDA events) per call."""
    import torch
    per_graph = len(fn_list)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        # warm up on the capture stream: the library sizes its per-stream workspace here
        for _ in range(max(warmup, 3)):
            for f in fn_list:
                f()
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            for f in fn_list:
                f()
    torch.cuda.current_stream().wait_stream(s)
    reps = max(1, steps // per_graph)
    for _ in range(2):
        g.replay()
    barrier_sync(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(reps):
        g.replay()
    end.record()
    barrier_sync(world)
    ms = start.elapsed_time(end)
    del g
    return ms / (reps * per_graph), reps * per_graph


def time_exact_steps(step_fns, steps, warmup, world):
    """Time exactly `steps` steps on the device.  Untimed: `warmup` eager calls, then the capture
    of one CUDA graph holding the `steps` calls (cycling over step_fns) and one replay of it.
    Timed: one more replay between CUDA events on the replay stream, max over ranks.  A device-side
    sleep ahead of the start event keeps the graph's host submission out of the timed region.
    Returns milliseconds per step."""
    import torch
    calls = [step_fns[i % len(step_fns)] for i in range(steps)]
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(max(warmup, 3)):
            step_fns[i % len(step_fns)]()
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            for f in calls:
                f()
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    barrier_sync(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(200000)
    start.record()
    g.replay()
    end.record()
    barrier_sync(world)
    ms = start.elapsed_time(end) / steps
    del g
    return max_over_ranks(ms, world)


def bench_config(world: int) -> dict:
    """The workload both arms measure (the native and the reference line carry the same dict)."""
    return {"workload": DECODE_WORKLOAD, "d_model": D_MODEL, "r": R, "d_ff": D_FF, "k": K, "tokens_per_step": 1,
            "weights": WEIGHTS_RECIPE,
            "l2": f"inputs larger than L2: steps cycle over {N_COPIES} weight copies "
                  f"({N_COPIES * 2 * D_MODEL * D_FF * 2 / 1e9:.2f} GB)",
            "parallelism": f"replicas x{world}"}


def oracle_baseline(seconds: float, T_sample: int = 1):
    """fp64 oracle on host cores: decode tokens/s per layer on the same synthetic layer."""
    import numpy as np

    import oracle
    from activation_sparse_transformer_predictor_b200 import synthetic
    w = synthetic.ffn_layer(D_MODEL, R, D_FF)
    bits = {k: synthetic.bf16_bits(v) for k, v in w.items()}
    cores = oracle.max_threads()
    batch = max(1, cores)
    done = 0
    t0 = time.perf_counter()
    layer_seed = 0
    while time.perf_counter() - t0 < seconds:
        q = synthetic.bf16_bits(synthetic.tokens(batch, D_MODEL, layer=1000 + layer_seed))
        oracle.spark_ffn(q, bits["K1"], bits["K2"], bits["V"], R, K, n_threads=cores)
        done += batch
        layer_seed += 1
    el = time.perf_counter() - t0
    return {"value": done / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} decode tokens (batches of {batch}, one per OpenMP thread) on one "
                      f"Gemma-shaped layer, {el:.1f} s wall"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from activation_sparse_transformer_predictor_b200 import synthetic
    w = synthetic.ffn_layer(D_MODEL, R, D_FF)
    bits = {k: synthetic.bf16_bits(v) for k, v in w.items()}
    cores = oracle.max_threads()
    q = synthetic.bf16_bits(synthetic.tokens(max(1, cores), D_MODEL))
    for _ in range(args.warmup):
        oracle.spark_ffn(q[:1], bits["K1"], bits["K2"], bits["V"], R, K, n_threads=1)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.spark_ffn(q[i % len(q):i % len(q) + 1], bits["K1"], bits["K2"], bits["V"], R, K, n_threads=1)
    el = time.perf_counter() - t0
    v = args.steps / el
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(args.gpus),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"{args.steps} decode tokens, one per step, single thread"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def run_case(args):
    """Plain launches of one workload (for ncu captures): warmup calls, then `steps` calls."""
    import torch

    import activation_sparse_transformer_predictor_b200 as spark
    from activation_sparse_transformer_predictor_b200 import synthetic
    dev = torch.device("cuda", 0)
    if args.case == "attention":
        import math as _m
        caches = []
        for c in range(4):
            host = synthetic.attention_inputs(8, 4, 4096, 256, layer=c)
            caches.append({n: t.to(dev) for n, t in host.items()})
        aout = torch.empty_like(caches[0]["q"])
        fn = lambda i: spark.attention_decode(caches[i % 4]["q"], caches[i % 4]["K"], caches[i % 4]["V"], 128, 256,
                                              scale=1.0 / _m.sqrt(256), out=aout)
        unit = "attention 8/4 heads x 4096 positions"
    elif args.case == "predictor":
        w = synthetic.ffn_layer(D_MODEL, R, D_FF)
        k1s = [w["K1"].to(dev)] + [w["K1"].to(dev).clone() for _ in range(3)]
        q = synthetic.tokens(args.tokens, D_MODEL, layer=1).to(dev)
        xo = torch.empty((args.tokens, D_FF), dtype=torch.float32, device=dev)
        fn = lambda i: spark.ffn_predictor(q, k1s[i % len(k1s)], out=xo)
        unit = f"predictor GEMM, T={args.tokens}"
    elif args.case == "topk_causal":
        rows, d, k = 8 * 4096, 4096, 256
        x = torch.randn(rows, d, device=dev, generator=torch.Generator(device=dev).manual_seed(5))
        out = torch.empty_like(x)
        fn = lambda i: spark.stat_topk_soft_threshold_causal(x, k, n_q=4096, out=out)
        unit = f"causal rows {rows} x {d}"
    elif args.case == "huber_bwd":
        rows, d, k = 8 * 4096, 4096, 256
        x = torch.randn(rows, d, device=dev, generator=torch.Generator(device=dev).manual_seed(5))
        g = torch.randn(rows, d, device=dev, generator=torch.Generator(device=dev).manual_seed(6))
        gx = torch.empty_like(x)
        fn = lambda i: spark.stat_topk_huber_backward(x, g, k, 0.25, grad_x=gx)
        unit = f"Huber backward rows {rows} x {d}"
    elif args.case == "noalloc":
        # the single-launch fused kernel at one token, through the allocation-free entry point
        from activation_sparse_transformer_predictor_b200 import _binding
        w = synthetic.ffn_layer(D_MODEL, R, D_FF)
        copies = [{n: t.to(dev) for n, t in w.items()}]
        copies += [{n: t.clone() for n, t in copies[0].items()} for _ in range(3)]
        q = synthetic.tokens(1, D_MODEL).to(dev)[0].contiguous()
        out = torch.empty_like(q)
        L = _binding.lib()

        def fn(i):
            c = copies[i % len(copies)]
            rc = L.spark_ffn_forward_noalloc(q.data_ptr(), c["K1"].data_ptr(), c["K2"].data_ptr(), c["V"].data_ptr(),
                                             D_MODEL, R, D_FF, K, out.data_ptr(), _binding.stream_handle())
            if rc != 0:
                raise _binding.SparkError("spark_ffn_forward_noalloc", rc)
        unit = "no-allocation decode (fused kernel), T=1"
    elif args.case == "topk":
        rows, d, k = 8 * 4096, 4096, 256
        x = torch.randn(rows, d, device=dev, generator=torch.Generator(device=dev).manual_seed(5))
        out = torch.empty_like(x)
        fn = lambda i: spark.stat_topk_soft_threshold(x, k, out=out)
        unit = f"rows {rows} x {d}"
    else:
        w = synthetic.ffn_layer(D_MODEL, R, D_FF)
        copies = [{n: t.to(dev) for n, t in w.items()}]
        if args.case == "decode":
            copies += [{n: t.clone() for n, t in copies[0].items()} for _ in range(N_COPIES - 1)]
            q = synthetic.tokens(1, D_MODEL).to(dev)[0].contiguous()
        else:
            q = synthetic.tokens(args.tokens, D_MODEL, layer=1).to(dev)
        out = torch.empty_like(q)
        fn = lambda i: spark.ffn_forward(q, copies[i % len(copies)]["K1"], copies[i % len(copies)]["K2"],
                                         copies[i % len(copies)]["V"], K, out=out)
        unit = f"{args.case}, T={1 if args.case == 'decode' else args.tokens}"
    for i in range(args.warmup):
        fn(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        fn(args.warmup + i)
    e1.record()
    e1.synchronize()
    assert spark.query_status() == 0
    print(f"case {unit}: {e0.elapsed_time(e1) * 1e3 / args.steps:.2f} us per call over {args.steps} calls")


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.case is not None:
        run_case(args)
        return
    import torch

    import activation_sparse_transformer_predictor_b200 as spark
    from activation_sparse_transformer_predictor_b200 import _binding, synthetic

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = peaks()

    # ---------------- inputs: one synthetic layer, cloned into N_COPIES distinct buffers
    w = synthetic.ffn_layer(D_MODEL, R, D_FF)
    base = {k: v.to(dev) for k, v in w.items()}
    copies = [{k: v.clone() for k, v in base.items()} for _ in range(N_COPIES)]
    q1 = synthetic.tokens(1, D_MODEL).to(dev)[0].contiguous()
    out1 = torch.empty_like(q1)
    L = _binding.lib()

    # measured active count on this input (deterministic), for the algorithmic byte count
    dbg = spark.ffn_forward_debug(q1, base["K1"], base["K2"], base["V"], K)
    m_active = int(dbg["active"].sum().item())
    bytes_per_token = D_FF * R * 2 + m_active * ((D_MODEL - R) + D_MODEL) * 2 + 2 * D_MODEL * 2

    def decode_step(c):
        def f():
            st = _binding.stream_handle()
            rc = L.spark_ffn_forward(q1.data_ptr(), c["K1"].data_ptr(), c["K2"].data_ptr(), c["V"].data_ptr(),
                                     D_MODEL, R, D_FF, K, out1.data_ptr(), st)
            if rc != 0:
                raise _binding.SparkError("spark_ffn_forward", rc)
        return f

    fns = [decode_step(c) for c in copies] * 8  # 128 calls per graph
    # the score kernel of each call streams its K1 slice while the previous
    # call's gather and reduce kernels run (programmatic dependent launch)
    spark.set_weight_overlap(True)
    with ClockSampler(local) as clk:
        ms_step = time_exact_steps(fns, args.steps, args.warmup, world)
        # the same calls over a longer graph (2560 calls): a steadier figure for the notes, and
        # enough decode load around the timed steps for the clock samples
        ms_long, _ = time_graph(fns, 2560, args.warmup, world)
        ms_long = max_over_ranks(ms_long, world)
    n_timed = args.steps
    assert spark.query_status() == 0
    # the same calls without the overlap
    spark.set_weight_overlap(False)
    ms_plain, _ = time_graph(fns, min(args.steps, 1280), args.warmup, world)
    ms_plain = max_over_ranks(ms_plain, world)
    assert spark.query_status() == 0
    tok_s = whole_job_rate(1, ms_step, world)
    achieved_gbs = bytes_per_token / (ms_step * 1e-3) / 1e9

    # ---------------- end to end through the C ABI with host buffers (spark_ffn_forward_host):
    # every step copies q from pinned host memory to the device, runs the forward and copies out back
    q_host = synthetic.tokens(1, D_MODEL)[0].contiguous().pin_memory()
    out_host = torch.empty_like(q_host).pin_memory()
    e2e_steps = min(args.steps, 2000)
    spark.set_weight_overlap(True)
    sh = _binding.stream_handle()
    wptr = [(c["K1"].data_ptr(), c["K2"].data_ptr(), c["V"].data_ptr()) for c in copies]
    qh, oh = q_host.data_ptr(), out_host.data_ptr()
    fh = L.spark_ffn_forward_host

    def host_steps(n):
        for i in range(n):
            k1, k2, v = wptr[i % N_COPIES]
            rc = fh(qh, k1, k2, v, 1, D_MODEL, R, D_FF, K, oh, sh)
            if rc != 0:
                raise _binding.SparkError("spark_ffn_forward_host", rc)

    host_steps(max(args.warmup, 3))
    torch.cuda.synchronize()
    barrier_sync(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    host_steps(e2e_steps)
    e1.record()
    barrier_sync(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    torch.cuda.synchronize()
    # the host buffer holds the last step's output: the device entry point's bits
    assert torch.equal(out_host, spark.ffn_forward(q_host.to(dev), base["K1"], base["K2"], base["V"], K).cpu())
    # the same through the public Python API (torch copies around spark.ffn_forward), for comparison
    q_dev = torch.empty_like(q1)
    for i in range(max(args.warmup, 3)):
        q_dev.copy_(q_host, non_blocking=True)
        o = spark.ffn_forward(q_dev, copies[i % N_COPIES]["K1"], copies[i % N_COPIES]["K2"],
                              copies[i % N_COPIES]["V"], K, out=out1)
        out_host.copy_(o, non_blocking=True)
    barrier_sync(world)
    e0.record()
    for i in range(e2e_steps):
        c = copies[i % N_COPIES]
        q_dev.copy_(q_host, non_blocking=True)
        o = spark.ffn_forward(q_dev, c["K1"], c["K2"], c["V"], K, out=out1)
        out_host.copy_(o, non_blocking=True)
    e1.record()
    barrier_sync(world)
    py_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    spark.set_weight_overlap(False)

    also = {
        "decode_T1_graph_of_2560_calls": {
            "tokens_per_s": whole_job_rate(1, ms_long, world), "us_per_call": ms_long * 1e3,
            "frac_of_hbm_peak": bytes_per_token / (ms_long * 1e-3) / 1e9 / hbm_gbs,
            "note": "the headline calls timed over a longer graph"},
        "decode_T1_without_weight_overlap": {
            "tokens_per_s": whole_job_rate(1, ms_plain, world), "us_per_call": ms_plain * 1e3,
            "frac_of_hbm_peak": bytes_per_token / (ms_plain * 1e-3) / 1e9 / hbm_gbs,
            "note": "score kernel launched after the previous call completes"},
    }
    if not args.no_extra:
        also.update(extra_workloads(spark, synthetic, torch, dev, base, copies, world, args, hbm_gbs))

    if rank == 0:
        cpu = oracle_baseline(args.cpu_seconds) if world == 1 or rank == 0 else None
        traffic = profile_traffic("ffn_decode_pg_gemma_T1.txt", DECODE_SOURCES)
        line = {
            "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": n_timed,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(world),
            "notes": {"active_neurons": m_active,
                      "timing": f"one CUDA graph of exactly {n_timed} library calls, replayed once between CUDA "
                                "events on the launch stream (after an untimed replay)",
                      "weight_overlap": "on (spark_set_weight_overlap): each call's score kernel streams K1 "
                                        "while the previous call's gather and reduce kernels run"},
            "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": achieved_gbs / hbm_gbs, "traffic": traffic, "peak_source": peak_src,
                         "frac_vs_8TBs": achieved_gbs / 8000.0,
                         "kernel": "decode_score_kernel + decode_gather_kernel + decode_reduce_kernel (one programmatic chain per step)",
                         "duration": "graph replay time per step (three kernels, gaps included)",
                         "algorithmic_bytes_per_launch": bytes_per_token},
            "cpu_baseline": cpu,
            "e2e": {"value": whole_job_rate(1, e2e_ms, world), "unit": "tokens/s", "h2d_bytes_per_step": D_MODEL * 2,
                    "d2h_bytes_per_step": D_MODEL * 2, "steps": e2e_steps,
                    "path": "C ABI with host buffers per step (spark_ffn_forward_host, weight overlap on): the "
                            "first kernel reads q from the pinned host buffer, the reduce kernel stores out into "
                            "the pinned host buffer; CUDA events around the steps",
                    "python_api_path": "torch pinned H2D copy, spark.ffn_forward, D2H copy per step",
                    "python_api_tokens_per_s": whole_job_rate(1, py_ms, world)},
            "gpu_launches": 3 * n_timed,  # score, gather and reduce kernel per timed call
            "clocks": clk.summary(),
            "also": also,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def extra_workloads(spark, synthetic, torch, dev, base, copies, world, args, hbm_gbs):
    from activation_sparse_transformer_predictor_b200 import _binding
    L = _binding.lib()
    bf16_tflops = peaks()[1]  # burst: each prefill call is timed by itself
    res = {}
    # mean number of active neurons per token on these inputs (for the method's own FLOP count)
    qm = synthetic.tokens(64, D_MODEL, layer=1).to(dev)
    m_mean = float(spark.ffn_forward_debug(qm, base["K1"], base["K2"], base["V"], K)["active"].sum().item()) / 64
    del qm
    # batched prefill, T = 256 and T = 4096 (one layer; whole-call throughput: predictor GEMM, theta,
    # gate GEMM, output GEMM and split-K reduce)
    for T, reps in ((16, 80), (64, 80), (256, 40), (1024, 16), (4096, 8)):
        q = synthetic.tokens(T, D_MODEL, layer=1).to(dev)
        out = torch.empty_like(q)

        def pre(q=q, out=out, T=T):
            rc = L.spark_ffn_forward_tokens(q.data_ptr(), base["K1"].data_ptr(), base["K2"].data_ptr(),
                                            base["V"].data_ptr(), T, D_MODEL, R, D_FF, K, out.data_ptr(),
                                            _binding.stream_handle())
            if rc != 0:
                raise _binding.SparkError("spark_ffn_forward_tokens", rc)

        ms, n = time_graph([pre] * 4, reps, args.warmup, world)
        ms = max_over_ranks(ms, world)
        # the method's own work: predictor 2 r d_ff, then 2 (d - r) + 2 d per active neuron
        aflops = T * (2.0 * R * D_FF + 2.0 * m_mean * (2 * D_MODEL - R))
        # what the kernels execute: predictor + gate (a) + two-part output, dense over the tile union
        xflops = 2.0 * T * D_FF * (R + (D_MODEL - R) + 2 * D_MODEL)
        # algorithmic bytes: K1 once, the expected union of the tokens' active K2 / V rows, q and out
        union = D_FF * (1.0 - (1.0 - K / D_FF) ** T)
        abytes = D_FF * R * 2 + union * ((D_MODEL - R) + D_MODEL) * 2 + 2 * T * D_MODEL * 2
        res[f"prefill_T{T}"] = {"tokens_per_s": whole_job_rate(T, ms, world), "ms_per_call": ms,
                                "algorithmic_tflops": aflops / (ms * 1e-3) / 1e12,
                                "frac_of_bf16_peak": aflops / (ms * 1e-3) / 1e12 / bf16_tflops,
                                "executed_tflops": xflops / (ms * 1e-3) / 1e12,
                                "executed_frac_of_bf16_peak": xflops / (ms * 1e-3) / 1e12 / bf16_tflops,
                                "mean_active_per_token": m_mean,
                                "algorithmic_bytes": abytes,
                                "frac_of_hbm_peak": abytes / (ms * 1e-3) / 1e9 / hbm_gbs,
                                "note": "one layer; whole call (three GEMMs, plus the threshold and split-K reduce "
                                        "kernels where they run separately); the masked products run as "
                                        "dense 128-token tiles (the union of per-token active sets covers "
                                        "~every neuron); per-kernel live spans are in the prefill profile"}
        del q, out
    # the predictor GEMM alone (spark_ffn_predictor: x = K1^T q[:r]), cycling over the 16 K1 copies
    for T in (256, 1024, 4096):
        q = synthetic.tokens(T, D_MODEL, layer=1).to(dev)
        xo = torch.empty((T, D_FF), dtype=torch.float32, device=dev)

        def pred(c, q=q, xo=xo, T=T):
            def f():
                rc = L.spark_ffn_predictor(q.data_ptr(), c["K1"].data_ptr(), T, D_MODEL, R, D_FF, xo.data_ptr(),
                                           _binding.stream_handle())
                if rc != 0:
                    raise _binding.SparkError("spark_ffn_predictor", rc)
            return f

        ms, n = time_graph([pred(c) for c in copies], 16 * max(1, 64 // (T // 256)), args.warmup, world)
        ms = max_over_ranks(ms, world)
        tf = 2.0 * T * R * D_FF / (ms * 1e-3) / 1e12
        res[f"predictor_gemm_T{T}"] = {"ms_per_call": ms, "tflops": tf, "frac_of_bf16_peak": tf / bf16_tflops,
                                       "peak": bf16_tflops, "peak_kind": "measured bf16 burst",
                                       "traffic": profile_traffic("umma_gemm_predictor_gemma_T256.txt", PRED_SOURCES)
                                       if T == 256 else None,
                                       "note": "GEMM 1 alone (tcgen05, fp32 x stored row-major), 2 T r d_ff flops "
                                               "per call, 16 K1 copies cycled (340 MB > L2)"}
        del q, xo
    # 26-layer decode stack (Gemma-2-2B depth), one token, residual + RMSNorm between layers
    import ctypes
    n_layers = 26
    layers = []
    for l in range(n_layers):
        wl = synthetic.ffn_layer(D_MODEL, R, D_FF, layer=l)
        layers.append(tuple(wl[n].to(dev) for n in ("K1", "K2", "V")))
    ptrs = [(ctypes.c_void_p * n_layers)(*[t[j].data_ptr() for t in layers]) for j in range(3)]
    h0 = synthetic.residual(1, D_MODEL)[0].to(dev)
    h = h0.clone()

    def stack():
        h.copy_(h0)
        rc = L.spark_ffn_decode_stack(h.data_ptr(), h.data_ptr(), ptrs[0], ptrs[1], ptrs[2], n_layers, D_MODEL, R,
                                      D_FF, K, 1e-6, None, None, _binding.stream_handle())
        if rc != 0:
            raise _binding.SparkError("spark_ffn_decode_stack", rc)

    ms, n = time_graph([stack] * 2, 20, args.warmup, world)
    ms = max_over_ranks(ms, world)
    stack_bytes = n_layers * (D_FF * R * 2 + 737 * (D_MODEL - R + D_MODEL) * 2 + 2 * D_MODEL * 2)
    res["stack_26_layers_T1"] = {"tokens_per_s": whole_job_rate(1, ms, world), "us_per_token": ms * 1e3,
                                 "us_per_layer": ms * 1e3 / n_layers,
                                 "achieved_GBs": stack_bytes / (ms * 1e-3) / 1e9,
                                 "frac_of_hbm_peak": stack_bytes / (ms * 1e-3) / 1e9 / hbm_gbs,
                                 "note": "26 distinct layers (2.21 GB of weights > L2): one score, gather and reduce "
                                         "kernel per layer, each layer's K1 streamed under the previous layer's "
                                         "gather and reduce; the reduce kernel writes h + out and the next score "
                                         "kernel forms q = RMSNorm(h); bytes counted as K1 + 737 active K2/V rows + "
                                         "q/out per layer"}
    del layers
    # Spark Attention, one decoding position: 8 query heads over 4 key/value heads, d_head 256 split
    # r = 128, 4096 cached positions, k_attn = 256 (Gemma-2-2B-like heads), 16 distinct caches cycled
    import math as _m
    H, KV, NC, DH, RA, KA = 8, 4, 4096, 256, 128, 256
    caches = []
    for c in range(16):
        host = synthetic.attention_inputs(H, KV, NC, DH, layer=c)
        caches.append({n: t.to(dev) for n, t in host.items()})
    aout = torch.empty_like(caches[0]["q"])

    def attn(c):
        def f():
            rc = L.spark_attention_decode(c["q"].data_ptr(), c["K"].data_ptr(), c["V"].data_ptr(), H, KV, NC, DH, RA,
                                          KA, 1.0 / _m.sqrt(DH), aout.data_ptr(), _binding.stream_handle())
            if rc != 0:
                raise _binding.SparkError("spark_attention_decode", rc)
        return f

    ms, n = time_graph([attn(c) for c in caches] * 4, 640, args.warmup, world)
    ms = max_over_ranks(ms, world)
    abytes = KV * NC * RA * 2 + H * KA * ((DH - RA) + DH) * 2 + 2 * H * DH * 2
    res["spark_attention_decode_8x4096"] = {
        "calls_per_s": whole_job_rate(1, ms, world), "us_per_call": ms * 1e3, "achieved_GBs": abytes / (ms * 1e-3) / 1e9,
        "frac_of_hbm_peak": abytes / (ms * 1e-3) / 1e9 / hbm_gbs, "algorithmic_bytes_per_call": abytes,
        "note": "one launch, one 16-CTA cluster per query head; bytes = predictor parts of all cached keys + "
                "K2 parts and value rows of ~256 selected keys per head + q/out; 16 caches (75 MB) cycled"}
    del caches
    # stat top-k on 8 x 4096 x 4096 fp32 rows, k = 256
    rows, d, k = 8 * 4096, 4096, 256
    xs = torch.randn(rows, d, device=dev, generator=torch.Generator(device=dev).manual_seed(5))
    xo = torch.empty_like(xs)

    def tk():
        rc = L.stat_topk_soft_threshold(xs.data_ptr(), rows, d, k, xo.data_ptr(), _binding.stream_handle())
        if rc != 0:
            raise _binding.SparkError("stat_topk_soft_threshold", rc)

    ms, n = time_graph([tk] * 2, 20, args.warmup, world)
    ms = max_over_ranks(ms, world)
    gbs = rows * d * 8 / (ms * 1e-3) / 1e9
    res["stat_topk_32768x4096"] = {"rows_per_s": whole_job_rate(rows, ms, world), "ms_per_call": ms, "achieved_GBs": gbs,
                                   "frac_of_hbm_peak": gbs / hbm_gbs,
                                   "traffic": profile_traffic("stat_topk_32768x4096.txt", TOPK_SOURCES),
                                   "note": "512 MiB read + 512 MiB written per call (> L2)"}
    # the same rows under a causal mask (square scores of one 4096-token prompt per head): row i of a head
    # sees i + 1 keys, rows with at most k of them pass through
    tc = torch.empty(rows, dtype=torch.float32, device=dev)

    def tkc():
        rc = L.stat_topk_soft_threshold_causal(xs.data_ptr(), rows, d, k, 4096, 0, xo.data_ptr(), tc.data_ptr(),
                                               _binding.stream_handle())
        if rc != 0:
            raise _binding.SparkError("stat_topk_soft_threshold_causal", rc)

    ms, n = time_graph([tkc] * 2, 20, args.warmup, world)
    ms = max_over_ranks(ms, world)
    cbytes = 8 * (4096 * 4097 // 2) * 4 + rows * d * 4 + rows * 4  # visible entries read, all written, theta
    gbs = cbytes / (ms * 1e-3) / 1e9
    res["stat_topk_causal_32768x4096"] = {"rows_per_s": whole_job_rate(rows, ms, world), "ms_per_call": ms,
                                          "achieved_GBs": gbs, "frac_of_hbm_peak": gbs / hbm_gbs,
                                          "algorithmic_bytes": cbytes,
                                          "traffic": profile_traffic("stat_topk_causal_32768x4096.txt", TOPK_SOURCES),
                                          "note": "8 heads x 4096 queries x 4096 keys, causal: the visible "
                                                  "entries (268 MB) read, every entry (537 MB) written"}
    # backward of the Huber-smoothed operator on the same rows (delta = 0.25): x and the upstream
    # gradient read, the gradient written, 12 bytes per element
    gs = torch.randn(rows, d, device=dev, generator=torch.Generator(device=dev).manual_seed(6))

    def hb():
        rc = L.stat_topk_huber_backward(xs.data_ptr(), gs.data_ptr(), rows, d, k, 0.25, xo.data_ptr(),
                                        _binding.stream_handle())
        if rc != 0:
            raise _binding.SparkError("stat_topk_huber_backward", rc)

    ms, n = time_graph([hb] * 2, 20, args.warmup, world)
    ms = max_over_ranks(ms, world)
    hbytes = rows * d * 12
    gbs = hbytes / (ms * 1e-3) / 1e9
    res["stat_topk_huber_backward_32768x4096"] = {
        "rows_per_s": whole_job_rate(rows, ms, world), "ms_per_call": ms, "achieved_GBs": gbs,
        "frac_of_hbm_peak": gbs / hbm_gbs, "algorithmic_bytes": hbytes,
        "traffic": profile_traffic("stat_topk_huber_backward_32768x4096.txt", TOPK_SOURCES),
        "note": "gradient of the Huber-smoothed statistical top-k (delta 0.25): x and grad_out read, grad_x "
                "written (1.61 GB per call)"}
    del gs
    return res


if __name__ == "__main__":
    main()
