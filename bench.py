"""Benchmark: int4 g128 batch-1 GEMV weight GB/s on the Qwen2.5-0.5B-shaped decode set.

One step = one decoded token's worth of linear layers: all 169 matrices of the set
(24 layers x q, k, v, o, gate, up, down + the 151936-row lm_head, 493,961,216 int4 g128
weights = 262.42 MB of codes + scales + zeros) in one wq_linear_set launch. `value` is
weight bytes per second with everything resident in HBM; `e2e` is the same through the
public API with the activations copied in from pinned host memory and the outputs
copied back inside the timed region. Secondary rows (lm_head formats, quantiser,
batch sweep, M=512 prefill GEMM) are reported under "rows".

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]
Under torchrun (N > 1) every rank runs an independent replica on its own GPU (the
decode set has no data-path exchange); rank 0 prints the JSON line with the
max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_weight_quantized_unpack_b200 import synth, workloads  # noqa: E402

METRIC = "int4 g128 batch-1 GEMV weight GB/s (% of HBM peak); M=512 GEMM TFLOPS"
INT4_BYTES_PER_WEIGHT = 0.5 + 4 / 128  # codes + fp16 scale + fp16 zero per 128 weights
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one gemv_stream_kernel launch
# over the 0.5B decode set, from one ncu capture of the kernel as it is now (None when the
# kernel changed after the capture); TRAFFIC_SOURCE names that capture
GEMV_TRAFFIC_BYTES = 263556352 + 3634432
TRAFFIC_SOURCE = ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --clock-control none "
                  "-k regex:gemv_stream -s 10 -c 1 python bench.py --steps 20 --warmup 5 --no-rows --quick")
L2_BYTES = 126 * 1000 * 1000


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return rank, ws


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(v, ws):
    """The largest of the ranks' values (every rank gets it): the job's step time."""
    if ws == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_gbs(nbytes_per_rank, ms_max, ws):
    """Whole-job rate in GB/s: each of ws ranks moved nbytes_per_rank in one step, and the
    job's step lasts as long as its slowest rank's (ms_max)."""
    return nbytes_per_rank * ws / ms_max / 1e6


class Clocks:
    """nvidia-smi sampling of SM clock and throttle reasons while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"wq_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            idx = str(torch.cuda.current_device())
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                idx = vis.split(",")[torch.cuda.current_device()]
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", idx, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------

def build_set(widx, copies, fmt="int4"):
    """Quantise `copies` independent copies of a workload's layer set on the GPU."""
    from bit_weight_quantized_unpack_b200 import wq
    wl = workloads.WORKLOADS[widx]
    mats = workloads.workload_mats(widx)
    K_tot = sum(m.K for m in mats)
    N_tot = sum(m.N for m in mats)
    sets = []
    for cidx in range(copies):
        x_all = torch.empty(K_tot, dtype=torch.float16, device="cuda")
        y_all = torch.empty(N_tot, dtype=torch.float16, device="cuda")
        ent, ko, no = [], 0, 0
        for i, m in enumerate(mats):
            seed = synth.sub_seed(wl["seed"] + 7919 * cidx, i, 0)
            W = synth.weights(m.N, m.K, wl["sigma"], seed, device="cuda")
            c, s, z = wq.alloc_packed(m.N, m.K, fmt)
            wq.wq_quantize(W, m.N, m.K, fmt, 32 if fmt == "int4h" else 128, c, s, z)
            del W
            x = x_all[ko:ko + m.K]
            x.copy_(synth.activations(1, m.K, synth.sub_seed(wl["seed"], i, 1), device="cuda")[0])
            ent.append((c, s, z, x, y_all[no:no + m.N], m.N, m.K))
            ko += m.K
            no += m.N
        sets.append({"desc": wq.make_linear_set(ent), "count": len(ent), "ent": ent,
                     "x_all": x_all, "y_all": y_all})
    torch.cuda.synchronize()
    weights = sum(m.N * m.K for m in mats)
    return sets, weights, K_tot, N_tot


def time_steps(step, steps, warmup, ws, clocks=None):
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(ws)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = clocks if clocks is not None else _Null()
    with ctx:
        torch.cuda.synchronize()
        ev0.record()
        for i in range(steps):
            step(i)
        ev1.record()
        torch.cuda.synchronize()
    barrier(ws)
    return ev0.elapsed_time(ev1) / steps  # ms per step on this rank


def step_stats(step, n, warm=3):
    """Per-step device times from one CUDA event between consecutive steps on the launching
    stream: median, p10 and p90 in ms (the pages' timing hygiene: median with p10 / p90)."""
    for i in range(warm):
        step(i)
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    evs[0].record()
    for i in range(n):
        step(i)
        evs[i + 1].record()
    torch.cuda.synchronize()
    d = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(n))

    def q(f):
        return d[min(n - 1, int(f * (n - 1) + 0.5))]
    return {"median_ms": q(0.5), "p10_ms": q(0.1), "p90_ms": q(0.9), "n": n}


def row_stats(step, n, nbytes, pk):
    """A bench row: per-launch median / p10 / p90 (ms) and the median's GB/s of nbytes."""
    st = step_stats(step, n)
    gbs = nbytes / st["median_ms"] / 1e6
    return {"ms": st["median_ms"], "p10_ms": st["p10_ms"], "p90_ms": st["p90_ms"], "GBps": gbs,
            "frac_hbm": gbs / pk["hbm_gbs"]}


def graph_of(calls):
    """A CUDA graph replaying `calls` (each enqueues work on torch's current stream); every
    call runs once before capture, so that the library's one-time set-up is done."""
    for f in calls:
        f()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in calls:
            f()
    torch.cuda.synchronize()
    return g


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        pass


def bench_rows(args, pk):
    """Secondary measurements of the other hot-path rows (1 GPU)."""
    from bit_weight_quantized_unpack_b200 import wq
    rows = {}
    N, K = 151936, 896
    wl = workloads.WORKLOADS[2]
    # lm_head alone, each format; rotating copies of the packed head so that one pass over
    # them reads at least 3 x L2 from HBM
    n_launch = 200 if not args.quick else 20
    for fmt in ("int4", "int4h", "int3", "int2", "ternary"):
        nb = wq.wq_codes_bytes(fmt, N, K) + wq.wq_scale_bytes(fmt, N, K) + wq.wq_zero_bytes(fmt, N, K)
        n_copies = max(4, -(-3 * L2_BYTES // nb))
        copies = []
        for cidx in range(1):
            W = synth.weights_with_outliers(N, K, wl["sigma"], synth.sub_seed(wl["seed"] + cidx, 0, 0),
                                            wl["outlier_frac"], wl["outlier_gain"], device="cuda")
            c, s, z = wq.alloc_packed(N, K, fmt)
            if fmt == "int4" and cidx == 0:
                # quantiser throughput (row a1/a2 measured on the int4 path)
                ev0, ev1 = torch.cuda.Event(True), torch.cuda.Event(True)
                wq.wq_quantize(W, N, K, fmt, 128, c, s, z)
                ev0.record()
                for _ in range(5):
                    wq.wq_quantize(W, N, K, fmt, 128, c, s, z)
                ev1.record()
                torch.cuda.synchronize()
                ms = ev0.elapsed_time(ev1) / 5
                rows["quantize_int4_lm_head"] = {"ms": ms, "W_GBps": N * K * 4 / ms / 1e6}
            wq.wq_quantize(W, N, K, fmt, 32 if fmt == "int4h" else 128, c, s, z)
            del W
            copies.append((c, s, z))
        # the other copies: the same bytes at other addresses (the stream's cost depends on
        # where the bytes come from, not on their values)
        copies += [tuple(None if t is None else t.clone() for t in copies[0]) for _ in range(n_copies - 1)]
        x = synth.activations(1, K, 99, device="cuda")[0]
        y = torch.empty(N, dtype=torch.float16, device="cuda")

        def step(i, copies=copies, fmt=fmt):
            c, s, z = copies[i % len(copies)]
            wq.wq_gemv(x, c, s, z, fmt, N, K, y)
        rows[f"gemv_lm_head_{fmt}"] = {**row_stats(step, n_launch, nb, pk), "copies": n_copies,
                                       "working_set_MB": n_copies * nb / 1e6}
        if fmt == "int4":
            # fused greedy pick: product and argmax in one launch, y not stored
            ws = torch.zeros(wq.wq_argmax_workspace_bytes(), dtype=torch.uint8, device="cuda")
            am = torch.zeros(1, dtype=torch.int32, device="cuda")

            def step_am(i, copies=copies):
                c, s, z = copies[i % len(copies)]
                wq.wq_gemv_argmax(x, c, s, z, "int4", N, K, None, am, ws, ws.numel())
            rows["gemv_argmax_lm_head_int4"] = row_stats(step_am, n_launch, nb, pk)
            # head rescoring: int4 head, top 8 candidates recomputed from an fp16 head copy
            topk = 8
            w16 = synth.weights_with_outliers(N, K, wl["sigma"], synth.sub_seed(wl["seed"], 0, 0),
                                              wl["outlier_frac"], wl["outlier_gain"], device="cuda").half()
            wsr = torch.empty(wq.wq_rescore_workspace_bytes(N, topk), dtype=torch.uint8, device="cuda")
            cand = torch.empty(topk, dtype=torch.int32, device="cuda")
            cl = torch.empty(topk, dtype=torch.float32, device="cuda")
            tok = torch.empty(1, dtype=torch.int32, device="cuda")

            def step_rs(i, copies=copies):
                c, s, z = copies[i % len(copies)]
                wq.wq_gemv_rescore(x, c, s, z, "int4", w16, N, K, topk, y, cand, cl, tok, wsr, wsr.numel())
            rows["gemv_rescore_lm_head_int4"] = {**row_stats(step_rs, n_launch, nb, pk), "topk": topk,
                                                 "launches": 3}
            del w16
        del copies
        torch.cuda.empty_cache()
    rows.update(bench_int4h_set(args, pk))
    rows.update(bench_config0(args, pk))
    rows.update(bench_per_matrix_graphs(args, pk))
    rows.update(bench_batch_sweep(args, pk))
    rows.update(bench_7b_set(args, pk))
    return rows


def bench_config0(args, pk):
    """The single 896 x 896 int4 matrix at batch 1, one wq_gemv per product, over enough
    copies (C) that one pass reads 3 x L2 from HBM. The launches of one pass are replayed as a
    CUDA graph (back to back on the GPU, no host gaps): per launch = pass / C."""
    from bit_weight_quantized_unpack_b200 import wq
    wl = workloads.WORKLOADS[0]
    N = K = 896
    nb = wq.wq_codes_bytes("int4", N, K) + wq.wq_scale_bytes("int4", N, K) + wq.wq_zero_bytes("int4", N, K)
    copies = 3 * L2_BYTES // nb + 1
    W = synth.weights(N, K, wl["sigma"], wl["seed"], device="cuda")
    c0, s0, z0 = wq.alloc_packed(N, K, "int4")
    wq.wq_quantize(W, N, K, "int4", 128, c0, s0, z0)
    C = c0.repeat(copies, 1) if c0.dim() == 2 else c0.view(1, -1).repeat(copies, 1)
    S = s0.view(1, -1).repeat(copies, 1)
    Z = z0.view(1, -1).repeat(copies, 1)
    x = synth.activations(1, K, synth.sub_seed(wl["seed"], 0, 1), device="cuda")[0]
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    g = graph_of([lambda i=i: wq.wq_gemv(x, C[i], S[i], Z[i], "int4", N, K, y) for i in range(copies)])
    st = step_stats(lambda i: g.replay(), 20 if not args.quick else 5)
    per = st["median_ms"] / copies
    out = {"gemv_single_896_int4": {"us_per_launch": per * 1e3, "p10_us": st["p10_ms"] / copies * 1e3,
                                    "p90_us": st["p90_ms"] / copies * 1e3, "GBps": nb / per / 1e6,
                                    "frac_hbm": nb / per / 1e6 / pk["hbm_gbs"], "copies": copies,
                                    "bytes_per_pass": nb * copies,
                                    "launch": "CUDA graph of one wq_gemv per copy"}}
    del C, S, Z, g
    torch.cuda.empty_cache()
    return out


def bench_per_matrix_graphs(args, pk):
    """One token of the 0.5B set (2 copies) and of the 7B set as a CUDA graph of one wq_gemv per
    matrix, beside the one-launch wq_linear_set (Whetstone README, "The baseline, and where the
    opportunity actually is": dispatch and launch overhead set the baseline's speed)."""
    from bit_weight_quantized_unpack_b200 import wq
    out = {}
    for widx, copies, name in ((1, 2, "qwen05b"), (3, 1, "qwen7b")):
        sets, weights, _, _ = build_set(widx, copies=copies)
        nbytes = weights * INT4_BYTES_PER_WEIGHT
        calls = [lambda e=e: wq.wq_gemv(e[3], e[0], e[1], e[2], "int4", e[5], e[6], e[4])
                 for st in sets for e in st["ent"]]
        g = graph_of(calls)
        gs = step_stats(lambda i: g.replay(), 20 if not args.quick else 5)
        ls = step_stats(lambda i: wq.wq_linear_set(sets[i % copies]["desc"], sets[0]["count"], "int4"),
                        100 if not args.quick else 10)
        per_tok_graph = gs["median_ms"] / copies
        out[f"per_matrix_graph_{name}_int4"] = {
            "ms_per_token": per_tok_graph, "GBps": nbytes / per_tok_graph / 1e6,
            "launches_per_token": len(calls) // copies,
            "grouped_ms_per_token": ls["median_ms"], "grouped_GBps": nbytes / ls["median_ms"] / 1e6,
            "grouped_p10_ms": ls["p10_ms"], "grouped_p90_ms": ls["p90_ms"],
            "speedup_grouped_vs_graph": per_tok_graph / ls["median_ms"]}
        del sets, g, calls
        torch.cuda.empty_cache()
    return out


def bench_int4h_set(args, pk):
    """The 0.5B decode set in hierarchical int4 (group-32 indices against a per-row fp16 pair,
    4.28 bits/weight): one wq_linear_set per token, 2 rotating copies (each larger than L2)."""
    from bit_weight_quantized_unpack_b200 import wq
    sets, weights, _, _ = build_set(1, copies=2, fmt="int4h")
    nbytes = sum(wq.wq_codes_bytes("int4h", m.N, m.K) + wq.wq_scale_bytes("int4h", m.N, m.K) +
                 wq.wq_zero_bytes("int4h", m.N, m.K) for m in workloads.workload_mats(1))

    def step(i):
        s = sets[i % len(sets)]
        wq.wq_linear_set(s["desc"], s["count"], "int4h")
    r = row_stats(step, 500 if not args.quick else 20, nbytes, pk)
    out = {"gemv_set_qwen05b_int4h": {**r, "bytes_per_token": nbytes, "implied_tok_s": 1e3 / r["ms"]}}
    del sets
    torch.cuda.empty_cache()
    return out


def bench_7b_set(args, pk):
    """One decoded token of the Qwen2.5-7B-shaped set (197 int4 matrices, 3.76 GB) in one
    wq_linear_set call; larger than L2 by itself, so one copy suffices."""
    sets, weights, _, _ = build_set(3, copies=1)
    nbytes = weights * INT4_BYTES_PER_WEIGHT
    s = sets[0]
    from bit_weight_quantized_unpack_b200 import wq

    def step(i):
        wq.wq_linear_set(s["desc"], s["count"], "int4")
    r = row_stats(step, 40 if not args.quick else 5, nbytes, pk)
    out = {"gemv_set_qwen7b_int4": {**r, "implied_tok_s": 1e3 / r["ms"]}}
    del sets, s
    torch.cuda.empty_cache()
    return out


def bench_batch_sweep(args, pk, Ms=(2, 4, 8, 16, 32, 64, 512, 2048)):
    """Batch sweep on the 0.5B set: M tokens through all 169 matrices in one wq_linear_set
    call per pass (one skinny-batch launch for 2 <= M <= 32,
    tensor-core launches of up to 80 matrices for larger M). The set's 262 MB exceed L2."""
    from bit_weight_quantized_unpack_b200 import wq
    wl = workloads.WORKLOADS[4]
    mats = workloads.workload_mats(4)
    packed = []
    for i, m in enumerate(mats):
        W = synth.weights(m.N, m.K, wl["sigma"], synth.sub_seed(wl["seed"], i, 0), device="cuda")
        c, s, z = wq.alloc_packed(m.N, m.K, "int4")
        wq.wq_quantize(W, m.N, m.K, "int4", 128, c, s, z)
        del W
        packed.append((c, s, z))
    weights = sum(m.N * m.K for m in mats)
    out = {}
    for M in Ms:
        X = [synth.activations(M, m.K, synth.sub_seed(wl["seed"], i, 1), device="cuda")
             for i, m in enumerate(mats)]
        Y = [torch.empty(M, m.N, dtype=torch.float16, device="cuda") for m in mats]
        desc = wq.make_linear_set([(c, s, z, x, y, m.N, m.K, M)
                                   for (c, s, z), m, x, y in zip(packed, mats, X, Y)])

        def one_pass(i, desc=desc):
            wq.wq_linear_set(desc, len(mats), "int4")
        steps = 20 if M >= 512 else 50
        st = step_stats(one_pass, steps if not args.quick else 5)
        ms = st["median_ms"]
        flops = 2.0 * M * weights
        gbs = weights * INT4_BYTES_PER_WEIGHT / ms / 1e6
        out[f"gemm_set_M{M}"] = {"ms": ms, "p10_ms": st["p10_ms"], "p90_ms": st["p90_ms"],
                                 "TFLOPS": flops / ms / 1e9,
                                 "frac_tensor": flops / ms / 1e9 / pk["bf16_tflops"],
                                 "weight_GBps": gbs, "frac_hbm": gbs / pk["hbm_gbs"],
                                 "kernel": ("gemv_stream_kernel" if M == 1 else
                                            "gemm_skinny_kernel" if M <= 32 else "gemm_tc_int4_kernel"),
                                 "launches_per_pass": (len(mats) + 79) // 80 if M > 32 else 1}
        del X, Y
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    rank, ws = dist_init()
    torch.cuda.init()
    from bit_weight_quantized_unpack_b200 import wq
    pk = peaks()
    sets, weights, K_tot, N_tot = build_set(1, copies=2)
    nbytes = weights * INT4_BYTES_PER_WEIGHT

    def step(i):
        s = sets[i % len(sets)]
        wq.wq_linear_set(s["desc"], s["count"], "int4")

    clocks = Clocks()
    ms = time_steps(step, args.steps, args.warmup, ws, clocks)
    ms_max = max_over_ranks(ms, ws)
    gbs = job_gbs(nbytes, ms_max, ws)  # whole job: every rank processed one set per step

    # e2e: pinned host activations in, outputs out, inside the timed region
    x_host = torch.empty(K_tot, dtype=torch.float16, pin_memory=True)
    x_host.copy_(sets[0]["x_all"].cpu())
    y_host = torch.empty(N_tot, dtype=torch.float16, pin_memory=True)

    def step_e2e(i):
        s = sets[i % len(sets)]
        s["x_all"].copy_(x_host, non_blocking=True)
        wq.wq_linear_set(s["desc"], s["count"], "int4")
        y_host.copy_(s["y_all"], non_blocking=True)

    e2e_steps = max(args.steps // 4, 10)
    ms_e2e = max_over_ranks(time_steps(step_e2e, e2e_steps, args.warmup, ws), ws)
    # per-launch spread of the same step (event between consecutive launches)
    launch_stats = step_stats(step, min(args.steps, 2000))

    rows = bench_rows(args, pk) if (rank == 0 and ws == 1 and not args.no_rows) else {}

    if rank == 0:
        cpu = cpu_baseline(args) if ws == 1 else None
        line = {
            "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16 x int4 -> f32", "data": "synthetic (seeded N(0,0.02^2) weights, N(0,1) fp16 x)",
            "config": {"workload": workloads.WORKLOADS[1]["name"], "matrices": len(sets[0]["ent"]),
                       "weights": weights, "weight_bytes_per_step": nbytes, "batch": 1,
                       "launch": "one wq_linear_set (persistent) per step",
                       "l2": "inputs larger than L2: 2 rotating copies of the set (525 MB)",
                       "parallelism": f"replicas x{ws}"},
            "implied_tok_s": round(1e3 / ms_max, 1),
            "launch_stats": {k: (round(v, 5) if isinstance(v, float) else v) for k, v in launch_stats.items()},
            "frac_of_hbm_peak": round(gbs / ws / pk["hbm_gbs"], 4),
            "roofline": {"bound": "hbm", "achieved": round(nbytes / ms / 1e6, 2),
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(nbytes / ms / 1e6 / pk["hbm_gbs"], 4),
                         "traffic": GEMV_TRAFFIC_BYTES, "traffic_source": TRAFFIC_SOURCE,
                         "kernel": "gemv_stream_kernel<4, 256>", "peak_source": pk["source"]},
            "e2e": {"value": round(job_gbs(nbytes, ms_e2e, ws), 2), "unit": "GB/s",
                    "h2d_bytes_per_step": 2 * K_tot, "d2h_bytes_per_step": 2 * N_tot},
            "gpu_launches": args.steps,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
            "gemm_m512_tflops": (round(rows["gemm_set_M512"]["TFLOPS"], 1) if "gemm_set_M512" in rows else None),
            "gemm_m512_frac_of_tensor_peak": (round(rows["gemm_set_M512"]["frac_tensor"], 4)
                                              if "gemm_set_M512" in rows else None),
            "gemm_m512": ({"TFLOPS": round(rows["gemm_set_M512"]["TFLOPS"], 1),
                           "frac_of_tensor_peak": round(rows["gemm_set_M512"]["frac_tensor"], 4),
                           "peak_tflops": pk["bf16_tflops"],
                           "workload": "qwen2.5-0.5b set, M=512, one wq_linear_set call per pass"}
                          if "gemm_set_M512" in rows else None),
            "rows": rows,
        }
        print(json.dumps(line), flush=True)
    barrier(ws)
    if ws > 1:
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------------------------------------
# oracle arms (host cores)
# ---------------------------------------------------------------------------------------

def _oracle_sample(rows_div=64):
    """A bounded sample of the decode set: every rows_div-th row of every matrix, with the
    oracle's own quantisation done before timing. Returns (list of (x, packed...), weights)."""
    import numpy as np
    from oracle import wq_oracle as O
    wl = workloads.WORKLOADS[1]
    sample, weights = [], 0
    for i, m in enumerate(workloads.workload_mats(1)):
        n = max(1, m.N // rows_div)
        W = synth.weights(n, m.K, wl["sigma"], synth.sub_seed(wl["seed"], i, 0) ^ 0xC0FFEE)
        x = synth.activations(1, m.K, synth.sub_seed(wl["seed"], i, 1))[0].numpy()
        sample.append((x, O.quantize(W.numpy(), "int4"), m.K))
        weights += n * m.K
    return sample, weights


def _threads():
    """Threads of the BLAS pool the oracle's float64 matrix product runs on (its
    dequantisation is single-threaded numpy)."""
    try:
        from threadpoolctl import threadpool_info
        return max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        return 1


def _cpu_fields():
    return {"cores": _threads(), "host_cores": os.cpu_count(),
            "parallel": "float64 matrix product on the BLAS pool (cores); dequantisation single-threaded"}


def cpu_baseline(args):
    from oracle import wq_oracle as O
    sample, weights = _oracle_sample(256 if args.quick else 64)
    t0 = time.perf_counter()
    reps = 0
    while True:
        for x, (p, s, z), K in sample:
            O.gemv_packed(x, "int4", p, s, z, K)
        reps += 1
        if time.perf_counter() - t0 > (2.0 if args.quick else 10.0):
            break
    dt = (time.perf_counter() - t0) / reps
    return {"value": round(weights * INT4_BYTES_PER_WEIGHT / dt / 1e9, 4), "unit": "GB/s",
            **_cpu_fields(), "kind": "oracle",
            "sample": f"every {256 if args.quick else 64}th row of each of the 169 matrices "
                      f"({weights} weights), dequantise + float64 product, {reps} reps"}


def run_reference(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import wq_oracle as O
    # size each step's sample so that warmup + steps take about --ref-budget-s of host time
    cal, cal_w = _oracle_sample(1024)
    t0 = time.perf_counter()
    for x, (p, s, z), K in cal:
        O.gemv_packed(x, "int4", p, s, z, K)
    t_cal = time.perf_counter() - t0
    budget = args.ref_budget_s / (args.steps + args.warmup)
    rows_div = int(min(max(1024 * t_cal / budget, 64), 1 << 20))
    sample, weights = _oracle_sample(rows_div)
    nbytes = weights * INT4_BYTES_PER_WEIGHT

    def step():
        for x, (p, s, z), K in sample:
            O.gemv_packed(x, "int4", p, s, z, K)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    v = round(nbytes / dt / 1e9, 4)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workloads.WORKLOADS[1]["name"],
                                            "sample": f"every {rows_div}th row of each matrix"},
            "cpu_baseline": {"value": v, "unit": "GB/s", **_cpu_fields(), "kind": "oracle",
                             "sample": f"every {rows_div}th row of each of the 169 matrices "
                                       f"({weights} weights)"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--quick", action="store_true", help="smaller rows / CPU sample")
    ap.add_argument("--no-rows", action="store_true", help="skip the secondary rows")
    ap.add_argument("--case", default=None, choices=["gemm_set", "int4h_set"],
                    help="time one secondary case alone (for profiling): gemm_set = the "
                         "0.5B set at --batch tokens through wq_linear_set; int4h_set = the "
                         "0.5B set in hierarchical int4 at batch 1")
    ap.add_argument("--batch", type=int, default=512)
    ap.add_argument("--ref-budget-s", type=float, default=90.0,
                    help="host seconds the reference arm's warmup + steps take (about)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.case == "gemm_set":
        torch.cuda.init()
        args.quick = False
        r = bench_batch_sweep(args, peaks(), Ms=(args.batch,))
        print(json.dumps({"case": args.case, "batch": args.batch, **r}), flush=True)
    elif args.case == "int4h_set":
        torch.cuda.init()
        args.quick = True
        r = bench_int4h_set(args, peaks())
        print(json.dumps({"case": args.case, **r}), flush=True)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
