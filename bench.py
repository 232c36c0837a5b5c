#!/usr/bin/env python
"""Benchmark of the routed-expert MoE layer on B200: one step = one whole layer (gate, route,
group, expert FFN, combine) over one batch of synthetic tokens.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--tokens T]
    python bench.py --impl reference ...     # the CPU oracle, timed on the host cores

Prints one JSON line (rank 0).  Timing: CUDA events on the launching stream, barrier +
synchronize on both sides of exactly K steps, max over ranks.  L2: every step reads a layer
other than the previous step's (rotation over resident layers whose weights total far more
than L2) and fresh activations, so no weight byte is served from L2 by a previous step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

PROFILES = os.path.join(ROOT, "profiles")
METRIC = "MoE-layer tokens/s and expert-weight HBM GB/s (fraction of roofline), 1 B200"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="coli", choices=["coli", "reference"])
    ap.add_argument("--workload", default="glm_decode", choices=list(synth.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=0, help="tokens per step (default: workload's first)")
    ap.add_argument("--layers", type=int, default=0, help="resident layers rotated (default 4)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="default workload only: skip the 2048-token prefill measurement")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile", action="store_true",
                    help="only run warmup+steps layer calls (for ncu captures); prints no JSON")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def record_bytes(wl):
    return synth.record_layout(wl.hidden, wl.inter, wl.fmt, wl.group)["bytes"]


def alg_bytes(wl, T, U):
    """Algorithmic bytes of one layer: unique experts' records (+ shared), router weight and
    bias, activations in, output out."""
    rec = record_bytes(wl)
    act = 4 if wl.act == "f32" else 2
    return ((U + wl.n_shared) * rec + wl.n_experts * wl.hidden * 4 + wl.n_experts * 4
            + T * wl.hidden * act + T * wl.hidden * 4)


def alg_flops(wl, T):
    return (T * wl.top_k + T * wl.n_shared) * 6 * wl.hidden * wl.inter + T * wl.n_experts * wl.hidden * 2


def max_over_ranks(value, dist, device):
    """The largest per-rank value (a timed region's device time) over all ranks; the value
    itself on one rank."""
    if dist is None:
        return value
    t = torch.tensor([value], device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, steps, tokens, ms_max):
    """Tokens of all ranks (each runs `steps` steps of `tokens` tokens) per second of the
    slowest rank's time."""
    return world * steps * tokens / (ms_max / 1e3)


def src_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


class Clocks:
    """nvidia-smi sampler around the loaded window."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1])); mx = float(r[2])
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except Exception:
                pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------- GPU arm ----------

# arithmetic of each execution path (coli_moe_layer_kernels -> path), for the `dtype` key
PATH_DTYPE = {
    1: "int8 x int8 tensor-core MMA (int32 accumulate) on 24-bit fixed-point activations, f32 epilogue",
    5: "f32 CUDA-core GEMV on dequantised codes",
    7: "int8 x int8 tensor-core MMA (int32 accumulate) on 16-bit fixed-point activations, f32 epilogue",
}
PATH_NAME = {1: "fused decode kernel", 5: "gate/route/group + GEMV expert kernels",
             7: "gate/route/group + tensor-core grouped GEMM"}


def workload_config(wl, T):
    """The `config` keys that name the workload (shared by both arms)."""
    return {
        "workload": {"glm_decode": "glm_decode (GLM-5.2-shaped decode layer)",
                     "glm_prefill": "glm_prefill (GLM-5.2-shaped 2048-token prefill layer, Zipf(1.1) popularity)"
                     }.get(wl.name, wl.name),
        "tokens_per_step": T, "hidden": wl.hidden, "expert_inter": wl.inter,
        "experts": wl.n_experts, "top_k": wl.top_k, "n_group": wl.n_group,
        "topk_group": wl.topk_group, "shared_experts": wl.n_shared,
        "weights": {4: "packed int4", 8: "int8", 2: "packed int2"}[wl.fmt] + " per-row f32 scales",
        "activations": wl.act,
    }


def measure(args, wl, T, n_layers, K, W, rank, world, dist, dev, label):
    """Time K whole-layer steps of workload `wl` at T tokens (after >= W warm-up steps), the
    expert FFN launches alone, and the end-to-end rate with host buffers.  Returns the result
    dict and the context the CPU baseline needs."""
    import quantized_routed_expert_noaux_b200 as q

    cfg = q.config_for(wl)
    layers = []
    for l in range(n_layers):
        ex = synth.make_expert_records(wl, device=dev, layer=l)
        sh = synth.make_shared_record(wl, device=dev, layer=l)
        Wr, b = synth.make_router(wl, device=dev, layer=l)
        layers.append((ex, sh, Wr, b, q.weights_for(Wr, b, ex, sh)))
    n_x = 64 if T <= 64 else 4
    xs = [synth.make_activations(wl, T, device=dev, step=1000 * rank + i) for i in range(n_x)]
    out = torch.empty(T, wl.hidden, dtype=torch.float32, device=dev)
    ids_all = torch.empty(K, T, wl.top_k, dtype=torch.int32, device=dev)
    ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()

    def step(i, ids=None):
        ex, sh, Wr, b, wts = layers[i % n_layers]
        q.coli_moe_layer(cfg, wts, xs[i % n_x], T, out, ids, None, ws, st.cuda_stream)

    if args.profile:
        q.coli_moe_clear_error(ws)
        for i in range(W + K):
            step(i)
        torch.cuda.synchronize()
        if q.coli_moe_error_word(ws):
            raise RuntimeError("device error word set")
        return None, None

    def barrier():
        if dist is not None:
            dist.barrier()

    clocks = Clocks(dev.index if dev.index is not None else 0)
    q.coli_moe_clear_error(ws)
    t_soak = time.time()
    i = 0
    while i < W or time.time() - t_soak < 1.0:  # >= W warm-up steps and >= 1 s under load
        step(i)
        i += 1
        if i % 256 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for k in range(K):
        step(k, ids_all[k])
    e1.record(st)
    torch.cuda.synchronize()
    barrier()
    ms = e0.elapsed_time(e1)
    clk = clocks.stop()
    err = q.coli_moe_error_word(ws)
    if err:
        raise RuntimeError(f"device error word {err:#x} after the timed region ({label})")
    ms_max = max_over_ranks(ms, dist, dev)

    # algorithmic bytes of the timed steps (unique experts per step from the routing written)
    ids_np = ids_all.cpu().numpy()
    U = np.array([len(np.unique(ids_np[k])) for k in range(K)])
    bytes_steps = sum(alg_bytes(wl, T, int(u)) for u in U)
    expert_bytes = sum((int(u) + wl.n_shared) * record_bytes(wl) for u in U)

    # live per-launch time of the expert FFN part (coli_moe_ffn on the same rotation), on the
    # launching stream
    offs = torch.empty(wl.n_experts + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * wl.top_k, dtype=torch.int32, device=dev)
    cnt = torch.empty(wl.n_experts, dtype=torch.int32, device=dev)
    uq = torch.empty(wl.n_experts, dtype=torch.int32, device=dev)
    nu = torch.empty(1, dtype=torch.int32, device=dev)
    lg = torch.empty(T, wl.n_experts, dtype=torch.float32, device=dev)
    tw = torch.empty(T, wl.top_k, dtype=torch.float32, device=dev)
    tid = torch.empty(T, wl.top_k, dtype=torch.int32, device=dev)
    n_ffn = min(K, 500)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_ffn)]
    for k in range(n_ffn):
        ex, sh, Wr, b, wts = layers[k % n_layers]
        x = xs[k % n_x]
        q.coli_moe_gate(cfg, Wr, x, T, lg, st.cuda_stream)
        q.coli_moe_route(cfg, lg, b, T, tid, tw, st.cuda_stream)
        q.coli_moe_group(cfg, tid, T, cnt, offs, perm, uq, nu, ws, st.cuda_stream)
        evs[k][0].record(st)
        q.coli_moe_ffn(cfg, wts, x, T, tw, offs, perm, uq, nu, out, ws, st.cuda_stream)
        evs[k][1].record(st)
    torch.cuda.synchronize()
    ffn_ms = sum(a.elapsed_time(b) for a, b in evs) / n_ffn
    U_mean = float(U[:n_ffn].mean()) if len(U) else 0.0
    act = 4 if wl.act == "f32" else 2
    ffn_bytes = (U_mean + wl.n_shared) * record_bytes(wl) + T * wl.hidden * act + T * wl.hidden * 4

    # end to end through the C ABI with host buffers: pinned H2D of x, layer, D2H of out
    x_host = [xs[i].cpu().pin_memory() for i in range(n_x)]
    out_host = torch.empty(T, wl.hidden, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(xs[0])
    K2 = min(K, 1000)
    barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(st)
    for k in range(K2):
        x_dev.copy_(x_host[k % n_x], non_blocking=True)
        ex, sh, Wr, b, wts = layers[k % n_layers]
        q.coli_moe_layer(cfg, wts, x_dev, T, out, None, None, ws, st.cuda_stream)
        out_host.copy_(out, non_blocking=True)
    f1.record(st)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), dist, dev)

    # the same layer calls replayed from a captured CUDA graph (no host launch path per step);
    # reported beside the per-call number, which stays the headline
    G = min(K, 40)
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(st)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for i in range(G):
            wts = layers[i % n_layers][4]
            q.coli_moe_layer(cfg, wts, xs[i % n_x], T, out, None, None, ws, side.cuda_stream)
    R = max(1, min(K, 2000) // G)
    graph.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record(st)
    for _ in range(R):
        graph.replay()
    r1.record(st)
    torch.cuda.synchronize()
    barrier()
    graph_ms = max_over_ranks(r0.elapsed_time(r1), dist, dev)
    del graph
    if q.coli_moe_error_word(ws):
        raise RuntimeError(f"device error word set during the graph replays ({label})")

    hbm, bf16, bf16s, peak_kind = peaks()
    tok_s = whole_job_rate(world, K, T, ms_max)
    traffic = None
    tf = os.path.join(PROFILES, f"{wl.name}_t{T}_traffic.json")
    if os.path.exists(tf):
        d = json.load(open(tf))
        cur = src_hash([os.path.join(ROOT, "quantized_routed_expert_noaux_b200", "csrc", f)
                        for f in d.get("sources", [])])
        if d.get("source_hash") == cur:
            traffic = d.get("traffic_bytes_per_launch")

    n_kern = q.coli_moe_layer_kernels(cfg, T)
    # Tensor-core path: int8 MMAs on two 8-bit activation slices, i.e. two int8 operations per
    # algorithmic multiply-add -- the bf16 tensor rate; ~1 ms launches back to back -> sustained
    # peak.  The bound is whichever of the flops and the bytes takes longer at the measured
    # peaks (small batches on that path are bound by HBM like decode).
    ffn_flops = (T * wl.top_k + T * wl.n_shared) * 6.0 * wl.hidden * wl.inter
    peak_t = bf16s if bf16s else bf16
    tc_kernel = "expert FFN (x quantisation, gate/up int8 GEMM, h quantisation, down int8 GEMM + combine)"
    if n_kern == 7 and ffn_flops / (peak_t * 1e12) > ffn_bytes / (hbm * 1e9):
        tf_s = ffn_flops / (ffn_ms / 1e3) / 1e12
        roofline = {
            "bound": "tensor", "kernel": tc_kernel, "achieved": round(tf_s, 1), "peak": peak_t,
            "unit": "TFLOP/s", "frac": round(tf_s / peak_t, 4), "traffic": traffic,
            "peak_source": f"{peak_kind} bf16_tflops{'_sustained' if bf16s else ''} (int8 with two "
                           f"activation slices runs algorithmic flops at the bf16 rate); frac of {peak_kind}",
            "launch_us": round(ffn_ms * 1e3, 2),
            "hbm_gbs_of_weights": round(ffn_bytes / (ffn_ms / 1e3) / 1e9, 1),
        }
    else:
        achieved = ffn_bytes / (ffn_ms / 1e3) / 1e9
        roofline = {
            "bound": "hbm",
            "kernel": ("fused decode layer kernel (FFN part)" if n_kern == 1 else
                       tc_kernel if n_kern == 7 else "expert FFN (gate/up GEMV + down GEMV with fused combine)"),
            "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "traffic": traffic,
            "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth); frac of {peak_kind}",
            "launch_us": round(ffn_ms * 1e3, 2),
        }
    # whole-layer roofline: max(bytes / HBM, flops / tensor peak) over the measured step time
    layer_flops = alg_flops(wl, T)
    t_roof = max(bytes_steps / K / (hbm * 1e9), layer_flops / (peak_t * 1e12))
    res = {
        "value": round(tok_s, 2),
        "unit": "tokens/s",
        "ms_per_step": round(ms_max / K, 6),
        "dtype": PATH_DTYPE[n_kern],
        "path": PATH_NAME[n_kern],
        "config": dict(workload_config(wl, T),
                       l2=f"rotation over {n_layers} resident layers ({n_layers * wl.n_experts * record_bytes(wl) / 1e9:.1f} GB of expert records) + fresh activations every step; no flush",
                       parallelism=f"replicas x{world}"),
        "expert_gbs": round(expert_bytes / (ms_max / 1e3) / 1e9, 1),
        "layer_gbs": round(bytes_steps / (ms_max / 1e3) / 1e9, 1),
        "layer_frac_of_hbm": round(bytes_steps / (ms_max / 1e3) / 1e9 / hbm, 4),
        "layer_roofline_us": round(t_roof * 1e6, 2),
        "layer_frac_of_roofline": round(t_roof / (ms_max / K / 1e3), 4),
        "unique_experts_mean": round(float(U.mean()), 2),
        "roofline": roofline,
        "e2e": {"value": round(whole_job_rate(world, K2, T, e2e_ms), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": int(xs[0].numel() * xs[0].element_size()),
                "d2h_bytes_per_step": int(out.numel() * 4)},
        "graph_replay": {"value": round(whole_job_rate(world, R * G, T, graph_ms), 2), "unit": "tokens/s",
                         "ms_per_step": round(graph_ms / (R * G), 6), "steps_per_graph": G,
                         "replays": R},
        "gpu_launches": n_kern * K,
        "clocks": clk,
    }
    return res, (wl, T, layers, xs)


def gpu_arm(args, rank, world, dist):
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[args.workload]
    T = args.tokens or wl.tokens[0]
    n_layers = args.layers or (4 if wl.hidden >= 2048 else 1)
    K, W = args.steps, args.warmup
    res, ctx = measure(args, wl, T, n_layers, K, W, rank, world, dist, dev, wl.name)
    if res is None:
        return None, None
    line = {"metric": METRIC, "value": res.pop("value"), "unit": res.pop("unit"), "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": res.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": res.pop("dtype"),
            "data": "synthetic (seeded; weights N(0,0.02) quantised per row, activations N(0,1))"}
    line.update(res)
    if args.workload == "glm_decode" and not args.no_prefill:
        # the second headline workload: the 2048-token prefill layer, its own timed region
        pwl = synth.WORKLOADS["glm_prefill"]
        pres, pctx = measure(args, pwl, pwl.tokens[0], 2, min(K, 20), max(W, 3), rank, world, dist,
                             dev, pwl.name)
        pres["steps"] = min(K, 20)
        line["prefill"] = pres
        ctx = ctx + (pctx,)
    return line, ctx


# ------------------------------------------------------------------------- CPU oracle -------

def _oracle_sample(wl, T_tokens, x_list, layers_dev, budget_s, device):
    """Run the oracle on a bounded sample of the workload's tokens; returns (tokens, seconds,
    threads)."""
    import oracle
    cfg = oracle.make_cfg(wl)
    threads = os.cpu_count() or 1
    ex, sh, Wr, b = layers_dev
    Wr_h, b_h = Wr.cpu(), b.cpu()
    cache = {}

    def recs_for(xh, n):
        lg = oracle.gate(cfg, Wr_h, xh, n)
        ids, _ = oracle.route(cfg, lg, b_h, n)
        for e in np.unique(ids):
            if int(e) not in cache:
                cache[int(e)] = ex[int(e)].cpu().numpy()
        table = [cache.get(e) for e in range(wl.n_experts)]
        return oracle.Records(table, None if sh is None else sh.cpu().numpy())

    # calibrate on one token
    x0 = x_list[0][:1].cpu()
    R = recs_for(x0, 1)
    t0 = time.time()
    oracle.layer(cfg, Wr_h, b_h, R, x0, 1, n_threads=1)
    per_tok = max(time.time() - t0, 1e-4)
    n = int(max(1, min(budget_s * threads / per_tok, 4096)))
    n = max(n, min(threads, 4096))
    xs = torch.cat([x.cpu() for x in x_list], 0)
    while xs.shape[0] < n:
        xs = torch.cat([xs, xs], 0)
    xs = xs[:n].contiguous()
    R = recs_for(xs, n)
    t0 = time.time()
    oracle.layer(cfg, Wr_h, b_h, R, xs, n, n_threads=threads)
    return n, time.time() - t0, threads


def cpu_baseline(wl, T, xs, layers, seconds):
    n, sec, thr = _oracle_sample(wl, T, xs[:8], layers[0][:4], seconds, None)
    return {"value": round(n / sec, 4), "unit": "tokens/s", "cores": thr, "kind": "oracle",
            "sample": f"{n} tokens of the same workload (layer 0), {sec:.1f} s wall on {thr} threads"}


def reference_arm(args):
    """The CPU oracle as the reference implementation, on the host cores."""
    wl = synth.WORKLOADS[args.workload]
    T = args.tokens or wl.tokens[0]
    device = "cuda" if torch.cuda.is_available() else "cpu"
    import oracle
    cfg = oracle.make_cfg(wl)
    threads = os.cpu_count() or 1
    K, W = args.steps, args.warmup
    # the oracle is slow: a step is a bounded sample of T tokens, the same batch shape
    ex = synth.make_expert_records(wl, device=device, experts=[])
    sh = synth.make_shared_record(wl, device=device)
    Wr, b = synth.make_router(wl, device=device)
    Wr_h, b_h = Wr.cpu(), b.cpu()
    per_step = []
    made = set()
    budget = 150.0
    t_start = time.time()
    steps_done = 0
    for k in range(W + K):
        x = synth.make_activations(wl, T, device=device, step=k).cpu()
        lg = oracle.gate(cfg, Wr_h, x, T)
        ids, _ = oracle.route(cfg, lg, b_h, T)
        need = [int(e) for e in np.unique(ids) if int(e) not in made]
        if need:
            synth.make_expert_records(wl, device=device, experts=need, out=ex)
            made.update(need)
        table = [ex[e].cpu().numpy() if e in made else None for e in range(wl.n_experts)]
        R = oracle.Records(table, None if sh is None else sh.cpu().numpy())
        t0 = time.time()
        oracle.layer(cfg, Wr_h, b_h, R, x, T, n_threads=threads)
        dt = time.time() - t0
        if k >= W:
            per_step.append(dt)
            steps_done += 1
        if time.time() - t_start > budget and steps_done >= 1:
            break
    sec = sum(per_step)
    val = steps_done * T / sec
    return {
        "metric": METRIC, "impl": "reference", "value": round(val, 4), "unit": "tokens/s",
        "n_gpus": 1, "steps": steps_done, "warmup": W, "ms_per_step": round(1e3 * sec / steps_done, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": dict(workload_config(wl, T), parallelism="host cores (oracle)"),
        # the oracle parallelises over tokens: a step of T tokens keeps min(T, threads) busy
        "cpu_baseline": {"value": round(val, 4), "unit": "tokens/s", "cores": min(threads, T),
                         "kind": "oracle",
                         "sample": f"{steps_done} steps of {T} token(s) each (run stopped after {budget:.0f} s if K was larger)"},
        "e2e": {"value": round(val, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(reference_arm(args)))
        return
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist_mod
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    res, ctx = gpu_arm(args, rank, world, dist)
    if res is None:
        return
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        wl, T, layers, xs = ctx[:4]
        res["cpu_baseline"] = cpu_baseline(wl, T, xs, layers, args.cpu_seconds)
        if len(ctx) > 4:
            pwl, pT, players, pxs = ctx[4]
            res["prefill"]["cpu_baseline"] = cpu_baseline(pwl, pT, pxs, players, args.cpu_seconds)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))


if __name__ == "__main__":
    main()
