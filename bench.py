"""Benchmark: the 64-layer tree-MTP verify step (27B-class dense model, NVFP4
W4A4 linears incl. the LM head, FP8 paged KV cache, 16-node tree, 23,552
cached tokens, kv_page_restore of the reused 96% prefix) on one B200 per rank.

One step = restore of the prefix pages + 64 layers + LM head + argmax, captured
as one CUDA graph.  `value` is verify steps/s over all ranks (replicas: each
rank verifies its own tree), timed on the device with CUDA events around K
graph replays, max over ranks.  `e2e` adds, per step, the host->device copy of
the step's inputs (16 hidden rows + parent array, pinned) and the
device->host read of the 16 argmax ids.  Weights (11.4 GB) far exceed L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

`--prefill S` times instead the suffix prefill of the last S prompt tokens
(positions ctx - S .. ctx - 1, after the restored prefix) through all layers
plus the last token's LM head, one CUDA graph per prefill, on one GPU.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HBM GB/s (% of B200 peak) for NVFP4 linear + tree attn at M=16; verify steps/s"
UNIT = "verify steps/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ctx", type=int, default=23552)
    ap.add_argument("--sweep", default="1024,8192,23552",
                    help="context lengths of the verify-step sweep (same weights), '' for none")
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--chain", type=int, default=0,
                    help="verify a linear-MTP chain of this many tokens instead of the 16-node tree")
    ap.add_argument("--prefill", type=int, default=0,
                    help="time the suffix prefill of this many tokens instead of the verify step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-range", action="store_true",
                    help="bracket one untimed step replay with cudaProfilerStart/Stop (for ncu --profile-from-start off)")
    ap.add_argument("--kernel-case", default=None,
                    choices=["linear_lmhead", "linear_gate_up", "linear_gate_up_swiglu", "linear_qkv", "linear_o",
                             "linear_down",
                             "linear_m1_2048", "wide_qkv", "wide_o", "wide_gate_up", "wide_down", "causal_attn", "attn",
                             "restore",
                             "quantize", "rmsnorm_quantize"],
                    help="run one kernel on a small case (for ncu captures) instead of the step")
    return ap.parse_args()


# ------------------------------------------------------------------ distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() and args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.distributed.get_backend() == "nccl" else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------------ clocks
class Clocks:
    """nvidia-smi sampling (200 ms) during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev):
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", uuid], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.strip().splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax, "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ peaks / traffic
def measured_peak():
    """HBM copy bandwidth (GB/s) and where it comes from: MEASURED_PEAKS.json's
    hbm_gbs when the file is there, else the profiling recipe's fallback figure."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    return 6650.0, "fallback 6,650 GB/s (no MEASURED_PEAKS.json)"


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("linear.cuh", "common.cuh", "quant.cuh"):          # the linear kernels and their epilogues
        h.update(open(os.path.join(ROOT, "nvfp4_skinny_gemm_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def attn_source_hash():
    h = hashlib.sha256()
    for f in ("attn.cuh", "common.cuh"):                          # the attention kernels' memory traffic
        h.update(open(os.path.join(ROOT, "nvfp4_skinny_gemm_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_attn_traffic():
    """DRAM bytes per tree-attention call (the split kernel), from the committed
    ncu summary, if it was taken on the current attention source (else None)."""
    p = os.path.join(ROOT, "profiles", "tree_attn_fp8kv_ctx23552_t16.md")
    if not os.path.exists(p):
        return None
    m = re.search(r"traffic_bytes_per_call_of_split:\s*([0-9.eE+]+)\s+source:\s*([0-9a-f]+)", open(p).read())
    if m and m.group(2) == attn_source_hash():
        return float(m.group(1))
    return None


def recorded_traffic():
    """DRAM bytes per linear launch of the step, from the committed ncu summary,
    if it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "nvfp4_linear_verify_step.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m = re.search(r"traffic_bytes_per_step_of_linears:\s*([0-9.eE+]+)\s+source:\s*([0-9a-f]+)", txt)
    if m and m.group(2) == kernel_source_hash():
        return float(m.group(1))
    return None


# ------------------------------------------------------------------ CPU baseline (oracle)
def oracle_sample(ctx, layers, seconds_hint=15.0):
    """Time the CPU oracle on a bounded sample of one verify step and
    extrapolate to a whole step.  Returns (steps/s, threads, description)."""
    import oracle
    from nvfp4_skinny_gemm_b200 import inputs as I
    T = I.TREE_NODES
    rng = np.random.default_rng(7)
    est = {}
    t_lin = 0.0
    ns = 1024
    for t, (name, (K, N)) in enumerate(I.LAYER_LINEARS.items()):
        w = I.weight_fp32(4, t, N, K, sub=0)
        wc, ws, gw = oracle.quantize(w)
        del w
        a = I.activation_bf16(4, 100 + t, T, K, 0.01).float().numpy()
        t0 = time.perf_counter()
        ac, asc, ga = oracle.quantize(a)
        im, inn = rng.integers(0, T, ns), rng.integers(0, N, ns)
        oracle.linear_sampled(ac, asc, ga, wc, ws, gw, im, inn)
        dt = time.perf_counter() - t0
        t_lin += dt * (T * N) / ns
        est[name] = dt * (T * N) / ns
    cache = I.kv_cache(4, ctx, T=T, Hkv=1)
    q = I.query_bf16(4, T, 6).float().numpy()
    parent = I.tree_parent(4)
    t0 = time.perf_counter()
    oracle.tree_attn(q, cache.k_pool, cache.v_pool, cache.page_table, ctx, parent, cache.k_scale, cache.v_scale)
    t_att = (time.perf_counter() - t0) * I.N_KV_HEADS
    pb, n_pages = 32768, 256
    src = np.random.default_rng(1).integers(0, 256, n_pages * pb, dtype=np.uint8)
    dst = np.zeros_like(src)
    ids = np.arange(n_pages, dtype=np.int32)
    t0 = time.perf_counter()
    oracle.kv_page_restore(src, ids, dst, ids, pb)
    n_restore = layers * 2 * math.ceil(round(0.96 * ctx) / 64)
    t_rst = (time.perf_counter() - t0) * n_restore / n_pages
    w = I.weight_fp32(4, 9, 4096, I.HIDDEN)
    wc, ws, gw = oracle.quantize(w)
    a = I.activation_bf16(4, 200, T, I.HIDDEN).float().numpy()
    t0 = time.perf_counter()
    ac, asc, ga = oracle.quantize(a)
    im, inn = rng.integers(0, T, ns), rng.integers(0, 4096, ns)
    oracle.linear_sampled(ac, asc, ga, wc, ws, gw, im, inn)
    t_head = (time.perf_counter() - t0) * T * I.VOCAB / ns
    step = layers * (t_lin + t_att) + t_head + t_rst
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    desc = (f"oracle (fp64 C, OpenMP) on one layer's linears ({ns} sampled outputs each of 16xN), "
            f"attention of 1 of 4 KV heads at ctx {ctx}, restore of {n_pages} of {n_restore} pages, "
            f"LM head {ns} sampled logits; extrapolated to {layers} layers + LM head + restore "
            f"({step:.1f} s per step)")
    return 1.0 / step, threads, desc


def oracle_sample_one_thread(ctx, layers, timeout=600):
    """The same bounded oracle sample on one OpenMP thread, in a fresh Python
    process (fork + exec, no CUDA state).  Returns its steps/s, or None if it
    could not run: the multi-threaded figure stays the reported baseline."""
    code = (f"import json, sys; sys.path.insert(0, {ROOT!r}); import bench; "
            f"v, t, _ = bench.oracle_sample({int(ctx)}, {int(layers)}); print(json.dumps([v, t]))")
    env = dict(os.environ, OMP_NUM_THREADS="1", CUDA_VISIBLE_DEVICES="")
    try:
        r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=timeout)
        v, threads = json.loads(r.stdout.strip().splitlines()[-1])
        return float(v) if threads == 1 else None
    except Exception:
        return None


# ------------------------------------------------------------------ reference arm
def run_reference(args, world, rank):
    if rank != 0:
        return
    vals, desc, threads = [], "", 1
    t0 = time.perf_counter()
    for _ in range(max(1, args.steps)):
        v, threads, desc = oracle_sample(args.ctx, args.layers)
        vals.append(v)
        if time.perf_counter() - t0 > 240:
            break
    v = float(np.median(vals))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": len(vals), "warmup": args.warmup, "ms_per_step": 1e3 / v,
            "ms_per_step_kind": "estimate: each step times a bounded oracle sample and extrapolates it "
                                "to a whole verify step (no step runs in full)",
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{args.layers}-layer 27B-class verify step, "
                               f"{f'linear-MTP chain of {T}' if args.chain else '16-node tree'}, ctx {args.ctx} FP8 paged KV, "
                                   f"NVFP4 W4A4 linears + LM head, kv_page_restore of 96% prefix",
                       "layers": args.layers, "ctx": args.ctx, "tree_nodes": 16, "parallelism": "replicas"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def capture(stream, fn):
    """One CUDA graph of fn()'s launches on `stream`."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def time_graph(graph, stream, reps, warm=3):
    """Seconds per replay: CUDA events on the launching stream around `reps`
    back-to-back replays, after `warm` untimed ones."""
    for _ in range(warm):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e-3 / reps


def linear_launches(model):
    """The step's 257 linear launches (same operands, shapes and order; with
    static scales gate+up is the launch that also does SwiGLU + NVFP4)."""
    from nvfp4_skinny_gemm_b200 import lib as nv
    for l, lay in enumerate(model.layers):
        model._linear(model.q_h.buf, model.q_h.g, lay["qkv"], model.qkv)
        model._linear(model.q_a.buf, model.q_a.g, lay["o"], model.h, residual=model.h)
        gu = lay["gate_up"]
        if model.static:
            g_f = model._site(l * model.SITES + 3)
            nv.linear_swiglu(model.q_h.buf, model.q_h.g, model.T, gu.prep, gu.g, gu.N // 2, gu.K, g_f, model.q_f.buf)
        else:
            g_f = model.q_f.g
            model._linear(model.q_h.buf, model.q_h.g, gu, model.gu)
        model._linear(model.q_f.buf, g_f, lay["down"], model.h, residual=model.h)
    model._linear(model.q_h.buf, model.q_h.g, model.lm_head, model.logits)


def attention_launches(model):
    """The step's attention calls (split and combine, with the static NVFP4
    output), one per layer over that layer's pools, back to back."""
    from nvfp4_skinny_gemm_b200 import inputs as I
    from nvfp4_skinny_gemm_b200 import lib as nv
    for l in range(model.n_layers):
        nv.tree_attn(model.qkv, model.k_pool(l), model.v_pool(l), model.page_table, model.L, model.parent,
                     model.k_scale[l], model.v_scale[l], out=model.attn, ld_q=model.qkv.stride(0), T=model.T,
                     Hq=I.N_Q_HEADS, g_act=model._site(l * model.SITES + 1), act=model.q_a.buf)


def run_ours(args, world, rank, local):
    from nvfp4_skinny_gemm_b200 import inputs as I
    from nvfp4_skinny_gemm_b200 import lib as nv
    from nvfp4_skinny_gemm_b200.step import VerifyModel

    dev = torch.device("cuda", torch.cuda.current_device())
    T = args.chain or I.TREE_NODES
    model = VerifyModel(n_layers=args.layers, ctx_len=args.ctx, T=T, weights="device", device=dev)
    h0 = I.bf16_normal(4, 300, (T, I.HIDDEN)).pin_memory()
    par0 = torch.from_numpy(I.chain_parent(T) if args.chain else I.tree_parent(4)).pin_memory()
    ids_host = torch.empty(T, dtype=torch.int32).pin_memory()
    stream = torch.cuda.Stream(device=dev)

    def load_inputs():
        model.h.copy_(h0, non_blocking=True)
        model.parent.copy_(par0, non_blocking=True)

    with torch.cuda.stream(stream):
        load_inputs()
        model.step()                                       # eager: allocates workspaces
        load_inputs()
        model.calibrate()                                  # static activation scales from one dynamic step
        load_inputs()
        model.step()
        torch.cuda.synchronize()
        rc, site = nv.device_status(stream)
        assert rc == 0, f"device status {rc} at site {site}"
        graph = capture(stream, model.step)
        lin_graph = capture(stream, lambda: linear_launches(model))     # the dominant kernel alone, same launches
        attn_graph = capture(stream, lambda: attention_launches(model))  # the attention calls alone
        load_inputs()
        for _ in range(max(3, args.warmup)):
            graph.replay()
        torch.cuda.synchronize()
        if args.profile_range:
            torch.cuda.profiler.start()
            graph.replay()
            torch.cuda.synchronize()
            torch.cuda.profiler.stop()

        # ---- device-timed step
        barrier(world)
        torch.cuda.synchronize()
        clocks = Clocks(dev)
        time.sleep(0.3)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        clk = clocks.stop()
        t_dev = max_over_ranks(ev0.elapsed_time(ev1) * 1e-3, world)
        rc, site = nv.device_status(stream)
        assert rc == 0, f"device status {rc} at site {site}"

        # ---- dominant kernel: all linear launches of one step, back to back;
        #      then the 64 attention calls of one step, back to back
        reps = max(3, min(20, args.steps))
        t_lin = time_graph(lin_graph, stream, reps)
        t_attn = time_graph(attn_graph, stream, reps)
        n_lin = 4 * model.n_layers + 1

        # ---- the step without the per-step prefix restore (the pages restore
        #      once per agent turn; the benchmarked step includes it)
        nr_graph = capture(stream, lambda: model.step(restore=False))
        t_nr = max_over_ranks(time_graph(nr_graph, stream, args.steps), world)
        del nr_graph

        # ---- end to end: pinned host inputs in, argmax ids out, every step.
        #      (1) queued back to back (stream throughput); (2) the host waits
        #      for each step's ids before issuing the next, as a decode loop
        #      that drafts the next tree from them must
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            load_inputs()
            graph.replay()
            ids_host.copy_(model.ids, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        t_e2e = max_over_ranks(e0.elapsed_time(e1) * 1e-3, world)
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            load_inputs()
            graph.replay()
            ids_host.copy_(model.ids, non_blocking=True)
            stream.synchronize()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        t_e2e_sync = max_over_ranks(e0.elapsed_time(e1) * 1e-3, world)

    peak, peak_kind = measured_peak()
    lin_bytes = model.linear_bytes()
    achieved = lin_bytes / t_lin / 1e9
    traffic = recorded_traffic()
    step_bytes = model.step_bytes()
    attn_bytes = model.attn_bytes()
    attn_gbs = attn_bytes / t_attn / 1e9
    value = world * args.steps / t_dev
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_dev / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block scales, f32 accumulate); fp8 e4m3 KV",
        "data": "synthetic",
        "config": {"workload": f"{args.layers}-layer 27B-class verify step, "
                               f"{f'linear-MTP chain of {T}' if args.chain else '16-node tree'}, ctx {args.ctx} FP8 paged KV, "
                               f"NVFP4 W4A4 linears + LM head, kv_page_restore of 96% prefix",
                   "layers": args.layers, "ctx": args.ctx, "tree_nodes": T, "hidden": I.HIDDEN,
                   "weights_gb": round(sum(l.nbytes for lay in model.layers for l in lay.values()) / 1e9
                                       + model.lm_head.nbytes / 1e9, 3),
                   "l2": "inputs larger than L2 (11.4 GB of weights streamed per step)",
                   "act_scales": "static per quantised tensor, calibrated on one dynamic-scale step",
                   "parallelism": f"replicas x{world}"},
        "step_pct_of_peak": round(100 * step_bytes / (t_dev / args.steps) / 1e9 / peak, 1),
        "roofline": {"kernel": "nvfp4_linear_kernel (all 257 linear launches of one step, back to back)",
                     "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": peak_kind,
                     "algorithmic_bytes_per_step": lin_bytes, "launches": n_lin,
                     "us_per_step_of_linears": round(t_lin * 1e6, 1),
                     "traffic": traffic},
        "roofline_attn": {"kernel": f"tree_attn_split_kernel + tree_attn_combine_kernel ({model.n_layers} calls "
                                    f"of one step, back to back)",
                          "bound": "hbm", "achieved": round(attn_gbs, 1), "peak": peak, "unit": "GB/s",
                          "frac": round(attn_gbs / peak, 4),
                          "peak_source": peak_kind,
                          "algorithmic_bytes_per_step": attn_bytes,
                          "algorithmic_bytes_per_call": attn_bytes // model.n_layers,
                          "us_per_call": round(t_attn / model.n_layers * 1e6, 2),
                          "traffic": recorded_attn_traffic() if args.ctx == 23552 else None,
                          "traffic_note": "DRAM bytes per call of the split kernel (ncu, 23,552-token "
                                          "context); the combine was not captured"},
        "no_restore": {"value": world / t_nr, "unit": UNIT, "ms_per_step": round(t_nr * 1e3, 3),
                       "note": "the same step without the per-step kv_page_restore of the prefix "
                               "(the pages restore once per agent turn)"},
        "clocks": clk,
        "e2e": {"value": world * args.steps / t_e2e, "unit": UNIT,
                "h2d_bytes_per_step": h0.numel() * 2 + par0.numel() * 4,
                "d2h_bytes_per_step": ids_host.numel() * 4,
                "mode": "steps queued back to back (stream throughput)"},
        "e2e_sync": {"value": world * args.steps / t_e2e_sync, "unit": UNIT,
                     "ms_per_step": round(t_e2e_sync / args.steps * 1e3, 3),
                     "mode": "the host waits for each step's argmax ids before issuing the next step"},
        "gpu_launches": model.launches_per_step() * args.steps,
    }
    line["step_hbm_gbs"] = round(step_bytes / (t_dev / args.steps) / 1e9, 1)
    line["node_tokens_per_s"] = round(T * value, 1)      # candidate tokens verified per second

    # ---- context sweep of the verify step (same weights; cache and page table rebuilt)
    del graph, lin_graph, attn_graph
    sweep = [{"ctx": args.ctx, "value": value, "ms_per_step": line["ms_per_step"],
              "step_hbm_gbs": line["step_hbm_gbs"], "pct_of_peak": line["step_pct_of_peak"]}]
    if args.sweep:
        for c in [int(x) for x in args.sweep.split(",") if int(x) != args.ctx]:
            with torch.cuda.stream(stream):
                model.set_context(c)
                load_inputs()
                model.step()
                torch.cuda.synchronize()
                g2 = capture(stream, model.step)
                t_c = max_over_ranks(time_graph(g2, stream, args.steps), world)
                rc, site = nv.device_status(stream)
                assert rc == 0, f"device status {rc} at site {site}"
                del g2
            sb = model.step_bytes()
            sweep.append({"ctx": c, "value": world / t_c, "ms_per_step": round(t_c * 1e3, 3),
                          "step_hbm_gbs": round(sb / t_c / 1e9, 1), "pct_of_peak": round(100 * sb / t_c / 1e9 / peak, 1)})
        sweep.sort(key=lambda d: d["ctx"])
    line["sweep"] = sweep

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        runs = [oracle_sample(args.ctx, args.layers) for _ in range(3)]
        med = sorted(runs, key=lambda r: r[0])[1]             # the median run, with its own description
        v, threads, desc = float(med[0]), med[1], med[2]
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": desc + "; median of 3 runs",
                                "runs": [r[0] for r in runs],
                                "value_one_thread": oracle_sample_one_thread(args.ctx, args.layers)}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ suffix prefill
def prefill_flops(S, start, layers):
    """FLOPs a suffix prefill of S tokens after `start` cached tokens must do:
    (NVFP4 linears over S rows + the LM head over the last row, QK^T and PV
    of causal attention: row i sees start + i + 1 positions)."""
    from nvfp4_skinny_gemm_b200 import inputs as I
    lin = 2.0 * S * sum(N * K for (K, N) in I.LAYER_LINEARS.values()) * layers + 2.0 * I.VOCAB * I.HIDDEN
    visible = S * (start + 1) + S * (S - 1) / 2
    attn = 4.0 * I.HEAD_DIM * I.N_Q_HEADS * visible * layers
    return lin, attn


def run_prefill(args):
    """Suffix prefill of S = args.prefill tokens after ctx - S cached tokens,
    timed with CUDA events around graph replays (weights far exceed L2).

    Roofline: the FLOPs the prefill must do (the NVFP4 linears over S rows, the
    LM head over the last row, QK^T and PV of the causal attention) at the
    tensor peaks of their types (FP4 linears, FP8 attention: the measured
    sustained bf16 GEMM peak times the nominal ratios 4 and 2)."""
    from nvfp4_skinny_gemm_b200 import inputs as I
    from nvfp4_skinny_gemm_b200 import lib as nv
    from nvfp4_skinny_gemm_b200.step import VerifyModel

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    S, L = args.prefill, args.ctx
    start = L - S
    model = VerifyModel(n_layers=args.layers, ctx_len=L, weights="device", device=dev)
    h_in = (I.bf16_normal(4, 303, (S, I.HIDDEN)) * 0.5).to(dev)
    h = torch.empty_like(h_in)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        model.h.copy_(I.bf16_normal(4, 300, (I.TREE_NODES, I.HIDDEN)).to(dev))
        model.parent.copy_(torch.from_numpy(I.tree_parent(4)).to(dev))
        model.step()                                       # eager: allocates workspaces
        model.calibrate()                                  # restore + one dynamic-scale step
        h.copy_(h_in)
        model.prefill(h, start)                            # eager: allocates the prefill buffers
        torch.cuda.synchronize()
        rc, site = nv.device_status(stream)
        assert rc == 0, f"device status {rc} at site {site}"
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            h.copy_(h_in)
            ids = model.prefill(h, start)
        for _ in range(max(3, args.warmup)):
            graph.replay()
        torch.cuda.synchronize()
        clocks = Clocks(dev)
        time.sleep(0.3)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        clk = clocks.stop()
        t = e0.elapsed_time(e1) * 1e-3 / args.steps
        rc, site = nv.device_status(stream)
        assert rc == 0, f"device status {rc} at site {site}"
        assert ids is not None and 0 <= int(ids.cpu()[0]) < I.VOCAB

        # ---- breakdown: the prefill's wide linears alone, then its causal
        #      attention calls alone (same shapes, same buffers, back to back)
        pf = model._pf
        scratch_h = torch.empty_like(h)

        def wide_linears():
            for lay in model.layers:
                for name, y in (("qkv", pf["qkv"][:S]), ("o", scratch_h), ("gate_up", pf["gu"][:S]),
                                ("down", scratch_h)):
                    lin = lay[name]
                    nv.linear_wide(pf["wide"], pf["g"], S, lin.prep, lin.g, lin.N, lin.K, y=y)

        def causal_attention():
            # the blocks of each layer as the prefill launches them (round its streams)
            for l in range(model.n_layers):
                model._causal_blocks(pf, l, pf["qkv"][:S], pf["attn"][:S], start, S)

        g_lin = capture(stream, wide_linears)
        g_att = capture(stream, causal_attention)
        t_lin = time_graph(g_lin, stream, max(2, args.steps))
        t_att = time_graph(g_att, stream, max(2, args.steps))
        rc, site = nv.device_status(stream)
        assert rc == 0, f"device status {rc} at site {site}"
        del g_lin, g_att

    lin_flops, attn_flops = prefill_flops(S, start, args.layers)
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) \
        if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    bf16 = float(peaks.get("bf16_tflops_sustained", 1400.0))
    kind = "measured" if "bf16_tflops_sustained" in peaks else "fallback"
    ideal = lin_flops / (4 * bf16 * 1e12) + attn_flops / (2 * bf16 * 1e12)
    flops = lin_flops + attn_flops
    line = {
        "metric": "suffix prefill tokens/s", "value": S / t, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block scales, f32 accumulate); fp8 e4m3 KV", "data": "synthetic",
        "config": {"workload": f"{args.layers}-layer suffix prefill of {S} tokens after {start} cached tokens, "
                               f"wide NVFP4 linears and causal attention in 128-query blocks, LM head on the "
                               f"last token",
                   "layers": args.layers, "ctx": L, "suffix": S, "parallelism": "single GPU",
                   "l2": "inputs larger than L2 (11.4 GB of weights)"},
        "roofline": {"bound": "tensor", "achieved": round(flops / t / 1e12, 1),
                     "peak": round(flops / ideal / 1e12, 1), "unit": "TFLOP/s", "frac": round(ideal / t, 4),
                     "peak_source": f"{kind} sustained bf16 GEMM x 4 (FP4 linears) and x 2 (FP8 attention), "
                                    f"weighted by their FLOPs",
                     "linear_tflop": round(lin_flops / 1e12, 2), "attention_tflop": round(attn_flops / 1e12, 2),
                     "traffic": None},
        "breakdown": {
            "wide_linears": {"ms": round(t_lin * 1e3, 3), "tflops": round(lin_flops / t_lin / 1e12, 1),
                             "frac": round(lin_flops / t_lin / (4 * bf16 * 1e12), 4),
                             "note": "all nvfp4_linear_wide launches of one prefill, back to back; frac of the "
                                     "FP4 peak (sustained bf16 x 4)"},
            "causal_attention": {"ms": round(t_att * 1e3, 3), "tflops": round(attn_flops / t_att / 1e12, 1),
                                 "frac": round(attn_flops / t_att / (2 * bf16 * 1e12), 4),
                                 "note": "all causal_attn_fp8kv launches of one prefill, back to back (each "
                                         "layer's blocks round the prefill's streams); frac of the FP8 peak "
                                         "(sustained bf16 x 2)"},
            "rest_ms": round((t - t_lin - t_att) * 1e3, 3)},
        "clocks": clk,
        "gpu_launches": model.prefill_launches(S) * args.steps,
    }
    print(json.dumps(line), flush=True)
    del graph


# ------------------------------------------------------------------ single-kernel cases
def run_kernel_case(args):
    """A few launches of one kernel on a small case (a few GB at most): the
    command that ncu captures for the per-kernel profiles."""
    from nvfp4_skinny_gemm_b200 import inputs as I
    from nvfp4_skinny_gemm_b200 import lib as nv
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(1)
    case = args.kernel_case
    if case.startswith("linear"):
        K, N = {"linear_lmhead": (I.HIDDEN, I.VOCAB), "linear_gate_up": I.LAYER_LINEARS["gate_up"],
                "linear_gate_up_swiglu": I.LAYER_LINEARS["gate_up"],
                "linear_qkv": I.LAYER_LINEARS["qkv"], "linear_o": I.LAYER_LINEARS["o"],
                "linear_down": I.LAYER_LINEARS["down"], "linear_m1_2048": (2048, 2048)}[case]
        M = 1 if case == "linear_m1_2048" else 16
        ncopy = max(1, math.ceil(400e6 / (N * K * 9 // 16)))     # rotate copies: > L2 per sweep
        ws = []
        for _ in range(ncopy):
            c = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
            sc = torch.randint(0x30, 0x40, (N, K // 16), dtype=torch.uint8, device=dev, generator=g)
            ws.append((nv.prepare_weight(c, sc, N, K), torch.full((1,), 0.01, device=dev)))
            del c, sc
        a = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        act = nv.act_buffer(K)
        _, _, ga = nv.quantize(a, act=act)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        fn = lambda i: nv.linear(act, ga, M, ws[i % ncopy][0], ws[i % ncopy][1], N, K, y=y)
        if case == "linear_gate_up_swiglu":                       # + SwiGLU + NVFP4 in the epilogue
            act_f, g_f = nv.act_buffer(N // 2), torch.full((1,), 0.01, device=dev)
            fn = lambda i: nv.linear_swiglu(act, ga, M, ws[i % ncopy][0], ws[i % ncopy][1], N // 2, K, g_f, act_f)
        nbytes = N * K * 9 // 16
    elif case.startswith("wide"):
        K, N = I.LAYER_LINEARS[case[5:]]
        S = 942
        wc = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
        wsc = torch.randint(0x30, 0x40, (N, K // 16), dtype=torch.uint8, device=dev, generator=g)
        w_p = nv.prepare_weight(wc, wsc, N, K)
        ncopy = max(1, math.ceil(250e6 / w_p.numel()))          # rotate copies: > L2 per sweep
        w_ps = [w_p] + [w_p.clone() for _ in range(ncopy - 1)]
        ac = torch.randint(0, 256, (S, K // 2), dtype=torch.uint8, device=dev, generator=g)
        asc = torch.randint(0x30, 0x40, (S, K // 16), dtype=torch.uint8, device=dev, generator=g)
        a_p = nv.prepare_weight(ac, asc, S, K)
        one = torch.full((1,), 0.01, device=dev)
        y = torch.empty(S, N, dtype=torch.bfloat16, device=dev)
        fn = lambda i: nv.linear_wide(a_p, one, S, w_ps[i % ncopy], one, N, K, y=y)
        nbytes = N * K * 9 // 16
    elif case == "causal_attn":
        start, T = 22610, 128
        cache = I.kv_cache(3, start, T=T)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
        kp, vp, pt, ks, vs = t(cache.k_pool), t(cache.v_pool), t(cache.page_table), t(cache.k_scale), t(cache.v_scale)
        q = I.query_bf16(3, T).to(dev)
        out = torch.empty(T, 24, 128, dtype=torch.bfloat16, device=dev)
        pools = [(kp, vp)] + [(kp.clone(), vp.clone()) for _ in range(7)]   # > L2 per sweep
        fn = lambda i: nv.causal_attn(q, pools[i % 8][0], pools[i % 8][1], pt, start, ks, vs, out=out)
        nbytes = (start + T) * 4 * 128 * 2
    elif case == "attn":
        cache = I.kv_cache(3, I.CTX_MAX)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
        kp, vp, pt, ks, vs = t(cache.k_pool), t(cache.v_pool), t(cache.page_table), t(cache.k_scale), t(cache.v_scale)
        par, q = t(I.tree_parent(3)), I.query_bf16(3).to(dev)
        out = torch.empty(16, 24, 128, dtype=torch.bfloat16, device=dev)
        pools = [(kp, vp)] + [(kp.clone(), vp.clone()) for _ in range(7)]   # > L2 per sweep
        fn = lambda i: nv.tree_attn(q, pools[i % 8][0], pools[i % 8][1], pt, I.CTX_MAX, par, ks, vs, out=out)
        nbytes = (I.CTX_MAX + 16) * 4 * 128 * 2
    elif case == "restore":
        pb, n = 32768, 354 * 128
        src = torch.empty((n + 64) * pb, dtype=torch.uint8, device=dev)
        dst = torch.empty((n + 64) * pb, dtype=torch.uint8, device=dev)
        sid = torch.randperm(n + 64, device=dev, generator=g)[:n].to(torch.int32)
        did = torch.randperm(n + 64, device=dev, generator=g)[:n].to(torch.int32)
        fn = lambda i: nv.kv_page_restore(src, sid, dst, did, pb)
        nbytes = 2 * n * pb
    elif case == "rmsnorm_quantize":                      # the step's RMSNorm + NVFP4, static scale
        x = torch.randn(16, I.HIDDEN, device=dev, generator=g).to(torch.bfloat16)
        nw = torch.ones(I.HIDDEN, dtype=torch.bfloat16, device=dev)
        act = nv.act_buffer(I.HIDDEN)
        out = (None, None, torch.empty(1, dtype=torch.float32, device=dev))
        g_in = torch.full((1,), 0.002, dtype=torch.float32, device=dev)
        fn = lambda i: nv.rmsnorm_quantize(x, nw, 1e-6, out, act=act, g_in=g_in)
        nbytes = x.numel() * 2 + act.numel()
    else:
        x = torch.randn(16, I.FFN, device=dev, generator=g).to(torch.bfloat16)
        fn = lambda i: nv.quantize(x)
        nbytes = x.numel() * 2
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(3):
        fn(i + 3)
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) * 1e-3 / 3
    # the same calls back to back in one CUDA graph (dependent launch between
    # them, as inside the step), operands rotated so that each sweep exceeds L2
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        graph = capture(stream, lambda: [fn(6 + i) for i in range(20)])
        t_graph = time_graph(graph, stream, 5) / 20
    del graph
    print(json.dumps({"kernel_case": case, "us_per_call_incl_launch": round(t * 1e6, 2),
                      "us_per_call_graph": round(t_graph * 1e6, 2), "algorithmic_bytes": nbytes,
                      "gbs_graph": round(nbytes / t_graph / 1e9, 1), "status": nv.device_status()[0]}), flush=True)


def main():
    args = parse()
    if args.kernel_case:
        torch.cuda.set_device(0)
        run_kernel_case(args)
        return
    if args.prefill > 0 and args.impl == "ours":
        run_prefill(args)
        return
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
