#!/usr/bin/env python
"""Throughput of the quantised MoE layer on B200: one JSON line on rank 0.

A step is one coli_moe_forward of one batch of synthetic tokens through one
layer (router, Q8_0(x), batch-union expert gate/up + SwiGLU + Q8_0(h), down,
combine).  Default workload: single-token decode of the GLM-5.2-shaped layer
(hidden 6144, intermediate 2048, 256 routed + 1 shared expert, top-8 of 8
groups keeping 4, packed int4 weights, Q8_0 activations).  To keep the expert
weights out of L2 between steps, `--layers` distinct copies of the layer
(different seeds, 4.86 GB of int4 weights each) are cycled step by step.

Each rank (one per GPU) runs its own replica on its own tokens: no collective
is on the data path (weak scaling); ranks only meet at the barriers that
bracket the timed region and in the max-over-ranks reduction of its length.

--impl reference times the oracle (the scalar C reference under oracle/) on
this host's cores on a bounded sample of the same workload.
"""
import argparse
import concurrent.futures as cf
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s and expert-weight HBM GB/s (int4, top-8 of 256) on 1 B200"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=40000)
    p.add_argument("--warmup", type=int, default=200)
    p.add_argument("--impl", default="coli", choices=["coli", "reference"])
    p.add_argument("--workload", default="glm52_decode_int4_t1", choices=sorted(synth.WORKLOADS))
    p.add_argument("--tokens", type=int, default=None, help="override tokens per step")
    p.add_argument("--bits", type=int, default=None, choices=[8, 4, 2])
    p.add_argument("--layers", type=int, default=8)
    p.add_argument("--n-routed", type=int, default=None,
                   help="override the routed expert count (smaller layers for profiling)")
    p.add_argument("--e2e-steps", type=int, default=2000)
    p.add_argument("--profile-steps", type=int, default=400)
    p.add_argument("--cpu-sample-tokens", type=int, default=None,
                   help="tokens in the CPU-baseline sample (default: one per host thread)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-graph", action="store_true")
    p.add_argument("--no-prefill", action="store_true",
                   help="skip the extra batch-union prefill measurement (2048 tokens)")
    p.add_argument("--prefill-steps", type=int, default=10)
    return p.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def over_ranks(value, op, device):
    """`value` combined over every rank of the process group ("max" or "sum");
    the value itself when there is no group or a single rank."""
    dist = torch.distributed
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank_step, steps, world, ms_max):
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank_step * steps * world / (ms_max / 1e3)


def sm_max_mhz():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["sm_max_mhz"])
    except Exception:
        return 1965.0


def source_sha():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "quantized_expert_ffn_noaux_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """dram bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (profiles/*.md lines 'traffic: <kernel>
    <workload> <src_sha> <bytes_per_launch>')."""
    sha = source_sha()
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for f in sorted(os.listdir(pdir)):
        if not f.endswith((".md", ".txt")):
            continue
        for ln in open(os.path.join(pdir, f)):
            parts = ln.strip().split()
            if len(parts) == 5 and parts[0] == "traffic:" and parts[1] == kernel \
                    and parts[2] == workload and parts[3] == sha:
                return float(parts[4])
    return None


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.sel = str(device)

    def start(self):
        try:
            self.path = "/tmp/coli_clocks_%d.csv" % os.getpid()
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        for ln in open(self.path):
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                "sw_power_cap"), f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ coli arm
def build_layers(cfg, n_layers, max_tokens, device, qe):
    layers = []
    E, S, bits = cfg["n_routed"], cfg["n_shared"], cfg["bits"]
    for ell in range(n_layers):
        W, b = synth.router(cfg, device=device, layer=ell)
        experts = []
        for e in range(E + S):
            g, u, d = synth.expert_fp32(cfg, e, device=device, layer=ell)
            experts.append(qe.Expert.quantise(g, u, d, bits))
            del g, u, d
        lc = synth.layer_cfg(cfg)
        lc["max_tokens"] = max_tokens
        layers.append(qe.MoELayer(lc, W, b, experts))
    torch.cuda.synchronize()
    return layers


def expert_bytes(cfg):
    H, I, b = cfg["hidden"], cfg["inter"], cfg["bits"]
    gate = I * (H * b // 8) + 4 * I
    down = H * (I * b // 8) + 4 * H
    return 2 * gate, down


def run_coli(args, cfg, rank, world, device):
    import quantized_expert_ffn_noaux_b200 as qe
    T = cfg["tokens"]
    L = args.layers
    layers = build_layers(cfg, L, T, device, qe)
    # one distinct batch per layer and rank (weak scaling: ranks see different tokens)
    xs = [synth.tokens(cfg, T=T, device=device, layer=ell, stream=rank) for ell in range(L)]
    outs = [torch.empty_like(x) for x in xs]
    # batch-union sizes (distinct experts incl. shared) per layer, from the router
    union = []
    for ell in range(L):
        idx, _ = layers[ell].router(xs[ell])
        union.append(len(set(idx.cpu().numpy().reshape(-1).tolist())) + cfg["n_shared"])
    gu_b, dn_b = expert_bytes(cfg)
    bytes_per_step = [u * (gu_b + dn_b) for u in union]

    stream = torch.cuda.Stream(device=device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for ell in range(L):  # eager warm-up sets kernel attributes before capture
            layers[ell].forward(xs[ell], outs[ell])
    torch.cuda.synchronize()
    graphs = []
    launches_before = qe.launch_count()
    if not args.no_graph:
        for ell in range(L):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
                layers[ell].forward(xs[ell], outs[ell])
            graphs.append(g)
        launches_per_step = (qe.launch_count() - launches_before) / L
    else:
        launches_per_step = None

    def step(s):
        ell = s % L
        if graphs:
            graphs[ell].replay()
        else:
            layers[ell].forward(xs[ell], outs[ell])

    with torch.cuda.stream(stream):
        for s in range(args.warmup):
            step(s)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sampler = ClockSampler(device)
    sampler.start()
    time.sleep(0.3)
    c0 = qe.launch_count()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for s in range(args.steps):
            step(s)
        ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    ms = ev0.elapsed_time(ev1)
    if launches_per_step is None:
        launches_per_step = (qe.launch_count() - c0) / args.steps
    gpu_launches = int(round(launches_per_step * args.steps))
    bytes_timed = sum(bytes_per_step[s % L] for s in range(args.steps))
    ms = over_ranks(ms, "max", device)
    bytes_timed = over_ranks(bytes_timed, "sum", device)
    value = job_tokens_per_s(T, args.steps, world, ms)
    gbs = bytes_timed / (ms / 1e3) / 1e9

    # ---- per-kernel times (events on the launching stream), eager steps
    for lay in layers:
        lay.profile(True)
    with torch.cuda.stream(stream):
        for s in range(args.profile_steps):
            layers[s % L].forward(xs[s % L], outs[s % L])
    torch.cuda.synchronize()
    ktimes = {}
    for lay in layers:
        for name, (n, kms) in lay.profile_read().items():
            a = ktimes.setdefault(name, [0, 0.0])
            a[0] += n
            a[1] += kms
        lay.profile(False)
    dom = max(ktimes.items(), key=lambda kv: kv[1][1])[0]
    n_dom, ms_dom = ktimes[dom]
    avg_ms = ms_dom / n_dom
    prof_bytes = [bytes_per_step[s % L] for s in range(args.profile_steps)]
    frac_gu = gu_b / (gu_b + dn_b)
    # router weights + bias (fp32) and the fp32 token rows read and written
    router_b = cfg["n_routed"] * cfg["hidden"] * 4 + cfg["n_routed"] * 4
    io_b = 2 * T * cfg["hidden"] * 4
    if dom.startswith("moe_decode"):
        # the whole layer in one launch: every union expert's three matrices
        alg = statistics.mean(prof_bytes) + router_b + io_b
    elif dom.startswith("gateup"):
        alg = statistics.mean(prof_bytes) * frac_gu
    elif dom.startswith("down"):
        alg = statistics.mean(prof_bytes) * (1 - frac_gu)
    else:
        alg = None
    peak, peak_kind = peaks()
    roofline = None
    if dom.startswith("gateup_tc") or dom.startswith("down_tc"):
        # The tensor-core grouped GEMMs are bound by the exact promotion of
        # every 32-block product (int -> fp64 convert + fp64 FMA), not by
        # HBM: that fp64 work against the fp64 lanes of the part.
        H, I = cfg["hidden"], cfg["inter"]
        pairs = T * (cfg["top_k"] + cfg["n_shared"])
        if dom.startswith("gateup"):
            blocks, macs = pairs * 2 * I * (H // 32), pairs * 2 * I * H
        else:
            blocks, macs = pairs * H * (I // 32), pairs * H * I
        nsm = torch.cuda.get_device_properties(device).multi_processor_count
        sm_mhz = sm_max_mhz()
        peak_fp64 = nsm * 64 * sm_mhz * 1e6 / 1e9
        ach = 2 * blocks / (avg_ms / 1e3) / 1e9
        roofline = {"bound": "alu", "achieved": round(ach, 1), "peak": round(peak_fp64, 1), "unit": "Gop/s",
                    "frac": round(ach / peak_fp64, 4), "traffic": recorded_traffic(dom, cfg["name"]),
                    "kernel": dom, "ops": "fp64 promotion of 32-block int8 products: convert + FMA",
                    "peak_source": "derived: %d SMs x 64 fp64 lanes x %.0f MHz (max SM clock)" % (nsm, sm_mhz),
                    "ops_per_launch": int(2 * blocks), "avg_launch_ms": round(avg_ms, 5),
                    "int8_tensor_tops": round(2 * macs / (avg_ms / 1e3) / 1e12, 2),
                    "int8_tensor_frac_of_nominal_4500": round(2 * macs / (avg_ms / 1e3) / 1e12 / 4500.0, 4)}
    elif alg is not None:
        ach = alg / (avg_ms / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                    "frac": round(ach / peak, 4), "traffic": recorded_traffic(dom, cfg["name"]),
                    "kernel": dom, "peak_source": peak_kind + " (MEASURED_PEAKS.json hbm_gbs)"
                    if peak_kind == "measured" else "fallback 6.65 TB/s",
                    "algorithmic_bytes_per_launch": int(alg), "avg_launch_ms": round(avg_ms, 5)}
    kernel_share = {k: {"launches": v[0], "ms": round(v[1], 3)} for k, v in ktimes.items()}

    # ---- end to end through the public API with host buffers
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty_like(x).pin_memory() for x in xh]
    n_e2e = min(args.e2e_steps, args.steps)
    with torch.cuda.stream(stream):
        for s in range(min(args.warmup, 20)):
            layers[s % L].forward_host(xh[s % L], yh[s % L])
        if world > 1:
            torch.distributed.barrier()
        t0 = time.perf_counter()
        for s in range(n_e2e):
            layers[s % L].forward_host(xh[s % L], yh[s % L])
        e2e_s = time.perf_counter() - t0
    e2e_s = over_ranks(e2e_s, "max", device)
    e2e = {"value": round(T * n_e2e * world / e2e_s, 2), "unit": "tokens/s",
           "h2d_bytes_per_step": int(xh[0].numel() * 4), "d2h_bytes_per_step": int(yh[0].numel() * 4),
           "steps": n_e2e, "api": "coli_moe_forward_host (pinned host buffers, synchronous)"}

    result = {
        "value": value, "ms_per_step": ms / args.steps, "expert_weight_gbs": round(gbs, 1),
        "gpu_launches": gpu_launches, "clocks": clocks, "roofline": roofline, "e2e": e2e,
        "kernels": kernel_share, "union_experts_per_step": statistics.mean(union),
        "graph": bool(graphs),
    }
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, layers[0], xs[0], args.cpu_sample_tokens, device)
    for lay in layers:
        lay.close()
    graphs.clear()
    return result, cpu


def run_prefill(args, device):
    """The batch-union prefill workload (2048 tokens through one layer of the
    same shape; every expert is active): throughput and the bounds of its
    dominant kernel, timed with CUDA events on the launching stream."""
    import quantized_expert_ffn_noaux_b200 as qe
    cfg = synth.workload("glm52_prefill_int4_t2048")
    T = cfg["tokens"]
    lay = build_layers(cfg, 1, T, device, qe)[0]
    x = synth.tokens(cfg, T=T, device=device)
    out = torch.empty_like(x)
    stream = torch.cuda.Stream(device=device)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            lay.forward(x, out)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.prefill_steps):
            lay.forward(x, out)
        ev1.record(stream)
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / args.prefill_steps
    lay.profile(True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            lay.forward(x, out)
    torch.cuda.synchronize()
    kt = lay.profile_read()
    lay.profile(False)
    lay.close()
    H, I, E, S, k = cfg["hidden"], cfg["inter"], cfg["n_routed"], cfg["n_shared"], cfg["top_k"]
    gu_b, dn_b = expert_bytes(cfg)
    weight_bytes = (E + S) * (gu_b + dn_b)          # every expert is active at 2048 tokens
    pairs = T * (k + S)
    macs = pairs * 3 * H * I                        # gate, up, down
    peak, peak_kind = peaks()
    nsm = torch.cuda.get_device_properties(device).multi_processor_count
    dom = max(kt.items(), key=lambda kv: kv[1][1])[0]
    n_dom, ms_dom = kt[dom]
    dom_ms = ms_dom / n_dom
    blocks = pairs * 2 * I * (H // 32) if dom.startswith("gateup") else pairs * H * (I // 32)
    dmacs = pairs * 2 * I * H if dom.startswith("gateup") else pairs * H * I
    peak_fp64 = nsm * 64 * sm_max_mhz() * 1e6 / 1e9
    ach = 2 * blocks / (dom_ms / 1e3) / 1e9
    return {
        "workload": cfg["name"], "tokens_per_step": T, "value": round(T / (ms / 1e3), 1),
        "unit": "tokens/s", "ms_per_step": round(ms, 4), "steps": args.prefill_steps,
        "expert_weight_gbs": round(weight_bytes / (ms / 1e3) / 1e9, 1),
        "hbm_frac_of_step": round(weight_bytes / (ms / 1e3) / 1e9 / peak, 4),
        "int8_tensor_tops": round(2 * macs / (ms / 1e3) / 1e12, 2),
        "int8_tensor_frac_of_nominal_4500": round(2 * macs / (ms / 1e3) / 1e12 / 4500.0, 4),
        "roofline": {"bound": "alu", "achieved": round(ach, 1), "peak": round(peak_fp64, 1),
                     "unit": "Gop/s", "frac": round(ach / peak_fp64, 4), "kernel": dom,
                     "ops": "fp64 promotion of 32-block int8 products: convert + FMA",
                     "peak_source": "derived: %d SMs x 64 fp64 lanes x %.0f MHz" % (nsm, sm_max_mhz()),
                     "avg_launch_ms": round(dom_ms, 4),
                     "int8_tensor_tops": round(2 * dmacs / (dom_ms / 1e3) / 1e12, 2),
                     "traffic": recorded_traffic(dom, cfg["name"])},
        "hbm_peak": peak, "hbm_peak_source": peak_kind,
        "kernels": {kname: {"launches": v[0], "ms": round(v[1], 3)} for kname, v in kt.items()},
    }


def oracle_layer_for(cfg, Wr, bias, needed, fp32_fn, threads):
    import oracle
    E, S = cfg["n_routed"], cfg["n_shared"]
    exs = [None] * (E + S)
    need = sorted(set(needed) | set(range(E, E + S)))

    def q(e):
        mats = [m.cpu().numpy() for m in fp32_fn(e)]
        return e, oracle.QExpert.quantise(*mats, bits=cfg["bits"])

    with cf.ThreadPoolExecutor(max_workers=threads) as pool:
        for e, qx in pool.map(q, need):
            exs[e] = qx
    return oracle.Layer(synth.layer_cfg(cfg), Wr, bias, exs)


def cpu_baseline(cfg, layer0, x0, n_tok, device):
    """The oracle on this host's cores: n_tok tokens of the workload (layer 0),
    one token per OpenMP thread (the oracle splits tokens over threads and
    nothing finer), plus one token on a single thread."""
    import oracle
    threads = os.cpu_count() or 1
    n_tok = threads if n_tok is None else n_tok
    W, b = synth.router(cfg, device=device, layer=0)
    Wr, bias = W.cpu().numpy(), b.cpu().numpy()
    x = synth.tokens(cfg, T=n_tok, device=device, layer=0, stream=10**6).cpu().numpy()
    probe = oracle.Layer(synth.layer_cfg(cfg), Wr, bias,
                         [None] * (cfg["n_routed"] + cfg["n_shared"]))
    need = set(probe.route(x)["idx"].reshape(-1).tolist())
    lay = oracle_layer_for(cfg, Wr, bias, need,
                           lambda e: synth.expert_fp32(cfg, e, device=device, layer=0), threads)
    t0 = time.perf_counter()
    lay.forward(x, nthreads=threads)
    dt = time.perf_counter() - t0
    t0 = time.perf_counter()
    lay.forward(x[:1], nthreads=1)
    dt1 = time.perf_counter() - t0
    used = min(threads, n_tok)
    return {"value": round(n_tok / dt, 4), "unit": "tokens/s", "cores": used, "kind": "oracle",
            "single_thread": {"value": round(1.0 / dt1, 4), "unit": "tokens/s", "cores": 1},
            "sample": "%d tokens of %s (layer 0) in one oracle forward on %d OpenMP threads, "
                      "one token per thread, %.1f s; single thread: 1 token, %.2f s" % (
                          n_tok, cfg["name"], used, dt, dt1)}


# ------------------------------------------------------------- reference arm
def run_reference(args, cfg):
    """The oracle as the reference arm: each step is one token of the workload
    through the oracle on this host (a bounded sample when the run would be long)."""
    import oracle
    threads = os.cpu_count() or 1
    T = cfg["tokens"]
    W, b = synth.router(cfg, device="cpu")
    Wr, bias = W.numpy(), b.numpy()
    n = args.steps + args.warmup
    xs = synth.tokens(cfg, T=min(n, 64) * T, device="cpu", stream=7).numpy().reshape(-1, T,
                                                                                   cfg["hidden"])
    probe = oracle.Layer(synth.layer_cfg(cfg), Wr, bias, [None] * (cfg["n_routed"] + cfg["n_shared"]))
    need = set()
    routes = []
    for x in xs:
        r = probe.route(x)
        routes.append(r["idx"])
        need |= set(r["idx"].reshape(-1).tolist())
    lay = oracle_layer_for(cfg, Wr, bias, need, lambda e: synth.expert_fp32(cfg, e, device="cpu"),
                           threads)
    # per-step work: all experts of the batch unless (steps + warmup) of them would take
    # longer than ~150 s; then each step runs m of the k + S slots and counts m/(k+S) of a batch
    slots = cfg["top_k"] + cfg["n_shared"]
    t0 = time.perf_counter()
    lay.forward(xs[0], nthreads=threads)
    per_batch = time.perf_counter() - t0
    m = slots
    if n * per_batch > 150.0:
        m = max(1, int(150.0 / (n * per_batch) * slots))
    H, I = cfg["hidden"], cfg["inter"]

    def one(i):
        x = xs[i % len(xs)]
        if m == slots:
            lay.forward(x, nthreads=threads)
            return
        xq, xd = oracle.quant_q8(x)
        for t in range(T):
            for j in range(m):
                e = routes[i % len(xs)][t][j] if j < cfg["top_k"] else cfg["n_routed"] + j - cfg["top_k"]
                oracle.expert(H, I, cfg["bits"], lay.experts[e], xq[t], xd[t])

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(args.warmup + i)
    dt = time.perf_counter() - t0
    value = T * args.steps * (m / slots) / dt
    used = 1 if m != slots else min(threads, T)  # OpenMP splits tokens, nothing finer
    sample = ("each step: one %d-token batch of %s through the oracle (%s); the oracle splits "
              "tokens over OpenMP threads, so %d of %d host threads work"
              % (T, cfg["name"], "all %d expert slots" % slots if m == slots else
                 "%d of %d expert slots per token, counted as %d/%d of a batch" % (m, slots, m, slots),
                 used, threads))
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": cfg["name"], "tokens_per_step": T, "bits": cfg["bits"]},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    over = {}
    if args.tokens is not None:
        over["tokens"] = args.tokens
    if args.bits is not None:
        over["bits"] = args.bits
    if args.n_routed is not None:
        over["n_routed"] = args.n_routed
    cfg = synth.workload(args.workload, **over)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, cfg)), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    res, cpu = run_coli(args, cfg, rank, world, device)
    prefill = None
    if world == 1 and not args.no_prefill and args.workload == "glm52_decode_int4_t1" \
            and args.n_routed is None:
        torch.cuda.empty_cache()
        prefill = run_prefill(args, device)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(res["value"], 2), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(res["ms_per_step"], 6), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": cfg["name"], "tokens_per_step": cfg["tokens"],
                       "hidden": cfg["hidden"], "inter": cfg["inter"],
                       "experts": "%d routed + %d shared, top-%d, %d groups keep %d" % (
                           cfg["n_routed"], cfg["n_shared"], cfg["top_k"], cfg["n_group"],
                           cfg["topk_group"]),
                       "bits": cfg["bits"], "layers_cycled": args.layers,
                       "l2": "inputs larger than L2: %d distinct layers (%.2f GB of weights "
                             "each) cycled step by step" % (
                                 args.layers, sum(expert_bytes(cfg)) *
                                 (cfg["n_routed"] + cfg["n_shared"]) / 1e9),
                       "parallelism": "replicas, dp%d" % world, "cuda_graph": res["graph"]},
            "expert_weight_gbs": res["expert_weight_gbs"],
            "union_experts_per_step": res["union_experts_per_step"],
            "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": res["e2e"],
            "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
            "prefill": prefill,
            "kernels": res["kernels"],
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
