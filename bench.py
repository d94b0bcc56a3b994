#!/usr/bin/env python3
"""Throughput of the MSA memory path on B200 (one JSON line on rank 0).

A step is one pass of the whole memory path over one batch of synthetic input:
msa_pool of the raw per-token K / V / Kr of every document into the bank, then
msa_layer_forward (route + top-k + index-driven gather + attention) for the
query of each layer.  The default workload is the 1M-token memory of the
Qwen3-4B-shaped layer (2048 documents x 512 tokens, Tq = 512 prefill tokens).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl msa|reference]

N > 1 runs under torchrun: each rank processes its own independent corpus and
queries (weak scaling, no data-path collective); times are the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import synth  # noqa: E402

METRIC = "MSA layer: routing memory-scan GB/s and query tokens/s at 1M–100M memory"
UNIT = "query tokens/s"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def workload_counts(cfg: synth.Config) -> dict:
    """Algorithmic work of one step (units: bytes, flops) for the roofline fields."""
    esz = 4 if cfg.dtype == "f32" else 2
    ntok, C = cfg.ntok, cfg.C
    row_in = (2 * cfg.Hkv * cfg.d + cfg.Hr * cfg.dr) * esz
    pool_bytes = ntok * row_in + C * row_in + C * cfg.Hr * 4
    route_bytes = C * cfg.Hr * cfg.dr * esz
    route_flops = 2.0 * cfg.B * cfg.Tq * cfg.Hr * cfg.dr * C
    # attention: every visible (query, key) pair costs 4 d flops (q.k and p.v)
    mem = cfg.Mmax  # every query's selected documents fill Mmax rows in these workloads
    pairs = sum(mem + cfg.Lloc - cfg.Tq + i + 1 for i in range(cfg.Tq))
    attn_flops = 4.0 * cfg.d * cfg.Hq * cfg.B * pairs
    return dict(pool_bytes=pool_bytes, route_bytes=route_bytes, route_flops=route_flops,
                attn_flops=attn_flops * cfg.layers, route_bytes_all=route_bytes * cfg.layers,
                route_flops_all=route_flops * cfg.layers)


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def traffic_record(kernel_file: str):
    """Per-launch DRAM bytes of the dominant kernel from a committed ncu summary,
    or None when the kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    src = os.path.join(ROOT, "routed_sparse_attention_chunk_b200", "csrc", kernel_file)
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    r = rec.get(kernel_file)
    if not r or r.get("source_sha256_16") != h:
        return None
    return r


def workload_config(args) -> synth.Config:
    cfg = synth.get_config(args.workload)
    if args.docs:
        cfg = cfg.scaled(D=args.docs, last_len=None, docs_per_slab=0)
    return cfg


# ----------------------------------------------------------------------------- GPU arm
class MSAWorkload:
    """Device buffers of one workload and its step (pool + every layer's fused forward)."""

    def __init__(self, cfg: synth.Config, device, seed: int):
        import routed_sparse_attention_chunk_b200 as msa
        self.msa, self.cfg, self.dev = msa, cfg, device
        dt = cfg.torch_dtype
        self.layers = [synth.gen_query(cfg, l, device, seed) for l in range(cfg.layers)]
        self.K, self.V, self.Kr = synth.gen_raw_slab(cfg, 0, cfg.D, device, seed, Qr0=self.layers[0]["Qr"][0])
        tok = synth.doc_tok_offsets(cfg)
        coff = msa.chunk_offsets(tok, cfg.P)
        self.D, self.C = cfg.D, int(coff[-1])
        self.tok_d = torch.from_numpy(tok).to(device)
        self.coff_d = torch.from_numpy(coff).to(device)
        self.rope = msa.rope_table(cfg.theta, cfg.d, int(np.diff(tok).max())).to(device)
        self.Kb = torch.empty((self.C, cfg.Hkv, cfg.d), dtype=dt, device=device)
        self.Vb = torch.empty_like(self.Kb)
        self.Krb = torch.empty((self.C, cfg.Hr, cfg.dr), dtype=dt, device=device)
        self.rn = torch.empty((self.C, cfg.Hr), dtype=torch.float32, device=device)
        self.flag = torch.zeros(1, dtype=torch.int32, device=device)
        B = cfg.B
        self.O = [torch.empty_like(L["Q"]) for L in self.layers]
        self.idx = [torch.empty((B, cfg.k), dtype=torch.int32, device=device) for _ in self.layers]
        nws = msa.layer_forward_workspace_size(B, cfg.Tq, cfg.Lloc, cfg.Hq, cfg.Hkv, cfg.d, cfg.Hr, self.D, cfg.k, cfg.Mmax)
        self.ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=device)

    def input_tensors(self):
        ts = [self.K, self.V, self.Kr]
        for L in self.layers:
            ts += [L["Qr"], L["Q"], L["Kloc"], L["Vloc"]]
        return ts

    def output_tensors(self):
        return self.O + self.idx

    def pool(self):
        c = self.cfg
        self.msa.pool(self.K, self.V, self.Kr, self.tok_d, self.coff_d, c.P, self.rope, self.Kb, self.Vb,
                      self.Krb, self.rn, self.flag)

    def layers_forward(self):
        c = self.cfg
        for l, L in enumerate(self.layers):
            self.msa.layer_forward(L["Qr"], self.Krb, self.rn, self.coff_d, c.k, L["Q"], L["Kloc"], L["Vloc"],
                                   self.Kb, self.Vb, c.Mmax, self.O[l], self.idx[l], self.ws, err_flag=self.flag)

    def step(self):
        self.pool()
        self.layers_forward()


def breakdown(w: MSAWorkload, counts: dict, peaks: dict, reps: int = 10) -> dict:
    """Per-step-kind times from the unfused entry points (outside the timed region)."""
    msa, c, dev = w.msa, w.cfg, w.dev
    L = w.layers[0]
    B = c.B
    ws = torch.empty(msa.route_topk_workspace_size(B, c.Tq, c.Hr, w.D, c.k), dtype=torch.uint8, device=dev)
    idx = torch.empty((B, c.k), dtype=torch.int32, device=dev)
    Km = torch.zeros((B, c.Mmax, c.Hkv, c.d), dtype=c.torch_dtype, device=dev)
    Vm = torch.zeros_like(Km)
    ml = torch.zeros(B, dtype=torch.int32, device=dev)
    O = torch.empty_like(L["Q"])
    aws_n = msa.sparse_attn_workspace_size(B, c.Tq, c.Lloc, c.Hq, c.Hkv, c.d, c.Mmax)
    aws = torch.empty(max(aws_n, 256), dtype=torch.uint8, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    fns = {
        "pool": w.pool,
        "route_topk": lambda: msa.route_topk(L["Qr"], w.Krb, w.rn, w.coff_d, c.k, idx, ws),
        "gather": lambda: msa.gather(idx, w.coff_d, w.Kb, w.Vb, Km, Vm, ml),
        "sparse_attn": lambda: msa.sparse_attn(L["Q"], L["Kloc"], L["Vloc"], Km, Vm, ml, O, ws=aws),
    }
    out = {}
    for name, fn in fns.items():
        fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1.0)  # cold L2 for every timed call
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        out[name] = {"ms": float(np.median(ts))}
    hbm = peaks["hbm_gbs"]
    tfl = peaks["bf16_tflops"]
    out["pool"].update(gbs=counts["pool_bytes"] / out["pool"]["ms"] / 1e6)
    out["pool"]["frac_hbm"] = out["pool"]["gbs"] / hbm
    r = out["route_topk"]
    r.update(scan_gbs=counts["route_bytes"] / r["ms"] / 1e6, tflops=counts["route_flops"] / r["ms"] / 1e9)
    r["frac_hbm"] = r["scan_gbs"] / hbm
    r["frac_tensor"] = r["tflops"] / tfl
    a = out["sparse_attn"]
    a.update(tflops=counts["attn_flops"] / c.layers / a["ms"] / 1e9)
    a["frac_tensor"] = a["tflops"] / tfl
    out["note"] = "unfused calls of layer 0, median of %d, L2 flushed before each" % reps
    return out


def run_gpu(args, rank, local_rank, world):
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    import routed_sparse_attention_chunk_b200 as msa
    cfg = workload_config(args)
    peaks, peak_kind = load_peaks()
    counts = workload_counts(cfg)
    w = MSAWorkload(cfg, device, seed=1000 * rank)
    in_bytes = sum(t.numel() * t.element_size() for t in w.input_tensors())
    flush = None if in_bytes > L2_BYTES else torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)

    # ---- warm-up, then exactly K timed steps
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(device)
    for _ in range(args.warmup):
        w.step()
    torch.cuda.synchronize()
    barrier(world, device)
    n0 = msa.kernel_launch_count()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_all0, t_all1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_all0.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.fill_(1.0)
        ev[i][0].record(stream)
        w.pool()
        ev[i][1].record(stream)
        w.layers_forward()
        ev[i][2].record(stream)
    t_all1.record(stream)
    torch.cuda.synchronize()
    launches = msa.kernel_launch_count() - n0
    clocks = sampler.stop()
    pool_ms = [a.elapsed_time(b) for a, b, _ in ev]
    layer_ms = [b.elapsed_time(c) for _, b, c in ev]
    step_ms_local = float(np.sum(pool_ms) + np.sum(layer_ms)) if flush is not None else t_all0.elapsed_time(t_all1)
    flag = int(w.flag.item())
    barrier(world, device)
    total_ms = max_over_ranks(step_ms_local, world, device)
    ms_per_step = total_ms / args.steps
    tokens_per_step = cfg.B * cfg.Tq * world
    value = tokens_per_step / (ms_per_step / 1e3)

    # ---- dominant kernel roofline (pool: HBM stream)
    pool_avg = float(np.mean(pool_ms))
    achieved = counts["pool_bytes"] / (pool_avg / 1e3) / 1e9
    tr = traffic_record("pool.cu")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": tr["dram_bytes_per_launch"] * (counts["pool_bytes"] / tr["alg_bytes_per_launch"]) if tr else None,
                "kernel": "pool_kernel (msa_pool)", "alg_bytes_per_launch": counts["pool_bytes"],
                "avg_launch_ms": round(pool_avg, 4), "peak_source": f"{peak_kind} hbm_gbs (copy test)"}

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        host_in = [t.detach().cpu().pin_memory() for t in w.input_tensors()]
        host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in w.output_tensors()]
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = sum(t.numel() * t.element_size() for t in host_out)
        dev_in, dev_out = w.input_tensors(), w.output_tensors()
        n_e2e = max(1, min(args.steps, args.e2e_steps))
        barrier(world, device)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            for d, h in zip(dev_in, host_in):
                d.copy_(h, non_blocking=True)
            w.step()
            for h, d in zip(host_out, dev_out):
                h.copy_(d, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device) / n_e2e
        e2e = {"value": round(tokens_per_step / (e2e_ms / 1e3), 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4), "steps": n_e2e}

    bd = breakdown(w, counts, peaks) if (rank == 0 and not args.no_breakdown) else None
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded generators; see workloads/synth.py)",
        "config": {"workload": f"{cfg.name}: {cfg.D} docs, {cfg.ntok} memory tokens, {cfg.C} chunks (P={cfg.P}), "
                               f"B={cfg.B} x Tq={cfg.Tq}, Lloc={cfg.Lloc}, Hq/Hkv/Hr={cfg.Hq}/{cfg.Hkv}/{cfg.Hr}, "
                               f"d={cfg.d}, k={cfg.k}, layers={cfg.layers}",
                   "step": "msa_pool of every raw token + msa_layer_forward per layer",
                   "l2": "inputs larger than L2" if flush is None else "L2 flushed between steps (not timed)",
                   "parallelism": f"{world} independent replica(s)" if world > 1 else "single GPU"},
        "route_scan_gbs": round(counts["route_bytes"] / (float(bd["route_topk"]["ms"]) / 1e3) / 1e9, 1) if bd else None,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "err_flag": flag,
        "breakdown": bd,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, budget_s=args.cpu_budget)
    if world > 1:
        import torch.distributed as dist
        barrier(world, device)
        dist.destroy_process_group()
    return result


# ----------------------------------------------------------------------------- CPU oracle arm
def oracle_step_sample(cfg: synth.Config, docs: int, tokens: int, seed: int = 0):
    """Time the oracle on a bounded sample of one step; returns (estimated full-step seconds, sample text).

    Pool: `docs` documents' raw tokens (time scaled by D / docs).  Query path of
    layer 0 (route over the full-size bank, top-k, gather, attention) for
    `tokens` query tokens (time scaled by Tq / tokens), times the layer count.
    """
    from oracle import msa_oracle as O
    wall0 = time.perf_counter()
    docs = max(1, min(docs, cfg.D))
    tokens = max(1, min(tokens, cfg.Tq))
    sub = cfg.scaled(D=docs, last_len=None, docs_per_slab=0, planted_doc=-1)
    K, V, Kr = synth.gen_raw_slab(sub, 0, docs, "cpu", seed)
    off = synth.doc_tok_offsets(sub)
    t0 = time.perf_counter()
    O.pool(K.double().numpy(), V.double().numpy(), Kr.double().numpy(), off, cfg.P, cfg.theta,
           out_bf16=cfg.dtype == "bf16")
    t_pool = (time.perf_counter() - t0) * cfg.D / docs
    # full-size bank for the query path (drawn, not pooled: only the time is used)
    rng = np.random.default_rng(seed)
    Krb = rng.standard_normal((cfg.C, cfg.Hr, cfg.dr)).astype(np.float32).astype(np.float64)
    coff = O.chunk_offsets(synth.doc_tok_offsets(cfg), cfg.P)
    q = synth.gen_query(cfg.scaled(Tq=tokens, Lloc=max(tokens, cfg.Lloc - cfg.Tq + tokens)), 0, "cpu", seed)
    Kb = rng.standard_normal((cfg.C, cfg.Hkv, cfg.d)).astype(np.float32)
    t0 = time.perf_counter()
    ds = O.route(q["Qr"].double().numpy(), Krb, coff)
    idx, _ = O.topk(ds, cfg.k)
    Km, Vm, ml = O.gather(idx, coff, Kb, Kb, cfg.Mmax)
    O.attention(q["Q"].double().numpy(), q["Kloc"].double().numpy(), q["Vloc"].double().numpy(), Km, Vm, ml)
    t_query = (time.perf_counter() - t0) * cfg.Tq / tokens * cfg.layers
    text = (f"oracle (numpy fp64) pool of {docs} of {cfg.D} documents scaled x{cfg.D / docs:.0f}; route over all "
            f"{cfg.C} chunks + top-k + gather + attention for {tokens} of {cfg.Tq} query tokens scaled "
            f"x{cfg.Tq / tokens:.0f}" + (f" and x{cfg.layers} layers" if cfg.layers > 1 else ""))
    return t_pool + t_query, text, time.perf_counter() - wall0


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg: synth.Config, budget_s: float = 20.0) -> dict:
    docs, tokens = 8, 16
    _, _, wall = oracle_step_sample(cfg, docs, tokens)           # calibration run
    grow = max(1.0, min(16.0, budget_s / max(wall, 1e-3)))
    est, text, wall = oracle_step_sample(cfg, int(docs * grow), int(tokens * grow))
    return {"value": round(cfg.B * cfg.Tq / est, 3), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": text + f"; sample wall {wall:.1f} s; host {os.cpu_count()} logical CPUs"}


def run_reference(args, rank, world):
    """The oracle arm: --steps K timed steps of a bounded sample, rank 0 only."""
    if rank != 0:
        return None
    cfg = workload_config(args)
    per_step = max(0.2, min(10.0, args.ref_budget / max(1, args.steps + args.warmup)))
    docs, tokens = 2, 4
    _, _, wall = oracle_step_sample(cfg, docs, tokens)          # calibration (counts as warm-up)
    grow = max(1.0, min(32.0, per_step / max(wall, 1e-3)))
    docs, tokens = int(docs * grow), int(tokens * grow)
    for _ in range(max(0, args.warmup - 1)):
        oracle_step_sample(cfg, docs, tokens)
    ests, texts = [], None
    wall0 = time.perf_counter()
    for _ in range(args.steps):
        e, texts, _ = oracle_step_sample(cfg, docs, tokens)
        ests.append(e)
    wall = time.perf_counter() - wall0
    est = float(np.mean(ests))
    value = cfg.B * cfg.Tq / est
    return {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(est * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generators; see workloads/synth.py)",
        "impl": "reference",
        "config": {"workload": cfg.name, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": texts + f"; {args.steps} steps in {wall:.1f} s wall (target {per_step:.1f} s/step)"},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="1m", choices=sorted(synth.CONFIGS))
    ap.add_argument("--docs", type=int, default=0, help="use only this many documents (smaller profiling case)")
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--ref-budget", type=float, default=120.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "msa":
        ap.error("--warmup must be >= 3")
    rank, local_rank, world = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_gpu(args, rank, local_rank, world)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
