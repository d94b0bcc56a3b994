#!/usr/bin/env python3
"""Throughput of the MSA memory path on B200 (one JSON line on rank 0).

A step is one pass of the query path of every layer over one batch of
synthetic input, on a memory bank pooled (msa_pool) before the timed region:
per layer msa_route_topk (cosine routing scan of the whole bank + top-k) and
msa_sparse_attn_indexed (attention over the selected documents' chunks read
in place from the bank by index, ++ the causal local KV) -- the two calls
msa_layer_forward makes.  Pooling is the offline stage of the pages'
inference pipeline; it is timed on its own and reported beside the step.
The default workload is the 100M-token memory bank (195,313 documents,
1,562,500 chunks, Tq = 64 query tokens, Qwen3-4B-shaped heads); on one GPU
the same line also carries stage results of the 16M-token decode batch, the
10M-token 16-layer prefill stack and the 1M-token layer, each with the SM
clock it ran at.

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
    """SM clock and throttle-reason samples (NVML, every ~2 ms) while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device: torch.device):
        import threading
        self.samples, self.max_mhz, self.err = [], None, None
        self._stop = threading.Event()
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self._h = nv.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
            self._nv = nv
        except Exception as e:  # no NVML: report that instead of clocks
            self._nv, self.err = None, f"nvml unavailable: {type(e).__name__}"
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)))
            except Exception:
                pass
            self._stop.wait(0.002)

    def start(self):
        if self._nv is not None:
            self._t.start()

    def stop(self) -> dict:
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err], "samples": 0}
        self._stop.set()
        self._t.join(timeout=5)
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        return {"sm_mhz": float(np.median(mhz)) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if bits & b], "samples": len(mhz)}


def sustained_region(timed_ms: float, clocks: dict) -> bool:
    """Whether the tensor roofline takes the sustained bf16 peak (measured as a
    seconds-long loop under the power cap) rather than the burst one: the timed
    region ran for over a second, or the power cap throttled it."""
    return timed_ms > 1000.0 or "sw_power_cap" in (clocks.get("reasons") or [])


def traffic_record(kernel_file: str, workload: str):
    """Per-launch DRAM bytes (read + write) of a kernel on a workload from the
    committed ncu summary profiles/traffic.json, or None when the record is
    missing or the kernel's source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    r = rec.get(f"{kernel_file}:{workload}")
    src = os.path.join(ROOT, "routed_sparse_attention_chunk_b200", "csrc", kernel_file)
    if not r or not os.path.exists(src):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != r.get("source_sha256_16"):
        return None
    return r


def workload_label(cfg: synth.Config) -> str:
    return (f"{cfg.name}: {cfg.D} docs, {cfg.ntok} memory tokens, {cfg.C} chunks (P={cfg.P}), "
            f"B={cfg.B} x Tq={cfg.Tq}, Lloc={cfg.Lloc}, Hq/Hkv/Hr={cfg.Hq}/{cfg.Hkv}/{cfg.Hr}, "
            f"d={cfg.d}, k={cfg.k}, layers={cfg.layers}")


def raw_bytes(cfg: synth.Config) -> int:
    """Bytes of the raw per-token K, V and Kr of the whole corpus."""
    return cfg.ntok * (2 * cfg.Hkv * cfg.d + cfg.Hr * cfg.dr) * (4 if cfg.dtype == "f32" else 2)


RAW_RESIDENT_MAX = 80e9  # a corpus this large is pooled slab by slab instead of held resident


def step_label(step_kind: str, unfused: bool = False) -> str:
    q = ("per layer msa_route_topk, msa_gather, msa_sparse_attn" if unfused else
         "per layer msa_route_topk + msa_sparse_attn_indexed (the calls of msa_layer_forward: routing scan + top-k, "
         "then attention over the selected chunks read in place from the bank)")
    return ("msa_pool of every raw token, then " + q) if step_kind == "full" else \
        (q + " over a bank pooled before timing")


def step_kind_for(cfg: synth.Config, args) -> str:
    """'query' (the query path over a bank pooled before timing) unless --step full asks for the
    offline pool inside the step too (only when the raw corpus fits the device next to the bank and
    the bank's K̄ / V̄ stay on the device)."""
    if getattr(args, "bank_kv", "device") == "host":
        return "query"
    if args.step == "full" and raw_bytes(cfg) <= RAW_RESIDENT_MAX:
        return "full"
    return "query"


def workload_config(args) -> synth.Config:
    cfg = synth.get_config(args.workload)
    if args.docs:
        cfg = cfg.scaled(D=args.docs, last_len=None)
    return cfg


# ----------------------------------------------------------------------------- GPU arm
class MSAWorkload:
    """Device buffers of one workload and its step.

    The bank (K̄, V̄, K̄r, 1/‖K̄r‖) is pooled at set-up: from a resident raw corpus
    in one msa_pool call when the corpus fits the device (then the pool can be
    timed on its own, or inside the step with step "full"), else slab by slab as
    the raw tokens are drawn (a 100M-token corpus cannot be resident), with the
    pool launches timed by events as they run.  The step per layer is
    msa_route_topk then msa_sparse_attn_indexed (unfused: msa_gather then
    msa_sparse_attn on the copied rows).
    """

    def __init__(self, cfg: synth.Config, device, seed: int, step_kind: str, bank_kv: str = "device",
                 unfused: bool = False, keep_raw: bool = False):
        import routed_sparse_attention_chunk_b200 as msa
        self.msa, self.cfg, self.dev, self.kind, self.unfused = msa, cfg, device, step_kind, unfused
        dt = cfg.torch_dtype
        self.layers = [synth.gen_query(cfg, l, device, seed) for l in range(cfg.layers)]
        tok = synth.doc_tok_offsets(cfg)
        coff = msa.chunk_offsets(tok, cfg.P)
        self.tok, self.coff = tok, coff
        self.D, self.C = cfg.D, int(coff[-1])
        self.tok_d = torch.from_numpy(tok).to(device)
        self.coff_d = torch.from_numpy(coff).to(device)
        self.rope = msa.rope_table(cfg.theta, cfg.d, int(np.diff(tok).max())).to(device)
        self.Kb = torch.empty((self.C, cfg.Hkv, cfg.d), dtype=dt, device=device)
        self.Vb = torch.empty_like(self.Kb)
        self.Krb = torch.empty((self.C, cfg.Hr, cfg.dr), dtype=dt, device=device)
        self.rn = torch.empty((self.C, cfg.Hr), dtype=torch.float32, device=device)
        self.flag = torch.zeros(1, dtype=torch.int32, device=device)
        self.raw = None
        self.slab_pool_ms = None  # pool launches of the slab-by-slab set-up, timed by events
        if (step_kind == "full" or keep_raw) and raw_bytes(cfg) <= RAW_RESIDENT_MAX:
            self._fill_raw(seed)
            self.pool()
            torch.cuda.synchronize()
        else:
            self._pool_slabs(seed)
        if bank_kv == "host":
            # host tier: K̄ / V̄ in page-locked host memory, read in place by the gather
            self.Kb = self.Kb.cpu().pin_memory()
            self.Vb = self.Vb.cpu().pin_memory()
            torch.cuda.empty_cache()
        B, c = cfg.B, cfg
        self.O = [torch.empty_like(L["Q"]) for L in self.layers]
        self.idx = [torch.empty((B, c.k), dtype=torch.int32, device=device) for _ in self.layers]
        self.rws = torch.empty(msa.route_topk_workspace_size(B, c.Tq, c.Hr, self.D, self.C, c.k), dtype=torch.uint8,
                               device=device)
        self.iws = torch.empty(max(256, msa.sparse_attn_indexed_workspace_size(B, c.Tq, c.Lloc, c.Hq, c.Hkv, c.d, c.k,
                                                                                c.Mmax)),
                               dtype=torch.uint8, device=device)
        n = msa.sparse_attn_workspace_size(B, c.Tq, c.Lloc, c.Hq, c.Hkv, c.d, c.Mmax)
        self.aws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
        if unfused:
            self.Km = torch.zeros((B, c.Mmax, c.Hkv, c.d), dtype=dt, device=device)
            self.Vm = torch.zeros_like(self.Km)
            self.ml = torch.zeros(B, dtype=torch.int32, device=device)
        self.pipe = None

    @property
    def stages(self):
        q = ("route_topk", "gather", "sparse_attn") if self.unfused else ("route_topk", "sparse_attn")
        return (("pool",) if self.kind == "full" else ()) + q

    def enable_pipeline(self):
        """Run the query path through the three-stream schedule (route of batch i+1, gather of batch
        i and attention of batch i-1 overlapped); a second topk_idx per layer lets route and gather of
        consecutive batches overlap."""
        from routed_sparse_attention_chunk_b200.pipeline import QueryPipeline
        c = self.cfg
        bank = dict(Krbar=self.Krb, kr_rnorm=self.rn, doc_chunk_off=self.coff_d, Kbar=self.Kb, Vbar=self.Vb)
        self.pipe = QueryPipeline(bank, c.k, c.Mmax, c.B, c.Tq, c.Lloc, c.Hq, c.Hkv, c.d, c.Hr, c.torch_dtype,
                                  self.dev, err_flag=self.flag)
        self.idx2 = [torch.empty_like(t) for t in self.idx]

    def pipelined_steps(self, n, marks=None):
        """n steps (every layer of each) enqueued through the schedule in one call, so consecutive steps
        overlap too; the caller's stream waits for all of it."""
        runs = []
        for i in range(n):
            for l, L in enumerate(self.layers):
                runs.append(dict(L, O=self.O[l], topk_idx=(self.idx[l] if (i * len(self.layers) + l) % 2 == 0
                                                            else self.idx2[l])))
        self.pipe.run(runs, marks)

    def _fill_raw(self, seed):
        """Resident raw K / V / Kr for the whole corpus, drawn slab by slab."""
        c, n = self.cfg, int(self.tok[-1])
        dt = c.torch_dtype
        self.raw = (torch.empty((n, c.Hkv, c.d), dtype=dt, device=self.dev),
                    torch.empty((n, c.Hkv, c.d), dtype=dt, device=self.dev),
                    torch.empty((n, c.Hr, c.dr), dtype=dt, device=self.dev))
        for lo, hi in synth.slab_bounds(c):
            t0, t1 = int(self.tok[lo]), int(self.tok[hi])
            for dst, src in zip(self.raw, synth.gen_raw_slab(c, lo, hi, self.dev, seed, Qr0=self.layers[0]["Qr"][0])):
                dst[t0:t1].copy_(src)
        torch.cuda.synchronize()

    def _pool_slabs(self, seed):
        c, msa = self.cfg, self.msa
        stream = torch.cuda.current_stream()
        evs = []
        for lo, hi in synth.slab_bounds(c):
            K, V, Kr = synth.gen_raw_slab(c, lo, hi, self.dev, seed, Qr0=self.layers[0]["Qr"][0])
            t = torch.from_numpy(self.tok[lo:hi + 1] - self.tok[lo]).to(self.dev)
            cs, ce = int(self.coff[lo]), int(self.coff[hi])
            ch = torch.from_numpy(self.coff[lo:hi + 1] - self.coff[lo]).to(self.dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            msa.pool(K, V, Kr, t, ch, c.P, self.rope, self.Kb[cs:ce], self.Vb[cs:ce], self.Krb[cs:ce],
                     self.rn[cs:ce], self.flag)
            e1.record(stream)
            evs.append((e0, e1))
            del K, V, Kr
        torch.cuda.synchronize()
        self.slab_pool_ms = [e0.elapsed_time(e1) for e0, e1 in evs]

    def input_tensors(self):
        ts = list(self.raw) if (self.raw is not None and self.kind == "full") else []
        for L in self.layers:
            ts += [L["Qr"], L["Q"], L["Kloc"], L["Vloc"]]
        return ts

    def output_tensors(self):
        return self.O + self.idx

    # the stages of one step
    def pool(self):
        c = self.cfg
        K, V, Kr = self.raw
        self.msa.pool(K, V, Kr, self.tok_d, self.coff_d, c.P, self.rope, self.Kb, self.Vb, self.Krb, self.rn,
                      self.flag)

    def route_topk(self, l):
        self.msa.route_topk(self.layers[l]["Qr"], self.Krb, self.rn, self.coff_d, self.cfg.k, self.idx[l], self.rws,
                            err_flag=self.flag)

    def gather(self, l):
        self.msa.gather(self.idx[l], self.coff_d, self.Kb, self.Vb, self.Km, self.Vm, self.ml, self.flag)

    def sparse_attn(self, l):
        L = self.layers[l]
        if self.unfused:
            self.msa.sparse_attn(L["Q"], L["Kloc"], L["Vloc"], self.Km, self.Vm, self.ml, self.O[l], ws=self.aws,
                                 err_flag=self.flag)
        else:
            self.msa.sparse_attn_indexed(L["Q"], L["Kloc"], L["Vloc"], self.idx[l], self.coff_d, self.Kb, self.Vb,
                                         self.cfg.Mmax, self.O[l], self.iws, err_flag=self.flag)

    def step(self, rec=None):
        """One step; rec(stage) records an event after each stage when given."""
        if self.kind == "full":
            self.pool()
            rec and rec("pool")
        for l in range(self.cfg.layers):
            self.route_topk(l)
            rec and rec("route_topk")
            if self.unfused:
                self.gather(l)
                rec and rec("gather")
            self.sparse_attn(l)
            rec and rec("sparse_attn")


def stage_roofline(name: str, ms: float, cfg: synth.Config, counts: dict, peaks: dict, peak_kind: str,
                   long_region: bool) -> dict:
    """Roofline object of one stage from its live per-launch time."""
    tfl = peaks.get("bf16_tflops_sustained" if long_region else "bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tfl_name = "bf16_tflops_sustained" if long_region else "bf16_tflops"
    hbm = peaks["hbm_gbs"]
    esz = 4 if cfg.dtype == "f32" else 2
    if name == "pool":
        return {"bound": "hbm", "achieved": counts["pool_bytes"] / ms / 1e6, "peak": hbm, "unit": "GB/s",
                "kernel": "pool_kernel (msa_pool)", "alg_bytes_per_launch": counts["pool_bytes"],
                "peak_source": f"{peak_kind} hbm_gbs"}
    if name == "route_topk":
        inten = counts["route_flops"] / counts["route_bytes"]
        if inten < tfl * 1e3 / hbm:
            return {"bound": "hbm", "achieved": counts["route_bytes"] / ms / 1e6, "peak": hbm, "unit": "GB/s",
                    "kernel": "msa_route_topk (query norms + tcgen05 scan + top-k)",
                    "alg_bytes_per_launch": counts["route_bytes"], "peak_source": f"{peak_kind} hbm_gbs"}
        return {"bound": "tensor", "achieved": counts["route_flops"] / ms / 1e9, "peak": tfl, "unit": "TFLOP/s",
                "kernel": "msa_route_topk (query norms + tcgen05 scan + top-k)",
                "alg_flops_per_launch": counts["route_flops"], "peak_source": f"{peak_kind} {tfl_name}"}
    if name == "sparse_attn":
        fl = counts["attn_flops"] / cfg.layers
        if cfg.Tq == 1:  # decode: the local and memory KV stream
            by = cfg.B * (cfg.Lloc + cfg.Mmax) * cfg.Hkv * cfg.d * esz * 2
            return {"bound": "hbm", "achieved": by / ms / 1e6, "peak": hbm, "unit": "GB/s",
                    "kernel": "msa_sparse_attn_indexed (plan + attn_decode_kernel + combine)",
                    "alg_bytes_per_launch": by, "peak_source": f"{peak_kind} hbm_gbs"}
        return {"bound": "tensor", "achieved": fl / ms / 1e9, "peak": tfl, "unit": "TFLOP/s",
                "kernel": "msa_sparse_attn_indexed (plan + attn_tc_kernel)", "alg_flops_per_launch": fl,
                "peak_source": f"{peak_kind} {tfl_name}"}
    by = 2 * 2 * cfg.B * cfg.Mmax * cfg.Hkv * cfg.d * esz
    return {"bound": "hbm", "achieved": by / ms / 1e6, "peak": hbm, "unit": "GB/s", "kernel": "gather_kernel",
            "alg_bytes_per_launch": by, "peak_source": f"{peak_kind} hbm_gbs"}


def timed_steps(w: MSAWorkload, steps: int, warmup: int, flush, world: int, device):
    """W untimed steps, then exactly K steps with an event after every stage.  Returns per-stage
    launch times (ms), the whole timed region (ms), NVML clocks during it and the launch count."""
    msa = w.msa
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(device)
    for _ in range(warmup):
        w.step()
    torch.cuda.synchronize()
    barrier(world, device)
    sampler.start()
    n0 = msa.kernel_launch_count()
    marks = []  # (stage, event) in launch order

    def rec(stage):
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        marks.append((stage, e))

    t_all0, t_all1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_all0.record(stream)
    for _ in range(steps):
        if flush is not None:
            flush.fill_(1.0)
        rec("start")
        w.step(rec)
    t_all1.record(stream)
    torch.cuda.synchronize()
    launches = msa.kernel_launch_count() - n0
    clocks = sampler.stop()
    stage_ms = {s: [] for s in w.stages}
    for (s0, e0), (s1, e1) in zip(marks[:-1], marks[1:]):
        if s1 != "start":
            stage_ms[s1].append(e0.elapsed_time(e1))
    return stage_ms, t_all0.elapsed_time(t_all1), clocks, launches


def timed_pool(w: MSAWorkload, launches: int, warmup: int, device):
    """msa_pool of the resident raw corpus on its own: per-launch times (ms) and clocks."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        w.pool()
    torch.cuda.synchronize()
    sampler = ClockSampler(device)
    sampler.start()
    ev = []
    for _ in range(launches):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        w.pool()
        e1.record(stream)
        ev.append((e0, e1))
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in ev], sampler.stop()


def read_stream_gbs(device, gib: int = 4) -> float:
    """Read-only HBM stream measured live: a torch sum over a `gib` GiB bf16 tensor (best of 5)."""
    x = torch.ones(gib * (1 << 29), dtype=torch.bfloat16, device=device)
    nbytes = x.numel() * x.element_size()
    best = float("inf")
    for _ in range(6):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch.sum(x, dtype=torch.float32)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del x
    torch.cuda.empty_cache()
    return nbytes / (best / 1e3) / 1e9


def stage_entry(name, times, cfg, counts, peaks, peak_kind, long_region, clocks, total=None) -> dict:
    """Per-stage summary: time per launch, achieved work rate and its fraction of the peak, and
    the launch's length in SM cycles at the median clock sampled while it ran."""
    per = float(np.mean(times))
    r = stage_roofline(name, per, cfg, counts, peaks, peak_kind, long_region)
    mhz = clocks.get("sm_mhz")
    out = {"ms_per_launch": round(per, 4), "launches": len(times), "bound": r["bound"],
           "achieved": round(r["achieved"], 2), "unit": r["unit"], "peak": r["peak"],
           "frac": round(r["achieved"] / r["peak"], 4), "peak_source": r["peak_source"],
           "sm_mhz": mhz, "kcycles_per_launch": round(per * mhz, 1) if mhz else None}
    if total:
        out["share"] = round(float(np.sum(times)) / total, 4)
    return out


def workload_extra(name: str, device, seed: int, peaks: dict, peak_kind: str, steps: int, warmup: int) -> dict:
    """Stage results of another workload, measured in the same run: the query-path step (W warm-up,
    K timed), each stage's achieved rate against its roofline, and the offline pool on its own."""
    cfg = synth.get_config(name)
    counts = workload_counts(cfg)
    keep_raw = raw_bytes(cfg) <= RAW_RESIDENT_MAX
    w = MSAWorkload(cfg, device, seed=seed, step_kind="query", keep_raw=keep_raw)
    in_bytes = w.Krb.numel() * w.Krb.element_size() + sum(t.numel() * t.element_size() for t in w.input_tensors())
    flush = None if in_bytes > L2_BYTES else torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    stage_ms, timed_ms, clocks, launches = timed_steps(w, steps, warmup, flush, 1, device)
    step_sum = sum(sum(v) for v in stage_ms.values())
    ms_per_step = (step_sum if flush is not None else timed_ms) / steps
    long_region = sustained_region(timed_ms, clocks)
    out = {"workload": workload_label(cfg), "step": step_label("query"), "steps": steps, "warmup": warmup,
           "ms_per_step": round(ms_per_step, 4), "value": round(cfg.B * cfg.Tq / (ms_per_step / 1e3), 1),
           "unit": UNIT, "clocks": clocks, "gpu_launches": int(launches),
           "l2": "inputs larger than L2" if flush is None else "L2 flushed between steps (not timed)",
           "stages": {s: stage_entry(s, v, cfg, counts, peaks, peak_kind, long_region, clocks, step_sum)
                      for s, v in stage_ms.items() if v}}
    if cfg.Tq > 1 and cfg.layers > 1:
        # the attention kernel alone: every layer's msa_sparse_attn_indexed back to back (its clock is
        # not the one the routing scan leaves it inside the step), W warm-up rounds, then K timed rounds
        stream = torch.cuda.current_stream()
        for _ in range(warmup):
            for l in range(cfg.layers):
                w.sparse_attn(l)
        torch.cuda.synchronize()
        sampler = ClockSampler(device)
        sampler.start()
        ev = []
        for _ in range(steps):
            for l in range(cfg.layers):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                w.sparse_attn(l)
                e1.record(stream)
                ev.append((e0, e1))
        torch.cuda.synchronize()
        aclocks = sampler.stop()
        at = [a.elapsed_time(b) for a, b in ev]
        out["sparse_attn_alone"] = stage_entry("sparse_attn", at, cfg, counts, peaks, peak_kind,
                                               sustained_region(float(np.sum(at)), aclocks), aclocks)
        out["sparse_attn_alone"]["clocks"] = aclocks
    if w.raw is not None:
        n = 3 if raw_bytes(cfg) > 20e9 else 10
        ptimes, pclocks = timed_pool(w, n, 2, device)
        out["offline_pool"] = stage_entry("pool", ptimes, cfg, counts, peaks, peak_kind,
                                          sustained_region(float(np.sum(ptimes)), pclocks), pclocks)
        out["offline_pool"]["clocks"] = pclocks
    elif w.slab_pool_ms:
        out["offline_pool"] = slab_pool_entry(w, cfg, counts, peaks, peak_kind)
    out["err_flag"] = int(w.flag.item())
    del w
    torch.cuda.empty_cache()
    return out


def slab_pool_entry(w: MSAWorkload, cfg, counts, peaks, peak_kind) -> dict:
    """The bank built slab by slab at set-up: total pool time over every slab (one pass, events)."""
    ms = float(np.sum(w.slab_pool_ms))
    gbs = counts["pool_bytes"] / ms / 1e6
    return {"ms_total": round(ms, 3), "slabs": len(w.slab_pool_ms), "achieved": round(gbs, 2), "unit": "GB/s",
            "peak": peaks["hbm_gbs"], "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": f"{peak_kind} hbm_gbs",
            "note": "one pass over the corpus while the bank is built (no warm-up); the slabs' raw tokens are drawn "
                    "between launches"}


def run_backward(args, rank, local_rank, world):
    """Backward of the query path: per layer msa_sparse_attn_backward + msa_gather_backward +
    msa_route_backward, the forward outputs (O, lse, the gathered rows) computed once before timing."""
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    import routed_sparse_attention_chunk_b200 as msa
    cfg = workload_config(args)
    counts = workload_counts(cfg)
    w = MSAWorkload(cfg, device, seed=1000 * rank, step_kind="query")
    B, c = cfg.B, cfg
    f32 = dict(dtype=torch.float32, device=device)
    dt = cfg.torch_dtype
    layers = []
    for l in range(cfg.layers):
        L = w.layers[l]
        w.route_topk(l)
        Km = torch.zeros((B, c.Mmax, c.Hkv, c.d), dtype=dt, device=device)
        Vm = torch.zeros_like(Km)
        ml = torch.zeros(B, dtype=torch.int32, device=device)
        msa.gather(w.idx[l], w.coff_d, w.Kb, w.Vb, Km, Vm, ml, w.flag)
        lse = torch.empty((B, c.Hq, c.Tq), **f32)
        msa.sparse_attn(L["Q"], L["Kloc"], L["Vloc"], Km, Vm, ml, w.O[l], lse, ws=w.aws, err_flag=w.flag)
        g = torch.Generator(device=device).manual_seed(7 + l)
        dO = (0.5 * torch.randn(L["Q"].shape, generator=g, device=device)).to(dt)
        layers.append((L, Km, Vm, ml, lse, dO))
    dQ = torch.empty((B, c.Tq, c.Hq, c.d), **f32)
    dKl, dVl = torch.empty((B, c.Lloc, c.Hkv, c.d), **f32), torch.empty((B, c.Lloc, c.Hkv, c.d), **f32)
    dKm, dVm = torch.empty((B, c.Mmax, c.Hkv, c.d), **f32), torch.empty((B, c.Mmax, c.Hkv, c.d), **f32)
    dKb, dVb = torch.zeros((w.C, c.Hkv, c.d), **f32), torch.zeros((w.C, c.Hkv, c.d), **f32)
    bws = torch.empty(max(256, msa.sparse_attn_backward_workspace_size(B, c.Tq, c.Hq)), dtype=torch.uint8,
                      device=device)
    # routing-score backward: the routing loss is not given, so its gradient per selected document is a
    # seeded synthetic input; dQr / dK̄r accumulate over the layers like dK̄ / dV̄
    d_score = [torch.randn((B, c.k), generator=torch.Generator(device=device).manual_seed(11 + l), device=device)
               for l in range(cfg.layers)]
    dQr = torch.zeros((B, c.Tq, c.Hr, c.dr), **f32)
    dKrb = torch.zeros((w.C, c.Hr, c.dr), **f32)
    rbws = torch.empty(max(256, msa.route_backward_workspace_size(B, c.Tq, c.k)), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    marks = []

    def rec(stage):
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        marks.append((stage, e))

    def step(r=None):
        for l, (L, Km, Vm, ml, lse, dO) in enumerate(layers):
            msa.sparse_attn_backward(L["Q"], L["Kloc"], L["Vloc"], Km, Vm, ml, w.O[l], lse, dO, dQ, dKl, dVl, dKm,
                                     dVm, bws, err_flag=w.flag)
            r and r("attn_backward")
            msa.gather_backward(w.idx[l], w.coff_d, dKm, dVm, ml, dKb, dVb, w.flag)
            r and r("gather_backward")
            msa.route_backward(L["Qr"], w.Krb, w.rn, w.coff_d, w.idx[l], d_score[l], dQr, dKrb, rbws, w.flag)
            r and r("route_backward")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world, device)
    sampler = ClockSampler(device)
    sampler.start()
    n0 = msa.kernel_launch_count()
    for _ in range(args.steps):
        rec("start")
        step(rec)
    torch.cuda.synchronize()
    launches = msa.kernel_launch_count() - n0
    clocks = sampler.stop()
    stage_ms = {"attn_backward": [], "gather_backward": [], "route_backward": []}
    for (s0, e0), (s1, e1) in zip(marks[:-1], marks[1:]):
        if s1 != "start":
            stage_ms[s1].append(e0.elapsed_time(e1))
    step_sum = sum(sum(v) for v in stage_ms.values())
    flag = int(w.flag.item())
    barrier(world, device)
    total_ms = max_over_ranks(step_sum, world, device)
    ms_per_step = total_ms / args.steps
    value = B * c.Tq * world / (ms_per_step / 1e3)
    per = float(np.mean(stage_ms["attn_backward"]))
    flops = 2.5 * counts["attn_flops"] / cfg.layers  # 10 d flops per visible (row, key) pair: s, dp, dq, dk, dv
    achieved = flops / per / 1e9
    gper = float(np.mean(stage_ms["gather_backward"]))
    rper = float(np.mean(stage_ms["route_backward"]))
    G = c.Hq // c.Hkv
    tensor = cfg.dtype == "bf16" and c.d == 128 and 128 % G == 0 and 128 // G >= 8
    if tensor:  # the tcgen05 dQ and dK / dV kernels: the bf16 tensor peak
        peaks, peak_kind = load_peaks()
        long_region = sustained_region(step_sum, clocks)
        pname = "bf16_tflops_sustained" if long_region else "bf16_tflops"
        peak = peaks.get(pname, FALLBACK_PEAKS["bf16_tflops"])
        bound, kname, psrc = "tensor", "attn_dq_tc_kernel + attn_dkv_tc_kernel (tcgen05)", f"{peak_kind} {pname}"
    else:  # CUDA-core fp32 peak from the unit counts and the maximum SM clock: SMs x 128 FMA lanes x 2 flops
        mhz = clocks.get("sm_max_mhz") or 1965
        peak = torch.cuda.get_device_properties(device).multi_processor_count * 128 * 2 * mhz * 1e6 / 1e12
        bound, kname = "alu", "bwd_dq_kernel + bwd_dkv_kernel (CUDA cores, fp32)"
        psrc = "derived: SMs x 128 fp32 lanes x 2 x max SM clock"
    return {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 (gradients; inputs " + cfg.dtype + ")", "data": "synthetic",
        "config": {"workload": workload_label(cfg), "step": "backward: per layer msa_sparse_attn_backward + "
                   "msa_gather_backward + msa_route_backward (forward outputs computed before timing; the routing "
                   "loss's gradient per selected document is a seeded synthetic input)", "parallelism": "single GPU"},
        "roofline": {"bound": bound, "achieved": round(achieved, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                     "kernel": kname, "alg_flops_per_launch": flops,
                     "peak_source": psrc, "frac": round(achieved / peak, 4),
                     "avg_launch_ms": round(per, 4), "traffic": None},
        "stages": {"attn_backward": {"ms_per_launch": round(per, 4)},
                   "gather_backward": {"ms_per_launch": round(gper, 4)},
                   "route_backward": {"ms_per_launch": round(rper, 4)}},
        "gpu_launches": launches, "clocks": clocks, "err_flag": flag,
    }


STATE_SHAPE = (32, 128, 128)  # a linear (DGA) layer's recurrent state: value heads x key dim x value dim


def run_state(args, rank, local_rank, world):
    """The linear (DGA) layers' memory injection: per query, the sum of its k
    selected documents' recurrent states (msa_state_gather_sum).  The states are a
    seeded synthetic bank of min(D, 8192) documents (the routing that picks them is
    timed by the forward pass); each step draws a fresh selection of k distinct
    documents per query, and L2 is flushed before every launch."""
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    import routed_sparse_attention_chunk_b200 as msa
    cfg = workload_config(args)
    dt = cfg.torch_dtype
    Dst = min(cfg.D, 8192)
    S = int(np.prod(STATE_SHAPE))
    g = torch.Generator(device=device).manual_seed(17 + 1000 * rank)
    states = torch.empty((Dst,) + STATE_SHAPE, dtype=dt, device=device)
    for i in range(0, Dst, 256):  # in slices, so no fp32 copy of the whole bank exists at once
        states[i:i + 256] = torch.randn((min(256, Dst - i),) + STATE_SHAPE, generator=g, device=device).to(dt)
    n_sel = args.warmup + args.steps
    sel = torch.stack([torch.stack([torch.randperm(Dst, generator=g, device=device)[:cfg.k] for _ in range(cfg.B)])
                       for _ in range(n_sel)]).to(torch.int32)
    out = torch.empty((cfg.B,) + STATE_SHAPE, dtype=torch.float32, device=device)
    flag = torch.zeros(1, dtype=torch.int32, device=device)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=device)  # 256 MB, twice the L2
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        flush.fill_(1.0)
        msa.state_gather_sum(states, sel[i], out, err_flag=flag)
    torch.cuda.synchronize()
    barrier(world, device)
    sampler = ClockSampler(device)
    sampler.start()
    n0 = msa.kernel_launch_count()
    ev = []
    for i in range(args.steps):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        msa.state_gather_sum(states, sel[args.warmup + i], out, err_flag=flag)
        e1.record(stream)
        ev.append((e0, e1))
    torch.cuda.synchronize()
    launches = msa.kernel_launch_count() - n0
    clocks = sampler.stop()
    step_sum = sum(e0.elapsed_time(e1) for e0, e1 in ev)
    barrier(world, device)
    total_ms = max_over_ranks(step_sum, world, device)
    ms_per_step = total_ms / args.steps
    esz = states.element_size()
    by = cfg.B * cfg.k * S * esz + cfg.B * S * 4  # the selected states read once, one fp32 state written
    peaks, peak_kind = load_peaks()
    achieved = by / (step_sum / args.steps) / 1e6
    value = cfg.B * cfg.Tq * world / (ms_per_step / 1e3)
    return {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype + " states, f32 sums", "data": "synthetic",
        "config": {"workload": workload_label(cfg),
                   "step": f"msa_state_gather_sum: per query the sum of {cfg.k} selected documents' recurrent "
                           f"states of {STATE_SHAPE[0]} x {STATE_SHAPE[1]} x {STATE_SHAPE[2]} from a bank of {Dst}",
                   "l2": "flushed before every launch", "parallelism": "single GPU"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "kernel": "state_sum_kernel (msa_state_gather_sum)", "alg_bytes_per_launch": by,
                     "peak_source": f"{peak_kind} hbm_gbs", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "avg_launch_ms": round(step_sum / args.steps, 4), "traffic": None},
        "gpu_launches": launches, "clocks": clocks, "err_flag": int(flag.item()),
    }


EXTRA_WORKLOADS = ("decode16m", "stack10m", "1m")
EXTRA_STEPS = {"decode16m": 30, "stack10m": 8, "1m": 30}


DGA_HEADS = (16, 32)  # key heads, value heads of the linear layers (d = 128); the pages give no head counts


GDR_TOKEN_MAX = 16  # msa_gated_delta_rule takes its token-by-token kernel up to this many query tokens


def run_dga(args, rank, local_rank, world):
    """The linear (DGA) layers' memory path for the workload's queries: per step, the sum of each
    query's k selected documents' recurrent states (msa_state_gather_sum, S_ext) and the gated delta
    rule over the query tokens from S_ext (msa_gated_delta_rule).  States, selections and token
    projections are seeded synthetic inputs; L2 is flushed before every step."""
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    import routed_sparse_attention_chunk_b200 as msa
    cfg = workload_config(args)
    dt = cfg.torch_dtype
    Hk, Hv = DGA_HEADS
    d = 128
    B, T = cfg.B, cfg.Tq
    Dst = min(cfg.D, 4096)
    g = torch.Generator(device=device).manual_seed(23 + 1000 * rank)
    states = torch.empty((Dst, Hv, d, d), dtype=dt, device=device)
    for i in range(0, Dst, 256):
        states[i:i + 256] = (0.1 * torch.randn((min(256, Dst - i), Hv, d, d), generator=g, device=device)).to(dt)
    sel = torch.stack([torch.randperm(Dst, generator=g, device=device)[:cfg.k] for _ in range(B)]).to(torch.int32)
    kk = torch.randn((B, T, Hk, d), generator=g, device=device)
    kk = (kk / kk.norm(dim=-1, keepdim=True)).to(dt)
    q = (torch.randn((B, T, Hk, d), generator=g, device=device) * 0.35).to(dt)
    v = torch.randn((B, T, Hv, d), generator=g, device=device).to(dt)
    lg = -0.3 * torch.rand((B, T, Hv), generator=g, device=device)
    beta = torch.rand((B, T, Hv), generator=g, device=device)
    S_ext = torch.empty((B, Hv, d, d), dtype=torch.float32, device=device)
    o = torch.empty((B, T, Hv, d), dtype=dt, device=device)
    flag = torch.zeros(1, dtype=torch.int32, device=device)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        msa.state_gather_sum(states, sel, S_ext, err_flag=flag)
        if ev is not None:
            ev.record(stream)
        msa.gated_delta_rule(q, kk, v, lg, beta, o, S_ext)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    barrier(world, device)
    sampler = ClockSampler(device)
    sampler.start()
    n0 = msa.kernel_launch_count()
    marks = []
    for _ in range(args.steps):
        flush.fill_(1.0)
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        step(e1)
        e2.record(stream)
        marks.append((e0, e1, e2))
    torch.cuda.synchronize()
    launches = msa.kernel_launch_count() - n0
    clocks = sampler.stop()
    sum_ms = [a.elapsed_time(b) for a, b, _ in marks]
    gdr_ms = [b.elapsed_time(c) for _, b, c in marks]
    step_local = sum(sum_ms) + sum(gdr_ms)
    barrier(world, device)
    ms_per_step = max_over_ranks(step_local, world, device) / args.steps
    value = B * T * world / (ms_per_step / 1e3)
    per = float(np.mean(gdr_ms))
    flops = 6.0 * d * d * Hv * B * T  # per token and value head: k^T h, the rank-1 update and h^T q
    mhz = clocks.get("sm_max_mhz") or 1965
    peak = torch.cuda.get_device_properties(device).multi_processor_count * 128 * 2 * mhz * 1e6 / 1e12
    S = Hv * d * d
    sum_bytes = B * cfg.k * S * states.element_size() + B * S * 4
    peaks, peak_kind = load_peaks()
    return {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype + " inputs, f32 state", "data": "synthetic",
        "config": {"workload": workload_label(cfg),
                   "step": f"linear (DGA) layer memory path: msa_state_gather_sum of {cfg.k} selected documents' "
                           f"states ({Hv} x {d} x {d}, from a bank of {Dst}) then msa_gated_delta_rule over {T} "
                           f"query tokens x {B} queries ({Hk} key heads, {Hv} value heads, d = {d})",
                   "l2": "flushed before every step", "parallelism": "single GPU"},
        "roofline": {"bound": "alu", "achieved": round(flops / per / 1e9, 2), "peak": round(peak, 1),
                     "unit": "TFLOP/s",
                     "kernel": ("gdr_token_kernel" if T <= GDR_TOKEN_MAX else "gdr_chunk_kernel") + " (msa_gated_delta_rule)",
                     "alg_flops_per_launch": flops,
                     "peak_source": "derived: SMs x 128 fp32 lanes x 2 x max SM clock",
                     "frac": round(flops / per / 1e9 / peak, 4), "avg_launch_ms": round(per, 4), "traffic": None},
        "stages": {"state_gather_sum": {"ms_per_launch": round(float(np.mean(sum_ms)), 4),
                                        "achieved": round(sum_bytes / float(np.mean(sum_ms)) / 1e6, 2),
                                        "unit": "GB/s", "peak": peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs"},
                   "gated_delta_rule": {"ms_per_launch": round(per, 4)}},
        "gpu_launches": launches, "clocks": clocks, "err_flag": int(flag.item()),
    }


def interleave_roofline(cfg: synth.Config, counts: dict, rounds: int, ms: float, peaks: dict, peak_kind: str,
                        long_region: bool) -> dict:
    """Roofline of one msa_interleave_forward call, taken against its `rounds` routing scans of the bank
    (the dominant work): the call is one C-ABI launch sequence, so the attention rounds and the
    router-query projections run inside the same time and the figure is a lower bound on the scans'
    rate.  The bound (HBM or tensor) is the routing stage's for the workload."""
    r = stage_roofline("route_topk", ms / rounds, cfg, counts, peaks, peak_kind, long_region)
    key = "alg_bytes_per_launch" if r["bound"] == "hbm" else "alg_flops_per_launch"
    r[key] = r[key] * rounds
    r["kernel"] = (f"msa_interleave_forward ({rounds} rounds: routing scans of the bank, plus the attention rounds "
                   "and router-query projections in the same time)")
    r["achieved"] = round(r["achieved"], 2)
    r["frac"] = round(r["achieved"] / r["peak"], 4)
    r["avg_launch_ms"] = round(ms, 4)
    r["traffic"] = None
    return r


def run_interleave(args, rank, local_rank, world):
    """Memory Interleave of the query path: per layer one msa_interleave_forward call of `--rounds`
    rounds (route, the k best documents no earlier round chose, attention over every round's documents
    ++ the local KV; the next round's router query is the round's output times a seeded W_route) over
    a bank pooled before timing."""
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    import routed_sparse_attention_chunk_b200 as msa
    cfg = workload_config(args)
    R = args.rounds
    if R < 1:
        raise SystemExit("--rounds must be >= 1")
    counts = workload_counts(cfg)
    w = MSAWorkload(cfg, device, seed=1000 * rank, step_kind="query")
    B, c = cfg.B, cfg
    dt = cfg.torch_dtype
    Mmax = R * c.Mmax  # every round's k documents fill Mmax rows in these workloads
    g = torch.Generator(device=device).manual_seed(77 + 1000 * rank)
    W = (torch.randn((c.Hq * c.d, c.Hr * c.dr), generator=g, device=device) / 64).to(dt) if R > 1 else None
    ws = torch.empty(max(256, msa.interleave_workspace_size(B, c.Tq, c.Lloc, c.Hq, c.Hkv, c.d, c.Hr, c.dr, w.D, w.C,
                                                            c.k, R, Mmax)), dtype=torch.uint8, device=device)
    idx = [torch.empty((B, R * c.k), dtype=torch.int32, device=device) for _ in w.layers]
    lse = torch.empty((B, c.Hq, c.Tq), dtype=torch.float32, device=device)
    in_bytes = w.Krb.numel() * w.Krb.element_size()  # every round scans the whole bank
    flush = None if in_bytes > L2_BYTES else torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def step(marks=None):
        for l, L in enumerate(w.layers):
            e0 = torch.cuda.Event(enable_timing=True) if marks is not None else None
            if e0 is not None:
                e0.record(stream)
            msa.interleave_forward(L["Qr"], w.Krb, w.rn, w.coff_d, c.k, R, W, L["Q"], L["Kloc"], L["Vloc"], w.Kb,
                                   w.Vb, Mmax, w.O[l], idx[l], ws, lse=lse, err_flag=w.flag)
            if e0 is not None:
                e1 = torch.cuda.Event(enable_timing=True)
                e1.record(stream)
                marks.append((e0, e1))

    for _ in range(args.warmup):
        if flush is not None:
            flush.fill_(1.0)
        step()
    torch.cuda.synchronize()
    barrier(world, device)
    sampler = ClockSampler(device)
    sampler.start()
    n0 = msa.kernel_launch_count()
    marks = []
    for _ in range(args.steps):
        if flush is not None:
            flush.fill_(1.0)
        step(marks)
    torch.cuda.synchronize()
    launches = msa.kernel_launch_count() - n0
    clocks = sampler.stop()
    call_ms = [a.elapsed_time(b) for a, b in marks]
    step_sum = float(np.sum(call_ms))
    flag = int(w.flag.item())
    barrier(world, device)
    ms_per_step = max_over_ranks(step_sum, world, device) / args.steps
    value = B * c.Tq * world / (ms_per_step / 1e3)
    peaks, peak_kind = load_peaks()
    per = float(np.mean(call_ms))
    roofline = interleave_roofline(cfg, counts, R, per, peaks, peak_kind, sustained_region(step_sum, clocks))
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded generators; see workloads/synth.py)",
        "config": {"workload": workload_label(cfg),
                   "step": f"Memory Interleave: per layer one msa_interleave_forward of {R} rounds (route + top-k of "
                           f"{c.k} new documents, attention over all rounds' documents ++ local KV; next router "
                           f"query = output x seeded W_route) over a bank pooled before timing",
                   "l2": "inputs larger than L2" if flush is None else "L2 flushed between steps (not timed)",
                   "parallelism": f"{world} independent replicas" if world > 1 else "single GPU"},
        "roofline": roofline,
        "stages": {"interleave_forward": {"ms_per_launch": round(per, 4), "launches": len(call_ms)}},
        "gpu_launches": int(launches), "clocks": clocks, "err_flag": flag,
    }
    if world > 1:
        import torch.distributed as dist
        barrier(world, device)
        dist.destroy_process_group()
    return result


def run_gpu(args, rank, local_rank, world):
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    import routed_sparse_attention_chunk_b200 as msa
    cfg = workload_config(args)
    step_kind = step_kind_for(cfg, args)
    peaks, peak_kind = load_peaks()
    counts = workload_counts(cfg)
    w = MSAWorkload(cfg, device, seed=1000 * rank, step_kind=step_kind, bank_kv=args.bank_kv,
                    unfused=args.unfused or args.bank_kv == "host")
    in_bytes = sum(t.numel() * t.element_size() for t in w.input_tensors())
    in_bytes += w.Krb.numel() * w.Krb.element_size()  # the scan reads the whole bank every step
    flush = None if in_bytes > L2_BYTES else torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)

    if args.pipeline:
        if step_kind != "query":
            raise SystemExit("--pipeline runs the query path over a bank pooled before timing (--step query)")
        w.enable_pipeline()
        return run_pipelined(args, rank, world, device, w, cfg, counts, peaks, peak_kind, flush)

    # ---- warm-up, then exactly K timed steps, an event after every stage
    stage_ms, timed_ms, clocks, launches = timed_steps(w, args.steps, args.warmup, flush, world, device)
    step_sum = sum(sum(v) for v in stage_ms.values())
    step_ms_local = step_sum if flush is not None else timed_ms
    flag = int(w.flag.item())
    barrier(world, device)
    total_ms = max_over_ranks(step_ms_local, world, device)
    ms_per_step = total_ms / args.steps
    tokens_per_step = cfg.B * cfg.Tq * world  # query tokens through the whole layer stack
    value = tokens_per_step / (ms_per_step / 1e3)

    # ---- roofline of the dominant stage (live per-launch times from the timed region)
    per_launch = {s: float(np.mean(v)) for s, v in stage_ms.items() if v}
    totals = {s: float(np.sum(v)) for s, v in stage_ms.items() if v}
    dom = max(totals, key=totals.get)
    long_region = sustained_region(timed_ms, clocks)
    roofline = stage_roofline(dom, per_launch[dom], cfg, counts, peaks, peak_kind, long_region)
    roofline["achieved"] = round(roofline["achieved"], 2)
    roofline["frac"] = round(roofline["achieved"] / roofline["peak"], 4)
    roofline["avg_launch_ms"] = round(per_launch[dom], 4)
    tr = traffic_record({"pool": "pool.cu", "route_topk": "route_tc.cu",
                         "sparse_attn": "attn_decode.cu" if cfg.Tq == 1 else "attn_tc.cu",
                         "gather": "gather.cu"}[dom], cfg.name)
    roofline["traffic"] = tr["dram_bytes_per_launch"] if tr else None
    if roofline["bound"] == "hbm" and world == 1:
        rs = read_stream_gbs(device)
        roofline["read_stream_gbs"] = round(rs, 1)
        roofline["frac_of_read_stream"] = round(roofline["achieved"] / rs, 4)
        roofline["read_stream_source"] = "measured in this run: torch sum over a 4 GiB bf16 tensor, best of 5"
    stages = {s: stage_entry(s, v, cfg, counts, peaks, peak_kind, long_region, clocks, step_sum)
              for s, v in stage_ms.items() if v}

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        host_in = [t.detach().cpu().pin_memory() for t in w.input_tensors()]
        host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in w.output_tensors()]
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = sum(t.numel() * t.element_size() for t in host_out)
        dev_in, dev_out = w.input_tensors(), w.output_tensors()
        n_e2e = max(1, min(args.steps, args.e2e_steps))
        stream = torch.cuda.current_stream()
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

    route_ms = per_launch.get("route_topk")
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded generators; see workloads/synth.py)",
        "config": {"workload": workload_label(cfg),
                   "step": step_label(step_kind, w.unfused),
                   **({"bank_kv": "pinned host memory, read in place by msa_gather"} if args.bank_kv == "host" else {}),
                   "l2": "inputs larger than L2" if flush is None else "L2 flushed between steps (not timed)",
                   "parallelism": f"{world} independent replicas" if world > 1 else "single GPU"},
        "route_scan_gbs": round(counts["route_bytes"] / (route_ms / 1e3) / 1e9, 1) if route_ms else None,
        "roofline": roofline,
        "stages": stages,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "err_flag": flag,
    }
    if step_kind == "query" and w.slab_pool_ms:
        result["offline_pool"] = slab_pool_entry(w, cfg, counts, peaks, peak_kind)
    extra = [x for x in (args.extra.split(",") if args.extra not in (None, "", "none") else [])
             if x and x != cfg.name]
    for x in extra:
        if x not in synth.CONFIGS:
            raise SystemExit(f"--extra: unknown workload {x}")
    if extra and world == 1 and args.bank_kv == "device" and not args.docs:
        del w
        torch.cuda.empty_cache()
        result["workloads"] = {}
        for name in extra:
            result["workloads"][name] = workload_extra(name, device, 0, peaks, peak_kind,
                                                       EXTRA_STEPS.get(name, 20), 3)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, budget_s=args.cpu_budget, with_pool=step_kind == "full")
    if world > 1:
        import torch.distributed as dist
        barrier(world, device)
        dist.destroy_process_group()
    return result


def host_link_gbs(device, mib: int = 256) -> float:
    """Page-locked host -> device copy bandwidth (copy engine, best of 5): the host link's measured peak."""
    h = torch.empty(mib << 20, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(mib << 20, dtype=torch.uint8, device=device)
    best = float("inf")
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        d.copy_(h, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    return (mib << 20) / (best / 1e3) / 1e9


def run_pipelined(args, rank, world, device, w, cfg, counts, peaks, peak_kind, flush):
    """Timed region: the K steps enqueued through the three-stream schedule in one call; per-stage
    launch times from events recorded on each stage's own stream."""
    import routed_sparse_attention_chunk_b200 as msa
    stream = torch.cuda.current_stream()
    link = host_link_gbs(device) if args.bank_kv == "host" else None
    sampler = ClockSampler(device)
    w.pipelined_steps(args.warmup)
    torch.cuda.synchronize()
    barrier(world, device)
    sampler.start()
    n0 = msa.kernel_launch_count()
    marks = []
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    w.pipelined_steps(args.steps, marks)
    t1.record(stream)
    torch.cuda.synchronize()
    launches = msa.kernel_launch_count() - n0
    clocks = sampler.stop()
    timed_ms = t0.elapsed_time(t1)
    flag = int(w.flag.item())
    barrier(world, device)
    ms_per_step = max_over_ranks(timed_ms, world, device) / args.steps
    tokens_per_step = cfg.B * cfg.Tq * world
    value = tokens_per_step / (ms_per_step / 1e3)
    stage_ms = {}
    for stage, e0, e1 in marks:
        stage_ms.setdefault(stage, []).append(e0.elapsed_time(e1))
    per_launch = {st: float(np.mean(v)) for st, v in stage_ms.items()}
    totals = {st: float(np.sum(v)) for st, v in stage_ms.items()}
    dom = max(totals, key=totals.get)
    long_region = sustained_region(timed_ms, clocks)
    if dom == "gather" and link is not None:
        esz = 4 if cfg.dtype == "f32" else 2
        rows = int(w.pipe.ml[(w.pipe.n - 1) % 2].sum())  # rows the last batch selected (every batch alike)
        by = 2 * rows * cfg.Hkv * cfg.d * esz  # K̄ and V̄ rows crossing the host link
        roofline = {"bound": "host_link", "achieved": by / per_launch[dom] / 1e6, "peak": round(link, 1),
                    "unit": "GB/s", "kernel": "gather_kernel (msa_gather, K̄ / V̄ in page-locked host memory)",
                    "alg_bytes_per_launch": by,
                    "peak_source": "measured in this run: page-locked host to device copy, 256 MiB, best of 5"}
    else:
        roofline = stage_roofline(dom, per_launch[dom], cfg, counts, peaks, peak_kind, long_region)
    roofline["achieved"] = round(roofline["achieved"], 2)
    roofline["frac"] = round(roofline["achieved"] / roofline["peak"], 4)
    roofline["avg_launch_ms"] = round(per_launch[dom], 4)
    roofline["traffic"] = None
    stages = {st: {"ms_per_launch": round(per_launch[st], 4),
                   "busy_per_step": round(totals[st] / args.steps / ms_per_step, 4)} for st in per_launch}

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
            w.pipelined_steps(1)
            for h, d in zip(host_out, dev_out):
                h.copy_(d, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device) / n_e2e
        e2e = {"value": round(tokens_per_step / (e2e_ms / 1e3), 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4), "steps": n_e2e,
               "note": "inputs copied in and outputs read back every step, so steps do not overlap"}
    route_ms = per_launch.get("route_topk")
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded generators; see workloads/synth.py)",
        "config": {"workload": workload_label(cfg),
                   "step": step_label("query") + "; three-stream schedule: route of batch i+1, gather of batch i "
                   "and attention of batch i-1 overlap",
                   **({"bank_kv": "pinned host memory, read in place by msa_gather"} if args.bank_kv == "host" else {}),
                   "l2": "inputs larger than L2" if flush is None else "L2 not flushed: steps overlap by design",
                   "parallelism": f"{world} independent replicas" if world > 1 else "single GPU"},
        "route_scan_gbs": round(counts["route_bytes"] / (route_ms / 1e3) / 1e9, 1) if route_ms else None,
        "roofline": roofline,
        "stages": stages,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "err_flag": flag,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, budget_s=args.cpu_budget, with_pool=False)
    if world > 1:
        import torch.distributed as dist
        barrier(world, device)
        dist.destroy_process_group()
    return result


# ----------------------------------------------------------------------------- CPU oracle arm
def oracle_step_sample(cfg: synth.Config, docs: int, tokens: int, seed: int = 0, with_pool: bool = True,
                       rdocs: int = 0):
    """Time the oracle on a bounded sample of one step; returns (estimated full-step seconds, sample text,
    sample wall seconds).

    Pool (only when the step includes it): `docs` documents' raw tokens, time
    scaled by D / docs.  Query path of layer 0 for `tokens` query tokens: the
    route over the chunks of `rdocs` documents (time scaled by C / their chunks
    and by Tq / tokens), the top-k over those documents' scores (scaled by
    D / rdocs), then gather + attention (scaled by Tq / tokens); times the
    layer count.
    """
    from oracle import msa_oracle as O
    wall0 = time.perf_counter()
    docs = max(1, min(docs, cfg.D))
    tokens = max(1, min(tokens, cfg.Tq))
    rdocs = max(cfg.k, min(rdocs or cfg.D, cfg.D))
    t_pool = 0.0
    if with_pool:
        sub = cfg.scaled(D=docs, last_len=None, docs_per_slab=0, planted_doc=-1)
        K, V, Kr = synth.gen_raw_slab(sub, 0, docs, "cpu", seed)
        off = synth.doc_tok_offsets(sub)
        t0 = time.perf_counter()
        O.pool(K.double().numpy(), V.double().numpy(), Kr.double().numpy(), off, cfg.P, cfg.theta,
               out_bf16=cfg.dtype == "bf16")
        t_pool = (time.perf_counter() - t0) * cfg.D / docs
    # a bank of the first rdocs documents' chunks (drawn, not pooled: only the time is used)
    coff = O.chunk_offsets(synth.doc_tok_offsets(cfg), cfg.P)
    scoff = coff[: rdocs + 1]
    Cs = int(scoff[-1])
    rng = np.random.default_rng(seed)
    Krb = rng.standard_normal((Cs, cfg.Hr, cfg.dr)).astype(np.float32).astype(np.float64)
    Kb = rng.standard_normal((Cs, cfg.Hkv, cfg.d)).astype(np.float32)
    q = synth.gen_query(cfg.scaled(Tq=tokens, Lloc=max(tokens, cfg.Lloc - cfg.Tq + tokens)), 0, "cpu", seed)
    t0 = time.perf_counter()
    ds = O.route(q["Qr"].double().numpy(), Krb, scoff)
    t_route = (time.perf_counter() - t0) * (cfg.C / Cs) * (cfg.Tq / tokens)
    t0 = time.perf_counter()
    idx, _ = O.topk(ds, cfg.k)
    t_topk = (time.perf_counter() - t0) * cfg.D / rdocs
    t0 = time.perf_counter()
    Km, Vm, ml = O.gather(idx, scoff, Kb, Kb, cfg.Mmax)
    O.attention(q["Q"].double().numpy(), q["Kloc"].double().numpy(), q["Vloc"].double().numpy(), Km, Vm, ml)
    t_attn = (time.perf_counter() - t0) * cfg.Tq / tokens
    est = t_pool + (t_route + t_topk + t_attn) * cfg.layers
    text = ((f"oracle (numpy fp64) pool of {docs} of {cfg.D} documents scaled x{cfg.D / docs:.0f}; " if with_pool
             else "oracle (numpy fp64), bank pooled outside the step; ") +
            f"route over {Cs} of {cfg.C} chunks ({rdocs} of {cfg.D} documents) for {tokens} of {cfg.Tq} query "
            f"tokens scaled x{cfg.C / Cs:.1f} x{cfg.Tq / tokens:.0f}, top-k scaled x{cfg.D / rdocs:.1f}, gather + "
            f"attention for {tokens} tokens scaled x{cfg.Tq / tokens:.0f}" +
            (f", x{cfg.layers} layers" if cfg.layers > 1 else ""))
    return est, text, time.perf_counter() - wall0


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg: synth.Config, budget_s: float = 20.0, with_pool: bool = True) -> dict:
    docs, tokens, rdocs = 8, 16, 512
    _, _, wall = oracle_step_sample(cfg, docs, tokens, with_pool=with_pool, rdocs=rdocs)   # calibration run
    grow = max(1.0, min(16.0, budget_s / max(wall, 1e-3)))
    est, text, wall = oracle_step_sample(cfg, int(docs * grow), int(tokens * grow), with_pool=with_pool,
                                         rdocs=int(rdocs * grow))
    return {"value": round(cfg.B * cfg.Tq / est, 3), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": text + f"; sample wall {wall:.1f} s; host {os.cpu_count()} logical CPUs"}


def run_reference(args, rank, world):
    """The oracle arm: --steps K timed steps of a bounded sample, rank 0 only."""
    if rank != 0:
        return None
    cfg = workload_config(args)
    kind = step_kind_for(cfg, args)
    wp = kind == "full"
    per_step = max(0.2, min(10.0, args.ref_budget / max(1, args.steps + args.warmup)))
    docs, tokens, rdocs = 2, 4, 256
    _, _, wall = oracle_step_sample(cfg, docs, tokens, with_pool=wp, rdocs=rdocs)   # calibration (a warm-up)
    grow = max(1.0, min(32.0, per_step / max(wall, 1e-3)))
    docs, tokens, rdocs = int(docs * grow), int(tokens * grow), int(rdocs * grow)
    for _ in range(max(0, args.warmup - 1)):
        oracle_step_sample(cfg, docs, tokens, with_pool=wp, rdocs=rdocs)
    ests, texts = [], None
    wall0 = time.perf_counter()
    for _ in range(args.steps):
        e, texts, _ = oracle_step_sample(cfg, docs, tokens, with_pool=wp, rdocs=rdocs)
        ests.append(e)
    wall = time.perf_counter() - wall0
    est = float(np.mean(ests))
    value = cfg.B * cfg.Tq / est
    return {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(est * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generators; see workloads/synth.py)",
        "impl": "reference",
        "config": {"workload": workload_label(cfg), "step": step_label(kind), "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": texts + f"; {args.steps} steps in {wall:.1f} s wall (target {per_step:.1f} s/step)"},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="100m", choices=sorted(synth.CONFIGS))
    ap.add_argument("--docs", type=int, default=0, help="use only this many documents (smaller profiling case)")
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="time msa_gather and msa_sparse_attn (copied rows) instead of msa_sparse_attn_indexed")
    ap.add_argument("--extra", default=None,
                    help="comma-separated workloads whose stage results join the line (one GPU only), or none; "
                         "default: " + ",".join(EXTRA_WORKLOADS) + " with the default 100m workload, none otherwise")
    ap.add_argument("--step", choices=["full", "query"], default=None,
                    help="full: pool + query path per step; query: bank pooled before timing")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="which_pass", choices=["forward", "backward", "state", "dga", "interleave"],
                    default="forward",
                    help="backward: time the backward of the query path instead of the forward step; "
                         "state: the linear layers' memory injection (sum of the selected documents' states); "
                         "dga: that injection and the gated delta rule; interleave: Memory Interleave rounds")
    ap.add_argument("--rounds", type=int, default=2, help="Memory Interleave rounds (with --pass interleave)")
    ap.add_argument("--bank-kv", choices=["device", "host"], default="device",
                    help="where the pooled K̄ / V̄ live (host: page-locked host memory, the query path only)")
    ap.add_argument("--pipeline", action="store_true",
                    help="query path through the three-stream schedule (route i+1 | gather i | attention i-1)")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--ref-budget", type=float, default=120.0)
    args = ap.parse_args()
    if args.extra is None:
        args.extra = ",".join(EXTRA_WORKLOADS) if (args.workload == "100m" and not args.docs) else ""
    if args.warmup < 3 and args.impl == "msa":
        ap.error("--warmup must be >= 3")
    rank, local_rank, world = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    elif args.which_pass == "backward":
        res = run_backward(args, rank, local_rank, world)
    elif args.which_pass == "state":
        res = run_state(args, rank, local_rank, world)
    elif args.which_pass == "dga":
        res = run_dga(args, rank, local_rank, world)
    elif args.which_pass == "interleave":
        res = run_interleave(args, rank, local_rank, world)
    else:
        res = run_gpu(args, rank, local_rank, world)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
