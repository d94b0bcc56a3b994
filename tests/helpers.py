"""Shared helpers of the parity tests: device-side setup through the C ABI, and
the comparison rules (tolerances, the top-k near-tie rule)."""
from __future__ import annotations

import numpy as np
import torch

import routed_sparse_attention_chunk_b200 as msa
from workloads import synth

# Tolerances (the fp32 numbers are relative with an rms floor, see close_rel)
TOL_F32_POOL = 1e-5      # pooled K̄ / V̄ / K̄r, fp32 storage
TOL_F32_SCORE = 1e-5     # document scores, fp32
TOL_BF16_ABS = 2e-2      # any bf16-stored output (pooled bank, attention output)
TOL_SCORE_ABS = 2e-5     # routing scores from bf16 inputs: exact products, fp32 sums
TOL_F32_ATTN = 1e-4      # attention output, fp32
NEAR_TIE = 1e-4          # top-k ranks may differ only where oracle scores are this close


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def close_rel(g: np.ndarray, o: np.ndarray, rel: float, what: str):
    """|g - o| <= rel * max(|o|, rms of o over its last axis), elementwise."""
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True))
    bound = rel * np.maximum(np.abs(o), rms) + 1e-30
    err = np.abs(g - o)
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} elements off; worst {np.max(err / bound):.3g}x the bound"


def close_abs(g, o, tol: float, what: str):
    err = np.abs(np.asarray(g, np.float64) - np.asarray(o, np.float64))
    assert np.all(err <= tol), f"{what}: max abs error {err.max():.3g} > {tol}"


def check_topk(gpu_idx: np.ndarray, gpu_score: np.ndarray | None, oracle_scores: np.ndarray, k: int,
               score_tol: float, what: str = "top-k"):
    """GPU top-k vs the oracle's document scores [B, D].

    Rank r must hold the oracle's rank-r document, except where the two documents'
    oracle scores differ by less than NEAR_TIE (then either order is correct).
    Every selected document must be distinct and in range, and the GPU's
    selected set must be a valid top-k set of the oracle scores up to NEAR_TIE.
    """
    from oracle import msa_oracle as O
    oi, ov = O.topk(oracle_scores, k)
    B, D = oracle_scores.shape
    for b in range(B):
        g = gpu_idx[b]
        assert len(set(g.tolist())) == k and g.min() >= 0 and g.max() < D, f"{what}: invalid indices {g}"
        kth = ov[b, -1]
        for r in range(k):
            if g[r] != oi[b, r]:
                assert np.isfinite(ov[b, r]) and abs(oracle_scores[b, g[r]] - ov[b, r]) < NEAR_TIE, \
                    f"{what}: row {b} rank {r}: gpu doc {g[r]} ({oracle_scores[b, g[r]]:.7f}) vs " \
                    f"oracle doc {oi[b, r]} ({ov[b, r]:.7f})"
        assert np.all(oracle_scores[b, g] >= kth - NEAR_TIE), f"{what}: row {b} selected a document below the k-th"
        if gpu_score is not None:
            o = oracle_scores[b, g]
            fin = np.isfinite(o)
            assert np.array_equal(np.asarray(gpu_score[b])[~fin], o[~fin]), f"{what}: -inf scores differ"
            close_abs(np.asarray(gpu_score[b])[fin], o[fin], score_tol, f"{what} scores")


def stream():
    return torch.cuda.current_stream()


def pool_on_gpu(cfg: synth.Config, K, V, Kr, doc_tok_off: np.ndarray, rope=None, kr_rnorm=True):
    """msa_pool of raw tensors already on the device; returns (Kbar, Vbar, Krbar, doc_chunk_off, rnorm, flag)."""
    dev = K.device
    coff = msa.chunk_offsets(doc_tok_off, cfg.P)
    C = int(coff[-1])
    max_len = int(np.diff(doc_tok_off).max()) if len(doc_tok_off) > 1 else 1
    if rope is None:
        rope = msa.rope_table(cfg.theta, cfg.d, max(max_len, 1)).to(dev)
    dt = K.dtype
    Kb = torch.empty((C, cfg.Hkv, cfg.d), dtype=dt, device=dev)
    Vb = torch.empty_like(Kb)
    Krb = torch.empty((C, cfg.Hr, cfg.dr), dtype=dt, device=dev)
    rn = torch.empty((C, cfg.Hr), dtype=torch.float32, device=dev) if kr_rnorm else None
    flag = torch.zeros(1, dtype=torch.int32, device=dev)
    msa.pool(K, V, Kr, torch.from_numpy(doc_tok_off).to(dev), torch.from_numpy(coff).to(dev), cfg.P, rope,
             Kb, Vb, Krb, rn, flag)
    return Kb, Vb, Krb, coff, rn, flag


def route_on_gpu(Qr, Krb, rn, coff: np.ndarray, k: int):
    dev = Qr.device
    B = Qr.shape[0]
    D = len(coff) - 1
    ws = torch.empty(msa.route_topk_workspace_size(B, Qr.shape[1], Qr.shape[2], D, Krb.shape[0], k), dtype=torch.uint8,
                     device=dev)
    idx = torch.empty((B, k), dtype=torch.int32, device=dev)
    sc = torch.empty((B, k), dtype=torch.float32, device=dev)
    ds = torch.empty((B, D), dtype=torch.float32, device=dev)
    flag = torch.zeros(1, dtype=torch.int32, device=dev)
    msa.route_topk(Qr, Krb, rn, torch.from_numpy(coff).to(dev), k, idx, ws, sc, ds, flag)
    return idx, sc, ds, flag


def attn_on_gpu(Q, Kl, Vl, Km, Vm, mem_len, scale=0.0, want_lse=True):
    dev = Q.device
    B, Tq, Hq, d = Q.shape
    O = torch.empty_like(Q)
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=dev) if want_lse else None
    n = msa.sparse_attn_workspace_size(B, Tq, Kl.shape[1], Hq, Kl.shape[2], d, Km.shape[1])
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    flag = torch.zeros(1, dtype=torch.int32, device=dev)
    msa.sparse_attn(Q, Kl, Vl, Km, Vm, mem_len, O, lse, scale, ws, flag)
    return O, lse, flag


def pool_bank_slabs(cfg: synth.Config, device, seed: int = 0, Qr0=None):
    """The bank of a whole workload pooled slab by slab on the device, as a large corpus is encoded
    (each slab's raw tokens drawn, pooled with slab-relative offsets, then freed).
    Returns (Kbar, Vbar, Krbar, doc_chunk_off, kr_rnorm, flag)."""
    tok = synth.doc_tok_offsets(cfg)
    coff = msa.chunk_offsets(tok, cfg.P)
    C = int(coff[-1])
    dt = cfg.torch_dtype
    rope = msa.rope_table(cfg.theta, cfg.d, int(np.diff(tok).max())).to(device)
    Kb = torch.empty((C, cfg.Hkv, cfg.d), dtype=dt, device=device)
    Vb = torch.empty_like(Kb)
    Krb = torch.empty((C, cfg.Hr, cfg.dr), dtype=dt, device=device)
    rn = torch.empty((C, cfg.Hr), dtype=torch.float32, device=device)
    flag = torch.zeros(1, dtype=torch.int32, device=device)
    for lo, hi in synth.slab_bounds(cfg):
        K, V, Kr = synth.gen_raw_slab(cfg, lo, hi, device, seed, Qr0=Qr0)
        t = torch.from_numpy(tok[lo:hi + 1] - tok[lo]).to(device)
        cs, ce = int(coff[lo]), int(coff[hi])
        ch = torch.from_numpy(coff[lo:hi + 1] - coff[lo]).to(device)
        msa.pool(K, V, Kr, t, ch, cfg.P, rope, Kb[cs:ce], Vb[cs:ce], Krb[cs:ce], rn[cs:ce], flag)
        del K, V, Kr
    return Kb, Vb, Krb, coff, rn, flag


def oracle_route_by_slabs(Qr64: np.ndarray, Krb: torch.Tensor, coff: np.ndarray, docs_per_slab: int) -> np.ndarray:
    """The oracle's document scores [B, D] over a device bank of any size: a document's score
    depends only on its own chunks, so the oracle's route runs on one slab of whole documents at
    a time (their stored bank bytes copied to the host and widened to fp64)."""
    from oracle import msa_oracle as O
    D = len(coff) - 1
    out = np.empty((Qr64.shape[0], D))
    for lo in range(0, D, docs_per_slab):
        hi = min(lo + docs_per_slab, D)
        cs, ce = int(coff[lo]), int(coff[hi])
        kb = Krb[cs:ce].to("cpu", torch.float64).numpy()
        out[:, lo:hi] = O.route(Qr64, kb, coff[lo:hi + 1] - cs)
    return out
