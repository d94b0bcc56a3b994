"""Parity of the backward of steps 5 and 4 against the fp64 oracle, through the C ABI.

Tolerances, from the arithmetic: every gradient is accumulated in fp32 from
inputs the oracle sees exactly (it reads the same fp32 / bf16 values in
fp64), over at most a few hundred keys or rows, so fp32 inputs agree to ~1e-5
of the gradient's scale (1e-4 allowed).  With bf16 storage the only rounded
quantity the kernels consume is the forward output O (bf16) in D_i = dO_i.O_i;
its 2^-9 relative rounding moves ds by about p * 2^-9 |D| and the gradients by
well under 1 % of their scale (5e-3 of the largest magnitude allowed).
"""
import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from oracle import msa_oracle as O
from workloads import synth

from .helpers import attn_on_gpu, pool_on_gpu, route_on_gpu, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BWD_F32 = 1e-4
TOL_BWD_BF16 = 5e-3


def _inputs(B, Tq, Lloc, Hq, Hkv, d, Mmax, mem_lens, dtype, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    r = lambda *s: (0.5 * torch.randn(s, generator=g, device=DEV)).to(dtype)
    Q, Kl, Vl = r(B, Tq, Hq, d), r(B, Lloc, Hkv, d), r(B, Lloc, Hkv, d)
    Km, Vm = r(B, max(Mmax, 1), Hkv, d), r(B, max(Mmax, 1), Hkv, d)
    dO = r(B, Tq, Hq, d)
    ml = torch.tensor(mem_lens, dtype=torch.int32, device=DEV)
    return Q, Kl, Vl, Km, Vm, ml, dO


def _backward_gpu(Q, Kl, Vl, Km, Vm, ml, dO):
    Og, lse, flag = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
    f = dict(dtype=torch.float32, device=DEV)
    dQ = torch.full(Q.shape, float("nan"), **f)           # every element must be written
    dKl, dVl = torch.full(Kl.shape, float("nan"), **f), torch.full(Vl.shape, float("nan"), **f)
    dKm, dVm = torch.full(Km.shape, float("nan"), **f), torch.full(Vm.shape, float("nan"), **f)
    B, Tq, Hq, _ = Q.shape
    ws = torch.empty(msa.sparse_attn_backward_workspace_size(B, Tq, Hq), dtype=torch.uint8, device=DEV)
    msa.sparse_attn_backward(Q, Kl, Vl, Km, Vm, ml, Og, lse, dO, dQ, dKl, dVl, dKm, dVm, ws, err_flag=flag)
    torch.cuda.synchronize()
    return (dQ, dKl, dVl, dKm, dVm), flag


def _check(gpu, ora, tol, names=("dQ", "dKloc", "dVloc", "dKmem", "dVmem")):
    for name, g, o in zip(names, gpu, ora):
        g = to64(g)
        assert np.isfinite(g).all(), f"{name}: element not written"
        scale = max(1.0, float(np.abs(o).max()))
        err = float(np.abs(g - o).max())
        assert err <= tol * scale, f"{name}: max error {err:.3e} > {tol * scale:.3e}"


@pytest.mark.parametrize("B,Tq,Lloc,Hq,Hkv,d,Mmax,mem_lens,dtype,tol", [
    (2, 5, 9, 4, 2, 64, 7, [7, 3], torch.float32, TOL_BWD_F32),                  # tiny, fp32
    (3, 40, 70, 32, 8, 128, 48, [48, 0, 17], torch.bfloat16, TOL_BWD_BF16),      # Qwen heads, ragged memory
    (1, 100, 130, 64, 8, 128, 40, [33], torch.bfloat16, TOL_BWD_BF16),           # G = 8, many tiles, odd sizes
    (2, 33, 33, 8, 8, 64, 16, [16, 5], torch.float32, TOL_BWD_F32),              # MHA, Tq = Lloc
    (2, 300, 420, 32, 8, 128, 200, [200, 77], torch.bfloat16, TOL_BWD_BF16),     # key tiles split over query chunks
    (1, 160, 160, 16, 16, 128, 0, [0], torch.bfloat16, TOL_BWD_BF16),            # MHA on the tensor cores, no memory
])
def test_attention_backward_matches_oracle(B, Tq, Lloc, Hq, Hkv, d, Mmax, mem_lens, dtype, tol):
    Q, Kl, Vl, Km, Vm, ml, dO = _inputs(B, Tq, Lloc, Hq, Hkv, d, Mmax, mem_lens, dtype, seed=B * 100 + Tq)
    gpu, flag = _backward_gpu(Q, Kl, Vl, Km, Vm, ml, dO)
    ora = O.attention_backward(to64(Q), to64(Kl), to64(Vl), to64(Km), to64(Vm), mem_lens, to64(dO))
    assert flag.item() == 0
    _check(gpu, ora, tol)
    for b, m in enumerate(mem_lens):   # memory rows past mem_len carry no gradient
        assert not gpu[3][b, m:].any() and not gpu[4][b, m:].any()


def test_gather_backward_matches_oracle_with_shared_documents():
    rng = np.random.default_rng(3)
    lengths = rng.integers(0, 6, size=40)
    coff = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    C, Hkv, d, k, B = int(coff[-1]), 8, 128, 6, 5
    nonempty = np.flatnonzero(lengths)
    idx = np.stack([rng.choice(nonempty[:12], size=k, replace=False) for _ in range(B)]).astype(np.int32)
    Mmax = int(max(lengths[r].sum() for r in idx))
    ml = np.array([lengths[r].sum() for r in idx], dtype=np.int32)
    dKm = rng.standard_normal((B, Mmax, Hkv, d)).astype(np.float32)
    dVm = rng.standard_normal((B, Mmax, Hkv, d)).astype(np.float32)
    t = lambda a: torch.from_numpy(a).to(DEV)
    dKb = torch.zeros((C, Hkv, d), dtype=torch.float32, device=DEV)
    dVb = torch.zeros_like(dKb)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.gather_backward(t(idx), t(coff), t(dKm), t(dVm), t(ml), dKb, dVb, flag)
    oK, oV = O.gather_backward(idx, coff, dKm, dVm, ml, C)
    torch.cuda.synchronize()
    assert flag.item() == 0
    assert np.allclose(to64(dKb), oK, atol=1e-5) and np.allclose(to64(dVb), oV, atol=1e-5)
    # the documents chosen by several queries really were shared
    assert len(np.unique(idx)) < idx.size


def test_layer_backward_chain_matches_oracle_chain():
    """Forward (layer) -> backward of attention -> backward of the gather, on a pooled bank,
    against the oracle's chain on the same bank bytes: the gradient of <dO, O> w.r.t. the
    bank's K̄ / V̄ through the selected chunks."""
    cfg = synth.get_config("1m").scaled(D=64, Tq=24, Lloc=40)
    q = synth.gen_query(cfg, 0, DEV)
    rng = np.random.default_rng(5)
    lengths = np.full(cfg.D, 2)
    coff = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    C = int(coff[-1])
    Kb = (0.5 * torch.randn((C, cfg.Hkv, cfg.d), device=DEV)).bfloat16()
    Vb = (0.5 * torch.randn((C, cfg.Hkv, cfg.d), device=DEV)).bfloat16()
    idx = np.stack([rng.choice(cfg.D, size=cfg.k, replace=False) for _ in range(cfg.B)]).astype(np.int32)
    t = lambda a: torch.from_numpy(a).to(DEV)
    Mmax = cfg.k * 2
    Km = torch.zeros((cfg.B, Mmax, cfg.Hkv, cfg.d), dtype=torch.bfloat16, device=DEV)
    Vm = torch.zeros_like(Km)
    ml = torch.zeros(cfg.B, dtype=torch.int32, device=DEV)
    msa.gather(t(idx), t(coff), Kb, Vb, Km, Vm, ml)
    dO = (0.5 * torch.randn(q["Q"].shape, device=DEV)).bfloat16()
    (dQ, dKl, dVl, dKm, dVm), flag = _backward_gpu(q["Q"], q["Kloc"], q["Vloc"], Km, Vm, ml, dO)
    dKb = torch.zeros((C, cfg.Hkv, cfg.d), dtype=torch.float32, device=DEV)
    dVb = torch.zeros_like(dKb)
    msa.gather_backward(t(idx), t(coff), dKm, dVm, ml, dKb, dVb, flag)
    torch.cuda.synchronize()
    assert flag.item() == 0
    oKm, oVm, oml = O.gather(idx, coff, to64(Kb), to64(Vb), Mmax)
    r = O.attention_backward(to64(q["Q"]), to64(q["Kloc"]), to64(q["Vloc"]), oKm, oVm, oml, to64(dO))
    oKb, oVb = O.gather_backward(idx, coff, r[3], r[4], oml, C)
    _check((dQ, dKb, dVb), (r[0], oKb, oVb), TOL_BWD_BF16, names=("dQ", "dKbar", "dVbar"))


def _route_bwd_case(B, Tq, Hr, dr, lengths, k, dtype, seed, idx=None):
    """Random Qr / K̄r and a selection; documents whose best (chunk, token) pair is within 1e-4 of
    the runner-up get d_score 0, so the argmax both sides take is unique wherever it matters."""
    rng = np.random.default_rng(seed)
    coff = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    C, D = int(coff[-1]), len(lengths)
    g = torch.Generator(device=DEV).manual_seed(seed)
    Qr = torch.randn((B, Tq, Hr, dr), generator=g, device=DEV).to(dtype)
    Krb = torch.randn((max(C, 1), Hr, dr), generator=g, device=DEV).to(dtype)[:C].contiguous()
    rn = torch.empty((C, Hr), dtype=torch.float32, device=DEV)
    msa.bank_rnorm(Krb, rn)
    if idx is None:
        idx = np.stack([rng.choice(D, size=k, replace=False) for _ in range(B)]).astype(np.int32)
    s = O.cosine_scores(to64(Qr), to64(Krb))                 # [B, Tq, C]
    dsc = rng.standard_normal((B, k)).astype(np.float32)
    for b in range(B):
        for r, j in enumerate(idx[b]):
            v = np.sort(s[b, :, coff[j]:coff[j + 1]].ravel())
            if v.size > 1 and v[-1] - v[-2] < 1e-4:
                dsc[b, r] = 0.0
    return Qr, Krb, rn, coff, idx, dsc


def _route_bwd_gpu(Qr, Krb, rn, coff, idx, dsc):
    B, Tq, Hr, dr = Qr.shape
    t = lambda a: torch.from_numpy(a).to(DEV)
    dQr = torch.zeros((B, Tq, Hr, dr), dtype=torch.float32, device=DEV)
    dKrb = torch.zeros((Krb.shape[0], Hr, dr), dtype=torch.float32, device=DEV)
    ws = torch.empty(msa.route_backward_workspace_size(B, Tq, idx.shape[1]), dtype=torch.uint8, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.route_backward(Qr, Krb, rn, t(coff), t(idx), t(dsc), dQr, dKrb, ws, flag)
    torch.cuda.synchronize()
    return dQr, dKrb, flag


@pytest.mark.parametrize("B,Tq,Hr,dr,maxlen,D,k,dtype", [
    (3, 5, 8, 128, 6, 30, 6, torch.float32),       # few pairs per document
    (2, 64, 8, 128, 40, 24, 8, torch.bfloat16),    # thousands of pairs: every split busy, ragged tail
    (4, 1, 4, 64, 9, 50, 16, torch.bfloat16),      # decode: one token, max over chunks only
    (2, 33, 1, 64, 3, 12, 12, torch.float32),      # Hr = 1, every document selected
    (2, 150, 3, 64, 5, 20, 6, torch.bfloat16),     # three token blocks (ragged), Hr not a multiple of 4
    (1, 200, 8, 128, 19, 10, 4, torch.float32),    # documents of more than 8 chunks: several chunk groups
])
def test_route_backward_matches_oracle(B, Tq, Hr, dr, maxlen, D, k, dtype):
    rng = np.random.default_rng(B * 1000 + Tq)
    lengths = rng.integers(1, maxlen + 1, size=D)
    lengths[D // 2] = 0                               # an empty document (no gradient if selected)
    Qr, Krb, rn, coff, idx, dsc = _route_bwd_case(B, Tq, Hr, dr, lengths, k, dtype, seed=B + Tq)
    dQr, dKrb, flag = _route_bwd_gpu(Qr, Krb, rn, coff, idx, dsc)
    oQ, oK = O.route_backward(to64(Qr), to64(Krb), coff, idx, dsc)
    assert flag.item() == 0
    assert (dsc != 0).sum() >= idx.size // 2          # most documents have a unique argmax
    _check((dQr, dKrb), (oQ, oK), TOL_BWD_F32, names=("dQr", "dKrbar"))


def test_route_backward_accumulates_over_shared_documents_after_routing():
    """Selection by the routing kernels themselves (so several queries pick the same documents);
    the gradients are added onto what dQr / dK̄r already hold.  64 selections from 40 documents
    must share some."""
    cfg = synth.get_config("1m").scaled(D=40, B=4, Tq=16, Lloc=32)
    q = synth.gen_query(cfg, 0, DEV)
    K, V, Kr = synth.gen_raw_slab(cfg, 0, cfg.D, DEV, Qr0=q["Qr"][0])
    Kb, Vb, Krb, coff, rn, flag = pool_on_gpu(cfg, K, V, Kr, synth.doc_tok_offsets(cfg))
    idx, _, _, _ = route_on_gpu(q["Qr"], Krb, rn, coff, cfg.k)
    idx = idx.cpu().numpy()
    Qr = q["Qr"]
    s = O.cosine_scores(to64(Qr), to64(Krb))
    rng = np.random.default_rng(9)
    dsc = rng.standard_normal(idx.shape).astype(np.float32)
    for b in range(idx.shape[0]):
        for r, j in enumerate(idx[b]):
            v = np.sort(s[b, :, coff[j]:coff[j + 1]].ravel())
            if v.size > 1 and v[-1] - v[-2] < 1e-4:
                dsc[b, r] = 0.0
    B, Tq, Hr, dr = Qr.shape
    t = lambda a: torch.from_numpy(a).to(DEV)
    base_q = torch.randn((B, Tq, Hr, dr), device=DEV)
    base_k = torch.randn((Krb.shape[0], Hr, dr), device=DEV)
    dQr, dKrb = base_q.clone(), base_k.clone()
    ws = torch.empty(msa.route_backward_workspace_size(B, Tq, cfg.k), dtype=torch.uint8, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.route_backward(Qr, Krb, rn, t(coff), t(idx), t(dsc), dQr, dKrb, ws, flag)
    torch.cuda.synchronize()
    oQ, oK = O.route_backward(to64(Qr), to64(Krb), coff, idx, dsc)
    assert flag.item() == 0
    assert len(np.unique(idx)) < idx.size
    _check((dQr - base_q, dKrb - base_k), (oQ, oK), TOL_BWD_F32, names=("dQr", "dKrbar"))
