"""End-to-end parity of one MSA layer's memory path (pool -> route -> top-k ->
gather -> attention, and the fused layer call) against the fp64 oracle run from
the same raw inputs."""
import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from oracle import msa_oracle as O
from workloads import synth

from .helpers import (TOL_BF16_ABS, TOL_F32_ATTN, TOL_SCORE_ABS, attn_on_gpu, check_topk, close_abs,
                      pool_on_gpu, route_on_gpu, to64)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer_gpu(cfg, q, Kb, Vb, Krb, rn, coff):
    B, Tq = cfg.B, cfg.Tq
    D = len(coff) - 1
    Mmax = cfg.Mmax
    ws = torch.empty(msa.layer_forward_workspace_size(B, Tq, cfg.Lloc, cfg.Hq, cfg.Hkv, cfg.d, cfg.Hr, D, Krb.shape[0],
                                                      cfg.k, Mmax),
                     dtype=torch.uint8, device=DEV)
    O_ = torch.empty_like(q["Q"])
    lse = torch.empty((B, cfg.Hq, Tq), dtype=torch.float32, device=DEV)
    idx = torch.empty((B, cfg.k), dtype=torch.int32, device=DEV)
    sc = torch.empty((B, cfg.k), dtype=torch.float32, device=DEV)
    ds = torch.empty((B, D), dtype=torch.float32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.layer_forward(q["Qr"], Krb, rn, torch.from_numpy(coff).to(DEV), cfg.k, q["Q"], q["Kloc"], q["Vloc"],
                      Kb, Vb, Mmax, O_, idx, ws, lse, sc, ds, 0.0, flag)
    return O_, lse, idx, sc, ds, flag


def _oracle_layer(cfg, q, K, V, Kr, bf16):
    off = synth.doc_tok_offsets(cfg)
    Kb, Vb, Krb, coff, _ = O.pool(to64(K), to64(V), to64(Kr), off, cfg.P, cfg.theta, out_bf16=bf16)
    r = O.layer_forward(to64(q["Qr"]), Krb, coff, cfg.k, to64(q["Q"]), to64(q["Kloc"]), to64(q["Vloc"]),
                        Kb, Vb, cfg.Mmax)
    return r, coff


@pytest.mark.parametrize("name,scale", [("tiny", {}), ("1m", dict(D=160, Tq=96, Lloc=160)),
                                        ("decode16m", dict(D=300, B=6, Lloc=300, docs_per_slab=0)),
                                        ("100m", dict(D=400, last_len=256, docs_per_slab=0)),
                                        ("stack10m", dict(D=120, Tq=80, Lloc=80, docs_per_slab=0))])
def test_layer_end_to_end(name, scale):
    cfg = synth.get_config(name).scaled(**scale)
    bf16 = cfg.dtype == "bf16"
    q = synth.gen_query(cfg, 0, DEV)
    K, V, Kr = synth.gen_raw_slab(cfg, 0, cfg.D, DEV, Qr0=q["Qr"][0])
    Kb, Vb, Krb, coff, rn, pflag = pool_on_gpu(cfg, K, V, Kr, synth.doc_tok_offsets(cfg))
    O_, lse, idx, sc, ds, flag = _layer_gpu(cfg, q, Kb, Vb, Krb, rn, coff)
    ref, ocoff = _oracle_layer(cfg, q, K, V, Kr, bf16)
    torch.cuda.synchronize()
    assert pflag.item() == 0 and flag.item() == 0
    assert np.array_equal(coff, ocoff)
    ods = ref["doc_scores"]
    # scores: fp32 bank -> 1e-5; bf16 bank -> both sides round the pooled means to
    # bf16, rarely differently, which moves a score by far less than 1e-4
    stol = 1e-5 if not bf16 else 1e-4
    fin = np.isfinite(ods)
    close_abs(to64(ds)[fin], ods[fin], stol, "doc scores")
    check_topk(idx.cpu().numpy(), to64(sc), ods, cfg.k, stol)
    gi = idx.cpu().numpy()
    if np.array_equal(gi, ref["topk_idx"]):
        close_abs(to64(O_), ref["O"], TOL_BF16_ABS if bf16 else TOL_F32_ATTN, "O")
        close_abs(to64(lse), ref["lse"], 2e-3 if bf16 else TOL_F32_ATTN, "lse")
    else:
        # near-tie swap: attention must match the oracle run on the GPU's selection
        Km, Vm, ml = O.gather(gi, coff, to64(Kb), to64(Vb), cfg.Mmax)
        Oo, _ = O.attention(to64(q["Q"]), to64(q["Kloc"]), to64(q["Vloc"]), Km, Vm, ml)
        close_abs(to64(O_), Oo, TOL_BF16_ABS if bf16 else TOL_F32_ATTN, "O (GPU selection)")
    if name == "tiny":
        assert gi[0, 0] == 17
    if name == "100m":
        planted = synth.planted_docs(cfg)
        assert set(planted.tolist()) <= set(gi[0].tolist())


def test_fused_layer_equals_unfused_calls():
    """msa_layer_forward reads the bank through indices; msa_gather + msa_sparse_attn copy first.
    Both run the same arithmetic on the same bytes, so the outputs are identical."""
    cfg = synth.get_config("1m").scaled(D=96, Tq=40, Lloc=70)
    q = synth.gen_query(cfg, 0, DEV)
    K, V, Kr = synth.gen_raw_slab(cfg, 0, cfg.D, DEV, Qr0=q["Qr"][0])
    Kb, Vb, Krb, coff, rn, _ = pool_on_gpu(cfg, K, V, Kr, synth.doc_tok_offsets(cfg))
    O1, lse1, idx1, sc1, ds1, _ = _layer_gpu(cfg, q, Kb, Vb, Krb, rn, coff)
    idx2, sc2, ds2, _ = route_on_gpu(q["Qr"], Krb, rn, coff, cfg.k)
    Km = torch.zeros((cfg.B, cfg.Mmax, cfg.Hkv, cfg.d), dtype=torch.bfloat16, device=DEV)
    Vm = torch.zeros_like(Km)
    ml = torch.zeros(cfg.B, dtype=torch.int32, device=DEV)
    msa.gather(idx2, torch.from_numpy(coff).to(DEV), Kb, Vb, Km, Vm, ml)
    O2, lse2, _ = attn_on_gpu(q["Q"], q["Kloc"], q["Vloc"], Km, Vm, ml)
    torch.cuda.synchronize()
    assert torch.equal(idx1, idx2) and torch.equal(sc1, sc2) and torch.equal(ds1, ds2)
    assert torch.equal(O1, O2) and torch.equal(lse1, lse2)


@pytest.mark.parametrize("name,scale", [("1m", dict(D=96, Tq=40, Lloc=70)),
                                        ("decode16m", dict(D=200, B=5, Lloc=256, docs_per_slab=0))])
def test_layer_ignores_stale_workspace_bytes(name, scale):
    """The gathered rows live in the caller's workspace; rows past a query's selection are masked,
    and the gather zeroes them, so a workspace full of NaN bit patterns (0xFF bytes) gives the same
    output as a zeroed one.  Mmax is larger than any selection, so every query has such rows."""
    cfg = synth.get_config(name).scaled(**scale)
    q = synth.gen_query(cfg, 0, DEV)
    K, V, Kr = synth.gen_raw_slab(cfg, 0, cfg.D, DEV, Qr0=q["Qr"][0])
    Kb, Vb, Krb, coff, rn, _ = pool_on_gpu(cfg, K, V, Kr, synth.doc_tok_offsets(cfg))
    D, Mmax = len(coff) - 1, cfg.Mmax + 200

    def run(fill):
        ws = torch.full((msa.layer_forward_workspace_size(cfg.B, cfg.Tq, cfg.Lloc, cfg.Hq, cfg.Hkv, cfg.d, cfg.Hr, D,
                                                          Krb.shape[0], cfg.k, Mmax),), fill, dtype=torch.uint8,
                        device=DEV)
        O_ = torch.empty_like(q["Q"])
        lse = torch.empty((cfg.B, cfg.Hq, cfg.Tq), dtype=torch.float32, device=DEV)
        idx = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device=DEV)
        flag = torch.zeros(1, dtype=torch.int32, device=DEV)
        msa.layer_forward(q["Qr"], Krb, rn, torch.from_numpy(coff).to(DEV), cfg.k, q["Q"], q["Kloc"], q["Vloc"],
                          Kb, Vb, Mmax, O_, idx, ws, lse, None, None, 0.0, flag)
        torch.cuda.synchronize()
        return O_, lse, idx, flag

    O0, lse0, idx0, f0 = run(0)
    O1, lse1, idx1, f1 = run(255)
    assert f0.item() == 0 and f1.item() == 0
    assert torch.isfinite(O1.float()).all()
    assert torch.equal(idx0, idx1) and torch.equal(O0, O1) and torch.equal(lse0, lse1)
