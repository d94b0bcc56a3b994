"""Parity at the workloads' full sizes: the 100M-token bank (195,313 documents,
1,562,500 chunks), the 16M-token decode batch, the 1M-token layer and the
10M-token corpus of the 16-layer stack, each built and run on the GPU exactly
as the benchmark builds and runs it, and compared with the fp64 oracle.

Step by step, as for every bf16 workload: the oracle routes over the GPU's
stored bank bytes (rounding the pooled means to bf16 can move a score by
~1e-3, more than the top-k near-tie allowance), and attends over the GPU's
selection.  The pool is checked on sampled documents, among them the last ones
of the 10M-token corpus, whose element offsets pass 2^31.

These tests hold up to ~70 GB of device memory and run the oracle for tens of
seconds each."""
import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from oracle import msa_oracle as O
from workloads import synth

from .helpers import (TOL_BF16_ABS, TOL_SCORE_ABS, check_topk, close_abs, oracle_route_by_slabs, pool_bank_slabs,
                      pool_on_gpu, to64)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(cfg, q, Kb, Vb, Krb, rn, coff):
    """msa_layer_forward (route + top-k, attention over the selected chunks read from the bank)."""
    B, D = cfg.B, len(coff) - 1
    ws = torch.empty(msa.layer_forward_workspace_size(B, cfg.Tq, cfg.Lloc, cfg.Hq, cfg.Hkv, cfg.d, cfg.Hr, D,
                                                      Krb.shape[0], cfg.k, cfg.Mmax), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(q["Q"])
    lse = torch.empty((B, cfg.Hq, cfg.Tq), dtype=torch.float32, device=DEV)
    idx = torch.empty((B, cfg.k), dtype=torch.int32, device=DEV)
    sc = torch.empty((B, cfg.k), dtype=torch.float32, device=DEV)
    ds = torch.empty((B, D), dtype=torch.float32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.layer_forward(q["Qr"], Krb, rn, torch.from_numpy(coff).to(DEV), cfg.k, q["Q"], q["Kloc"], q["Vloc"],
                      Kb, Vb, cfg.Mmax, out, idx, ws, lse, sc, ds, 0.0, flag)
    torch.cuda.synchronize()
    return out, lse, idx, sc, ds, int(flag.item())


def _attention_on_selection(cfg, q, Kb, Vb, coff, gi, b_rows=None):
    """The oracle's attention over the GPU's selection, from the GPU bank's bytes of those documents."""
    rows = b_rows if b_rows is not None else range(cfg.B)
    outs, lses = [], []
    for b in rows:
        chunks = np.concatenate([np.arange(coff[j], coff[j + 1]) for j in gi[b]])
        sel = torch.from_numpy(chunks).to(DEV)
        Km = to64(Kb[sel])[None]
        Vm = to64(Vb[sel])[None]
        o, l = O.attention(to64(q["Q"][b:b + 1]), to64(q["Kloc"][b:b + 1]), to64(q["Vloc"][b:b + 1]), Km, Vm,
                           np.array([len(chunks)]))
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def test_100m_bank_full_route_topk_and_attention():
    cfg = synth.get_config("100m")
    q = synth.gen_query(cfg, 0, DEV)
    Kb, Vb, Krb, coff, rn, pflag = pool_bank_slabs(cfg, DEV, Qr0=q["Qr"][0])
    assert Krb.shape[0] == 1_562_500 and len(coff) - 1 == 195_313
    out, lse, idx, sc, ds, flag = _layer(cfg, q, Kb, Vb, Krb, rn, coff)
    assert pflag.item() == 0 and flag == 0
    ods = oracle_route_by_slabs(to64(q["Qr"]), Krb, coff, 20_000)
    close_abs(to64(ds), ods, TOL_SCORE_ABS, "document scores, all 195,313 documents")
    gi = idx.cpu().numpy()
    check_topk(gi, to64(sc), ods, cfg.k, TOL_SCORE_ABS)
    planted = synth.planted_docs(cfg)
    assert set(planted.tolist()) <= set(gi[0].tolist()), "a planted document is missing from the top 16"
    close_abs(to64(ds)[0, planted], np.ones(len(planted)), 1e-5, "planted documents' scores")
    Oo, lo = _attention_on_selection(cfg, q, Kb, Vb, coff, gi)
    close_abs(to64(out), Oo, TOL_BF16_ABS, "O")
    close_abs(to64(lse), lo, 2e-3, "lse")


def test_decode16m_full_batch():
    cfg = synth.get_config("decode16m")
    q = synth.gen_query(cfg, 0, DEV)
    Kb, Vb, Krb, coff, rn, pflag = pool_bank_slabs(cfg, DEV, Qr0=q["Qr"][0])
    out, lse, idx, sc, ds, flag = _layer(cfg, q, Kb, Vb, Krb, rn, coff)
    assert pflag.item() == 0 and flag == 0
    ods = oracle_route_by_slabs(to64(q["Qr"]), Krb, coff, 8192)
    close_abs(to64(ds), ods, TOL_SCORE_ABS, "document scores of 64 queries")
    gi = idx.cpu().numpy()
    check_topk(gi, to64(sc), ods, cfg.k, TOL_SCORE_ABS)
    Oo, lo = _attention_on_selection(cfg, q, Kb, Vb, coff, gi)
    close_abs(to64(out), Oo, TOL_BF16_ABS, "O")
    close_abs(to64(lse), lo, 2e-3, "lse")


def test_1m_full_layer_and_sampled_pool():
    cfg = synth.get_config("1m")
    q = synth.gen_query(cfg, 0, DEV)
    K, V, Kr = synth.gen_raw_slab(cfg, 0, cfg.D, DEV, Qr0=q["Qr"][0])
    tok = synth.doc_tok_offsets(cfg)
    Kb, Vb, Krb, coff, rn, pflag = pool_on_gpu(cfg, K, V, Kr, tok)
    out, lse, idx, sc, ds, flag = _layer(cfg, q, Kb, Vb, Krb, rn, coff)
    assert pflag.item() == 0 and flag == 0
    # pool: 48 sampled documents, the first and last among them
    rng = np.random.default_rng(1)
    docs = np.unique(np.concatenate([[0, 1, cfg.D - 2, cfg.D - 1], rng.choice(cfg.D, 44, replace=False)]))
    _check_pooled_docs(cfg, K, V, Kr, tok, coff, Kb, Vb, Krb, rn, docs)
    ods = oracle_route_by_slabs(to64(q["Qr"]), Krb, coff, cfg.D)
    close_abs(to64(ds), ods, TOL_SCORE_ABS, "document scores")
    gi = idx.cpu().numpy()
    check_topk(gi, to64(sc), ods, cfg.k, TOL_SCORE_ABS)
    Oo, lo = _attention_on_selection(cfg, q, Kb, Vb, coff, gi)
    close_abs(to64(out), Oo, TOL_BF16_ABS, "O")
    close_abs(to64(lse), lo, 2e-3, "lse")


def _check_pooled_docs(cfg, K, V, Kr, tok, coff, Kb, Vb, Krb, rn, docs):
    """The oracle's pool of each listed document's raw tokens (copied from the device) against the
    device bank's rows of that document."""
    for j in docs.tolist():
        t0, t1 = int(tok[j]), int(tok[j + 1])
        c0, c1 = int(coff[j]), int(coff[j + 1])
        ok, ov, okr, ocoff, orn = O.pool(to64(K[t0:t1]), to64(V[t0:t1]), to64(Kr[t0:t1]),
                                         np.array([0, t1 - t0]), cfg.P, cfg.theta, out_bf16=True)
        assert np.array_equal(ocoff, np.array([0, c1 - c0]))
        close_abs(to64(Kb[c0:c1]), ok, TOL_BF16_ABS, f"K̄ of document {j}")
        close_abs(to64(Vb[c0:c1]), ov, TOL_BF16_ABS, f"V̄ of document {j}")
        close_abs(to64(Krb[c0:c1]), okr, TOL_BF16_ABS, f"K̄r of document {j}")
        # the norms describe the stored bank bytes exactly (fp32 sums of exact squares)
        kb = to64(Krb[c0:c1])
        ref = 1.0 / np.maximum(np.sqrt((kb * kb).sum(-1)), 1e-12)
        np.testing.assert_allclose(to64(rn[c0:c1]), ref, rtol=1e-5, err_msg=f"1/|K̄r| of document {j}")


def test_stack10m_full_corpus_pool_and_one_layer():
    cfg = synth.get_config("stack10m")
    q = synth.gen_query(cfg, 0, DEV)
    tok = synth.doc_tok_offsets(cfg)
    n = int(tok[-1])
    K = torch.empty((n, cfg.Hkv, cfg.d), dtype=torch.bfloat16, device=DEV)
    V = torch.empty_like(K)
    Kr = torch.empty((n, cfg.Hr, cfg.dr), dtype=torch.bfloat16, device=DEV)
    for lo, hi in synth.slab_bounds(cfg):
        t0, t1 = int(tok[lo]), int(tok[hi])
        for dst, src in zip((K, V, Kr), synth.gen_raw_slab(cfg, lo, hi, DEV, Qr0=q["Qr"][0])):
            dst[t0:t1].copy_(src)
    # one msa_pool call over the whole 61 GB corpus: element offsets pass 2^31 from token 2^31 / 1024 on
    Kb, Vb, Krb, coff, rn, pflag = pool_on_gpu(cfg, K, V, Kr, tok)
    torch.cuda.synchronize()
    assert pflag.item() == 0 and Krb.shape[0] == 160_000
    first_past = int(np.searchsorted(tok, (1 << 31) // (cfg.Hkv * cfg.d)))  # first document past 2^31 elements
    rng = np.random.default_rng(2)
    docs = np.unique(np.concatenate([[0, first_past - 1, first_past, cfg.D - 2, cfg.D - 1],
                                     rng.choice(cfg.D, 45, replace=False)]))
    assert (tok[docs + 1] * cfg.Hkv * cfg.d > (1 << 31)).sum() >= 10
    _check_pooled_docs(cfg, K, V, Kr, tok, coff, Kb, Vb, Krb, rn, docs)
    del K, V, Kr
    torch.cuda.empty_cache()
    out, lse, idx, sc, ds, flag = _layer(cfg, q, Kb, Vb, Krb, rn, coff)
    assert flag == 0
    ods = oracle_route_by_slabs(to64(q["Qr"]), Krb, coff, 1000)
    close_abs(to64(ds), ods, TOL_SCORE_ABS, "document scores (4096 query rows, CTA-pair scan)")
    gi = idx.cpu().numpy()
    check_topk(gi, to64(sc), ods, cfg.k, TOL_SCORE_ABS)
    Oo, lo = _attention_on_selection(cfg, q, Kb, Vb, coff, gi)
    close_abs(to64(out), Oo, TOL_BF16_ABS, "O (4096 tokens x 32 heads)")
    close_abs(to64(lse), lo, 2e-3, "lse")
