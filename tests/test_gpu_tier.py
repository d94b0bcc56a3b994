"""Host tier of the pooled K̄ / V̄ ("MSA: Memory Sparse Attention" README,
"Inference Pipeline": the pooled K̄ / V̄ can stay in host memory while K̄r
stays on the GPU for routing; only the selected documents' rows are loaded).

The bank's K̄ / V̄ live in page-locked host memory and msa_gather /
msa_layer_forward read the selected rows in place.  The kernels are the ones
the device-resident bank uses, so the results must be identical byte for byte,
and the gather must match the oracle exactly.
"""
import ctypes

import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from routed_sparse_attention_chunk_b200 import _lib
from oracle import msa_oracle as O
from workloads import synth

from .helpers import pool_on_gpu, route_on_gpu, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bank(cfg):
    q = synth.gen_query(cfg, 0, DEV)
    K, V, Kr = synth.gen_raw_slab(cfg, 0, cfg.D, DEV, Qr0=q["Qr"][0])
    Kb, Vb, Krb, coff, rn, flag = pool_on_gpu(cfg, K, V, Kr, synth.doc_tok_offsets(cfg))
    torch.cuda.synchronize()
    assert flag.item() == 0
    return q, Kb, Vb, Krb, coff, rn


def _gather(idx, coff, Kb, Vb, cfg):
    Km = torch.zeros((cfg.B, cfg.Mmax, cfg.Hkv, cfg.d), dtype=Kb.dtype, device=DEV)
    Vm = torch.zeros_like(Km)
    ml = torch.zeros(cfg.B, dtype=torch.int32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.gather(idx, torch.from_numpy(coff).to(DEV), Kb, Vb, Km, Vm, ml, flag)
    torch.cuda.synchronize()
    return Km, Vm, ml, flag


def test_gather_from_pinned_host_bank_is_bitexact():
    cfg = synth.get_config("decode16m").scaled(D=200, B=5, Lloc=256, docs_per_slab=0)
    q, Kb, Vb, Krb, coff, rn = _bank(cfg)
    idx, _, _, _ = route_on_gpu(q["Qr"], Krb, rn, coff, cfg.k)
    Kh, Vh = Kb.cpu().pin_memory(), Vb.cpu().pin_memory()
    assert not Kh.is_cuda and Kh.is_pinned()
    Km_d, Vm_d, ml_d, _ = _gather(idx, coff, Kb, Vb, cfg)
    Km_h, Vm_h, ml_h, flag = _gather(idx, coff, Kh, Vh, cfg)
    assert flag.item() == 0
    assert torch.equal(ml_h, ml_d)
    for b in range(cfg.B):
        n = int(ml_d[b])
        assert torch.equal(Km_h[b, :n], Km_d[b, :n]) and torch.equal(Vm_h[b, :n], Vm_d[b, :n])
    # and against the oracle's gather of the same bank bytes
    oK, oV, oml = O.gather(idx.cpu().numpy(), coff, to64(Kh), to64(Vh), cfg.Mmax)
    assert np.array_equal(ml_h.cpu().numpy(), oml)
    for b in range(cfg.B):
        n = int(oml[b])
        assert np.array_equal(to64(Km_h[b, :n]), oK[b, :n]) and np.array_equal(to64(Vm_h[b, :n]), oV[b, :n])


def test_layer_forward_with_pinned_host_bank_equals_device_bank():
    cfg = synth.get_config("1m").scaled(D=120, Tq=48, Lloc=96)
    q, Kb, Vb, Krb, coff, rn = _bank(cfg)
    Kh, Vh = Kb.cpu().pin_memory(), Vb.cpu().pin_memory()

    def run(Kbank, Vbank):
        D = len(coff) - 1
        ws = torch.empty(msa.layer_forward_workspace_size(cfg.B, cfg.Tq, cfg.Lloc, cfg.Hq, cfg.Hkv, cfg.d, cfg.Hr, D,
                                                          Krb.shape[0], cfg.k, cfg.Mmax), dtype=torch.uint8, device=DEV)
        O_ = torch.empty_like(q["Q"])
        idx = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device=DEV)
        flag = torch.zeros(1, dtype=torch.int32, device=DEV)
        msa.layer_forward(q["Qr"], Krb, rn, torch.from_numpy(coff).to(DEV), cfg.k, q["Q"], q["Kloc"], q["Vloc"],
                          Kbank, Vbank, cfg.Mmax, O_, idx, ws, err_flag=flag)
        torch.cuda.synchronize()
        return O_, idx, flag

    O_d, idx_d, _ = run(Kb, Vb)
    O_h, idx_h, flag = run(Kh, Vh)
    assert flag.item() == 0
    assert torch.equal(idx_h, idx_d)
    assert torch.equal(O_h, O_d)


def test_pageable_host_bank_is_refused_before_any_launch():
    cfg = synth.get_config("decode16m").scaled(D=40, B=2, Lloc=128, docs_per_slab=0)
    q, Kb, Vb, Krb, coff, rn = _bank(cfg)
    idx, _, _, _ = route_on_gpu(q["Qr"], Krb, rn, coff, cfg.k)
    Kp, Vp = Kb.cpu(), Vb.cpu()          # ordinary (pageable) host memory
    assert not Kp.is_pinned()
    with pytest.raises(ValueError):      # the binding
        _gather(idx, coff, Kp, Vp, cfg)
    Km = torch.zeros((cfg.B, cfg.Mmax, cfg.Hkv, cfg.d), dtype=Kb.dtype, device=DEV)
    ml = torch.zeros(cfg.B, dtype=torch.int32, device=DEV)
    coff_d = torch.from_numpy(coff).to(DEV)
    st = _lib.load().msa_gather(1, idx.data_ptr(), cfg.B, cfg.k, coff_d.data_ptr(), len(coff) - 1, Krb.shape[0],
                                Kp.data_ptr(), Vp.data_ptr(), cfg.Hkv, cfg.d, cfg.Mmax, Km.data_ptr(), Km.data_ptr(),
                                ml.data_ptr(), None, None)
    assert st == -1                      # MSA_ERR_INVALID_ARG, nothing launched
    torch.cuda.synchronize()


def test_pipelined_host_tier_equals_sequential_calls():
    """The three-stream schedule (route of batch i+1, host gather of batch i and attention of
    batch i-1 overlapped) gives the outputs of the sequential calls, bit for bit, for a run of
    distinct batches, also when the caller reuses two topk_idx tensors in turn."""
    from routed_sparse_attention_chunk_b200.pipeline import QueryPipeline
    cfg = synth.get_config("decode16m").scaled(D=200, B=5, Lloc=256, docs_per_slab=0)
    q, Kb, Vb, Krb, coff, rn = _bank(cfg)
    coff_d = torch.from_numpy(coff).to(DEV)
    batches = [synth.gen_query(cfg, 0, DEV, seed) for seed in range(6)]
    ref = []
    for bt in batches:
        idx, _, _, _ = route_on_gpu(bt["Qr"], Krb, rn, coff, cfg.k)
        Km, Vm, ml, _ = _gather(idx, coff, Kb, Vb, cfg)
        O_ = torch.empty_like(bt["Q"])
        ws = torch.empty(max(256, msa.sparse_attn_workspace_size(cfg.B, cfg.Tq, cfg.Lloc, cfg.Hq, cfg.Hkv, cfg.d,
                                                                 cfg.Mmax)), dtype=torch.uint8, device=DEV)
        msa.sparse_attn(bt["Q"], bt["Kloc"], bt["Vloc"], Km, Vm, ml, O_, ws=ws)
        torch.cuda.synchronize()
        ref.append((idx.clone(), O_))
    Kh, Vh = Kb.cpu().pin_memory(), Vb.cpu().pin_memory()
    bank = dict(Krbar=Krb, kr_rnorm=rn, doc_chunk_off=coff_d, Kbar=Kh, Vbar=Vh)
    for reuse in (False, True):
        pipe = QueryPipeline(bank, cfg.k, cfg.Mmax, cfg.B, cfg.Tq, cfg.Lloc, cfg.Hq, cfg.Hkv, cfg.d, cfg.Hr,
                             Kb.dtype, DEV)
        ring = [torch.empty((cfg.B, cfg.k), dtype=torch.int32, device=DEV) for _ in range(2)]
        runs = [dict(bt, O=torch.empty_like(bt["Q"]),
                     topk_idx=ring[i % 2] if reuse else torch.empty((cfg.B, cfg.k), dtype=torch.int32, device=DEV))
                for i, bt in enumerate(batches)]
        marks = []
        pipe.run(runs[:2], marks)
        pipe.run(runs[2:], marks)         # the event rings continue across calls
        torch.cuda.synchronize()
        assert pipe.flag.item() == 0
        assert len(marks) == 3 * len(runs)
        for i, (r, (idx, O_)) in enumerate(zip(runs, ref)):
            assert torch.equal(r["O"], O_), f"batch {i} (reuse={reuse})"
            if not reuse:
                assert torch.equal(r["topk_idx"], idx)
