"""msa_sparse_attn_indexed: attention over the selected documents' chunks read in
place from the bank by index (steps 4 and 5 fused) against the fp64 oracle's
gather followed by its attention, on the same bytes.

Documents here have chunk counts that are not multiples of 8 (the runs of
chunk rows the kernels load are then padded with masked rows), selections that
overflow Mmax (rows past it are dropped and flagged), and indices outside the
bank (skipped and flagged).  With 8-chunk documents the index-driven path gives
the gathered path's output bit for bit."""
import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from oracle import msa_oracle as O
from workloads import synth

from .helpers import TOL_BF16_ABS, attn_on_gpu, close_abs, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bank(n_chunks, Hkv, d, seed):
    coff = np.concatenate([[0], np.cumsum(n_chunks)]).astype(np.int64)
    C = int(coff[-1])
    Kb = synth.gen_bank_bf16(C, Hkv, d, DEV, seed, "Kbar")
    Vb = synth.gen_bank_bf16(C, Hkv, d, DEV, seed, "Vbar")
    return Kb, Vb, coff


def _selection(B, D, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(D, size=k, replace=False) for _ in range(B)]).astype(np.int32)


def _queries(B, Tq, Lloc, Hq, Hkv, d, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    r = lambda *s: (0.5 * torch.randn(s, generator=g, device=DEV)).bfloat16()
    return r(B, Tq, Hq, d), r(B, Lloc, Hkv, d), r(B, Lloc, Hkv, d)


def _indexed(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax):
    B, Tq, Hq, d = Q.shape
    k = idx.shape[1]
    ws = torch.empty(msa.sparse_attn_indexed_workspace_size(B, Tq, Kl.shape[1], Hq, Kl.shape[2], d, k, Mmax),
                     dtype=torch.uint8, device=DEV)
    out = torch.empty_like(Q)
    lse = torch.empty((B, Hq, Tq), dtype=torch.float32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx_d = torch.from_numpy(np.ascontiguousarray(idx)).to(DEV)
    msa.sparse_attn_indexed(Q, Kl, Vl, idx_d, torch.from_numpy(coff).to(DEV), Kb, Vb, Mmax, out, ws, lse,
                            err_flag=flag)
    torch.cuda.synchronize()
    return out, lse, int(flag.item())


def _oracle(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax, D):
    """Oracle gather of the in-range selections, rows past Mmax dropped, then its attention."""
    kept = [[j for j in row if 0 <= j < D] for row in idx]
    big = max(sum(int(coff[j + 1] - coff[j]) for j in row) for row in kept) + 1
    # the oracle's gather takes a rectangular index list: pad short rows with an empty document
    # (none here has zero chunks), so gather each query on its own
    B = len(kept)
    Kg = np.zeros((B, Mmax) + tuple(Kb.shape[1:]))
    Vg = np.zeros_like(Kg)
    ml = np.zeros(B, dtype=np.int64)
    Kb64, Vb64 = to64(Kb), to64(Vb)
    for b, row in enumerate(kept):
        Km, Vm, n = O.gather(np.array([row], dtype=np.int64), coff, Kb64, Vb64, big)
        m = min(int(n[0]), Mmax)
        Kg[b, :m], Vg[b, :m], ml[b] = Km[0, :m], Vm[0, :m], m
    return O.attention(to64(Q), to64(Kl), to64(Vl), Kg, Vg, ml)


@pytest.mark.parametrize("B,Tq,Lloc,Hq,Hkv,k,Mmax,seed", [
    (2, 96, 160, 32, 8, 16, 400, 1),     # prefill, GQA 4 heads x 32 tokens per CTA, several memory tiles
    (1, 200, 200, 16, 4, 9, 200, 2),      # prefill, GQA 4, a selection longer than Mmax (dropped, flagged)
    (6, 1, 300, 32, 8, 16, 300, 3),       # decode, 4 query rows per KV head
    (3, 2, 260, 32, 8, 5, 80, 4),         # decode, 8 rows per KV head, overflow
    (2, 16, 48, 8, 8, 7, 64, 5),          # prefill MHA (G = 1: 8-token blocks)
    (3, 24, 90, 32, 8, 11, 256, 6),       # one ragged block of rows per KV head, two memory tiles
    (1, 160, 160, 64, 8, 16, 512, 7),     # G = 8: ten 16-token blocks, four memory tiles
    (2, 60, 120, 40, 8, 10, 200, 8),      # G = 5: no tensor-core tiling, the gathered path (no overflow)
    (2, 8, 300, 32, 8, 12, 256, 9),       # 8 tokens x G = 4: neither a prefill block nor decode rows
])
def test_indexed_attention_ragged_documents(B, Tq, Lloc, Hq, Hkv, k, Mmax, seed):
    rng = np.random.default_rng(seed)
    D = 60
    n = rng.integers(1, 21, size=D)                       # 1..20 chunks: partial runs of 8
    Kb, Vb, coff = _bank(n, Hkv, 128, seed)
    idx = _selection(B, D, k, seed)
    Q, Kl, Vl = _queries(B, Tq, Lloc, Hq, Hkv, 128, seed)
    out, lse, flag = _indexed(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax)
    Oo, lo = _oracle(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax, D)
    overflow = any(sum(int(n[j]) for j in row) > Mmax for row in idx)
    assert flag == (msa.FLAG_OVERFLOW if overflow else 0)
    close_abs(to64(out), Oo, TOL_BF16_ABS, "O")
    close_abs(to64(lse), lo, 2e-3, "lse")


def test_indexed_attention_flags_and_skips_bad_indices():
    rng = np.random.default_rng(7)
    D, B, Tq, Lloc, Hq, Hkv, k, Mmax = 40, 3, 64, 64, 32, 8, 6, 200
    n = rng.integers(1, 13, size=D)
    Kb, Vb, coff = _bank(n, Hkv, 128, 7)
    idx = _selection(B, D, k, 7)
    idx[0, 2] = -1          # below the bank
    idx[2, 5] = D + 3       # past the last document
    Q, Kl, Vl = _queries(B, Tq, Lloc, Hq, Hkv, 128, 7)
    out, lse, flag = _indexed(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax)
    Oo, lo = _oracle(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax, D)
    assert flag & msa.FLAG_INDEX_OOB
    close_abs(to64(out), Oo, TOL_BF16_ABS, "O")
    close_abs(to64(lse), lo, 2e-3, "lse")


@pytest.mark.parametrize("B,Tq,Lloc", [(1, 100, 180), (8, 1, 512)])
def test_indexed_equals_gathered_for_8_chunk_documents(B, Tq, Lloc):
    """8-chunk documents fill whole runs, so the keys sit at the gathered positions.  Prefill
    shapes then run the same arithmetic in the same order as gather + attention: bit for bit.
    Decode shapes reserve room for padded runs (one more memory tile per KV head), which moves
    where the CTAs split the keys, so only the fp32 summation order differs."""
    D, Hq, Hkv, k = 50, 32, 8, 16
    Mmax = 8 * k
    Kb, Vb, coff = _bank(np.full(D, 8), Hkv, 128, 9)
    idx = _selection(B, D, k, 9)
    Q, Kl, Vl = _queries(B, Tq, Lloc, Hq, Hkv, 128, 9)
    out, lse, flag = _indexed(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax)
    Km = torch.zeros((B, Mmax, Hkv, 128), dtype=torch.bfloat16, device=DEV)
    Vm = torch.zeros_like(Km)
    ml = torch.zeros(B, dtype=torch.int32, device=DEV)
    idx_d = torch.from_numpy(idx).to(DEV)
    msa.gather(idx_d, torch.from_numpy(coff).to(DEV), Kb, Vb, Km, Vm, ml)
    O2, lse2, f2 = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
    torch.cuda.synchronize()
    assert flag == 0 and f2.item() == 0
    if Tq > 1:
        assert torch.equal(out, O2) and torch.equal(lse, lse2)
    else:
        close_abs(to64(out), to64(O2), 4e-3, "O (decode: summation order)")
        close_abs(to64(lse), to64(lse2), 1e-5, "lse (decode: summation order)")


def test_indexed_host_bank_matches_device_bank():
    """K̄ / V̄ in page-locked host memory take the gathered path; the result equals the device bank's."""
    rng = np.random.default_rng(11)
    D, B, Tq, Lloc, Hq, Hkv, k, Mmax = 30, 2, 40, 90, 32, 8, 5, 120
    n = rng.integers(1, 17, size=D)
    Kb, Vb, coff = _bank(n, Hkv, 128, 11)
    idx = _selection(B, D, k, 11)
    Q, Kl, Vl = _queries(B, Tq, Lloc, Hq, Hkv, 128, 11)
    out_d, lse_d, f_d = _indexed(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax)
    out_h, lse_h, f_h = _indexed(Q, Kl, Vl, idx, coff, Kb.cpu().pin_memory(), Vb.cpu().pin_memory(), Mmax)
    assert f_d == 0 and f_h == 0
    Oo, lo = _oracle(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax, D)
    close_abs(to64(out_h), Oo, TOL_BF16_ABS, "O (host bank)")
    close_abs(to64(out_d), to64(out_h), TOL_BF16_ABS, "O (device vs host bank)")


def test_indexed_fp32_takes_the_gathered_path():
    rng = np.random.default_rng(13)
    D, B, Tq, Lloc, Hq, Hkv, k, Mmax = 20, 2, 24, 40, 4, 2, 3, 40
    n = rng.integers(1, 9, size=D)
    coff = np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
    C = int(coff[-1])
    g = torch.Generator(device=DEV).manual_seed(13)
    Kb = torch.randn((C, Hkv, 64), generator=g, device=DEV)
    Vb = torch.randn((C, Hkv, 64), generator=g, device=DEV)
    Q = torch.randn((B, Tq, Hq, 64), generator=g, device=DEV)
    Kl = torch.randn((B, Lloc, Hkv, 64), generator=g, device=DEV)
    Vl = torch.randn((B, Lloc, Hkv, 64), generator=g, device=DEV)
    idx = _selection(B, D, k, 13)
    out, lse, flag = _indexed(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax)
    Oo, lo = _oracle(Q, Kl, Vl, idx, coff, Kb, Vb, Mmax, D)
    assert flag == 0
    close_abs(to64(out), Oo, 1e-4, "O (fp32)")
