"""Step-by-step parity of the CUDA path against the fp64 oracle, through the C ABI.

Inputs are drawn on the device by the seeded generators, copied to the host
for the oracle; the oracle never sees a CUDA result.  Sizes span several tiles
and ragged tails while the oracle still finishes in seconds.
"""
import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from oracle import msa_oracle as O
from workloads import synth

from .helpers import (NEAR_TIE, TOL_BF16_ABS, TOL_F32_ATTN, TOL_F32_POOL, TOL_F32_SCORE, TOL_SCORE_ABS,
                      attn_on_gpu, check_topk, close_abs, close_rel, pool_on_gpu, route_on_gpu, to64)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _raw(cfg, seed=0):
    q = synth.gen_query(cfg, 0, DEV, seed)
    K, V, Kr = synth.gen_raw_slab(cfg, 0, cfg.D, DEV, seed, Qr0=q["Qr"][0])
    return q, K, V, Kr


def _ragged_offsets(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


# ---------------------------------------------------------------- step 1: pool
def test_pool_tiny_fp32():
    cfg = synth.get_config("tiny")
    q, K, V, Kr = _raw(cfg)
    off = synth.doc_tok_offsets(cfg)
    Kb, Vb, Krb, coff, rn, flag = pool_on_gpu(cfg, K, V, Kr, off)
    oK, oV, oKr, ocoff, orn = O.pool(to64(K), to64(V), to64(Kr), off, cfg.P, cfg.theta)
    torch.cuda.synchronize()
    assert flag.item() == 0
    assert np.array_equal(coff, ocoff)
    close_rel(to64(Kb), oK, TOL_F32_POOL, "Kbar")
    close_rel(to64(Vb), oV, TOL_F32_POOL, "Vbar")
    close_rel(to64(Krb), oKr, TOL_F32_POOL, "Krbar")
    close_rel(to64(rn), orn, TOL_F32_POOL, "kr_rnorm")


@pytest.mark.parametrize("lengths", [
    [500] * 24,                                          # the 10M stack's documents: 7 x 64 + 52
    [1, 64, 65, 0, 127, 128, 129, 500, 3, 0, 64, 1000],   # ragged, empty, single-token documents
])
def test_pool_bf16_ragged(lengths):
    cfg = synth.get_config("stack10m").scaled(D=len(lengths), docs_per_slab=0)
    off = _ragged_offsets(lengths)
    n = int(off[-1])
    g = torch.Generator(device=DEV).manual_seed(7)
    K = (0.5 * torch.randn((n, 8, 128), generator=g, device=DEV)).bfloat16()
    V = (0.5 * torch.randn((n, 8, 128), generator=g, device=DEV)).bfloat16()
    Kr = torch.randn((n, 8, 128), generator=g, device=DEV).bfloat16()
    Kb, Vb, Krb, coff, rn, flag = pool_on_gpu(cfg, K, V, Kr, off)
    oK, oV, oKr, ocoff, orn = O.pool(to64(K), to64(V), to64(Kr), off, cfg.P, cfg.theta, out_bf16=True)
    torch.cuda.synchronize()
    assert flag.item() == 0
    assert np.array_equal(coff, ocoff)
    close_abs(to64(Kb), oK, TOL_BF16_ABS, "Kbar")
    close_abs(to64(Vb), oV, TOL_BF16_ABS, "Vbar")
    close_abs(to64(Krb), oKr, TOL_BF16_ABS, "Krbar")
    # the bf16 rounding of the mean is the same rounding in nearly every element
    assert np.mean(to64(Kb) == oK) > 0.99 and np.mean(to64(Krb) == oKr) > 0.99
    # kr_rnorm is 1/||stored Krbar||: exact property, and close to the oracle's own
    Kg = to64(Krb)
    close_rel(to64(rn), 1.0 / np.maximum(np.linalg.norm(Kg, axis=-1), 1e-12), 1e-6, "rnorm property")
    close_rel(to64(rn), orn, 1e-2, "rnorm vs oracle")


def test_pool_flags_long_document_and_bad_offsets():
    cfg = synth.get_config("tiny").scaled(D=3)
    off = _ragged_offsets([10, 100, 20])
    n = int(off[-1])
    K = torch.randn((n, 2, 64), device=DEV)
    rope = msa.rope_table(cfg.theta, 64, 50).to(DEV)           # doc 1 (100 tokens) is too long
    Kb, Vb, Krb, coff, rn, flag = pool_on_gpu(cfg, K, K, K, off, rope=rope)
    torch.cuda.synchronize()
    assert flag.item() & msa.FLAG_INDEX_OOB
    oK, _, _, _, _ = O.pool(to64(K), to64(K), to64(K), off, cfg.P, cfg.theta)
    close_rel(to64(Kb)[0], oK[0], TOL_F32_POOL, "doc 0 still pooled")
    # offsets that disagree with P: document 0 given two chunks instead of one
    bad = torch.tensor([0, 2, 4, 5], dtype=torch.int64, device=DEV)
    Kb2 = torch.empty((5, 2, 64), device=DEV)
    flag2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.pool(K, K, K, torch.from_numpy(off).to(DEV), bad, cfg.P, msa.rope_table(cfg.theta, 64, 128).to(DEV),
             Kb2, torch.empty_like(Kb2), torch.empty_like(Kb2), None, flag2)
    torch.cuda.synchronize()
    assert flag2.item() & msa.FLAG_OFFSETS


# ---------------------------------------------------------------- steps 2-3: route + top-k
def test_route_topk_tiny_fp32_planted():
    cfg = synth.get_config("tiny")
    q, K, V, Kr = _raw(cfg)
    off = synth.doc_tok_offsets(cfg)
    Kb, Vb, Krb, coff, rn, _ = pool_on_gpu(cfg, K, V, Kr, off)
    idx, sc, ds, flag = route_on_gpu(q["Qr"], Krb, rn, coff, cfg.k)
    _, _, oKr, _, _ = O.pool(to64(K), to64(V), to64(Kr), off, cfg.P, cfg.theta)
    ods = O.route(to64(q["Qr"]), oKr, coff)
    torch.cuda.synchronize()
    assert flag.item() == 0
    close_rel(to64(ds), ods, TOL_F32_SCORE, "doc scores")
    check_topk(idx.cpu().numpy(), to64(sc), ods, cfg.k, 1e-5)
    assert idx[0, 0].item() == 17 and abs(sc[0, 0].item() - 1.0) < 1e-5


def _bank_case(C_docs, Hr, dr, seed):
    """A drawn bf16 bank with ragged documents (0..9 chunks), and its rnorm from the library."""
    rng = np.random.default_rng(seed)
    n = rng.integers(0, 10, size=C_docs)
    n[rng.integers(0, C_docs)] = 0
    coff = _ragged_offsets(n)
    C = int(coff[-1])
    Krb = synth.gen_bank_bf16(C, Hr, dr, DEV, seed)
    rn = torch.empty((C, Hr), dtype=torch.float32, device=DEV)
    msa.bank_rnorm(Krb, rn)
    return Krb, rn, coff


@pytest.mark.parametrize("B,Tq,Hr,dr,D,k", [
    (1, 512, 8, 128, 300, 16),    # 1M-token workload's query shape
    (64, 1, 8, 128, 700, 16),     # batched decode
    (1, 64, 8, 128, 1500, 16),    # 100M workload's query shape
    (3, 37, 4, 64, 257, 5),       # odd sizes, dr = 64
    (2, 9, 1, 128, 40, 40),       # one router head, k = D
    (4, 2, 8, 128, 20000, 32),    # largest k of the warp-level top-k, three slices merged
    (3, 3, 8, 128, 17000, 33),    # smallest k of the block-level top-k, three slices
    (2, 5, 2, 64, 9000, 1),       # k = 1 over two slices
    (64, 1, 2, 64, 32768, 16),    # four whole slices per query (256 threads x 32 documents each)
    (1, 4, 2, 64, 20, 20),        # fewer documents than a warp, k = D
    (1, 512, 8, 128, 9000, 16),   # ~40K chunks, 4 blocks of 128 query rows
    (2, 300, 1, 128, 9000, 16),   # blocks that span two queries, ragged last block
    (1, 600, 2, 64, 9000, 16),    # dr = 64, ragged last block
    # CTA-pair scan (blocks of 256 rows inside one query)
    (3, 512, 8, 128, 1500, 16),   # several queries, Tq a multiple of 256
    (1, 4096, 8, 128, 300, 16),   # the 16-layer workload's query length: 16 row blocks
    (1, 256, 3, 128, 1001, 7),    # one row block, three router heads
    (1, 300, 8, 128, 20, 4),      # under 128 chunks: the pair's second CTA holds none
])
def test_route_topk_bf16(B, Tq, Hr, dr, D, k):
    Krb, rn, coff = _bank_case(D, Hr, dr, seed=B * 1000 + Tq)
    g = torch.Generator(device=DEV).manual_seed(11)
    Qr = torch.randn((B, Tq, Hr, dr), generator=g, device=DEV).bfloat16()
    idx, sc, ds, flag = route_on_gpu(Qr, Krb, rn, coff, k)
    ods = O.route(to64(Qr), to64(Krb), coff)
    torch.cuda.synchronize()
    assert flag.item() == 0
    gds = to64(ds)
    empty = np.isneginf(ods)
    assert np.array_equal(np.isneginf(gds), empty)
    close_abs(gds[~empty], ods[~empty], TOL_SCORE_ABS, "doc scores")
    check_topk(idx.cpu().numpy(), to64(sc), ods, k, TOL_SCORE_ABS)


def test_topk_exact_ties_prefer_lower_index():
    # 40 documents of one chunk, bank rows copied so that scores tie exactly
    base = synth.gen_bank_bf16(5, 2, 64, DEV, 3)
    Krb = base[torch.tensor([i % 5 for i in range(40)], device=DEV)].contiguous()
    rn = torch.empty((40, 2), dtype=torch.float32, device=DEV)
    msa.bank_rnorm(Krb, rn)
    coff = np.arange(41, dtype=np.int64)
    Qr = torch.randn((1, 3, 2, 64), device=DEV).bfloat16()
    idx, sc, ds, _ = route_on_gpu(Qr, Krb, rn, coff, 12)
    ods = O.route(to64(Qr), to64(Krb), coff)
    oi, _ = O.topk(ods, 12)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), oi)   # exact: equal scores resolved by index


def test_topk_many_slices_merge():
    # three slices of the per-row filter plus the last-CTA merge, two query rows
    Krb, rn, coff = _bank_case(70000, 2, 64, seed=21)
    g = torch.Generator(device=DEV).manual_seed(12)
    Qr = torch.randn((2, 3, 2, 64), generator=g, device=DEV).bfloat16()
    idx, sc, ds, flag = route_on_gpu(Qr, Krb, rn, coff, 16)
    ods = O.route(to64(Qr), to64(Krb), coff)
    torch.cuda.synchronize()
    assert flag.item() == 0
    check_topk(idx.cpu().numpy(), to64(sc), ods, 16, TOL_SCORE_ABS)


def test_topk_more_slices_than_one_merge_round():
    # 600,000 one-chunk documents: 74 slices of 8192, more lists than the last CTA
    # merges at once in shared memory (64), so the merge runs in two batches
    D, k = 600000, 16
    g = torch.Generator(device=DEV).manual_seed(31)
    Krb = (torch.randn((D, 1, 64), generator=g, device=DEV)).bfloat16()
    rn = torch.empty((D, 1), dtype=torch.float32, device=DEV)
    msa.bank_rnorm(Krb, rn)
    coff = np.arange(D + 1, dtype=np.int64)
    Qr = torch.randn((1, 1, 1, 64), generator=g, device=DEV).bfloat16()
    idx, sc, ds, flag = route_on_gpu(Qr, Krb, rn, coff, k)
    ods = O.route(to64(Qr), to64(Krb), coff)
    torch.cuda.synchronize()
    assert flag.item() == 0
    check_topk(idx.cpu().numpy(), to64(sc), ods, k, TOL_SCORE_ABS)


def test_topk_filter_overflow_takes_streaming_path():
    # k = 100 over four slices of 8192 one-chunk documents; in a slice the
    # filter's 256 threads hold 32 documents each (document i of the slice is
    # item i // 256 of thread i % 256).  In every slice the documents of threads
    # 0..99 score high and rise with (thread, item), so several thousand keys
    # pass the threshold and each slice falls back to the streamed block sort.
    D, k, dr, S, T = 4 * 8192, 100, 64, 8192, 256
    idx_all = np.arange(D)
    local = idx_all % S
    t, m = local % T, local // T
    heavy = t < k
    a = np.where(heavy, 1.0 + (t * 32 + m) / 4096.0, -1.0)
    bank = np.zeros((D, 1, dr), dtype=np.float32)
    bank[:, 0, 0] = a
    bank[:, 0, 1] = 1.0
    Krb = torch.from_numpy(bank).to(DEV).bfloat16()
    rn = torch.empty((D, 1), dtype=torch.float32, device=DEV)
    msa.bank_rnorm(Krb, rn)
    coff = np.arange(D + 1, dtype=np.int64)
    qr = np.zeros((1, 1, 1, dr), dtype=np.float32)
    qr[..., 0] = 1.0
    Qr = torch.from_numpy(qr).to(DEV).bfloat16()
    idx, sc, ds, flag = route_on_gpu(Qr, Krb, rn, coff, k)
    ods = O.route(to64(Qr), to64(Krb), coff)
    oi, _ = O.topk(ods, k)
    torch.cuda.synchronize()
    assert flag.item() == 0
    # each slice's survivor count, from the oracle's scores: keys >= the k-th
    # largest per-thread maximum, keys ordered by (score, lower index)
    for sl in range(D // S):
        sc_sl, ix_sl, t_sl = ods[0, sl * S:(sl + 1) * S], idx_all[sl * S:(sl + 1) * S], t[sl * S:(sl + 1) * S]
        order = np.lexsort((ix_sl, -sc_sl))            # rank 0 = largest key
        rank = np.empty(S, dtype=np.int64)
        rank[order] = np.arange(S)
        thread_best = np.array([rank[t_sl == i].min() for i in range(T)])
        tau_rank = np.sort(thread_best)[k - 1]
        assert int((rank <= tau_rank).sum()) > 2048
    assert np.array_equal(idx.cpu().numpy(), oi)


# ---------------------------------------------------------------- step 4: gather
def test_gather_bitexact_and_flags():
    rng = np.random.default_rng(5)
    D = 50
    n = rng.integers(0, 9, size=D)
    coff = _ragged_offsets(n)
    C = int(coff[-1])
    Kb = synth.gen_bank_bf16(C, 8, 128, DEV, 1, "K")
    Vb = synth.gen_bank_bf16(C, 8, 128, DEV, 1, "V")
    B, k, Mmax = 4, 6, 6 * 8
    sel = np.stack([rng.choice(D, k, replace=False) for _ in range(B)]).astype(np.int32)
    Km = torch.zeros((B, Mmax, 8, 128), dtype=torch.bfloat16, device=DEV)
    Vm = torch.zeros_like(Km)
    ml = torch.zeros(B, dtype=torch.int32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    coff_d = torch.from_numpy(coff).to(DEV)
    msa.gather(torch.from_numpy(sel).to(DEV), coff_d, Kb, Vb, Km, Vm, ml, flag)
    oKm, oVm, oml = O.gather(sel, coff, to64(Kb), to64(Vb), Mmax)
    torch.cuda.synchronize()
    assert flag.item() == 0
    assert np.array_equal(ml.cpu().numpy(), oml)
    for b in range(B):
        m = int(oml[b])
        assert np.array_equal(to64(Km)[b, :m], oKm[b, :m]) and np.array_equal(to64(Vm)[b, :m], oVm[b, :m])
    # an out-of-range document index is skipped and flagged; too many rows are dropped and flagged
    sel2 = sel.copy()
    sel2[1, 2] = D + 7
    flag.zero_()
    msa.gather(torch.from_numpy(sel2).to(DEV), coff_d, Kb, Vb, Km, Vm, ml, flag)
    torch.cuda.synchronize()
    assert flag.item() & msa.FLAG_INDEX_OOB
    Km_small = torch.zeros((B, 3, 8, 128), dtype=torch.bfloat16, device=DEV)
    flag.zero_()
    msa.gather(torch.from_numpy(sel).to(DEV), coff_d, Kb, Vb, Km_small, torch.zeros_like(Km_small), ml, flag)
    torch.cuda.synchronize()
    assert flag.item() & msa.FLAG_OVERFLOW
    assert ml.max().item() <= 3


def test_gather_zeroes_rows_past_the_selection():
    """Rows [mem_len, Mmax) of the output are set to zero (they start as NaN here), so the
    attention kernels, which multiply masked rows by zero weights, stay finite."""
    rng = np.random.default_rng(8)
    D = 40
    n = rng.integers(1, 5, size=D)
    coff = _ragged_offsets(n)
    C = int(coff[-1])
    Kb = synth.gen_bank_bf16(C, 8, 128, DEV, 2, "K")
    Vb = synth.gen_bank_bf16(C, 8, 128, DEV, 2, "V")
    B, k, Mmax = 3, 5, 150
    sel = np.stack([rng.choice(D, k, replace=False) for _ in range(B)]).astype(np.int32)
    Km = torch.full((B, Mmax, 8, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    Vm = torch.full_like(Km, float("nan"))
    ml = torch.zeros(B, dtype=torch.int32, device=DEV)
    msa.gather(torch.from_numpy(sel).to(DEV), torch.from_numpy(coff).to(DEV), Kb, Vb, Km, Vm, ml)
    torch.cuda.synchronize()
    for b in range(B):
        m = int(ml[b])
        assert 0 < m < Mmax
        assert not Km[b, m:].float().abs().sum() and not Vm[b, m:].float().abs().sum()
    oKm, oVm, oml = O.gather(sel, coff, to64(Kb), to64(Vb), Mmax)
    for Tq, Lloc in ((1, 300), (100, 150)):      # decode and prefill kernels
        g = torch.Generator(device=DEV).manual_seed(Tq)
        Q = (0.5 * torch.randn((B, Tq, 32, 128), generator=g, device=DEV)).bfloat16()
        Kl = (0.5 * torch.randn((B, Lloc, 8, 128), generator=g, device=DEV)).bfloat16()
        Vl = (0.5 * torch.randn((B, Lloc, 8, 128), generator=g, device=DEV)).bfloat16()
        Og, lse, flag = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
        Oo, _ = O.attention(to64(Q), to64(Kl), to64(Vl), oKm, oVm, oml)
        torch.cuda.synchronize()
        assert flag.item() == 0
        close_abs(to64(Og), Oo, TOL_BF16_ABS, f"O (Tq={Tq})")


# ---------------------------------------------------------------- step 5: attention
def _attn_inputs(B, Tq, Lloc, Hq, Hkv, d, Mmax, mem_lens, dtype, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    r = lambda *s: (0.5 * torch.randn(s, generator=g, device=DEV)).to(dtype)
    Q, Kl, Vl = r(B, Tq, Hq, d), r(B, Lloc, Hkv, d), r(B, Lloc, Hkv, d)
    Km, Vm = r(B, max(Mmax, 1), Hkv, d), r(B, max(Mmax, 1), Hkv, d)
    ml = torch.tensor(mem_lens, dtype=torch.int32, device=DEV)
    return Q, Kl, Vl, Km, Vm, ml


def test_attention_tiny_fp32():
    Q, Kl, Vl, Km, Vm, ml = _attn_inputs(1, 32, 32, 4, 2, 64, 16, [16], torch.float32, 1)
    Og, lse, flag = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
    Oo, olse = O.attention(to64(Q), to64(Kl), to64(Vl), to64(Km), to64(Vm), [16])
    torch.cuda.synchronize()
    assert flag.item() == 0
    close_abs(to64(Og), Oo, TOL_F32_ATTN, "O")
    close_abs(to64(lse), olse, TOL_F32_ATTN, "lse")


@pytest.mark.parametrize("B,Tq,Lloc,Hq,Hkv,d,Mmax,mem_lens", [
    (1, 200, 300, 32, 8, 128, 128, [128]),           # prefill, ragged tiles, Lloc > Tq
    (2, 130, 130, 8, 8, 64, 40, [0, 40]),            # MHA, d = 64, one row with no memory
    (4, 1, 1000, 32, 8, 128, 128, [128, 0, 77, 5]),  # decode
    (1, 64, 64, 32, 8, 128, 128, [128]),             # the 100M workload's query shape
])
def test_attention_bf16(B, Tq, Lloc, Hq, Hkv, d, Mmax, mem_lens):
    Q, Kl, Vl, Km, Vm, ml = _attn_inputs(B, Tq, Lloc, Hq, Hkv, d, Mmax, mem_lens, torch.bfloat16, 2)
    Og, lse, flag = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
    Oo, olse = O.attention(to64(Q), to64(Kl), to64(Vl), to64(Km), to64(Vm), mem_lens)
    torch.cuda.synchronize()
    assert flag.item() == 0
    close_abs(to64(Og), Oo, TOL_BF16_ABS, "O")
    close_abs(to64(lse), olse, 2e-3, "lse")


@pytest.mark.parametrize("B,Tq,Lloc,Hq,Hkv,Mmax,mem_lens", [
    (3, 100, 260, 32, 8, 160, [128, 0, 77]),      # G=4: ragged memory tiles, one row without memory
    (1, 300, 300, 8, 8, 128, [128]),              # G=1 (MHA): 128 tokens per block
    (2, 50, 400, 64, 8, 256, [256, 200]),         # G=8: 16 tokens per block, two memory tiles
    (1, 1030, 1030, 32, 8, 128, [128]),           # many local tiles, a partial last block
    (4, 480, 480, 32, 8, 128, [128, 0, 100, 128]),  # odd block count, ragged memory across the batch
    (2, 1100, 1300, 32, 8, 256, [256, 37]),       # local history longer than the query, partial last block
    (1, 600, 600, 64, 8, 128, [128]),             # G=8: 16 tokens per tile, many tiles
    (2, 512, 512, 40, 40, 64, [64, 30]),          # G=1 with 40 heads: 128 tokens per tile
    (2, 20, 300, 32, 8, 128, [128, 50]),          # one ragged block of rows per KV head
    (1, 33, 33, 32, 8, 0, [0]),                   # two blocks, the second with one token, no memory
])
def test_attention_bf16_tensor_core_tiling(B, Tq, Lloc, Hq, Hkv, Mmax, mem_lens):
    Q, Kl, Vl, Km, Vm, ml = _attn_inputs(B, Tq, Lloc, Hq, Hkv, 128, Mmax, mem_lens, torch.bfloat16, 4)
    Og, lse, flag = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
    Oo, olse = O.attention(to64(Q), to64(Kl), to64(Vl), to64(Km), to64(Vm), mem_lens)
    torch.cuda.synchronize()
    assert flag.item() == 0
    close_abs(to64(Og), Oo, TOL_BF16_ABS, "O")
    close_abs(to64(lse), olse, 2e-3, "lse")


@pytest.mark.parametrize("B,Tq,Lloc,Hq,Hkv,Mmax,mem_lens", [
    (5, 1, 4096, 32, 8, 128, [128, 0, 77, 1, 128]),   # the batched-decode shape, ragged memory
    (2, 4, 700, 32, 8, 200, [200, 13]),               # 4 tokens x G=4: 16 rows, causal inside the block
    (3, 2, 300, 64, 8, 128, [5, 128, 64]),             # G=8, 2 tokens: 16 rows
    (2, 3, 129, 8, 8, 0, [0, 0]),                      # MHA, no memory at all
])
def test_attention_bf16_decode_shapes(B, Tq, Lloc, Hq, Hkv, Mmax, mem_lens):
    Q, Kl, Vl, Km, Vm, ml = _attn_inputs(B, Tq, Lloc, Hq, Hkv, 128, Mmax, mem_lens, torch.bfloat16, 5)
    Og, lse, flag = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
    Oo, olse = O.attention(to64(Q), to64(Kl), to64(Vl), to64(Km), to64(Vm), mem_lens)
    torch.cuda.synchronize()
    assert flag.item() == 0
    close_abs(to64(Og), Oo, TOL_BF16_ABS, "O")
    close_abs(to64(lse), olse, 2e-3, "lse")


@pytest.mark.parametrize("B,Tq,Lloc,Hq,Hkv,Mmax,mem_lens,dtype", [
    (2, 8, 300, 32, 8, 128, [128, 40], torch.bfloat16),      # 8 tokens x G=4: too few for a tensor-core block, too many rows to decode
    (1, 70, 150, 40, 8, 64, [50], torch.bfloat16),           # G=5 does not divide a block of 128 rows
    (3, 1, 500, 40, 8, 128, [128, 0, 60], torch.bfloat16),   # G=5 decode: 5 real rows of the 8-row kernel
    (2, 40, 100, 32, 1, 32, [32, 7], torch.bfloat16),        # G=32: 4 tokens per block, under the tensor-core minimum
    (1, 50, 90, 8, 2, 40, [40], torch.float32),              # fp32 at d = 128
])
def test_attention_shapes_outside_the_tensor_core_tiles(B, Tq, Lloc, Hq, Hkv, Mmax, mem_lens, dtype):
    Q, Kl, Vl, Km, Vm, ml = _attn_inputs(B, Tq, Lloc, Hq, Hkv, 128, Mmax, mem_lens, dtype, 6)
    Og, lse, flag = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
    Oo, olse = O.attention(to64(Q), to64(Kl), to64(Vl), to64(Km), to64(Vm), mem_lens)
    torch.cuda.synchronize()
    assert flag.item() == 0
    tol = TOL_F32_ATTN if dtype == torch.float32 else TOL_BF16_ABS
    close_abs(to64(Og), Oo, tol, "O")
    close_abs(to64(lse), olse, TOL_F32_ATTN if dtype == torch.float32 else 2e-3, "lse")


def test_attention_bad_mem_len_is_flagged_not_faulted():
    Q, Kl, Vl, Km, Vm, ml = _attn_inputs(1, 4, 4, 2, 1, 64, 8, [9999], torch.bfloat16, 3)
    Og, lse, flag = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
    torch.cuda.synchronize()
    assert flag.item() & msa.FLAG_INDEX_OOB
    Oo, _ = O.attention(to64(Q), to64(Kl), to64(Vl), to64(Km), to64(Vm), [8])   # clamped to Mmax
    close_abs(to64(Og), Oo, TOL_BF16_ABS, "O with clamped mem_len")
