"""msa_route_topk_noalloc: the routing + top-k entry point for callers that
cannot allocate device memory when they call the library (for example a plugin
whose host framework owns all device memory).  It must give the same answer as
msa_route_topk with a caller workspace, call after call, although every call
reuses the same library-owned scratch; and it must refuse a problem that does
not fit that scratch before doing any work.

This file is named so that pytest collects it last."""
import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from routed_sparse_attention_chunk_b200 import _lib
from workloads import synth

from .helpers import TOL_SCORE_ABS, close_abs, route_on_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bank(D, Hr, dr, seed, chunks_per_doc=None):
    rng = np.random.default_rng(seed)
    n = np.full(D, chunks_per_doc) if chunks_per_doc else rng.integers(1, 9, size=D)
    coff = np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
    Krb = synth.gen_bank_bf16(int(coff[-1]), Hr, dr, DEV, seed)
    rn = torch.empty((int(coff[-1]), Hr), dtype=torch.float32, device=DEV)
    msa.bank_rnorm(Krb, rn)
    return Krb, rn, coff


def _noalloc(Qr, Krb, rn, coff, k):
    B, D = Qr.shape[0], len(coff) - 1
    idx = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
    sc = torch.zeros((B, k), dtype=torch.float32, device=DEV)
    ds = torch.zeros((B, D), dtype=torch.float32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.route_topk_noalloc(Qr, Krb, rn, torch.from_numpy(coff).to(DEV), k, idx, sc, ds, flag)
    return idx, sc, ds, flag


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    # call 1: three queries over a larger bank; call 2: one different query over a
    # smaller bank, so stale per-document maxima left by call 1 would show up;
    # call 3: 20,000 documents, three top-k slices merged through per-query
    # counters and candidates that live in the shared scratch between calls
    cases = [(3, 40, 8, 128, 900, 16, 1), (1, 5, 8, 128, 300, 8, 2), (2, 3, 8, 128, 20000, 16, 3)]
    for B, Tq, Hr, dr, D, k, seed in cases:
        Krb, rn, coff = _bank(D, Hr, dr, seed)
        g = torch.Generator(device=DEV).manual_seed(100 + seed)
        Qr = torch.randn((B, Tq, Hr, dr), generator=g, device=DEV).bfloat16()
        i1, s1, d1, f1 = route_on_gpu(Qr, Krb, rn, coff, k)
        i2, s2, d2, f2 = _noalloc(Qr, Krb, rn, coff, k)
        torch.cuda.synchronize()
        assert f1.item() == 0 and f2.item() == 0
        assert torch.equal(i1, i2)
        close_abs(s2.cpu().numpy(), s1.cpu().numpy(), TOL_SCORE_ABS, "top-k scores")
        close_abs(d2.cpu().numpy(), d1.cpu().numpy(), TOL_SCORE_ABS, "document scores")


def _largest_fitting_docs(B, Tq, Hr, chunks_per_doc, k):
    lo, hi = 1, 1 << 26
    while lo < hi:
        m = (lo + hi + 1) // 2
        if msa.route_topk_workspace_size(B, Tq, Hr, m, chunks_per_doc * m, k) <= msa.NOALLOC_SCRATCH_BYTES:
            lo = m
        else:
            hi = m - 1
    return lo


def test_noalloc_size_bound_just_under_and_just_over():
    # one one-token query, one 64-wide router head, documents of 8 chunks: the
    # largest document count whose routing workspace fits the fixed scratch runs
    # (and matches the workspace entry point); one more document is refused
    B, Tq, Hr, dr, cpd, k = 1, 1, 1, 64, 8, 16
    D = _largest_fitting_docs(B, Tq, Hr, cpd, k)
    assert 400_000 < D < 500_000  # about 465,800: the header's stated bound for this shape
    Krb, rn, coff = _bank(D, Hr, dr, 5, chunks_per_doc=cpd)
    g = torch.Generator(device=DEV).manual_seed(105)
    Qr = torch.randn((B, Tq, Hr, dr), generator=g, device=DEV).bfloat16()
    i1, s1, d1, f1 = route_on_gpu(Qr, Krb, rn, coff, k)
    i2, s2, d2, f2 = _noalloc(Qr, Krb, rn, coff, k)
    torch.cuda.synchronize()
    assert f1.item() == 0 and f2.item() == 0
    assert torch.equal(i1, i2)
    close_abs(d2.cpu().numpy(), d1.cpu().numpy(), TOL_SCORE_ABS, "document scores")
    lib = _lib.load()
    fake = 0x10000
    assert lib.msa_route_topk_workspace_size(B, Tq, Hr, D + 1, cpd * (D + 1), k) > msa.NOALLOC_SCRATCH_BYTES
    st = lib.msa_route_topk_noalloc(1, fake, B, Tq, Hr, dr, fake, fake, fake, D + 1, cpd * (D + 1), k,
                                    None, fake, None, None, None)
    assert st == -5


def test_noalloc_rejects_a_problem_larger_than_its_scratch():
    lib = _lib.load()
    B, Tq, Hr, D, k = 64, 1, 8, 1 << 17, 16          # 64 x 131072 document keys alone are 32 MiB
    need = lib.msa_route_topk_workspace_size(B, Tq, Hr, D, 4 * D, k)
    assert need > msa.NOALLOC_SCRATCH_BYTES
    # the size check comes before any use of the (never dereferenced) pointers
    fake = 0x10000
    st = lib.msa_route_topk_noalloc(1, fake, B, Tq, Hr, 128, fake, fake, fake, D, 4 * D, k,
                                    None, fake, None, None, None)
    assert st == -5
    assert b"scratch" in lib.msa_status_string(st)
