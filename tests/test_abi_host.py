"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point that include/msa.h declares, its host helpers agree with the
oracle, and bad arguments are rejected before anything is launched.

Every rejected call below has exactly one bad argument, and that argument is
checked before any CUDA call in the entry point, so no device work is queued
even when a GPU is present (the fake device pointers are never dereferenced).
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from routed_sparse_attention_chunk_b200 import _lib
from oracle import msa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, WORKSPACE = 0, -1, -2, -3
FAKE = 0x10000  # 16-byte aligned, never dereferenced (validation fails first)


def declared_functions():
    src = open(os.path.join(ROOT, "include", "msa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    lib = _lib.load()
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"libmsa.so does not export {n}"
    assert set(names) == set(_lib.SIGNATURES), "binding signatures out of step with msa.h"


def test_status_strings_and_version():
    lib = _lib.load()
    for st in (OK, INVALID, UNSUPPORTED, WORKSPACE, -4, 12345):
        assert lib.msa_status_string(st)
    assert re.fullmatch(rb"\d+\.\d+\.\d+", lib.msa_version())


def test_rope_table_matches_oracle_angles():
    t = msa.rope_table(1e6, 128, 600).numpy()
    ang = O.rope_angles(np.arange(600), 128, 1e6)
    np.testing.assert_allclose(t[..., 0], np.cos(ang).astype(np.float32), rtol=0, atol=1.2e-7)
    np.testing.assert_allclose(t[..., 1], np.sin(ang).astype(np.float32), rtol=0, atol=1.2e-7)
    lib = _lib.load()
    buf = (ctypes.c_float * 8)()
    assert lib.msa_rope_table_host(1e6, 3, 4, buf) == INVALID
    assert lib.msa_rope_table_host(-1.0, 4, 1, buf) == INVALID
    assert lib.msa_rope_table_host(1e6, 4, 0, buf) == INVALID


def test_chunk_offsets_match_oracle():
    off = np.array([0, 500, 1000, 1064, 1065, 1065, 1200], dtype=np.int64)
    for P in (1, 7, 64, 4096):
        assert np.array_equal(msa.chunk_offsets(off, P), O.chunk_offsets(off, P))
    with pytest.raises(msa.MSAError):
        msa.chunk_offsets(np.array([0, 5, 3]), 64)


def _pool(**kw):
    a = dict(dt=1, K=FAKE, V=FAKE, Kr=FAKE, tok=FAKE, chk=FAKE, D=4, Ntok=100, C=4, Hkv=8, d=128, Hr=8,
             dr=128, P=64, rope=FAKE, max_len=64, Kb=FAKE, Vb=FAKE, Krb=FAKE, rn=None, flag=None)
    a.update(kw)
    return _lib.load().msa_pool(*a.values(), None)


def test_pool_rejects_bad_arguments():
    assert _pool(d=96) == UNSUPPORTED
    assert _pool(dr=32) == UNSUPPORTED
    assert _pool(P=0) == INVALID
    assert _pool(P=5000) == UNSUPPORTED
    assert _pool(K=None) == INVALID
    assert _pool(V=FAKE + 8) == INVALID           # misaligned
    assert _pool(dt=7) == INVALID
    assert _pool(C=0, K=None) == OK                # nothing to do, nothing launched


def _route(**kw):
    a = dict(dt=1, Qr=FAKE, B=1, Tq=4, Hr=8, dr=128, Krb=FAKE, rn=FAKE, chk=FAKE, D=10, C=20, k=3,
             ds=None, idx=FAKE, sc=None, ws=FAKE, wsb=1 << 20, flag=None)
    a.update(kw)
    return _lib.load().msa_route_topk(*a.values(), None)


def test_route_rejects_bad_arguments():
    assert _route(k=11) == INVALID          # k > D
    assert _route(k=0) == INVALID
    assert _route(Hr=9) == UNSUPPORTED
    assert _route(dr=96) == UNSUPPORTED
    assert _route(Tq=0) == INVALID
    assert _route(idx=None) == INVALID
    assert _route(Qr=FAKE + 2) == INVALID
    assert _route(ws=None) == WORKSPACE
    need = _lib.load().msa_route_topk_workspace_size(1, 4, 8, 10, 20, 3)
    assert need > 0 and _route(wsb=need - 1) == WORKSPACE
    assert _route(B=0) == OK


def _attn(**kw):
    a = dict(dt=1, Q=FAKE, Kl=FAKE, Vl=FAKE, B=1, Tq=8, Lloc=8, Hq=32, Hkv=8, d=128, Km=FAKE, Vm=FAKE,
             ml=FAKE, Mmax=16, scale=0.0, O=FAKE, lse=None, ws=FAKE, wsb=1 << 20, flag=None)
    a.update(kw)
    return _lib.load().msa_sparse_attn(*a.values(), None)


def test_attention_rejects_bad_arguments():
    assert _attn(Hq=30) == INVALID          # Hq % Hkv != 0
    assert _attn(Lloc=4) == INVALID         # Lloc < Tq
    assert _attn(d=80) == UNSUPPORTED
    assert _attn(Mmax=-1) == INVALID
    assert _attn(O=None) == INVALID
    assert _attn(ml=None) == INVALID
    assert _attn(Kl=FAKE + 4) == INVALID
    assert _attn(B=0) == OK


def test_gather_and_layer_reject_bad_arguments():
    lib = _lib.load()
    g = dict(dt=1, idx=FAKE, B=2, k=4, chk=FAKE, D=10, C=30, Kb=FAKE, Vb=FAKE, Hkv=8, d=128, Mmax=32,
             Km=FAKE, Vm=FAKE, ml=FAKE, flag=None)
    assert lib.msa_gather(*dict(g, d=100).values(), None) == UNSUPPORTED
    assert lib.msa_gather(*dict(g, ml=None).values(), None) == INVALID
    assert lib.msa_gather(*dict(g, Km=FAKE + 1).values(), None) == INVALID
    need = lib.msa_layer_forward_workspace_size(1, 8, 8, 32, 8, 128, 8, 10, 20, 3, 24)
    assert need > lib.msa_route_topk_workspace_size(1, 8, 8, 10, 20, 3)
    L = dict(dt=1, Qr=FAKE, Hr=8, dr=128, Krb=FAKE, rn=FAKE, chk=FAKE, D=10, C=20, k=3, Q=FAKE, Kl=FAKE,
             Vl=FAKE, B=1, Tq=8, Lloc=8, Hq=32, Hkv=8, d=128, Kb=FAKE, Vb=FAKE, Mmax=24, scale=0.0, O=FAKE,
             lse=None, idx=FAKE, sc=None, ds=None, ws=FAKE, wsb=need, flag=None)
    assert lib.msa_layer_forward(*dict(L, wsb=need - 1).values(), None) == WORKSPACE
    assert lib.msa_layer_forward(*dict(L, Hq=33).values(), None) == INVALID
    assert lib.msa_layer_forward(*dict(L, k=0).values(), None) == INVALID
    assert lib.msa_layer_forward(*dict(L, Kb=None).values(), None) == INVALID


def test_binding_rejects_host_and_strided_tensors():
    x = torch.zeros((4, 8, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        msa.bank_rnorm(x, torch.zeros((4, 8)))
    with pytest.raises(TypeError):
        msa._dt(torch.zeros(2, dtype=torch.float16))


def test_backward_entry_points_reject_bad_arguments():
    lib = _lib.load()
    bw = dict(dt=1, Q=FAKE, Kl=FAKE, Vl=FAKE, B=1, Tq=8, Lloc=8, Hq=32, Hkv=8, d=128, Km=FAKE, Vm=FAKE, ml=FAKE,
              Mmax=16, scale=0.0, O=FAKE, lse=FAKE, dO=FAKE, dQ=FAKE, dKl=FAKE, dVl=FAKE, dKm=FAKE, dVm=FAKE,
              ws=FAKE, wsb=lib.msa_sparse_attn_backward_workspace_size(1, 8, 32), flag=None)
    call = lambda **kw: lib.msa_sparse_attn_backward(*dict(bw, **kw).values(), None)
    assert call(d=96) == UNSUPPORTED
    assert call(Lloc=4) == INVALID            # Lloc < Tq
    assert call(lse=None) == INVALID          # the forward's lse is required
    assert call(dKm=None) == INVALID          # memory gradients required when Mmax > 0
    assert call(dO=FAKE + 4) == INVALID       # misaligned
    assert call(wsb=3) == WORKSPACE
    assert call(B=0) == OK
    assert lib.msa_sparse_attn_backward_workspace_size(2, 5, 4) >= 2 * 5 * 4 * 4
    gb = dict(idx=FAKE, B=2, k=4, chk=FAKE, D=10, C=30, dKm=FAKE, dVm=FAKE, ml=FAKE, Hkv=8, d=128, Mmax=32,
              dKb=FAKE, dVb=FAKE, flag=None)
    gcall = lambda **kw: lib.msa_gather_backward(*dict(gb, **kw).values(), None)
    assert gcall(d=100) == UNSUPPORTED
    assert gcall(dKb=None) == INVALID
    assert gcall(k=0) == INVALID
    assert gcall(B=0) == OK
    rb = dict(dt=1, Qr=FAKE, B=2, Tq=4, Hr=8, dr=128, Krb=FAKE, rn=FAKE, chk=FAKE, D=10, C=30, k=4, idx=FAKE,
              dsc=FAKE, dQr=FAKE, dKrb=FAKE, ws=FAKE, wsb=lib.msa_route_backward_workspace_size(2, 4, 4), flag=None)
    rcall = lambda **kw: lib.msa_route_backward(*dict(rb, **kw).values(), None)
    assert rcall(dr=96) == UNSUPPORTED
    assert rcall(Hr=9) == UNSUPPORTED
    assert rcall(k=11) == INVALID             # k > D
    assert rcall(dsc=None) == INVALID         # the upstream gradient is required
    assert rcall(dKrb=None) == INVALID
    assert rcall(Qr=FAKE + 4) == INVALID      # misaligned
    assert rcall(wsb=0) == WORKSPACE
    assert rcall(B=0) == OK
    assert lib.msa_route_backward_workspace_size(2, 4, 4) >= 2 * 4 * 8
    assert lib.msa_route_backward_workspace_size(2, 130, 4) >= 2 * 4 * 8 * 3   # a candidate per 64 tokens


def test_state_gather_sum_rejects_bad_arguments():
    lib = _lib.load()
    a = dict(dt=1, st=FAKE, D=10, S=64, idx=FAKE, B=2, k=3, out=FAKE, flag=None)
    assert lib.msa_state_gather_sum(*dict(a, S=60).values(), None) == UNSUPPORTED     # bf16: S % 8
    assert lib.msa_state_gather_sum(*dict(a, dt=0, S=62).values(), None) == UNSUPPORTED  # fp32: S % 4
    assert lib.msa_state_gather_sum(*dict(a, B=70000).values(), None) == UNSUPPORTED
    assert lib.msa_state_gather_sum(*dict(a, dt=7).values(), None) == INVALID
    assert lib.msa_state_gather_sum(*dict(a, k=0).values(), None) == INVALID
    assert lib.msa_state_gather_sum(*dict(a, D=0).values(), None) == INVALID
    assert lib.msa_state_gather_sum(*dict(a, out=None).values(), None) == INVALID
    assert lib.msa_state_gather_sum(*dict(a, out=FAKE + 4).values(), None) == INVALID
    assert lib.msa_state_gather_sum(*dict(a, B=0).values(), None) == OK              # nothing to do


def test_noalloc_checks_arguments_before_its_size():
    # msa_route_topk_noalloc runs msa_route_topk's argument checks first, so an
    # invalid argument reports its own error even when the problem is also too
    # large for the fixed scratch; a valid oversize problem reports TOO_LARGE
    lib = _lib.load()
    B, Tq, Hr, D, k = 64, 1, 8, 1 << 17, 16
    call = lambda qr, dr, kk: lib.msa_route_topk_noalloc(1, qr, B, Tq, Hr, dr, FAKE, FAKE, FAKE, D, 4 * D, kk,
                                                         None, FAKE, None, None, None)
    assert call(FAKE, 96, k) == UNSUPPORTED      # dr = 96
    assert call(None, 128, k) == INVALID         # no Qr
    assert call(FAKE, 128, D + 1) == INVALID     # k > D
    assert call(FAKE, 128, k) == -5              # MSA_ERR_TOO_LARGE


def _largest_fitting_docs(B, Tq, Hr, chunks_per_doc, k):
    lo, hi = 1, 1 << 26
    while lo < hi:
        m = (lo + hi + 1) // 2
        if msa.route_topk_workspace_size(B, Tq, Hr, m, chunks_per_doc * m, k) <= msa.NOALLOC_SCRATCH_BYTES:
            lo = m
        else:
            hi = m - 1
    return lo


def test_noalloc_bounds_in_the_header_are_exact():
    # msa.h states the largest document counts the allocation-free entry point takes for two
    # shapes (documents of 8 chunks, Hr = 8, k = 16); they are the exact boundary of the library's
    # own size function, and its size formula holds to the 256-byte rounding of each part
    text = open(os.path.join(ROOT, "include", "msa.h")).read()
    text = re.sub(r"\s+", " ", re.sub(r"\n\s*\*", " ", text))  # comment lines joined
    one = int(re.search(r"fits up to ([0-9,]+) documents", text).group(1).replace(",", ""))
    many = int(re.search(r"64 one-token queries up to ([0-9,]+) documents", text).group(1).replace(",", ""))
    assert _largest_fitting_docs(1, 64, 8, 8, 16) == one
    assert _largest_fitting_docs(64, 1, 8, 8, 16) == many
    for B, Tq, D in ((1, 64, one), (64, 1, many), (3, 7, 9000), (2, 1, 100)):
        Hr, k, C = 8, 16, 8 * D
        nslice = -(-D // 8192)
        formula = 4 * (B * D + B) + 4 * C + 4 * B * Tq * Hr + (8 * B * k * nslice if D > 8192 else 0)
        got = msa.route_topk_workspace_size(B, Tq, Hr, D, C, k)
        assert formula <= got <= formula + 4 * 255
