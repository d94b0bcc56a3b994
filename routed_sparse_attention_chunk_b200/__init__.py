"""Python binding of the MSA memory-path library (include/msa.h) for B200.

Argument marshalling only: every function takes caller-allocated torch tensors,
checks that they are contiguous CUDA tensors of the right dtype (the bank's
K̄ / V̄ may instead be pinned host tensors: the host tier, read in place), and
passes raw pointers and sizes to the C ABI in libmsa.so on the current (or
given) stream.
All computation happens in the library's CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import torch

from . import _lib

F32, BF16 = 0, 1
FLAG_INDEX_OOB, FLAG_OFFSETS, FLAG_TIMEOUT, FLAG_OVERFLOW = 1, 2, 4, 8
DTYPES = {torch.float32: F32, torch.bfloat16: BF16}


class MSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = _lib.load().msa_status_string(status).decode()
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


def _dt(t: torch.Tensor) -> int:
    if t.dtype not in DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return DTYPES[t.dtype]


def _p(t, dtype=None, host_ok=False):
    """Device pointer of a contiguous CUDA tensor (None -> NULL).  With host_ok, a
    page-locked CPU tensor is accepted too (the device reads it in place)."""
    if t is None:
        return None
    if not t.is_cuda and not (host_ok and t.is_pinned()):
        raise ValueError("the MSA library takes CUDA tensors" + (" or pinned CPU tensors" if host_ok else ""))
    if not t.is_contiguous():
        raise ValueError("the MSA library takes contiguous tensors")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    return t.data_ptr()


def _s(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _call(name: str, *args) -> None:
    st = getattr(_lib.load(), name)(*args)
    if st != 0:
        raise MSAError(name, st)


def version() -> str:
    return _lib.load().msa_version().decode()


def kernel_launch_count() -> int:
    """Kernels the library has launched in this process (msa_kernel_launch_count)."""
    return int(_lib.load().msa_kernel_launch_count())


def testing_set_wait_polls(polls: int) -> None:
    """Test hook (msa_testing_set_wait_polls): polls of the prefill attention kernel's pipeline
    waits; 0 makes every such wait expire at once, a negative value restores the default."""
    _lib.load().msa_testing_set_wait_polls(int(polls))


def rope_table(theta: float, d: int, max_len: int) -> torch.Tensor:
    """Host fp32 [max_len, d/2, 2] table of (cos, sin) built in fp64 by the library."""
    out = torch.empty((max_len, d // 2, 2), dtype=torch.float32)
    _call("msa_rope_table_host", float(theta), d, max_len, out.data_ptr())
    return out


def chunk_offsets(doc_tok_off, P: int):
    """Host int64 [D+1] chunk offsets for host int64 token offsets (msa_chunk_offsets_host)."""
    import numpy as np
    tok = np.ascontiguousarray(np.asarray(doc_tok_off, dtype=np.int64))
    out = np.empty_like(tok)
    _call("msa_chunk_offsets_host", tok.ctypes.data, len(tok) - 1, P, out.ctypes.data)
    return out


def pool(K, V, Kr, doc_tok_off, doc_chunk_off, P, rope_cs, Kbar, Vbar, Krbar, kr_rnorm=None,
         err_flag=None, stream=None):
    """Step 1: RoPE + chunk-mean pooling (msa_pool)."""
    D = doc_tok_off.numel() - 1
    _call("msa_pool", _dt(K), _p(K), _p(V, K.dtype), _p(Kr, K.dtype), _p(doc_tok_off, torch.int64),
          _p(doc_chunk_off, torch.int64), D, K.shape[0], Kbar.shape[0], K.shape[1], K.shape[2],
          Kr.shape[1], Kr.shape[2], P, _p(rope_cs, torch.float32), rope_cs.shape[0],
          _p(Kbar, K.dtype), _p(Vbar, K.dtype), _p(Krbar, K.dtype), _p(kr_rnorm, torch.float32),
          _p(err_flag, torch.int32), _s(stream))


def bank_rnorm(Krbar, kr_rnorm, stream=None):
    _call("msa_bank_rnorm", _dt(Krbar), _p(Krbar), Krbar.shape[0], Krbar.shape[1], Krbar.shape[2],
          _p(kr_rnorm, torch.float32), _s(stream))


def route_topk_workspace_size(B: int, Tq: int, Hr: int, D: int, C: int, k: int) -> int:
    return _lib.load().msa_route_topk_workspace_size(B, Tq, Hr, D, C, k)


def route_topk(Qr, Krbar, kr_rnorm, doc_chunk_off, k, topk_idx, ws, topk_score=None, doc_scores=None,
               err_flag=None, stream=None):
    """Steps 2+3: cosine routing and top-k (msa_route_topk).  Qr [B, Tq, Hr, dr]."""
    B, Tq, Hr, dr = Qr.shape
    _call("msa_route_topk", _dt(Qr), _p(Qr), B, Tq, Hr, dr, _p(Krbar, Qr.dtype), _p(kr_rnorm, torch.float32),
          _p(doc_chunk_off, torch.int64), doc_chunk_off.numel() - 1, Krbar.shape[0], k,
          _p(doc_scores, torch.float32), _p(topk_idx, torch.int32), _p(topk_score, torch.float32),
          _p(ws), ws.numel() * ws.element_size(), _p(err_flag, torch.int32), _s(stream))


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024  # MSA_NOALLOC_SCRATCH_BYTES in msa.h


def route_topk_noalloc(Qr, Krbar, kr_rnorm, doc_chunk_off, k, topk_idx, topk_score=None, doc_scores=None,
                       err_flag=None, stream=None):
    """msa_route_topk_noalloc: route_topk with the library's fixed scratch instead of a workspace.

    For callers that cannot allocate device memory at call time.  Overlapping
    calls on the GPU race on the shared scratch; see include/msa.h.
    """
    B, Tq, Hr, dr = Qr.shape
    _call("msa_route_topk_noalloc", _dt(Qr), _p(Qr), B, Tq, Hr, dr, _p(Krbar, Qr.dtype),
          _p(kr_rnorm, torch.float32), _p(doc_chunk_off, torch.int64), doc_chunk_off.numel() - 1,
          Krbar.shape[0], k, _p(doc_scores, torch.float32), _p(topk_idx, torch.int32),
          _p(topk_score, torch.float32), _p(err_flag, torch.int32), _s(stream))


def gather(topk_idx, doc_chunk_off, Kbar, Vbar, Kmem, Vmem, mem_len, err_flag=None, stream=None):
    """Step 4: copy the selected documents' chunks (msa_gather).  Kmem [B, Mmax, Hkv, d]."""
    B, k = topk_idx.shape
    _call("msa_gather", _dt(Kbar), _p(topk_idx, torch.int32), B, k, _p(doc_chunk_off, torch.int64),
          doc_chunk_off.numel() - 1, Kbar.shape[0], _p(Kbar, host_ok=True), _p(Vbar, Kbar.dtype, host_ok=True),
          Kbar.shape[1],
          Kbar.shape[2], Kmem.shape[1], _p(Kmem, Kbar.dtype), _p(Vmem, Kbar.dtype),
          _p(mem_len, torch.int32), _p(err_flag, torch.int32), _s(stream))


def state_gather_sum(states, topk_idx, S_ext, err_flag=None, stream=None):
    """Linear (DGA) layers' memory injection (msa_state_gather_sum): S_ext[b] = sum of
    the selected documents' recurrent states.  states [D, ...] bf16 or fp32;
    topk_idx int32 [B, k]; S_ext fp32 [B, ...] with the states' trailing shape."""
    D = states.shape[0]
    S = states.numel() // D if D else 0
    B, k = topk_idx.shape
    if S_ext.numel() != B * S:
        raise ValueError("S_ext must hold one state per query")
    _call("msa_state_gather_sum", _dt(states), _p(states), D, S, _p(topk_idx, torch.int32), B, k,
          _p(S_ext, torch.float32), _p(err_flag, torch.int32), _s(stream))


def sparse_attn_workspace_size(B, Tq, Lloc, Hq, Hkv, d, Mmax) -> int:
    return _lib.load().msa_sparse_attn_workspace_size(B, Tq, Lloc, Hq, Hkv, d, Mmax)


def sparse_attn(Q, Kloc, Vloc, Kmem, Vmem, mem_len, O, lse=None, scale=0.0, ws=None, err_flag=None,
                stream=None):
    """Step 5: attention over [memory ++ causal local] (msa_sparse_attn).  Q [B, Tq, Hq, d]."""
    B, Tq, Hq, d = Q.shape
    _call("msa_sparse_attn", _dt(Q), _p(Q), _p(Kloc, Q.dtype), _p(Vloc, Q.dtype), B, Tq, Kloc.shape[1], Hq,
          Kloc.shape[2], d, _p(Kmem, Q.dtype), _p(Vmem, Q.dtype), _p(mem_len, torch.int32), Kmem.shape[1],
          float(scale), _p(O, Q.dtype), _p(lse, torch.float32), _p(ws),
          0 if ws is None else ws.numel() * ws.element_size(), _p(err_flag, torch.int32), _s(stream))


def sparse_attn_indexed_workspace_size(B, Tq, Lloc, Hq, Hkv, d, k, Mmax) -> int:
    return _lib.load().msa_sparse_attn_indexed_workspace_size(B, Tq, Lloc, Hq, Hkv, d, k, Mmax)


def sparse_attn_indexed(Q, Kloc, Vloc, topk_idx, doc_chunk_off, Kbar, Vbar, Mmax, O, ws, lse=None, scale=0.0,
                        err_flag=None, stream=None):
    """Steps 4+5 fused (msa_sparse_attn_indexed): attention over the selected documents' chunks,
    read in place from the bank K̄ / V̄ [C, Hkv, d] by index, and the causal local rows."""
    B, Tq, Hq, d = Q.shape
    k = topk_idx.shape[1]
    _call("msa_sparse_attn_indexed", _dt(Q), _p(Q), _p(Kloc, Q.dtype), _p(Vloc, Q.dtype), B, Tq, Kloc.shape[1], Hq,
          Kloc.shape[2], d, _p(topk_idx, torch.int32), k, _p(doc_chunk_off, torch.int64), doc_chunk_off.numel() - 1,
          Kbar.shape[0], _p(Kbar, Q.dtype, host_ok=True), _p(Vbar, Q.dtype, host_ok=True), Mmax, float(scale),
          _p(O, Q.dtype), _p(lse, torch.float32), _p(ws), ws.numel() * ws.element_size(),
          _p(err_flag, torch.int32), _s(stream))


def sparse_attn_backward_workspace_size(B, Tq, Hq) -> int:
    return _lib.load().msa_sparse_attn_backward_workspace_size(B, Tq, Hq)


def sparse_attn_backward(Q, Kloc, Vloc, Kmem, Vmem, mem_len, O, lse, dO, dQ, dKloc, dVloc, dKmem, dVmem, ws,
                         scale=0.0, err_flag=None, stream=None):
    """Backward of step 5 (msa_sparse_attn_backward): fp32 gradients of Q, Kloc, Vloc, Kmem, Vmem."""
    B, Tq, Hq, d = Q.shape
    f = torch.float32
    _call("msa_sparse_attn_backward", _dt(Q), _p(Q), _p(Kloc, Q.dtype), _p(Vloc, Q.dtype), B, Tq, Kloc.shape[1], Hq,
          Kloc.shape[2], d, _p(Kmem, Q.dtype), _p(Vmem, Q.dtype), _p(mem_len, torch.int32), Kmem.shape[1],
          float(scale), _p(O, Q.dtype), _p(lse, f), _p(dO, Q.dtype), _p(dQ, f), _p(dKloc, f), _p(dVloc, f),
          _p(dKmem, f), _p(dVmem, f), _p(ws), ws.numel() * ws.element_size(), _p(err_flag, torch.int32), _s(stream))


def gather_backward(topk_idx, doc_chunk_off, dKmem, dVmem, mem_len, dKbar, dVbar, err_flag=None, stream=None):
    """Backward of step 4 (msa_gather_backward): adds the gathered rows' gradients into dKbar / dVbar."""
    B, k = topk_idx.shape
    f = torch.float32
    _call("msa_gather_backward", _p(topk_idx, torch.int32), B, k, _p(doc_chunk_off, torch.int64),
          doc_chunk_off.numel() - 1, dKbar.shape[0], _p(dKmem, f), _p(dVmem, f), _p(mem_len, torch.int32),
          dKbar.shape[1], dKbar.shape[2], dKmem.shape[1], _p(dKbar, f), _p(dVbar, f), _p(err_flag, torch.int32),
          _s(stream))


def route_backward_workspace_size(B, Tq, k) -> int:
    return _lib.load().msa_route_backward_workspace_size(B, Tq, k)


def route_backward(Qr, Krbar, kr_rnorm, doc_chunk_off, topk_idx, d_score, dQr, dKrbar, ws, err_flag=None,
                   stream=None):
    """Backward of step 2 (msa_route_backward): adds the selected documents' routing-score gradients
    d_score [B, k] into dQr [B, Tq, Hr, dr] and dKrbar [C, Hr, dr] (fp32)."""
    B, Tq, Hr, dr = Qr.shape
    k = topk_idx.shape[1]
    f = torch.float32
    _call("msa_route_backward", _dt(Qr), _p(Qr), B, Tq, Hr, dr, _p(Krbar, Qr.dtype), _p(kr_rnorm, f),
          _p(doc_chunk_off, torch.int64), doc_chunk_off.numel() - 1, Krbar.shape[0], k,
          _p(topk_idx, torch.int32), _p(d_score, f), _p(dQr, f), _p(dKrbar, f), _p(ws),
          ws.numel() * ws.element_size(), _p(err_flag, torch.int32), _s(stream))


def layer_forward_workspace_size(B, Tq, Lloc, Hq, Hkv, d, Hr, D, C, k, Mmax) -> int:
    return _lib.load().msa_layer_forward_workspace_size(B, Tq, Lloc, Hq, Hkv, d, Hr, D, C, k, Mmax)


def layer_forward(Qr, Krbar, kr_rnorm, doc_chunk_off, k, Q, Kloc, Vloc, Kbar, Vbar, Mmax, O, topk_idx, ws,
                  lse=None, topk_score=None, doc_scores=None, scale=0.0, err_flag=None, stream=None):
    """Steps 2-5 in one call (msa_layer_forward): route + top-k, then attention over the selected
    documents' chunks read in place from the bank by index (msa_sparse_attn_indexed)."""
    B, Tq, Hr, dr = Qr.shape
    Hq, d = Q.shape[2], Q.shape[3]
    _call("msa_layer_forward", _dt(Qr), _p(Qr), Hr, dr, _p(Krbar, Qr.dtype), _p(kr_rnorm, torch.float32),
          _p(doc_chunk_off, torch.int64), doc_chunk_off.numel() - 1, Krbar.shape[0], k,
          _p(Q, Qr.dtype), _p(Kloc, Qr.dtype), _p(Vloc, Qr.dtype), B, Tq, Kloc.shape[1], Hq, Kloc.shape[2], d,
          _p(Kbar, Qr.dtype, host_ok=True), _p(Vbar, Qr.dtype, host_ok=True), Mmax, float(scale), _p(O, Qr.dtype),
          _p(lse, torch.float32),
          _p(topk_idx, torch.int32), _p(topk_score, torch.float32), _p(doc_scores, torch.float32),
          _p(ws), ws.numel() * ws.element_size(), _p(err_flag, torch.int32), _s(stream))


def interleave_workspace_size(B, Tq, Lloc, Hq, Hkv, d, Hr, dr, D, C, k, rounds, Mmax) -> int:
    return _lib.load().msa_interleave_workspace_size(B, Tq, Lloc, Hq, Hkv, d, Hr, dr, D, C, k, rounds, Mmax)


def interleave_forward(Qr0, Krbar, kr_rnorm, doc_chunk_off, k, rounds, W_route, Q, Kloc, Vloc, Kbar, Vbar, Mmax, O,
                       topk_idx, ws, lse=None, O_rounds=None, Qr_rounds=None, topk_score=None, scale=0.0,
                       err_flag=None, stream=None):
    """Memory Interleave (msa_interleave_forward): `rounds` rounds of route -> k new documents ->
    attention over every round's documents; the next round's router query is O_r x W_route.
    topk_idx int32 [B, rounds * k]; W_route [Hq * d, Hr * dr] (None when rounds == 1)."""
    B, Tq, Hr, dr = Qr0.shape
    Hq, d = Q.shape[2], Q.shape[3]
    _call("msa_interleave_forward", _dt(Qr0), _p(Qr0), Hr, dr, _p(Krbar, Qr0.dtype), _p(kr_rnorm, torch.float32),
          _p(doc_chunk_off, torch.int64), doc_chunk_off.numel() - 1, Krbar.shape[0], k, rounds,
          _p(W_route, Qr0.dtype), _p(Q, Qr0.dtype), _p(Kloc, Qr0.dtype), _p(Vloc, Qr0.dtype), B, Tq, Kloc.shape[1],
          Hq, Kloc.shape[2], d, _p(Kbar, Qr0.dtype, host_ok=True), _p(Vbar, Qr0.dtype, host_ok=True), Mmax,
          float(scale), _p(O, Qr0.dtype), _p(lse, torch.float32), _p(O_rounds, Qr0.dtype), _p(Qr_rounds, Qr0.dtype),
          _p(topk_idx, torch.int32), _p(topk_score, torch.float32), _p(ws), ws.numel() * ws.element_size(),
          _p(err_flag, torch.int32), _s(stream))


def gated_delta_rule(q, k, v, g, beta, o, h0=None, hT=None, scale=0.0, stream=None):
    """The linear (DGA) layers' query path (msa_gated_delta_rule): the gated delta rule over the
    query tokens from the initial state h0 (S_ext).  q, k [B, T, Hk, 128]; v, o [B, T, Hv, 128];
    g, beta fp32 [B, T, Hv]; h0, hT fp32 [B, Hv, 128, 128] or None."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    f = torch.float32
    _call("msa_gated_delta_rule", _dt(q), _p(q), _p(k, q.dtype), _p(v, q.dtype), _p(g, f), _p(beta, f), B, T, Hk, Hv,
          dk, dv, _p(h0, f), float(scale), _p(o, q.dtype), _p(hT, f), _s(stream))
