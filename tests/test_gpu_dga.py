"""The linear (DGA) layers' query path on the GPU: msa_gated_delta_rule (the
chunked gated delta rule, 64-token chunks) from an initial state, against the
oracle's token-by-token recurrence in fp64 on the same input bytes; and the
whole memory path of those layers (the selected documents' states summed by
msa_state_gather_sum into S_ext, then the rule from S_ext) against the
oracle's dga_query."""
import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from oracle import msa_oracle as O

from .helpers import close_rel, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(B, T, Hk, Hv, dt, seed, with_h0=True):
    g = torch.Generator(device=DEV).manual_seed(seed)
    r = lambda *s: torch.randn(s, generator=g, device=DEV)
    k = r(B, T, Hk, 128)
    k = k / k.norm(dim=-1, keepdim=True)          # the model normalises keys before the rule
    q = r(B, T, Hk, 128) / 128 ** 0.5 * 4
    v = r(B, T, Hv, 128)
    lg = -0.3 * torch.rand((B, T, Hv), generator=g, device=DEV)   # log gates in [-0.3, 0]
    beta = 0.1 + 0.9 * torch.rand((B, T, Hv), generator=g, device=DEV)
    h0 = r(B, Hv, 128, 128) if with_h0 else None
    return q.to(dt), k.to(dt), v.to(dt), lg, beta, h0


def _gpu(q, k, v, lg, beta, h0, scale=0.0):
    B, T, Hk, _ = q.shape
    Hv = v.shape[2]
    o = torch.empty((B, T, Hv, 128), dtype=q.dtype, device=DEV)
    hT = torch.empty((B, Hv, 128, 128), dtype=torch.float32, device=DEV)
    msa.gated_delta_rule(q, k, v, lg, beta, o, h0, hT, scale)
    torch.cuda.synchronize()
    return o, hT


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,T,Hk,Hv", [(2, 150, 2, 4),    # three chunks, the last one ragged (22 tokens)
                                       (1, 64, 1, 1),     # exactly one chunk
                                       (3, 1, 2, 2),      # one decode token (the token-by-token kernel)
                                       (2, 16, 2, 4),     # the token-by-token kernel's longest sequence
                                       (1, 17, 1, 2),     # one token more: a single ragged chunk
                                       (1, 1000, 1, 2)])  # sixteen chunks
def test_chunked_rule_matches_the_recurrence(dt, B, T, Hk, Hv):
    q, k, v, lg, beta, h0 = _inputs(B, T, Hk, Hv, dt, seed=T + Hv)
    o, hT = _gpu(q, k, v, lg, beta, h0)
    oo, oh = O.gated_delta_rule(to64(q), to64(k), to64(v), to64(lg), to64(beta), to64(h0), scale=128 ** -0.5)
    close_rel(to64(hT), oh, 1e-4, "state after the last token")
    close_rel(to64(o), oo, 1e-4 if dt == torch.float32 else 8e-3, "outputs")


def test_zero_initial_state_and_explicit_scale():
    q, k, v, lg, beta, _ = _inputs(1, 90, 2, 2, torch.bfloat16, seed=3, with_h0=False)
    o, hT = _gpu(q, k, v, lg, beta, None, scale=0.25)
    oo, oh = O.gated_delta_rule(to64(q), to64(k), to64(v), to64(lg), to64(beta), None, scale=0.25)
    close_rel(to64(hT), oh, 1e-4, "state")
    close_rel(to64(o), oo, 8e-3, "outputs")


def test_dga_memory_path_from_the_selected_documents_states():
    """S_ext = the sum of each query's selected documents' states (msa_state_gather_sum, states laid
    out [Hv, dk, dv]), then the rule over the query tokens from S_ext (msa_gated_delta_rule)."""
    B, T, Hk, Hv, D, kk = 2, 100, 1, 2, 40, 6
    g = torch.Generator(device=DEV).manual_seed(21)
    states = (0.3 * torch.randn((D, Hv, 128, 128), generator=g, device=DEV)).bfloat16()
    idx = torch.stack([torch.randperm(D, generator=g, device=DEV)[:kk] for _ in range(B)]).to(torch.int32)
    S_ext = torch.empty((B, Hv, 128, 128), dtype=torch.float32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.state_gather_sum(states, idx, S_ext, err_flag=flag)
    q, k, v, lg, beta, _ = _inputs(B, T, Hk, Hv, torch.bfloat16, seed=22, with_h0=False)
    o, hT = _gpu(q, k, v, lg, beta, S_ext)
    assert flag.item() == 0
    oo, oh = O.dga_query(to64(states), idx.cpu().numpy(), to64(q), to64(k), to64(v), to64(lg), to64(beta),
                         scale=128 ** -0.5)
    close_rel(to64(hT), oh, 1e-4, "state")
    close_rel(to64(o), oo, 8e-3, "outputs")
