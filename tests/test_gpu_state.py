"""Parity of the linear (DGA) layers' memory injection (msa_state_gather_sum)
against the fp64 oracle: each query's initial state is the sum of its
selected documents' recurrent states ("MSA x Qwen3.5" model card,
"Architecture summary")."""
import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from oracle import msa_oracle as O

from .helpers import TOL_F32_POOL, close_rel, route_on_gpu, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _states(D, shape, dtype, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return torch.randn((D,) + shape, generator=g, device=DEV).to(dtype)


@pytest.mark.parametrize("dtype,D,shape,B,k", [
    (torch.bfloat16, 37, (4, 16, 32), 5, 7),      # k under one batch of loads, repeats allowed
    (torch.bfloat16, 50, (3, 10, 80), 3, 20),     # k over two batches, ragged; 300 vectors: a partial CTA
    (torch.float32, 23, (2, 8, 12), 4, 9),        # fp32 states
    (torch.bfloat16, 64, (16, 64, 64), 2, 16),    # a head-shaped state of 16 x 64 x 64
])
def test_state_gather_sum_matches_oracle(dtype, D, shape, B, k):
    st = _states(D, shape, dtype, seed=D + k)
    rng = np.random.default_rng(D * 7 + k)
    idx = rng.integers(0, D, size=(B, k)).astype(np.int32)
    out = torch.full((B,) + shape, float("nan"), dtype=torch.float32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.state_gather_sum(st, torch.from_numpy(idx).to(DEV), out, err_flag=flag)
    ref = O.state_gather_sum(to64(st), idx)
    torch.cuda.synchronize()
    assert flag.item() == 0
    close_rel(to64(out), ref, TOL_F32_POOL, "S_ext")


def test_state_gather_sum_flags_and_skips_bad_indices():
    D, shape = 12, (2, 4, 8)
    st = _states(D, shape, torch.bfloat16, seed=5)
    idx = np.array([[3, D, 1], [-1, 4, 4]], dtype=np.int32)
    out = torch.empty((2,) + shape, dtype=torch.float32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.state_gather_sum(st, torch.from_numpy(idx).to(DEV), out, err_flag=flag)
    torch.cuda.synchronize()
    assert flag.item() & msa.FLAG_INDEX_OOB
    ref = np.stack([O.state_gather_sum(to64(st), np.array([[3, 1]]))[0],
                    O.state_gather_sum(to64(st), np.array([[4, 4]]))[0]])
    close_rel(to64(out), ref, TOL_F32_POOL, "S_ext without the bad selections")


def test_state_gather_sum_of_a_routed_selection():
    # the selection the routing kernels make, fed straight to the state sum
    D, Hr, dr = 40, 2, 64
    g = torch.Generator(device=DEV).manual_seed(9)
    Krb = torch.randn((D * 3, Hr, dr), generator=g, device=DEV).bfloat16()
    rn = torch.empty((D * 3, Hr), dtype=torch.float32, device=DEV)
    msa.bank_rnorm(Krb, rn)
    coff = np.arange(0, D * 3 + 1, 3, dtype=np.int64)
    Qr = torch.randn((3, 5, Hr, dr), generator=g, device=DEV).bfloat16()
    idx, _, _, rflag = route_on_gpu(Qr, Krb, rn, coff, 6)
    st = _states(D, (4, 32, 16), torch.bfloat16, seed=11)
    out = torch.empty((3, 4, 32, 16), dtype=torch.float32, device=DEV)
    msa.state_gather_sum(st, idx, out, err_flag=rflag)
    torch.cuda.synchronize()
    assert rflag.item() == 0
    close_rel(to64(out), O.state_gather_sum(to64(st), idx.cpu().numpy()), TOL_F32_POOL, "S_ext")
