"""The device-side error path of a tensor-core kernel: every pipeline wait of the
prefill attention kernel made to run out (a test-only poll limit of 0), so the
call must drain its own copies and tensor-core work, free its tensor memory,
report MSA_FLAG_TIMEOUT and return -- with no fault and no wait left open, and
with the next call, at the default limit, correct."""
import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from oracle import msa_oracle as O

from .helpers import TOL_BF16_ABS, attn_on_gpu, close_abs, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("Tq", [128, 24])  # four blocks of rows per KV head; one ragged block
def test_expired_waits_raise_the_timeout_flag_and_the_next_call_is_correct(Tq):
    g = torch.Generator(device=DEV).manual_seed(5)
    B, Lloc, Hq, Hkv, M = 1, 256, 32, 8, 64
    r = lambda *s: (0.5 * torch.randn(s, generator=g, device=DEV)).bfloat16()
    Q, Kl, Vl, Km, Vm = r(B, Tq, Hq, 128), r(B, Lloc, Hkv, 128), r(B, Lloc, Hkv, 128), r(B, M, Hkv, 128), \
        r(B, M, Hkv, 128)
    ml = torch.full((B,), M, dtype=torch.int32, device=DEV)
    try:
        msa.testing_set_wait_polls(0)
        _, _, flag = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
        torch.cuda.synchronize()
    finally:
        msa.testing_set_wait_polls(-1)
    assert flag.item() & msa.FLAG_TIMEOUT
    out, lse, flag2 = attn_on_gpu(Q, Kl, Vl, Km, Vm, ml)
    torch.cuda.synchronize()
    assert flag2.item() == 0
    Oo, lo = O.attention(to64(Q), to64(Kl), to64(Vl), to64(Km), to64(Vm), np.array([M]))
    close_abs(to64(out), Oo, TOL_BF16_ABS, "O after the expired call")
