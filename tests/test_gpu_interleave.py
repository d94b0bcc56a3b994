"""msa_interleave_forward (Memory Interleave: rounds of route -> k new documents ->
attention over every round's documents, the next router query a given linear
map of the round's output) against the fp64 oracle, round by round.

Step by step, as for every bf16 path: round r of the oracle routes with the
router query the GPU stored for that round (checked itself against the
oracle's map of the GPU's previous output, to one bf16 rounding), passes over
the documents the GPU selected in earlier rounds, and attends over the GPU's
union of selections, from the GPU's bank bytes."""
import numpy as np
import pytest
import torch

import routed_sparse_attention_chunk_b200 as msa
from oracle import msa_oracle as O
from workloads import synth

from .helpers import TOL_BF16_ABS, TOL_SCORE_ABS, check_topk, close_abs, pool_on_gpu, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _setup(name, scale, seed=0):
    cfg = synth.get_config(name).scaled(**scale)
    q = synth.gen_query(cfg, 0, DEV, seed)
    K, V, Kr = synth.gen_raw_slab(cfg, 0, cfg.D, DEV, seed, Qr0=q["Qr"][0])
    Kb, Vb, Krb, coff, rn, pflag = pool_on_gpu(cfg, K, V, Kr, synth.doc_tok_offsets(cfg))
    g = torch.Generator(device=DEV).manual_seed(seed + 77)
    W = (torch.randn((cfg.Hq * cfg.d, cfg.Hr * cfg.dr), generator=g, device=DEV) / 64).to(cfg.torch_dtype)
    torch.cuda.synchronize()
    assert pflag.item() == 0
    return cfg, q, Kb, Vb, Krb, coff, rn, W


def _run(cfg, q, Kb, Vb, Krb, rn, coff, W, rounds, Mmax):
    B, D, k = cfg.B, len(coff) - 1, cfg.k
    dt = cfg.torch_dtype
    ws = torch.empty(msa.interleave_workspace_size(B, cfg.Tq, cfg.Lloc, cfg.Hq, cfg.Hkv, cfg.d, cfg.Hr, cfg.dr, D,
                                                   Krb.shape[0], k, rounds, Mmax), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(q["Q"])
    lse = torch.empty((B, cfg.Hq, cfg.Tq), dtype=torch.float32, device=DEV)
    O_r = torch.empty((max(rounds - 1, 1),) + tuple(q["Q"].shape), dtype=dt, device=DEV) if rounds > 1 else None
    Qr_r = torch.empty((max(rounds - 1, 1),) + tuple(q["Qr"].shape), dtype=dt, device=DEV) if rounds > 1 else None
    idx = torch.empty((B, rounds * k), dtype=torch.int32, device=DEV)
    sc = torch.empty((B, rounds * k), dtype=torch.float32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.interleave_forward(q["Qr"], Krb, rn, torch.from_numpy(coff).to(DEV), k, rounds,
                           W if rounds > 1 else None, q["Q"], q["Kloc"], q["Vloc"], Kb, Vb, Mmax, out, idx, ws,
                           lse=lse, O_rounds=O_r, Qr_rounds=Qr_r, topk_score=sc, err_flag=flag)
    torch.cuda.synchronize()
    return out, lse, O_r, Qr_r, idx, sc, int(flag.item())


def test_one_round_is_the_layer():
    cfg, q, Kb, Vb, Krb, coff, rn, W = _setup("1m", dict(D=120, Tq=48, Lloc=80))
    out, lse, _, _, idx, sc, flag = _run(cfg, q, Kb, Vb, Krb, rn, coff, W, 1, cfg.Mmax)
    D = len(coff) - 1
    ws = torch.empty(msa.layer_forward_workspace_size(cfg.B, cfg.Tq, cfg.Lloc, cfg.Hq, cfg.Hkv, cfg.d, cfg.Hr, D,
                                                      Krb.shape[0], cfg.k, cfg.Mmax), dtype=torch.uint8, device=DEV)
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse)
    idx2 = torch.empty((cfg.B, cfg.k), dtype=torch.int32, device=DEV)
    msa.layer_forward(q["Qr"], Krb, rn, torch.from_numpy(coff).to(DEV), cfg.k, q["Q"], q["Kloc"], q["Vloc"], Kb, Vb,
                      cfg.Mmax, out2, idx2, ws, lse2)
    torch.cuda.synchronize()
    assert flag == 0
    assert torch.equal(idx, idx2) and torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("name,scale,rounds", [
    ("1m", dict(D=160, Tq=64, Lloc=96, k=4), 3),                     # prefill rounds
    ("decode16m", dict(D=400, B=8, Lloc=300, k=5, docs_per_slab=0), 2),  # decode rounds, 8 queries
    ("tiny", dict(), 3),                                              # fp32, d = 64 (the gathered path)
])
def test_rounds_match_the_oracle_step_by_step(name, scale, rounds):
    cfg, q, Kb, Vb, Krb, coff, rn, W = _setup(name, scale)
    k = cfg.k
    Mmax = rounds * cfg.Mmax
    out, lse, O_r, Qr_r, idx, sc, flag = _run(cfg, q, Kb, Vb, Krb, rn, coff, W, rounds, Mmax)
    assert flag == 0
    bf16 = cfg.dtype == "bf16"
    gi = idx.cpu().numpy()
    assert all(len(set(row.tolist())) == rounds * k for row in gi), "rounds must select disjoint documents"
    Krb64, Kb64, Vb64 = to64(Krb), to64(Kb), to64(Vb)
    W64 = to64(W)
    outs = [to64(O_r[r]) for r in range(rounds - 1)] + [to64(out)]
    for r in range(rounds):
        if r == 0:
            qr = to64(q["Qr"])
        else:
            qr = to64(Qr_r[r - 1])
            # the stored router query is the oracle's map of the GPU's previous output, rounded once
            want = O.round_query(outs[r - 1], W64, cfg.Hr, cfg.dr)
            if bf16:
                close_abs(qr, O.round_to_bf16(want), 2 ** -7 * np.abs(want).max(), f"Qr of round {r}")
            else:
                close_abs(qr, want, 1e-5 * np.abs(want).max(), f"Qr of round {r}")
        ds = O.exclude_selected(O.route(qr, Krb64, coff), [row[:r * k].tolist() for row in gi])
        tol = TOL_SCORE_ABS if bf16 else 1e-5
        check_topk(gi[:, r * k:(r + 1) * k], to64(sc)[:, r * k:(r + 1) * k], ds, k, tol, f"round {r} top-k")
        Km, Vm, ml = O.gather(gi[:, :(r + 1) * k], coff, Kb64, Vb64, Mmax)
        Oo, lo = O.attention(to64(q["Q"]), to64(q["Kloc"]), to64(q["Vloc"]), Km, Vm, ml)
        close_abs(outs[r], Oo, TOL_BF16_ABS if bf16 else 1e-4, f"O of round {r}")
        if r == rounds - 1:
            close_abs(to64(lse), lo, 2e-3 if bf16 else 1e-4, "lse of the last round")
