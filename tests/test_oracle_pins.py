"""Pins for the fp64 oracle: closed forms, textbook cases, a library routine, brute force.

None of these re-types an oracle formula: each checks the oracle against a fact
that the pages or the mathematics fix independently of how the oracle computes it.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.spatial.distance as ssd
import torch
import torch.nn.functional as F

from oracle import msa_oracle as O
from workloads import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def load_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rest = line.split("=", 1)
            vals[key.strip()] = np.array([float(x) for x in rest.split()])
    return vals


# ------------------------------------------------------------------ bf16 rounding
def _bf16_decode(bits):
    """Value of a bf16 bit pattern from the format's definition (1 / 8 / 7 bits)."""
    s = (bits >> 15) & 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0:
        v = m * 2.0 ** (-133)
    else:
        v = (1 + m / 128.0) * 2.0 ** (e - 127)
    return -v if s else v


def test_bf16_rounding_fixed_points_and_midpoints():
    finite = [b for b in range(0x0000, 0x7F80)]  # every non-negative finite pattern
    vals = np.array([_bf16_decode(b) for b in finite])
    assert np.array_equal(O.round_to_bf16(vals), vals)
    assert np.array_equal(O.round_to_bf16(-vals), -vals)
    lo, hi = vals[:-1], vals[1:]
    mid = (lo + hi) / 2
    even = np.array([(b & 1) == 0 for b in finite[:-1]])
    expect = np.where(even, lo, hi)
    assert np.array_equal(O.round_to_bf16(mid), expect)
    gap = hi - lo
    assert np.array_equal(O.round_to_bf16(mid - gap * 1e-3), lo)
    assert np.array_equal(O.round_to_bf16(mid + gap * 1e-3), hi)


# ------------------------------------------------------------------ RoPE
def test_rope_position_zero_is_identity():
    x = rng.standard_normal((5, 3, 16))
    assert np.array_equal(O.rope_rotate(x, np.zeros(5, int), 1e6), x)


def test_rope_keeps_pair_lengths():
    x = rng.standard_normal((7, 2, 32))
    y = O.rope_rotate(x, np.arange(7) * 37, 1e4)
    n = lambda a: a[..., :16] ** 2 + a[..., 16:] ** 2
    np.testing.assert_allclose(n(y), n(x), rtol=1e-12)


def test_rope_relative_position_identity():
    d = 64
    q, k = rng.standard_normal((1, 1, d)), rng.standard_normal((1, 1, d))
    for m, n in [(5, 3), (100, 7), (511, 510), (9, 0)]:
        lhs = np.sum(O.rope_rotate(q, [m], 1e6) * O.rope_rotate(k, [n], 1e6))
        rhs = np.sum(O.rope_rotate(q, [m - n], 1e6) * k)
        assert abs(lhs - rhs) < 1e-10


def test_rope_quarter_turn_by_hand():
    g = load_golden("rope_quarter_turn.txt")
    theta = float(g["theta"][0])
    x = g["x"].reshape(1, 1, 4)
    y = O.rope_rotate(x, [1], theta)[0, 0]
    np.testing.assert_allclose(y, g["expected"], atol=1e-12)


def test_document_positions_restart():
    off = np.array([0, 3, 3, 8])
    assert O.doc_positions(off).tolist() == [0, 1, 2, 0, 1, 2, 3, 4]


# ------------------------------------------------------------------ pooling
def _ragged_offsets():
    return np.array([0, 500, 1000, 1064, 1065, 1200], dtype=np.int64)


def test_chunk_offsets_ceil():
    off = _ragged_offsets()
    assert O.chunk_offsets(off, 64).tolist() == [0, 8, 16, 17, 18, 21]


def test_pool_constant_input_pools_to_itself():
    off = _ragged_offsets()
    n = int(off[-1])
    c = rng.standard_normal((1, 2, 8))
    V = np.repeat(c, n, axis=0)
    Kz = np.zeros((n, 2, 8))
    Kb, Vb, Krb, _, _ = O.pool(Kz, V, V, off, 64, 1e6)
    np.testing.assert_allclose(Vb, np.repeat(c, len(Vb), 0), rtol=1e-14)
    np.testing.assert_allclose(Krb, np.repeat(c, len(Vb), 0), rtol=1e-14)


def test_pool_ramp_mean_closed_form_and_tail():
    off = _ragged_offsets()
    n = int(off[-1])
    ranges = O.chunk_token_ranges(off, 64)
    V = np.zeros((n, 1, 4))
    for s, e, _ in ranges:
        V[s:e, 0, :] = np.arange(e - s)[:, None]      # 0, 1, ..., |c|-1 inside each chunk
    _, Vb, _, _, _ = O.pool(np.zeros_like(V), V, V, off, 64, 1e6)
    expect = np.array([(e - s - 1) / 2 for s, e, _ in ranges])
    np.testing.assert_allclose(Vb[:, 0, 0], expect, rtol=1e-14)
    # document 0 has 500 tokens: 7 full chunks and a 52-token tail averaging 0..51
    assert ranges[7][1] - ranges[7][0] == 52 and Vb[7, 0, 0] == 25.5


def test_pool_is_linear():
    off = _ragged_offsets()
    n = int(off[-1])
    X = [rng.standard_normal((n, 2, 8)) for _ in range(6)]
    a, b = 0.7, -1.9
    P1 = O.pool(X[0], X[1], X[2], off, 64, 1e6)
    P2 = O.pool(X[3], X[4], X[5], off, 64, 1e6)
    P3 = O.pool(a * X[0] + b * X[3], a * X[1] + b * X[4], a * X[2] + b * X[5], off, 64, 1e6)
    for i in range(3):
        np.testing.assert_allclose(P3[i], a * P1[i] + b * P2[i], atol=1e-12)


def test_pool_rotates_k_at_document_local_positions():
    # With P = 1 each chunk is one token: K̄ is that token rotated at its position
    # inside its own document, V̄ and K̄r are not rotated.
    off = np.array([0, 3, 7])
    K = rng.standard_normal((7, 2, 8))
    Kb, Vb, Krb, _, _ = O.pool(K, K, K, off, 1, 10.0)
    np.testing.assert_array_equal(Vb, K)
    np.testing.assert_array_equal(Krb, K)
    for t, p in enumerate([0, 1, 2, 0, 1, 2, 3]):
        ang = p * 10.0 ** (-2 * np.arange(4) / 8)
        lo, hi = K[t, :, :4], K[t, :, 4:]
        exp = np.concatenate([lo * np.cos(ang) - hi * np.sin(ang), hi * np.cos(ang) + lo * np.sin(ang)], -1)
        np.testing.assert_allclose(Kb[t], exp, atol=1e-12)


def test_pool_rnorm_is_inverse_norm_of_stored_bank():
    off = np.array([0, 64, 130])
    X = rng.standard_normal((130, 3, 16))
    _, _, Krb, _, rn = O.pool(X, X, X, off, 64, 1e6, out_bf16=True)
    assert np.array_equal(O.round_to_bf16(Krb), Krb)
    for c in range(Krb.shape[0]):
        for h in range(3):
            assert abs(rn[c, h] * math.sqrt(sum(v * v for v in Krb[c, h])) - 1) < 1e-13


# ------------------------------------------------------------------ cosine routing
def test_cosine_in_range_and_textbook_for_one_head():
    Qr = rng.standard_normal((2, 5, 1, 12))
    Kb = rng.standard_normal((9, 1, 12))
    s = O.cosine_scores(Qr, Kb)
    assert np.all(np.abs(s) <= 1 + 1e-15)
    for b, t, c in itertools.product(range(2), range(5), range(9)):
        assert abs(s[b, t, c] - (1 - ssd.cosine(Qr[b, t, 0], Kb[c, 0]))) < 1e-12


def test_cosine_identical_negated_and_scale_invariant():
    Kb = rng.standard_normal((4, 3, 16))
    Qr = np.stack([Kb[2], -Kb[1]])[None]                  # [1, 2, 3, 16]
    s = O.cosine_scores(Qr, Kb)
    assert abs(s[0, 0, 2] - 1) < 1e-14 and abs(s[0, 1, 1] + 1) < 1e-14
    s2 = O.cosine_scores(3.7 * Qr, 0.2 * Kb)
    np.testing.assert_allclose(s2, s, atol=1e-14)


def test_head_mean_then_token_max_hand_case():
    g = load_golden("route_hand_case.txt")
    Qr = g["Qr"].reshape(1, 2, 2, 2)
    Kb = g["Krbar"].reshape(1, 2, 2)
    ds = O.route(Qr, Kb, np.array([0, 1]))
    assert abs(ds[0, 0] - g["doc_score"][0]) < 1e-12
    assert abs(ds[0, 0] - g["max_then_mean"][0]) > 0.2   # the other order gives a different number


def test_document_score_is_max_over_its_chunks():
    Kb = rng.standard_normal((6, 2, 8))
    Qr = rng.standard_normal((1, 3, 2, 8))
    off = np.array([0, 2, 2, 6])                          # doc 1 is empty
    ds = O.route(Qr, Kb, off)
    per_chunk = [max(np.mean([1 - ssd.cosine(Qr[0, t, h], Kb[c, h]) for h in range(2)])
                     for t in range(3)) for c in range(6)]
    assert abs(ds[0, 0] - max(per_chunk[0:2])) < 1e-12
    assert ds[0, 1] == -np.inf
    assert abs(ds[0, 2] - max(per_chunk[2:6])) < 1e-12


def test_planted_document_scores_one_and_is_selected():
    cfg = synth.get_config("tiny")
    q = synth.gen_query(cfg)
    K, V, Kr = synth.gen_raw_slab(cfg, 0, cfg.D, Qr0=q["Qr"][0])
    off = synth.doc_tok_offsets(cfg)
    _, _, Krb, coff, _ = O.pool(K.numpy(), V.numpy(), Kr.numpy(), off, cfg.P, cfg.theta)
    ds = O.route(q["Qr"].numpy(), Krb, coff)
    assert abs(ds[0, 17] - 1.0) < 1e-12
    assert ds[0].max() == ds[0, 17]
    idx, _ = O.topk(ds, cfg.k)
    assert idx[0, 0] == 17


# ------------------------------------------------------------------ top-k
@pytest.mark.parametrize("D,k", [(5, 1), (6, 2), (9, 3), (12, 3)])
def test_topk_equals_bruteforce(D, k):
    for trial in range(20):
        row = rng.integers(-4, 5, size=D).astype(float) if trial % 2 else rng.standard_normal(D)
        idx, val = O.topk(row[None], k)
        assert list(idx[0]) == O.topk_bruteforce(row, k)
        assert np.array_equal(val[0], row[idx[0]])


def test_topk_sorted_and_ties_prefer_lower_index():
    row = np.array([0.5, 0.9, 0.5, 0.9, 0.1, 0.5])
    idx, _ = O.topk(row[None], 4)
    assert idx[0].tolist() == [1, 3, 0, 2]
    full = np.lexsort((np.arange(6), -row))
    assert idx[0].tolist() == full[:4].tolist()


# ------------------------------------------------------------------ gather
def test_gather_copies_selected_chunks_in_rank_order():
    off = np.array([0, 3, 4, 4, 9])
    Kb = rng.standard_normal((9, 2, 4))
    Vb = rng.standard_normal((9, 2, 4))
    Km, Vm, ml = O.gather(np.array([[3, 0, 2], [1, 3, 0]]), off, Kb, Vb, 10)
    assert ml.tolist() == [8, 9]
    assert np.array_equal(Km[0, :8], Kb[[4, 5, 6, 7, 8, 0, 1, 2]])
    assert np.array_equal(Vm[1, :9], Vb[[3, 4, 5, 6, 7, 8, 0, 1, 2]])
    assert not Km[0, 8:].any()


# ------------------------------------------------------------------ attention
def _sdpa(Q, K, V, mask, scale):
    """torch's fp64 CPU scaled_dot_product_attention as the independent routine. Q [Tq,H,d]."""
    q = torch.from_numpy(Q).permute(1, 0, 2)[None]
    k = torch.from_numpy(K).permute(1, 0, 2)[None]
    v = torch.from_numpy(V).permute(1, 0, 2)[None]
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(mask),
                                       scale=scale, enable_gqa=q.shape[1] != k.shape[1])
    return o[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("Tq,Lloc,M,Hq,Hkv", [(7, 7, 0, 4, 2), (5, 11, 0, 2, 2), (6, 9, 13, 8, 2), (1, 20, 4, 4, 1)])
def test_attention_matches_sdpa(Tq, Lloc, M, Hq, Hkv):
    d = 16
    Q = rng.standard_normal((1, Tq, Hq, d))
    Kl, Vl = rng.standard_normal((2, 1, Lloc, Hkv, d))
    Km, Vm = rng.standard_normal((2, 1, M + 3, Hkv, d))   # 3 pad rows past mem_len
    Oo, lse = O.attention(Q, Kl, Vl, Km, Vm, [M])
    pos = Lloc - Tq + np.arange(Tq)
    mask = np.concatenate([np.ones((Tq, M), bool), np.arange(Lloc)[None] <= pos[:, None]], 1)
    ref = _sdpa(Q[0], np.concatenate([Km[0, :M], Kl[0]]), np.concatenate([Vm[0, :M], Vl[0]]),
                mask, 1 / math.sqrt(d))
    np.testing.assert_allclose(Oo[0], ref, atol=1e-12)


def test_attention_no_memory_is_plain_causal_attention():
    Q = rng.standard_normal((1, 9, 2, 8))
    Kl, Vl = rng.standard_normal((2, 1, 9, 2, 8))
    Oo, _ = O.attention(Q, Kl, Vl, np.zeros((1, 4, 2, 8)), np.zeros((1, 4, 2, 8)), [0])
    q = torch.from_numpy(Q[0]).permute(1, 0, 2)
    ref = F.scaled_dot_product_attention(q, torch.from_numpy(Kl[0]).permute(1, 0, 2),
                                         torch.from_numpy(Vl[0]).permute(1, 0, 2), is_causal=True)
    np.testing.assert_allclose(Oo[0], ref.permute(1, 0, 2).numpy(), atol=1e-12)


def test_attention_identical_keys_give_mean_of_values_and_weights_sum_to_one():
    Tq, Lloc, M, d = 4, 6, 5, 8
    key = rng.standard_normal(d)
    Kl = np.broadcast_to(key, (1, Lloc, 1, d)).copy()
    Km = np.broadcast_to(key, (1, M, 1, d)).copy()
    Vl, Vm = rng.standard_normal((1, Lloc, 1, d)), rng.standard_normal((1, M, 1, d))
    Q = rng.standard_normal((1, Tq, 2, d))
    Oo, lse = O.attention(Q, Kl, Vl, Km, Vm, [M])
    for i in range(Tq):
        vis = np.concatenate([Vm[0, :, 0], Vl[0, : Lloc - Tq + i + 1, 0]])
        np.testing.assert_allclose(Oo[0, i, 0], vis.mean(0), atol=1e-12)
        # equal logits: the normaliser is logit + log(number of visible keys)
        logit = Q[0, i, 1] @ key / math.sqrt(d)
        assert abs(lse[0, 1, i] - (logit + math.log(len(vis)))) < 1e-12


def test_attention_hand_case():
    g = load_golden("attention_hand_case.txt")
    d = 2
    Q = g["q"].reshape(1, 1, 1, d)
    Kl = g["k_local"].reshape(1, 1, 1, d)
    Vl = g["v_local"].reshape(1, 1, 1, d)
    Km = g["k_mem"].reshape(1, 1, 1, d)
    Vm = g["v_mem"].reshape(1, 1, 1, d)
    Oo, _ = O.attention(Q, Kl, Vl, Km, Vm, [1], scale=1.0)
    np.testing.assert_allclose(Oo[0, 0, 0], g["out"], atol=1e-12)


# ------------------------------------------------------------------ composed layer
def test_layer_with_all_documents_is_dense_attention_over_bank():
    cfg = synth.get_config("tiny").scaled(D=6, L=100, k=6)
    q = synth.gen_query(cfg)
    K, V, Kr = synth.gen_raw_slab(cfg, 0, cfg.D, Qr0=q["Qr"][0])
    off = synth.doc_tok_offsets(cfg)
    Kb, Vb, Krb, coff, _ = O.pool(K.numpy(), V.numpy(), Kr.numpy(), off, cfg.P, cfg.theta)
    r = O.layer_forward(q["Qr"].numpy(), Krb, coff, cfg.k, q["Q"].numpy(), q["Kloc"].numpy(),
                        q["Vloc"].numpy(), Kb, Vb, Mmax=int(coff[-1]))
    assert r["mem_len"][0] == coff[-1]
    # attention is invariant to the order of the (unmasked) memory rows: compare with
    # dense attention over the whole bank in natural order
    Od, _ = O.attention(q["Q"].numpy(), q["Kloc"].numpy(), q["Vloc"].numpy(), Kb[None], Vb[None],
                        [int(coff[-1])])
    np.testing.assert_allclose(r["O"], Od, atol=1e-12)


# ---------------------------------------------------------------- backward of steps 5 and 4
def _fd_case(seed=0):
    rng = np.random.default_rng(seed)
    B, Tq, Lloc, Hq, Hkv, d, Mmax = 2, 3, 5, 4, 2, 4, 3
    Q = rng.standard_normal((B, Tq, Hq, d))
    Kl, Vl = rng.standard_normal((B, Lloc, Hkv, d)), rng.standard_normal((B, Lloc, Hkv, d))
    Km, Vm = rng.standard_normal((B, Mmax, Hkv, d)), rng.standard_normal((B, Mmax, Hkv, d))
    ml = np.array([3, 1])
    dO = rng.standard_normal((B, Tq, Hq, d))
    return [Q, Kl, Vl, Km, Vm], ml, dO


def test_attention_backward_matches_central_differences():
    """Every input element: d<dO, O>/dx by central differences of the forward oracle."""
    xs, ml, dO = _fd_case()
    grads = O.attention_backward(*xs, ml, dO)

    def loss(ys):
        return float((O.attention(*ys, ml)[0] * dO).sum())

    eps = 1e-6
    for which, (x, gx) in enumerate(zip(xs, grads)):
        num = np.zeros_like(x)
        for i in np.ndindex(x.shape):
            keep = x[i]
            x[i] = keep + eps
            up = loss(xs)
            x[i] = keep - eps
            dn = loss(xs)
            x[i] = keep
            num[i] = (up - dn) / (2 * eps)
        assert np.allclose(gx, num, atol=1e-7, rtol=1e-6), which


def test_attention_backward_unseen_keys_get_no_gradient():
    xs, ml, dO = _fd_case(1)
    dQ, dKl, dVl, dKm, dVm = O.attention_backward(*xs, ml, dO)
    # memory rows past mem_len and, with Lloc - Tq = 2, local rows 3 and 4 only
    # for later tokens: row 4 is seen by the last token alone
    assert not dKm[1, 1:].any() and not dVm[1, 1:].any()
    xs[0][:, -1] = 0.0
    dO[:, -1] = 0.0   # the last token contributes nothing, so local row 4 gets nothing
    _, dKl, dVl, _, _ = O.attention_backward(*xs, ml, dO)
    assert not dKl[:, 4].any() and not dVl[:, 4].any()


def test_gather_backward_is_the_adjoint_of_gather():
    rng = np.random.default_rng(7)
    off = np.array([0, 2, 2, 5, 6, 9])          # documents of 2, 0, 3, 1, 3 chunks
    C, Hkv, d, Mmax = 9, 2, 3, 8
    idx = np.array([[2, 0, 4], [4, 3, 2], [1, 0, 3]])
    Kb, Vb = rng.standard_normal((C, Hkv, d)), rng.standard_normal((C, Hkv, d))
    Km, Vm, ml = O.gather(idx, off, Kb, Vb, Mmax)
    yK, yV = rng.standard_normal(Km.shape), rng.standard_normal(Vm.shape)
    for b in range(3):
        yK[b, ml[b]:] = 0.0
        yV[b, ml[b]:] = 0.0
    gK, gV = O.gather_backward(idx, off, yK, yV, ml, C)
    assert math.isclose((Km * yK).sum(), (Kb * gK).sum(), rel_tol=1e-12)
    assert math.isclose((Vm * yV).sum(), (Vb * gV).sum(), rel_tol=1e-12)
    # chunk 6..8 (document 4) is selected by queries 0 and 1: both gradients land
    assert np.allclose(gK[6], yK[0, 5] + yK[1, 0])


def test_route_backward_matches_central_differences():
    """d/dx of sum_r g[b, r] * score(b, topk[b, r]) by central differences (distinct maxima)."""
    rng = np.random.default_rng(11)
    B, Tq, Hr, dr = 2, 3, 2, 4
    off = np.array([0, 2, 3, 6, 6, 8])                 # documents of 2, 1, 3, 0, 2 chunks
    C = int(off[-1])
    Qr = rng.standard_normal((B, Tq, Hr, dr))
    Kb = rng.standard_normal((C, Hr, dr))
    idx = np.array([[2, 0, 3], [4, 1, 2]])            # document 3 is empty: no gradient from it
    g = rng.standard_normal((B, 3))
    dQ, dK = O.route_backward(Qr, Kb, off, idx, g)

    def loss(q, k):
        sc = O.route(q, k, off)
        return float(sum(g[b, r] * sc[b, j] for b in range(B) for r, j in enumerate(idx[b]) if np.isfinite(sc[b, j])))

    eps = 1e-6
    for x, gx, args in ((Qr, dQ, 0), (Kb, dK, 1)):
        num = np.zeros_like(x)
        for i in np.ndindex(x.shape):
            keep = x[i]
            x[i] = keep + eps
            up = loss(Qr, Kb)
            x[i] = keep - eps
            dn = loss(Qr, Kb)
            x[i] = keep
            num[i] = (up - dn) / (2 * eps)
        assert np.allclose(gx, num, atol=1e-7, rtol=1e-6), args
    # only the argmax token of each selected document is touched
    assert np.count_nonzero(np.abs(dQ).sum(axis=(2, 3))) <= 2 * 2


# ---------------------------------------------------------------- DGA state injection (reading R16)
def test_state_gather_sum_single_selection_returns_the_state():
    rng = np.random.default_rng(21)
    st = rng.standard_normal((7, 2, 3, 4))
    out = O.state_gather_sum(st, np.array([[5], [0], [6]]))
    assert np.array_equal(out[0], st[5]) and np.array_equal(out[1], st[0]) and np.array_equal(out[2], st[6])


def test_state_gather_sum_one_hot_states_count_selections():
    D = 6
    st = np.eye(D).reshape(D, D)                   # document j's state is the unit vector e_j
    idx = np.array([[3, 1, 3, 5], [0, 0, 0, 2]])     # repeats count twice / three times
    out = O.state_gather_sum(st, idx)
    assert np.array_equal(out[0], [0, 1, 0, 2, 0, 1])
    assert np.array_equal(out[1], [3, 0, 1, 0, 0, 0])


def test_state_gather_sum_order_invariant_linear_and_total():
    rng = np.random.default_rng(22)
    D = 9
    st = rng.standard_normal((D, 5, 3))
    idx = np.array([[4, 2, 7], [1, 8, 0]])
    a = O.state_gather_sum(st, idx)
    assert np.allclose(a, O.state_gather_sum(st, idx[:, ::-1]), rtol=0, atol=1e-12)
    assert np.allclose(O.state_gather_sum(2.5 * st, idx), 2.5 * a, rtol=1e-14, atol=0)
    every = O.state_gather_sum(st, np.arange(D)[None, :])
    assert np.allclose(every[0], np.sum(st, axis=0), rtol=1e-14, atol=1e-14)
    with pytest.raises(ValueError):
        O.state_gather_sum(st, np.array([[D]]))


# ------------------------------------------------------------------ Memory Interleave (reading R17)
def _interleave_case(seed, D=12, Tq=3, Lloc=5, Hq=4, Hkv=2, d=8, Hr=2, dr=8):
    r = np.random.default_rng(seed)
    n = r.integers(1, 4, size=D)
    coff = np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
    C = int(coff[-1])
    return dict(
        Qr0=r.standard_normal((1, Tq, Hr, dr)), Krbar=r.standard_normal((C, Hr, dr)), coff=coff,
        Q=r.standard_normal((1, Tq, Hq, d)), Kloc=r.standard_normal((1, Lloc, Hkv, d)),
        Vloc=r.standard_normal((1, Lloc, Hkv, d)), Kbar=r.standard_normal((C, Hkv, d)),
        Vbar=r.standard_normal((C, Hkv, d)), W=r.standard_normal((Hq * d, Hr * dr)), n=n)


def _run_interleave(c, k, rounds, W=None, Mmax=None):
    return O.interleave(c["Qr0"], c["Krbar"], c["coff"], k, rounds, c["W"] if W is None else W, c["Q"], c["Kloc"],
                        c["Vloc"], c["Kbar"], c["Vbar"], Mmax or int(c["n"].sum()))


def test_interleave_one_round_is_the_layer():
    c = _interleave_case(1)
    a = _run_interleave(c, 3, 1)
    b = O.layer_forward(c["Qr0"], c["Krbar"], c["coff"], 3, c["Q"], c["Kloc"], c["Vloc"], c["Kbar"], c["Vbar"],
                        int(c["n"].sum()))
    assert np.array_equal(a["topk_idx"], b["topk_idx"])
    assert np.array_equal(a["O"], b["O"]) and np.array_equal(a["lse"], b["lse"])


def test_interleave_zero_map_selects_lowest_free_documents():
    # with W = 0 every later router query is zero, every cosine is 0 (norm floor), all
    # documents tie and the tie rule takes the lowest-index documents not yet selected
    c = _interleave_case(2, D=14)
    k, R = 3, 4
    res = _run_interleave(c, k, R, W=np.zeros_like(c["W"]))
    sel = res["topk_idx"][0]
    taken = set(sel[:k].tolist())
    for r in range(1, R):
        free = [j for j in range(14) if j not in taken]
        assert sel[r * k:(r + 1) * k].tolist() == free[:k]
        taken |= set(free[:k])
        assert np.all(res["topk_score"][0, r * k:(r + 1) * k] == 0.0)


def test_interleave_rounds_match_bruteforce_over_free_documents():
    # each round's selection is the best k-subset (largest score sum, then lower indices)
    # among the documents no earlier round took, by enumeration
    c = _interleave_case(3, D=9)
    k, R = 2, 3
    res = _run_interleave(c, k, R)
    sel = res["topk_idx"][0]
    assert len(set(sel.tolist())) == R * k, "rounds must select disjoint documents"
    taken = []
    for r in range(R):
        sc = O.route(res["Qr_rounds"][r], c["Krbar"], c["coff"])[0]
        free = [j for j in range(9) if j not in taken]
        best = max(itertools.combinations(free, k), key=lambda sub: (sum(sc[j] for j in sub), [-j for j in sub]))
        assert sorted(sel[r * k:(r + 1) * k].tolist()) == sorted(best)
        taken += sel[r * k:(r + 1) * k].tolist()


def test_round_query_one_hot_map_and_linearity():
    r = np.random.default_rng(4)
    B, Tq, Hq, d, Hr, dr = 2, 3, 2, 4, 3, 2
    Op = r.standard_normal((B, Tq, Hq, d))
    W = np.zeros((Hq * d, Hr * dr))
    W[5, 3] = 1.0   # output component (head 1, dim 1) -> router component (head 1, dim 1)
    W[2, 0] = 2.0   # (head 0, dim 2) -> twice into (head 0, dim 0)
    q = O.round_query(Op, W, Hr, dr)
    assert q.shape == (B, Tq, Hr, dr)
    np.testing.assert_array_equal(q[:, :, 1, 1], Op[:, :, 1, 1])
    np.testing.assert_array_equal(q[:, :, 0, 0], 2.0 * Op[:, :, 0, 2])
    assert np.count_nonzero(q) == np.count_nonzero(Op[:, :, 1, 1]) + np.count_nonzero(Op[:, :, 0, 2])
    W2 = r.standard_normal(W.shape)
    np.testing.assert_allclose(O.round_query(Op, 3 * W - W2, Hr, dr),
                               3 * O.round_query(Op, W, Hr, dr) - O.round_query(Op, W2, Hr, dr), atol=1e-12)


def test_interleave_attends_over_the_union_of_rounds():
    # Q = 0 makes every visible key weigh the same; each document's value rows are its
    # one-hot id and the local values are zero, so round r's output counts the chunks of
    # every document selected up to round r: n_j / (memory rows + visible local rows)
    D, k, R, Tq, Lloc = 10, 2, 3, 2, 3
    c = _interleave_case(5, D=D, Tq=Tq, Lloc=Lloc, Hq=2, Hkv=1, d=16)
    c["Q"] = np.zeros_like(c["Q"])
    c["Vloc"] = np.zeros_like(c["Vloc"])
    doc_of_chunk = np.repeat(np.arange(D), c["n"])
    c["Vbar"] = np.zeros_like(c["Vbar"])
    c["Vbar"][np.arange(len(doc_of_chunk)), 0, doc_of_chunk] = 1.0
    res = _run_interleave(c, k, R)
    sel = res["topk_idx"][0]
    for r in range(R):
        union = sel[:(r + 1) * k]
        M = int(c["n"][union].sum())
        for t in range(Tq):
            vis = M + (Lloc - Tq + t) + 1
            want = np.zeros(16)
            want[union] = c["n"][union] / vis
            for h in range(2):
                np.testing.assert_allclose(res["O_rounds"][r][0, t, h], want, atol=1e-12)


# ------------------------------------------------------------------ gated delta rule (reading R18)
def _gdr_case(seed, B=1, T=9, Hk=1, Hv=1, dk=6, dv=6, unit_keys=True):
    r = np.random.default_rng(seed)
    k = r.standard_normal((B, T, Hk, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    return dict(q=r.standard_normal((B, T, Hk, dk)), k=k, v=r.standard_normal((B, T, Hv, dv)),
                g=-r.uniform(0.0, 0.3, (B, T, Hv)), beta=r.uniform(0.1, 1.0, (B, T, Hv)),
                h0=r.standard_normal((B, Hv, dk, dv)))


def test_gdr_zero_write_strength_decays_the_initial_state():
    # beta = 0: nothing is written, h_t = exp(g_1 + ... + g_t) h0 and o_t = scale h_t^T q_t
    c = _gdr_case(1, T=7)
    o, h = O.gated_delta_rule(c["q"], c["k"], c["v"], c["g"], np.zeros_like(c["beta"]), c["h0"], scale=0.5)
    G = np.cumsum(c["g"][0, :, 0])
    for t in range(7):
        np.testing.assert_allclose(o[0, t, 0], 0.5 * math.exp(G[t]) * c["h0"][0, 0].T @ c["q"][0, t, 0], atol=1e-12)
    np.testing.assert_allclose(h[0, 0], math.exp(G[-1]) * c["h0"][0, 0], atol=1e-12)


def test_gdr_full_write_recalls_the_value_at_its_key():
    # unit gate, beta = 1, a unit key: (I - k k^T) erases what the state held at k, then k v^T
    # writes v there, so h^T k = v exactly whatever h0 was; reading with q = k returns scale v
    c = _gdr_case(2, T=1)
    c["q"] = c["k"].copy()
    o, h = O.gated_delta_rule(c["q"], c["k"], c["v"], np.zeros((1, 1, 1)), np.ones((1, 1, 1)), c["h0"], scale=2.0)
    np.testing.assert_allclose(h[0, 0].T @ c["k"][0, 0, 0], c["v"][0, 0, 0], atol=1e-12)
    np.testing.assert_allclose(o[0, 0, 0], 2.0 * c["v"][0, 0, 0], atol=1e-12)


def test_gdr_orthonormal_keys_overwrite_exactly_their_rows():
    # keys e_2, e_0, e_2: rows 0 and 2 end as the last value written at them, the rest are h0's
    dk = dv = 5
    c = _gdr_case(3, T=3, dk=dk, dv=dv)
    k = np.zeros((1, 3, 1, dk))
    for t, row in enumerate((2, 0, 2)):
        k[0, t, 0, row] = 1.0
    _, h = O.gated_delta_rule(c["q"], k, c["v"], np.zeros((1, 3, 1)), np.ones((1, 3, 1)), c["h0"])
    want = c["h0"][0, 0].copy()
    want[0] = c["v"][0, 1, 0]
    want[2] = c["v"][0, 2, 0]
    np.testing.assert_allclose(h[0, 0], want, atol=1e-12)


def test_gdr_output_is_affine_in_the_initial_state():
    c = _gdr_case(4, T=6)
    run = lambda h0: O.gated_delta_rule(c["q"], c["k"], c["v"], c["g"], c["beta"], h0)[0]
    base = run(np.zeros_like(c["h0"]))
    np.testing.assert_allclose(run(3 * c["h0"]) - base, 3 * (run(c["h0"]) - base), atol=1e-10)


def test_gdr_value_heads_share_their_key_head():
    # two value heads on one key head with the same values, gates and strengths give the same output
    c = _gdr_case(5, T=8, Hk=2, Hv=4)
    for a, b in ((0, 1), (2, 3)):
        for name in ("v", "g", "beta"):
            c[name][:, :, b] = c[name][:, :, a]
        c["h0"][:, b] = c["h0"][:, a]
    o, _ = O.gated_delta_rule(c["q"], c["k"], c["v"], c["g"], c["beta"], c["h0"])
    np.testing.assert_allclose(o[:, :, 1], o[:, :, 0], atol=1e-12)
    np.testing.assert_allclose(o[:, :, 3], o[:, :, 2], atol=1e-12)
    assert np.abs(o[:, :, 0] - o[:, :, 2]).max() > 1e-3


@pytest.mark.parametrize("T,chunk", [(37, 8), (64, 64), (70, 16), (5, 64)])
def test_gdr_chunked_form_equals_the_recurrence(T, chunk):
    c = _gdr_case(6, B=2, T=T, Hk=2, Hv=4, dk=8, dv=6)
    o1, h1 = O.gated_delta_rule(c["q"], c["k"], c["v"], c["g"], c["beta"], c["h0"], scale=0.7)
    o2, h2 = O.gated_delta_rule_chunked(c["q"], c["k"], c["v"], c["g"], c["beta"], c["h0"], scale=0.7, chunk=chunk)
    np.testing.assert_allclose(o2, o1, atol=1e-10)
    np.testing.assert_allclose(h2, h1, atol=1e-10)


def test_dga_query_starts_from_the_selected_documents_states():
    r = np.random.default_rng(7)
    c = _gdr_case(7, B=2, T=4, Hk=1, Hv=2)
    states = r.standard_normal((5, 2, 6, 6))
    idx = np.array([[1, 3], [4, 4]])
    o, h = O.dga_query(states, idx, c["q"], c["k"], c["v"], c["g"], c["beta"])
    h0 = np.stack([states[1] + states[3], 2 * states[4]])
    o2, h2 = O.gated_delta_rule(c["q"], c["k"], c["v"], c["g"], c["beta"], h0)
    np.testing.assert_allclose(o, o2, atol=1e-12)
    np.testing.assert_allclose(h, h2, atol=1e-12)
