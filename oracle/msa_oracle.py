"""Plain fp64 CPU oracle for the memory path of one Memory Sparse Attention layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

What the method computes, and where it is stated
-------------------------------------------------
* "MSA: Memory Sparse Attention" README, section "Architecture": document latent
  states K / V / K_r are compressed by chunk-mean pooling; a router scores
  relevance by cosine similarity, averaged over router heads and then maximised
  over the query's tokens; the top-k documents are selected and their compressed
  K / V are concatenated with the query's local K / V for attention.
* Same README, Figure 2 caption: the MSA layer uses document-wise ("parallel")
  RoPE on the memory side.  The blog post "MSA" (moses-y.github.io), section
  "What This Does": document-wise RoPE keeps positions from drifting between
  training and inference.
* Same README, section "Inference Pipeline", stages 1-2: memory is encoded
  offline into chunk-pooled (K̄, V̄, K̄_r); online, the query's Q_r is matched
  against K̄_r, the top-k documents are picked, and only their K̄ / V̄ are loaded
  and concatenated with the local context.
* "MSA × Qwen3.5" model card, section "Architecture summary": full-attention MSA
  layers concatenate the top-k chunks' K / V with the local KV in sparse
  attention.

The pages print no formulas.  Where they leave a step open this module takes
the plainest reading and says so at the function (the list of readings):
  R1 RoPE is the rotate-half form, ω_i = θ^(-2i/d) for i < d/2, applied to K only
     (not V, not K_r), at the token's position inside its own document.
  R2 A chunk is P consecutive tokens of one document; the last chunk of a
     document may be shorter and is averaged over its actual token count.
  R3 Cosine uses max(‖x‖, 1e-12) as the norm (only artificial zero vectors reach it).
  R4 A document's score is the maximum of its chunks' scores; every token of one
     query shares one top-k set; batch rows are independent.
  R5 Top-k output is sorted by score descending, ties broken by lower index.
  R6 Attention keys are [selected memory rows (no mask)] ++ [local rows, causal,
     bottom-right aligned: query token i sits at local position Lloc - Tq + i];
     q-head h reads KV head floor(h / (Hq / Hkv)); the scale is 1/sqrt(d).
  R7 Stored bf16 values are the fp64 result rounded to nearest, ties to even.
  R14 The backward of the query path (the pages train MSA end to end through the
     sparse attention but print no gradient) is the exact derivative of R6's
     attention, and the gather's adjoint adds each gathered row's gradient back
     into its chunk; the top-k choice itself carries no gradient.
  R15 The routing score's gradient (the model card names an auxiliary routing
     loss but does not define it) is taken for an upstream gradient of the
     selected documents' scores: the max passes it to its argmax (token, chunk),
     first in (chunk, token) order on ties, and the cosine's derivative spreads it
     over that token's Qr and that chunk's K̄r.
  R16 The linear (DGA) layers' memory injection ("MSA x Qwen3.5" model card,
     "Architecture summary": the top-k documents' recurrent states are summed
     into S_ext, the initial state of the query path's gated delta rule) sums
     each query's selected documents' states elementwise; how a document's state
     is produced, and the delta rule that consumes S_ext, are defined outside
     the pages and are not part of this module.
  R17 Memory Interleave (README, Figure 3 caption: an optional multi-round
     interleave for multi-hop questions; FAQ "What is Memory Interleave?":
     multi-round reasoning that jumps across scattered memory segments) is read
     as R rounds of the memory path: round r routes its router query over the
     bank, selects the k best documents not selected in an earlier round, and
     attends over every round's documents so far (round order, then rank
     order); the next round's router query is a given linear map W of this
     round's attention output (the pages produce it with the model, which is not
     available; W stands in for it).
  R18 The linear (DGA) layers' query path consumes S_ext as the initial state of
     the gated delta rule (model card, "Architecture summary").  The pages do not
     define that rule; it is the recurrence of Gated DeltaNet (Yang, Kautz and
     Hatamizadeh, "Gated Delta Networks: Improving Mamba2 with Delta Rule", ICLR
     2025), written here per value head with the state h (key dim x value dim, the
     transpose of the paper's S):
         h_t = exp(g_t) (I - beta_t k_t k_t^T) h_{t-1} + beta_t k_t v_t^T
         o_t = h_t^T (scale q_t)
     with h_0 = S_ext, log gates g_t <= 0 and write strengths beta_t given; a
     value head h reads key head h / (Hv / Hk).  Keys are used as given (the
     model normalises them before the rule).

Layouts are row-major with the innermost dimension last:
  K, V [Ntok, Hkv, d]; Kr [Ntok, Hr, dr]; doc_tok_off int64 [D+1]
  Kbar, Vbar [C, Hkv, d]; Krbar [C, Hr, dr]; doc_chunk_off int64 [D+1]
  Qr [B, Tq, Hr, dr]; doc_scores [B, D]; topk_idx int [B, k]
  Q [B, Tq, Hq, d]; Kloc, Vloc [B, Lloc, Hkv, d]; Kmem, Vmem [B, M, Hkv, d]

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
closed forms, textbook special cases, an independent library routine or brute
force (see the docstring of each function for which).
"""
from __future__ import annotations

import itertools
import math

import numpy as np

NORM_EPS = 1e-12  # reading R3


# ----------------------------------------------------------------------------
# storage rounding (reading R7)
# ----------------------------------------------------------------------------
def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp64 values rounded to the nearest bfloat16 (8 significant bits), ties to even.

    Written from the definition of the format: 1 sign bit, 8 exponent bits, 7
    stored mantissa bits.  Values below the smallest normal bf16 are rounded on
    the subnormal grid (spacing 2^-133).  Pinned by exhaustive comparison with
    the bit pattern decoding in tests.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    m, e = np.frexp(x[nz])  # x = m * 2**e, 0.5 <= |m| < 1
    # normal bf16: 8 significant bits -> scale the mantissa by 2**8
    e_min = -125  # frexp exponent of the smallest normal bf16 (2**-126 = 0.5 * 2**-125)
    shift = np.where(e < e_min, 8 - (e_min - e), 8)
    r = np.round(np.ldexp(m, shift))  # np.round is round-half-to-even
    out[nz] = np.ldexp(r, e - shift)
    return out


# ----------------------------------------------------------------------------
# step 1: document-wise RoPE + chunk-mean pooling
# ----------------------------------------------------------------------------
def rope_angles(positions: np.ndarray, d: int, theta: float) -> np.ndarray:
    """Angle p * ω_i for each position p and i < d/2, with ω_i = θ^(-2i/d) (reading R1)."""
    i = np.arange(d // 2, dtype=np.float64)
    omega = theta ** (-2.0 * i / d)
    return np.asarray(positions, dtype=np.float64)[:, None] * omega[None, :]


def rope_rotate(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE of x [T, H, d] with token positions [T] (reading R1).

    For i < d/2 the pair (x_i, x_{i+d/2}) turns by the angle p * ω_i:
      x_i'       = x_i cos - x_{i+d/2} sin
      x_{i+d/2}' = x_{i+d/2} cos + x_i sin
    Pins: position 0 is the identity; each pair keeps its length; the
    relative-position identity <R_m q, R_n k> = <R_{m-n} q, k>; a hand-made
    quarter turn.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = rope_angles(positions, d, theta)[:, None, :]  # [T, 1, d/2]
    c, s = np.cos(ang), np.sin(ang)
    lo, hi = x[..., : d // 2], x[..., d // 2 :]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


def chunk_offsets(doc_tok_off: np.ndarray, P: int) -> np.ndarray:
    """doc_chunk_off [D+1]: document j owns chunks [off[j], off[j+1]), n_j = ceil(L_j / P) (R2)."""
    L = np.diff(np.asarray(doc_tok_off, dtype=np.int64))
    n = (L + P - 1) // P
    return np.concatenate([[0], np.cumsum(n)]).astype(np.int64)


def chunk_token_ranges(doc_tok_off: np.ndarray, P: int):
    """List of (start, end, doc) token ranges, one per chunk, in chunk order (R2)."""
    out = []
    for j in range(len(doc_tok_off) - 1):
        s, e = int(doc_tok_off[j]), int(doc_tok_off[j + 1])
        for c0 in range(s, e, P):
            out.append((c0, min(c0 + P, e), j))
    return out


def doc_positions(doc_tok_off: np.ndarray) -> np.ndarray:
    """Position of every token inside its own document, restarting at 0 (R1, document-wise RoPE)."""
    off = np.asarray(doc_tok_off, dtype=np.int64)
    ntok = int(off[-1])
    pos = np.arange(ntok, dtype=np.int64)
    doc = np.searchsorted(off, pos, side="right") - 1
    return pos - off[doc]


def pool(K, V, Kr, doc_tok_off, P: int, theta: float, out_bf16: bool = False):
    """Step 1, offline memory encoding: RoPE on K, then chunk means of K', V and Kr.

    "MSA: Memory Sparse Attention" README, "Architecture" (chunk-mean pooling of
    K / V / K_r) and "Inference Pipeline" stage 1 (cache chunk-pooled K̄, V̄, K̄_r);
    Figure 2 caption (document-wise RoPE).  Readings R1, R2, R7.

    Returns (Kbar, Vbar, Krbar, doc_chunk_off, kr_rnorm) with kr_rnorm[c, h] =
    1 / max(‖Krbar[c, h]‖, 1e-12) taken from the (possibly bf16-rounded) stored Krbar.
    Pins: a constant input pools to itself; pooling is linear; a ramp 0..n-1 pools
    to (n-1)/2; a 52-token tail chunk averages over 52 tokens.
    """
    off = np.asarray(doc_tok_off, dtype=np.int64)
    Kp = rope_rotate(K, doc_positions(off), theta)
    V = np.asarray(V, dtype=np.float64)
    Kr = np.asarray(Kr, dtype=np.float64)
    ranges = chunk_token_ranges(off, P)
    starts = np.array([r[0] for r in ranges], dtype=np.int64)
    counts = np.array([r[1] - r[0] for r in ranges], dtype=np.float64)
    if len(ranges) == 0:
        z = lambda a: np.zeros((0,) + a.shape[1:])
        return z(K), z(V), z(Kr), chunk_offsets(off, P), np.zeros((0, Kr.shape[1]))
    # np.add.reduceat sums each [starts[c], starts[c+1]) slice; chunks tile the
    # token axis contiguously, so these are exactly the chunk sums.
    mean = lambda a: np.add.reduceat(a, starts, axis=0) / counts[:, None, None]
    Kbar, Vbar, Krbar = mean(Kp), mean(V), mean(Kr)
    if out_bf16:
        Kbar, Vbar, Krbar = round_to_bf16(Kbar), round_to_bf16(Vbar), round_to_bf16(Krbar)
    rnorm = 1.0 / np.maximum(np.sqrt((Krbar * Krbar).sum(-1)), NORM_EPS)
    return Kbar, Vbar, Krbar, chunk_offsets(off, P), rnorm


# ----------------------------------------------------------------------------
# step 2: cosine routing
# ----------------------------------------------------------------------------
def cosine_scores(Qr, Krbar) -> np.ndarray:
    """s[b, t, c] = (1/Hr) Σ_h cos(Qr[b, t, h], Krbar[c, h]).

    README "Architecture": relevance by cosine similarity, mean-pooled over heads
    (reading R3 for the norm clamp).  Pins: values in [-1, 1]; identical vectors
    give 1, negated give -1; invariant to positive scaling of either side; Hr = 1
    is the textbook cosine (scipy).
    """
    Qr = np.asarray(Qr, dtype=np.float64)
    Kb = np.asarray(Krbar, dtype=np.float64)
    qn = Qr / np.maximum(np.linalg.norm(Qr, axis=-1, keepdims=True), NORM_EPS)
    kn = Kb / np.maximum(np.linalg.norm(Kb, axis=-1, keepdims=True), NORM_EPS)
    Hr = Qr.shape[2]
    s = np.zeros(Qr.shape[:2] + (Kb.shape[0],))
    for h in range(Hr):
        s += qn[:, :, h, :] @ kn[:, h, :].T  # [B, Tq, C]
    return s / Hr


def route(Qr, Krbar, doc_chunk_off) -> np.ndarray:
    """Step 2: doc_score[b, j] = max over chunks c of document j of max over tokens t of s[b, t, c].

    README "Architecture": head mean first, then the token-wise max; the document
    score is the max over the document's chunks (reading R4).  A document with no
    chunks scores -inf.  Pins: the order head-mean-then-max matters and is checked
    on a hand case; a document whose K_r tokens all equal a query token scores 1.
    """
    s = cosine_scores(Qr, Krbar)          # [B, Tq, C]
    m = s.max(axis=1)                     # token-wise max -> [B, C]
    off = np.asarray(doc_chunk_off, dtype=np.int64)
    D = len(off) - 1
    out = np.full((m.shape[0], D), -np.inf)
    for j in range(D):
        if off[j + 1] > off[j]:
            out[:, j] = m[:, off[j] : off[j + 1]].max(axis=1)
    return out


# ----------------------------------------------------------------------------
# step 3: top-k documents
# ----------------------------------------------------------------------------
def topk(doc_scores, k: int):
    """Step 3: the k best documents per row, sorted by (score desc, index asc) (reading R5).

    README "Architecture" / "Inference Pipeline" stage 2: select the top-k
    documents.  Pins: brute force over every k-subset on small rows; agreement
    with a full stable sort.
    """
    sc = np.asarray(doc_scores, dtype=np.float64)
    B, D = sc.shape
    idx = np.zeros((B, k), dtype=np.int64)
    val = np.zeros((B, k))
    for b in range(B):
        order = sorted(range(D), key=lambda j: (-sc[b, j], j))[:k]
        idx[b] = order
        val[b] = sc[b, order]
    return idx, val


def topk_bruteforce(doc_scores_row, k: int):
    """Reference for tiny rows: the k-subset with the largest score sum, then sorted (R5)."""
    row = list(doc_scores_row)
    best, best_key = None, None
    for sub in itertools.combinations(range(len(row)), k):
        # maximise the sum; among equal sums prefer the lexicographically smallest index set
        key = (sum(row[j] for j in sub), tuple(-j for j in sub))
        if best_key is None or key > best_key:
            best, best_key = sub, key
    return sorted(best, key=lambda j: (-row[j], j))


# ----------------------------------------------------------------------------
# step 4: gather the selected documents' chunks
# ----------------------------------------------------------------------------
def gather(topk_idx, doc_chunk_off, Kbar, Vbar, Mmax: int):
    """Step 4: concatenate the selected documents' chunks, in rank order (README stage 2).

    Within a document the chunks keep their order.  Rows past mem_len[b] are zero.
    Pins: the copy is exact; mem_len equals the sum of the selected n_j.
    """
    idx = np.asarray(topk_idx, dtype=np.int64)
    off = np.asarray(doc_chunk_off, dtype=np.int64)
    Kb, Vb = np.asarray(Kbar), np.asarray(Vbar)
    B = idx.shape[0]
    Km = np.zeros((B, Mmax) + Kb.shape[1:], dtype=Kb.dtype)
    Vm = np.zeros((B, Mmax) + Vb.shape[1:], dtype=Vb.dtype)
    mem_len = np.zeros(B, dtype=np.int64)
    for b in range(B):
        rows = [c for j in idx[b] for c in range(off[j], off[j + 1])]
        n = len(rows)
        if n > Mmax:
            raise ValueError("selected documents exceed Mmax rows")
        Km[b, :n], Vm[b, :n] = Kb[rows], Vb[rows]
        mem_len[b] = n
    return Km, Vm, mem_len


def state_gather_sum(states, topk_idx):
    """Reading R16: S_ext[b] = sum over the query's selected documents j of states[j].

    states [D, ...] (one recurrent state per document, any trailing shape),
    topk_idx int [B, k] -> S_ext [B, ...] in fp64.  Every selected index must lie
    in [0, D); a document selected twice counts twice.
    Pins: one selected document gives its state back exactly; one-hot states
    count how often each document is selected; the sum is invariant under the
    order of the selection and linear in the states; selecting every document
    once gives numpy's sum over all documents.
    """
    st = np.asarray(states, dtype=np.float64)
    idx = np.asarray(topk_idx, dtype=np.int64)
    if idx.size and (idx.min() < 0 or idx.max() >= st.shape[0]):
        raise ValueError("selected document index out of range")
    out = np.zeros((idx.shape[0],) + st.shape[1:], dtype=np.float64)
    for b in range(idx.shape[0]):
        for j in idx[b]:
            out[b] += st[j]
    return out


# ----------------------------------------------------------------------------
# step 5: sparse attention over [memory ++ causal local]
# ----------------------------------------------------------------------------
def attention(Q, Kloc, Vloc, Kmem, Vmem, mem_len, scale=None):
    """Step 5: softmax(scale q·kᵀ) v over [memory rows ++ causal local rows] (reading R6).

    "MSA × Qwen3.5" card, "Architecture summary" (full layers: concat top-k
    chunks' K/V with local KV in sparse attention); README "Architecture".
    Returns (O [B, Tq, Hq, d], lse [B, Hq, Tq]) with lse the natural-log
    normaliser of the scaled logits.
    Pins: no memory rows equals plain causal attention and matches torch's
    scaled_dot_product_attention in fp64; identical keys return the mean of V;
    Hq = Hkv is plain multi-head attention; every row's weights sum to 1.
    """
    Q = np.asarray(Q, dtype=np.float64)
    Kl, Vl = np.asarray(Kloc, dtype=np.float64), np.asarray(Vloc, dtype=np.float64)
    Km, Vm = np.asarray(Kmem, dtype=np.float64), np.asarray(Vmem, dtype=np.float64)
    B, Tq, Hq, d = Q.shape
    Lloc, Hkv = Kl.shape[1], Kl.shape[2]
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    group = Hq // Hkv
    O = np.zeros_like(Q)
    lse = np.zeros((B, Hq, Tq))
    for b in range(B):
        M = int(mem_len[b])
        for h in range(Hq):
            g = h // group
            keys = np.concatenate([Km[b, :M, g], Kl[b, :, g]], axis=0)   # [M + Lloc, d]
            vals = np.concatenate([Vm[b, :M, g], Vl[b, :, g]], axis=0)
            logits = scale * (Q[b, :, h] @ keys.T)                       # [Tq, M + Lloc]
            pos = Lloc - Tq + np.arange(Tq)
            visible = np.concatenate(
                [np.ones((Tq, M), bool), np.arange(Lloc)[None, :] <= pos[:, None]], axis=1)
            logits = np.where(visible, logits, -np.inf)
            mx = logits.max(axis=1, keepdims=True)
            w = np.exp(logits - mx)
            den = w.sum(axis=1, keepdims=True)
            O[b, :, h] = (w / den) @ vals
            lse[b, h] = (mx + np.log(den))[:, 0]
    return O, lse


# ----------------------------------------------------------------------------
# backward of steps 5 and 4 (the differentiable part of the query path)
# ----------------------------------------------------------------------------
def attention_backward(Q, Kloc, Vloc, Kmem, Vmem, mem_len, dO, scale=None):
    """Gradient of attention()'s output O for an upstream gradient dO (reading R14).

    MSA is trained end to end through its sparse attention ("MSA: Memory Sparse
    Attention" README, Figure 2 caption and "Architecture": top-k selection is
    fused with sparse attention so the layer stays differentiable).  With
    s = scale q·kᵀ over the same visible keys as the forward, p = softmax(s),
    o = p v:
        dv_j = sum_i p_ij do_i          dp_ij = do_i · v_j
        ds_ij = p_ij (dp_ij - sum_l p_il dp_il)
        dq_i = scale sum_j ds_ij k_j    dk_j = scale sum_i ds_ij q_i
    summed over the q-heads of a GQA group for the shared K/V.  Returns
    (dQ, dKloc, dVloc, dKmem, dVmem) in fp64; memory rows past mem_len[b] get 0.
    Pins: central finite differences of sum(dO * O) on a small case; the
    gradients of keys no query sees are zero.
    """
    Q = np.asarray(Q, dtype=np.float64)
    Kl, Vl = np.asarray(Kloc, dtype=np.float64), np.asarray(Vloc, dtype=np.float64)
    Km, Vm = np.asarray(Kmem, dtype=np.float64), np.asarray(Vmem, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    B, Tq, Hq, d = Q.shape
    Lloc, Hkv = Kl.shape[1], Kl.shape[2]
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    group = Hq // Hkv
    dQ = np.zeros_like(Q)
    dKl, dVl = np.zeros_like(Kl), np.zeros_like(Vl)
    dKm, dVm = np.zeros_like(Km), np.zeros_like(Vm)
    for b in range(B):
        M = int(mem_len[b])
        for h in range(Hq):
            g = h // group
            keys = np.concatenate([Km[b, :M, g], Kl[b, :, g]], axis=0)
            vals = np.concatenate([Vm[b, :M, g], Vl[b, :, g]], axis=0)
            logits = scale * (Q[b, :, h] @ keys.T)
            pos = Lloc - Tq + np.arange(Tq)
            visible = np.concatenate(
                [np.ones((Tq, M), bool), np.arange(Lloc)[None, :] <= pos[:, None]], axis=1)
            logits = np.where(visible, logits, -np.inf)
            w = np.exp(logits - logits.max(axis=1, keepdims=True))
            P = w / w.sum(axis=1, keepdims=True)                   # [Tq, M + Lloc]
            dP = dO[b, :, h] @ vals.T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            dQ[b, :, h] = scale * (dS @ keys)
            dkeys = scale * (dS.T @ Q[b, :, h])
            dvals = P.T @ dO[b, :, h]
            dKm[b, :M, g] += dkeys[:M]
            dVm[b, :M, g] += dvals[:M]
            dKl[b, :, g] += dkeys[M:]
            dVl[b, :, g] += dvals[M:]
    return dQ, dKl, dVl, dKm, dVm


def gather_backward(topk_idx, doc_chunk_off, dKmem, dVmem, mem_len, C: int):
    """Adjoint of gather(): add every gathered row's gradient back into its chunk.

    A chunk selected by several queries accumulates all their gradients.
    Returns (dKbar, dVbar) [C, Hkv, d] in fp64.  Pin: the adjoint identity
    <gather(x), y> = <x, gather_backward(y)> for random x and y.
    """
    idx = np.asarray(topk_idx, dtype=np.int64)
    off = np.asarray(doc_chunk_off, dtype=np.int64)
    dKm, dVm = np.asarray(dKmem, dtype=np.float64), np.asarray(dVmem, dtype=np.float64)
    dKb = np.zeros((C,) + dKm.shape[2:])
    dVb = np.zeros((C,) + dVm.shape[2:])
    for b in range(idx.shape[0]):
        rows = [c for j in idx[b] for c in range(off[j], off[j + 1])][:int(mem_len[b])]
        for r, c in enumerate(rows):
            dKb[c] += dKm[b, r]
            dVb[c] += dVm[b, r]
    return dKb, dVb


def route_backward(Qr, Krbar, doc_chunk_off, topk_idx, d_score):
    """Gradient of the selected documents' scores (reading R15).

    score(b, j) = max over chunks c of j and tokens t of s[b, t, c] with
    s = (1/Hr) sum_h cos(Qr[b, t, h], K̄r[c, h]) (route()).  Given d_score[b, r],
    the upstream gradient of score(b, topk_idx[b, r]) (e.g. from an auxiliary
    routing loss), the max passes it to its argmax (the first pair in (chunk,
    token) order on ties) and the cosine's derivative
        d cos(q, k) / dq = k / (|q| |k|) - cos(q, k) q / |q|^2
    distributes it to that token's Qr and that chunk's K̄r, per head, with 1/Hr.
    Returns (dQr [B, Tq, Hr, dr], dKrbar [C, Hr, dr]) in fp64.  Documents with
    no chunks get no gradient.  Pin: central finite differences of
    sum_r d_score[b, r] * score(b, topk_idx[b, r]) on a case with distinct maxima.
    """
    Qr = np.asarray(Qr, dtype=np.float64)
    Kb = np.asarray(Krbar, dtype=np.float64)
    off = np.asarray(doc_chunk_off, dtype=np.int64)
    idx = np.asarray(topk_idx, dtype=np.int64)
    g = np.asarray(d_score, dtype=np.float64)
    B, Tq, Hr, dr = Qr.shape
    dQ = np.zeros_like(Qr)
    dK = np.zeros_like(Kb)
    s = cosine_scores(Qr, Kb)                                   # [B, Tq, C]
    for b in range(B):
        for r, j in enumerate(idx[b]):
            a, e = int(off[j]), int(off[j + 1])
            if e <= a:
                continue
            sc = s[b, :, a:e].T                                 # [chunks, Tq]: chunk-major order
            c_rel, t = np.unravel_index(int(np.argmax(sc)), sc.shape)
            c = a + int(c_rel)
            for h in range(Hr):
                q, k = Qr[b, t, h], Kb[c, h]
                nq, nk = max(np.linalg.norm(q), NORM_EPS), max(np.linalg.norm(k), NORM_EPS)
                cos = float(q @ k) / (nq * nk)
                w = g[b, r] / Hr
                dQ[b, t, h] += w * (k / (nq * nk) - cos * q / nq ** 2)
                dK[c, h] += w * (q / (nq * nk) - cos * k / nk ** 2)
    return dQ, dK


# ----------------------------------------------------------------------------
# the linear (DGA) layers' query path: gated delta rule from S_ext (reading R18)
# ----------------------------------------------------------------------------
def gated_delta_rule(q, k, v, g, beta, h0=None, scale=1.0):
    """The gated delta rule of reading R18, token by token (the definition).

    q, k [B, T, Hk, dk]; v [B, T, Hv, dv]; g, beta [B, T, Hv]; h0 [B, Hv, dk, dv]
    or None (zeros).  Returns (o [B, T, Hv, dv], h_T [B, Hv, dk, dv]) in fp64.
    Pins: beta = 0 decays h0 by the cumulative gate; with unit gates, beta = 1 and
    a unit key the state returns v at that key; orthonormal keys overwrite
    exactly their rows of h0; the output is affine in h0; the chunked form below
    agrees.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    g, beta = np.asarray(g, dtype=np.float64), np.asarray(beta, dtype=np.float64)
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    grp = Hv // Hk
    h = np.zeros((B, Hv, dk, dv)) if h0 is None else np.array(h0, dtype=np.float64, copy=True)
    o = np.zeros((B, T, Hv, dv))
    for b in range(B):
        for hv in range(Hv):
            hk = hv // grp
            H = h[b, hv]
            for t in range(T):
                kt, qt, vt = k[b, t, hk], q[b, t, hk], v[b, t, hv]
                a, bt = math.exp(g[b, t, hv]), beta[b, t, hv]
                H = a * (H - bt * np.outer(kt, kt @ H)) + bt * np.outer(kt, vt)
                o[b, t, hv] = H.T @ (scale * qt)
            h[b, hv] = H
    return o, h


def gated_delta_rule_chunked(q, k, v, g, beta, h0=None, scale=1.0, chunk: int = 64):
    """The same rule computed chunk by chunk (the form the GPU kernel uses), for cross-checking.

    Within a chunk of C tokens, with G_i the cumulative log gate from the chunk's
    start, the state after token i is exp(G_i) h0 + sum_{j <= i} exp(G_i - G_j) k_j u_j^T,
    where the new-value rows u solve the unit lower-triangular system
        u_i + beta_i sum_{j < i} exp(G_i - G_j) (k_i . k_j) u_j = beta_i (v_i - exp(G_i) h0^T k_i),
    so o_i = scale (exp(G_i) h0^T q_i + sum_{j <= i} exp(G_i - G_j) (q_i . k_j) u_j) and the
    chunk ends with h = exp(G_C) h0 + sum_j exp(G_C - G_j) k_j u_j^T.  (Derived from the
    recurrence by induction over i; it is the chunkwise form of the Gated DeltaNet paper.)
    Pin: equal to gated_delta_rule up to rounding.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    g, beta = np.asarray(g, dtype=np.float64), np.asarray(beta, dtype=np.float64)
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    grp = Hv // Hk
    h = np.zeros((B, Hv, dk, dv)) if h0 is None else np.array(h0, dtype=np.float64, copy=True)
    o = np.zeros((B, T, Hv, dv))
    for b in range(B):
        for hv in range(Hv):
            hk = hv // grp
            H = h[b, hv]
            for c0 in range(0, T, chunk):
                c1 = min(c0 + chunk, T)
                K, Q, V = k[b, c0:c1, hk], q[b, c0:c1, hk], v[b, c0:c1, hv]
                G = np.cumsum(g[b, c0:c1, hv])
                bt = beta[b, c0:c1, hv]
                n = c1 - c0
                decay = np.exp(np.minimum(G[:, None] - G[None, :], 0.0))  # exp(G_i - G_j) for j <= i
                A = np.tril(np.ones((n, n)), -1) * decay * (K @ K.T)
                rhs = bt[:, None] * (V - np.exp(G)[:, None] * (K @ H))
                U = np.linalg.solve(np.eye(n) + bt[:, None] * A, rhs)
                P = np.tril(np.ones((n, n))) * decay * (Q @ K.T)
                o[b, c0:c1, hv] = scale * (np.exp(G)[:, None] * (Q @ H) + P @ U)
                H = math.exp(G[-1]) * H + (np.exp(G[-1] - G)[:, None] * K).T @ U
            h[b, hv] = H
    return o, h


def dga_query(states, topk_idx, q, k, v, g, beta, scale=1.0):
    """The linear layers' memory path (model card, "Architecture summary"; readings R16, R18):
    S_ext = state_gather_sum(states, topk_idx) is the initial state of the gated delta rule over
    the query tokens.  states [D, Hv, dk, dv].  Returns (o, h_T)."""
    return gated_delta_rule(q, k, v, g, beta, state_gather_sum(states, topk_idx), scale)


# ----------------------------------------------------------------------------
# Memory Interleave (reading R17)
# ----------------------------------------------------------------------------
def exclude_selected(doc_scores, selected):
    """Scores with each query's already-selected documents set to -inf (R17: a round
    selects documents no earlier round selected).  selected: per query, a list of
    document indices.  Pin: with every other score equal, top-k then returns the
    lowest-index documents outside the excluded set."""
    out = np.array(doc_scores, dtype=np.float64, copy=True)
    for b, docs in enumerate(selected):
        if len(docs):
            out[b, np.asarray(docs, dtype=np.int64)] = -np.inf
    return out


def round_query(O_prev, W, Hr: int, dr: int):
    """Next round's router query (R17): Qr[b, t] = O_prev[b, t] (as one Hq*d vector) times W [Hq*d, Hr*dr],
    reshaped to [B, Tq, Hr, dr].  Pins: a one-hot W copies one output component to one
    router component; the map is linear."""
    O_prev = np.asarray(O_prev, dtype=np.float64)
    B, Tq = O_prev.shape[:2]
    flat = O_prev.reshape(B * Tq, -1)
    return (flat @ np.asarray(W, dtype=np.float64)).reshape(B, Tq, Hr, dr)


def interleave(Qr0, Krbar, doc_chunk_off, k: int, rounds: int, W, Q, Kloc, Vloc, Kbar, Vbar, Mmax: int,
               scale=None, O_feed=None, qr_store=None):
    """Memory Interleave over R = rounds rounds (reading R17), in the README's pipeline order per round.

    Returns a dict with topk_idx / topk_score [B, rounds * k] (round r in columns
    [r k, (r + 1) k)), O / lse of the last round, O_rounds (every round's output)
    and Qr_rounds (every round's router query).  O_feed (list of arrays) supplies
    the round outputs the next router queries are computed from instead of this
    function's own (for step-by-step comparison with a device that stores them in
    bf16); qr_store (a function) rounds each computed router query the way the
    device stores it.  Pins: one round is layer_forward; the rounds' selections
    are disjoint; with W = 0 every later round selects the lowest-index documents
    not yet selected; brute force over the k-subsets outside the excluded set.
    """
    Qr = np.asarray(Qr0, dtype=np.float64)
    B = Qr.shape[0]
    Hr, dr = Qr.shape[2], Qr.shape[3]
    chosen = [[] for _ in range(B)]
    idx_all = np.zeros((B, rounds * k), dtype=np.int64)
    sc_all = np.zeros((B, rounds * k))
    outs, lses, qrs = [], [], []
    for r in range(rounds):
        qrs.append(Qr)
        ds = exclude_selected(route(Qr, Krbar, doc_chunk_off), chosen)
        ti, ts = topk(ds, k)
        idx_all[:, r * k:(r + 1) * k] = ti
        sc_all[:, r * k:(r + 1) * k] = ts
        for b in range(B):
            chosen[b] += [int(j) for j in ti[b]]
        Km, Vm, ml = gather(np.array(chosen, dtype=np.int64), doc_chunk_off, Kbar, Vbar, Mmax)
        O_r, lse_r = attention(Q, Kloc, Vloc, Km, Vm, ml, scale)
        outs.append(O_r)
        lses.append(lse_r)
        if r + 1 < rounds:
            src = O_feed[r] if O_feed is not None else O_r
            Qr = round_query(src, W, Hr, dr)
            if qr_store is not None:
                Qr = qr_store(Qr)
    return dict(topk_idx=idx_all, topk_score=sc_all, O=outs[-1], lse=lses[-1], O_rounds=outs, Qr_rounds=qrs)


# ----------------------------------------------------------------------------
# steps 2-5 composed: one MSA layer's query path over a pooled bank
# ----------------------------------------------------------------------------
def layer_forward(Qr, Krbar, doc_chunk_off, k: int, Q, Kloc, Vloc, Kbar, Vbar, Mmax: int, scale=None):
    """Route -> top-k -> gather -> attention, in the README's "Inference Pipeline" order.

    Returns a dict with doc_scores, topk_idx, topk_score, mem_len, O, lse.
    """
    ds = route(Qr, Krbar, doc_chunk_off)
    ti, ts = topk(ds, k)
    Km, Vm, ml = gather(ti, doc_chunk_off, Kbar, Vbar, Mmax)
    O, lse = attention(Q, Kloc, Vloc, Km, Vm, ml, scale)
    return dict(doc_scores=ds, topk_idx=ti, topk_score=ts, mem_len=ml, O=O, lse=lse)
