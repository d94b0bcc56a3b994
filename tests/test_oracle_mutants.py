"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each one.

Each mutant is the oracle function's own source with one textual edit, compiled
into the oracle module's namespace; the pin that should catch it must then fail.
"""
import inspect
import textwrap

import pytest

from oracle import msa_oracle as O
import tests.test_oracle_pins as pins

MUTANTS = [
    # (function, original text, planted mistake, pin that must fail, pin args)
    ("rope_rotate", "lo * c - hi * s, hi * c + lo * s", "lo * c + hi * s, hi * c - lo * s",
     "test_rope_quarter_turn_by_hand", ()),
    ("doc_positions", "return pos - off[doc]", "return pos",
     "test_pool_rotates_k_at_document_local_positions", ()),
    ("pool", "/ counts[:, None, None]", "/ float(P)",
     "test_pool_ramp_mean_closed_form_and_tail", ()),
    ("route", "m = s.max(axis=1)", "m = s.max(axis=1) * 0 + s.mean(axis=1)",
     "test_planted_document_scores_one_and_is_selected", ()),
    ("route", "s = cosine_scores(Qr, Krbar)",
     "s = np.mean([cosine_scores(Qr[:, :, h:h + 1], Krbar[:, h:h + 1]).max(axis=1, keepdims=True)"
     " for h in range(np.asarray(Qr).shape[2])], axis=0)",
     "test_head_mean_then_token_max_hand_case", ()),
    ("cosine_scores", "s / Hr", "s",
     "test_cosine_identical_negated_and_scale_invariant", ()),
    ("cosine_scores", "qn[:, :, h, :] @ kn[:, h, :].T", "Qr[:, :, h, :] @ Kb[:, h, :].T",
     "test_cosine_identical_negated_and_scale_invariant", ()),
    ("topk", "key=lambda j: (-sc[b, j], j)", "key=lambda j: (-sc[b, j], -j)",
     "test_topk_sorted_and_ties_prefer_lower_index", ()),
    ("gather", "for c in range(off[j], off[j + 1])", "for c in range(off[j], off[j + 1] - 1)",
     "test_gather_copies_selected_chunks_in_rank_order", ()),
    ("attention", "<= pos[:, None]", "< pos[:, None]",
     "test_attention_matches_sdpa", (7, 7, 0, 4, 2)),
    ("attention", "g = h // group", "g = h % Hkv",
     "test_attention_matches_sdpa", (6, 9, 13, 8, 2)),
    ("attention", "pos = Lloc - Tq + np.arange(Tq)", "pos = np.arange(Tq)",
     "test_attention_matches_sdpa", (5, 11, 0, 2, 2)),
    ("attention", "[np.ones((Tq, M), bool),", "[np.arange(M)[None, :] <= np.arange(Tq)[:, None],",
     "test_attention_matches_sdpa", (6, 9, 13, 8, 2)),
    ("attention_backward", "dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))", "dS = P * dP",
     "test_attention_backward_matches_central_differences", ()),
    ("attention_backward", "dvals = P.T @ dO[b, :, h]", "dvals = P.T @ dO[b, :, g]",
     "test_attention_backward_matches_central_differences", ()),
    ("attention_backward", "dkeys = scale * (dS.T @ Q[b, :, h])", "dkeys = dS.T @ Q[b, :, h]",
     "test_attention_backward_matches_central_differences", ()),
    ("gather_backward", "dKb[c] += dKm[b, r]", "dKb[c] = dKm[b, r]",
     "test_gather_backward_is_the_adjoint_of_gather", ()),
    ("route_backward", "dQ[b, t, h] += w * (k / (nq * nk) - cos * q / nq ** 2)", "dQ[b, t, h] += w * k / (nq * nk)",
     "test_route_backward_matches_central_differences", ()),
    ("route_backward", "sc = s[b, :, a:e].T", "sc = s[b, :, a:e]",
     "test_route_backward_matches_central_differences", ()),
    ("state_gather_sum", "out[b] += st[j]", "out[b] = st[j]",
     "test_state_gather_sum_one_hot_states_count_selections", ()),
    ("state_gather_sum", "for j in idx[b]:", "for j in sorted(set(idx[b].tolist())):",
     "test_state_gather_sum_one_hot_states_count_selections", ()),
    ("interleave", "ds = exclude_selected(route(Qr, Krbar, doc_chunk_off), chosen)",
     "ds = route(Qr, Krbar, doc_chunk_off)", "test_interleave_rounds_match_bruteforce_over_free_documents", ()),
    ("interleave", "chosen[b] += [int(j) for j in ti[b]]", "chosen[b] = [int(j) for j in ti[b]]",
     "test_interleave_attends_over_the_union_of_rounds", ()),
    ("exclude_selected", "= -np.inf", "= 0.0", "test_interleave_zero_map_selects_lowest_free_documents", ()),
    ("round_query", "flat = O_prev.reshape(B * Tq, -1)", "flat = O_prev.transpose(0, 2, 1, 3).reshape(B * Tq, -1)",
     "test_round_query_one_hot_map_and_linearity", ()),
    ("gated_delta_rule", "H = a * (H - bt * np.outer(kt, kt @ H)) + bt * np.outer(kt, vt)",
     "H = a * H + bt * np.outer(kt, vt)", "test_gdr_full_write_recalls_the_value_at_its_key", ()),
    ("gated_delta_rule", "o[b, t, hv] = H.T @ (scale * qt)", "o[b, t, hv] = H @ (scale * qt)",
     "test_gdr_zero_write_strength_decays_the_initial_state", ()),
    ("gated_delta_rule", "hk = hv // grp", "hk = hv % Hk", "test_gdr_value_heads_share_their_key_head", ()),
    ("gated_delta_rule", "a, bt = math.exp(g[b, t, hv]), beta[b, t, hv]", "a, bt = 1.0, beta[b, t, hv]",
     "test_gdr_zero_write_strength_decays_the_initial_state", ()),
    ("gated_delta_rule_chunked", "A = np.tril(np.ones((n, n)), -1) * decay * (K @ K.T)",
     "A = np.tril(np.ones((n, n)), -1) * (K @ K.T)", "test_gdr_chunked_form_equals_the_recurrence", (37, 8)),
    ("state_gather_sum", "out[b] += st[j]", "out[b] = st[j]", "test_dga_query_starts_from_the_selected_documents_states",
     ()),
]


def _mutant(fn_name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(O, fn_name)))
    assert old in src, f"mutation anchor not found in {fn_name}"
    ns = {}
    exec(compile(src.replace(old, new, 1), f"<mutant {fn_name}>", "exec"), O.__dict__, ns)
    return ns[fn_name]


@pytest.mark.parametrize("fn,old,new,pin,args", MUTANTS, ids=[f"{m[0]}:{i}" for i, m in enumerate(MUTANTS)])
def test_pin_catches_planted_mistake(monkeypatch, fn, old, new, pin, args):
    monkeypatch.setattr(O, fn, _mutant(fn, old, new))
    with pytest.raises(AssertionError):
        getattr(pins, pin)(*args)
