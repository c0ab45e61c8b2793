"""Mutation checks on the oracle's pins.

Each case plants one plausible mistake in a copy of one oracle function and
requires at least one pin of test_oracle_pins.py to fail on it.  Examples of
such mistakes are a dropped term, a wrong sign, an off-by-one index or range,
swapped roles of two operands, or the wrong tie rule.  A case is one textual
edit of the function's source.  The edit must match exactly once, so a later
change to the oracle that removes the snippet fails here loudly instead of
passing silently.  The mistakes are planted in the CPU oracle only; nothing
here touches the GPU path.
"""
import __future__
import functools
import inspect
import textwrap

import pytest

import oracle
import oracle.kascade_oracle as K
import test_oracle_pins as P


def _mutant(name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(K, name)))
    assert src.count(old) == 1, f"{name}: snippet not found exactly once: {old!r}"
    ns = dict(vars(K))  # the module's globals; calls to other oracle functions stay unmutated
    code = compile(src.replace(old, new), f"<mutant of {name}>", "exec",
                   flags=__future__.annotations.compiler_flag, dont_inherit=True)
    exec(code, ns)
    return ns[name]


def _p(fn, *args):
    return functools.partial(fn, *args)


TOPK_PINS = [_p(P.test_topk_vs_rank_definition, s) for s in range(8)] + [P.test_topk_closed_cases]
DECODE_PINS = [_p(P.test_decode_anchor_brute_force, 0), P.test_decode_anchor_matches_sdpa_and_pooled_sums_to_one]
PREFILL_PINS = [P.test_prefill_anchor_matches_causal_sdpa, _p(P.test_prefill_anchor_pooled_brute_force, 0)]
REUSE_D_PINS = [P.test_decode_reuse_full_set_is_dense, P.test_decode_reuse_brute_force_with_head_map]
REUSE_P_PINS = [P.test_prefill_reuse_full_prefix_is_dense, P.test_prefill_reuse_brute_force]
DP_PINS = [_p(P.test_dp_matches_exhaustive, L) for L in (3, 5, 7)] + [
    P.test_dp_uses_weights_and_similarity, P.test_dp_single_anchor_value_is_total_weight,
    P.test_dp_ties_keep_earliest_anchors]
SIM_PINS = [P.test_similarity_identity_and_bounds, P.test_similarity_hand_example]
REMAP_PINS = [P.test_head_remap_recovers_permutation, P.test_head_remap_direction_hand_example]
K_PINS = [P.test_k_rule_golden, P.test_k_rule_closed_form_everywhere]

# (label, function, snippet, replacement, pins of which at least one must fail)
CASES = [
    # Top-k size rule (k equation; readings R1, R2)
    ("k: 0.1 n floored", "k_for_len", "tenth = (n + 5) // 10", "tenth = n // 10", K_PINS),
    ("k: 0.1 n rounded up", "k_for_len", "tenth = (n + 5) // 10", "tenth = (n + 9) // 10", K_PINS),
    ("k: no 128 floor", "k_for_len", "min(max(tenth, k_min), n)", "min(tenth, n)", K_PINS),
    ("k: no cap at n", "k_for_len", "min(max(tenth, k_min), n)", "max(tenth, k_min)", K_PINS),
    # Top-k selection (R3, R4)
    ("topk: ties to the higher index", "topk_select", "np.lexsort((np.arange(n), -v",
     "np.lexsort((-np.arange(n), -v", TOPK_PINS),
    ("topk: smallest values", "topk_select", "-v.astype(np.float64)))", "v.astype(np.float64)))", TOPK_PINS),
    ("topk: one index short", "topk_select", "order[:k]", "order[:max(k - 1, 0)]", TOPK_PINS),
    ("topk: selection order, not ascending", "topk_select", "np.sort(order[:k])", "(order[:k])", TOPK_PINS),
    ("topk rows: row length ignored", "topk_rows", "scores[r, : int(lens[r])]", "scores[r]",
     [P.test_topk_rows_tail_is_minus_one]),
    # softmax attention shared by the decode calls
    ("attention: scale dropped", "_softmax_attention", "s = scale * (q @ keys.T)", "s = q @ keys.T", DECODE_PINS),
    ("attention: unnormalised output", "_softmax_attention", "return p @ values", "return e @ values",
     DECODE_PINS),
    ("attention: lse without the log", "_softmax_attention", "(m + np.log(l))", "(m + l)", DECODE_PINS),
    ("attention: lse of the wrong sign", "_softmax_attention", "(m + np.log(l))", "(m - np.log(l))",
     DECODE_PINS),
    # decode anchor (R5, R6)
    ("decode anchor: pooled sum, not mean", "decode_anchor", "pb[h] = p.mean(axis=0)",
     "pb[h] = p.sum(axis=0)", DECODE_PINS),
    ("decode anchor: pooled from one query head", "decode_anchor", "pb[h] = p.mean(axis=0)", "pb[h] = p[0]",
     DECODE_PINS),
    ("decode anchor: GQA group shifted", "decode_anchor", "heads = slice(h * G, (h + 1) * G)",
     "heads = slice(h, h + G)", DECODE_PINS),
    ("decode anchor: last key dropped", "decode_anchor", "T = int(seq_len[b])", "T = int(seq_len[b]) - 1",
     DECODE_PINS),
    # decode reuse (head map, R7)
    ("decode reuse: head map ignored", "decode_reuse", "J = idx[b, a, : int(idx_k[b, a])]",
     "J = idx[b, h, : int(idx_k[b, h])]", REUSE_D_PINS),
    ("decode reuse: anchor head's K/V", "decode_reuse", "kb[h, J], vb[h, J]", "kb[a, J], vb[a, J]",
     REUSE_D_PINS),
    ("decode reuse: one index short", "decode_reuse", ": int(idx_k[b, a])]", ": int(idx_k[b, a]) - 1]",
     REUSE_D_PINS),
    # prefill anchor (causal rows, tile pooling)
    ("prefill anchor: strict causal mask", "prefill_anchor", "causal = cols[None, :] <= rows[:, None]",
     "causal = cols[None, :] < rows[:, None]", PREFILL_PINS),
    ("prefill anchor: pooled / tile only", "prefill_anchor", "acc / (tile * G)", "acc / tile", PREFILL_PINS),
    ("prefill anchor: pooled keys shifted", "prefill_anchor", "acc += p[:, :start].sum(axis=0)",
     "acc += p[:, 1:start + 1].sum(axis=0)", PREFILL_PINS),
    ("prefill anchor: lse of the wrong sign", "prefill_anchor", "lse[g, rows] = (m + np.log(l))[:, 0]",
     "lse[g, rows] = (m - np.log(l))[:, 0]", [_p(P.test_prefill_anchor_pooled_brute_force, 0)]),
    # prefill reuse (prefix indices + causal diagonal block)
    ("prefill reuse: diagonal block not causal", "prefill_reuse", "causal = diag[None, :] <= rows[:, None]",
     "causal = diag[None, :] >= 0 * rows[:, None]", REUSE_P_PINS),
    ("prefill reuse: head map ignored", "prefill_reuse", "J = idx[t, a, : int(idx_k[t, a])]",
     "J = idx[t, h, : int(idx_k[t, h])]", REUSE_P_PINS),
    ("prefill reuse: diagonal block shifted", "prefill_reuse", "keys = np.concatenate([J, diag])",
     "keys = np.concatenate([J, diag - 1])", REUSE_P_PINS),
    # layer schedule (R9)
    ("schedule: following anchor", "anchor_for_layer", "prior = [a for a in anchors if a <= layer]",
     "prior = [a for a in anchors if a >= layer] or [0]", [P.test_schedule_golden]),
    ("schedule: strictly preceding anchor", "anchor_for_layer", "if a <= layer]", "if a < layer] or [0]",
     [P.test_schedule_golden]),
    # similarity (sim equation)
    ("sim: ratio inverted", "similarity", "row_b[ia].sum() / row_b[ib].sum()",
     "row_b[ib].sum() / row_b[ia].sum()", SIM_PINS),
    ("sim: mass from layer a", "similarity", "row_b[ia].sum() / row_b[ib].sum()",
     "row_a[ia].sum() / row_a[ib].sum()", SIM_PINS),
    ("sim: indices of layer b only", "similarity", "ia = topk_select(row_a, k)", "ia = topk_select(row_b, k)",
     SIM_PINS),
    # weighted similarity and DP (Algorithm 1; R13, R14)
    ("weights on the anchor layer", "weighted_similarity_matrix", "float(w[l]) * sim[i, l]",
     "float(w[i]) * sim[i, l]", DP_PINS),
    ("weights dropped", "weighted_similarity_matrix", "float(w[l]) * sim[i, l]", "sim[i, l]", DP_PINS),
    ("dp: cover includes layer j", "select_anchors_dp", "run += S[i, j - 1]", "run += S[i, min(j, L - 1)]",
     DP_PINS),
    ("dp: ties keep the last i", "select_anchors_dp", "if val > best:", "if val >= best:", DP_PINS),
    ("dp: i starts at m", "select_anchors_dp", "for i in range(m - 1, j):", "for i in range(m, j):", DP_PINS),
    # head remap
    ("remap: similarity direction swapped", "head_remap", "similarity(p_anchor[a], p_reuse[h], k)",
     "similarity(p_reuse[h], p_anchor[a], k)", REMAP_PINS),
    ("remap: ties to the higher head", "head_remap", "out[h] = int(np.argmax(scores))",
     "out[h] = len(scores) - 1 - int(np.argmax(scores[::-1]))", REMAP_PINS),
]


@pytest.mark.parametrize("label,name,old,new,pins", CASES, ids=[c[0] for c in CASES])
def test_a_pin_catches_the_planted_mistake(monkeypatch, label, name, old, new, pins):
    mutant = _mutant(name, old, new)
    monkeypatch.setattr(K, name, mutant)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, mutant)
    failed = []
    for pin in pins:
        try:
            pin()
        except Exception as e:  # an assertion, or the mutant breaking outright
            failed.append(f"{getattr(pin, 'func', pin).__name__}: {type(e).__name__}")
    assert failed, f"no pin fails on the planted mistake '{label}'"


def test_unmutated_copies_pass_every_pin(monkeypatch):
    # the rewrite machinery itself changes nothing: identity edits pass all pins
    for name in sorted({c[1] for c in CASES}):
        src = textwrap.dedent(inspect.getsource(getattr(K, name)))
        first = src.splitlines()[0]
        copy = _mutant(name, first, first)
        monkeypatch.setattr(K, name, copy)
        if hasattr(oracle, name):
            monkeypatch.setattr(oracle, name, copy)
    for pins in (TOPK_PINS, DECODE_PINS, PREFILL_PINS, REUSE_D_PINS, REUSE_P_PINS, DP_PINS, SIM_PINS,
                 REMAP_PINS, K_PINS, [P.test_schedule_golden, P.test_topk_rows_tail_is_minus_one]):
        for pin in pins:
            pin()
