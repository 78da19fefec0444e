"""Planted mistakes in the oracle must be caught by its pins.

Each mutant replaces one oracle helper with a plausibly wrong version (a
dropped scale, a dropped gate bias, a flipped sign in the gate Jacobian, an
off-by-one causal mask or history length, ties to the wrong index, a dropped
term of the log-sum-exp) and the listed pins must fail under it. This runs
on the CPU only and never touches the CUDA path.
"""
import math

import numpy as np
import pytest

from oracle import sas_oracle as O
from tests import test_oracle as P
from tests import test_oracle_variants as V
from tests import test_oracle_paged as PG
from tests import test_oracle_selector as SEL


def _no_scale(d, scale):
    return 1.0


def _key_set_no_bias(j, b, T, sel_row, logg_row, use_gates):
    cols, bias, nh = ORIG["_key_set"](j, b, T, sel_row, logg_row, use_gates)
    return cols, np.zeros_like(bias), nh


def _dscores_sign(da, gates_row, n):
    out = ORIG["dscores_row"](da, gates_row, n)
    g = np.asarray(gates_row[:n], np.float64)
    return out + 2 * g * sum(da.values())


def _mask_strict(Qb, Kc, bias, nh, scale, row0, col0_cur):
    return ORIG["_block_logits"](Qb, Kc, bias, nh, scale, row0 - 1, col0_cur)


def _topk_high_ties(s_row_f32, n, K):
    vals = [float(np.float32(x)) for x in s_row_f32[:n]]
    order = sorted(range(n), key=lambda m: (-vals[m], -m))
    sel = order[:min(K, n)]
    return sel + [-1] * (K - len(sel))


def _lse_one_more(s_row, n):
    s = np.asarray(s_row, np.float64)
    m = min(n + 1, len(s))
    if n == 0:
        return s[:0]
    full = s[:m]
    lse = full.max() + math.log(np.exp(full - full.max()).sum())
    return s[:n] - lse


def _lse_max_only(X):
    return X.max(axis=1)


ORIG = {name: getattr(O, name) for name in
        ("_default_scale", "_key_set", "dscores_row", "_block_logits", "topk_row",
         "log_gates_row", "_lse_rows")}

ORIG_V = {name: getattr(O, name) for name in
          ("dscores_row_phi", "log_gates_row_phi", "attn_bwd_outer_block", "_col_gates",
           "decode_paged")}


def _paged_pages_reversed(q, kpages, vpages, page_indptr, page_indices, seq_lens, idx, logg, b,
                          scale=0.0, use_gates=False):
    ix = np.asarray(page_indices).copy()
    for bi in range(len(page_indptr) - 1):
        lo, hi = page_indptr[bi], page_indptr[bi + 1]
        ix[lo:hi] = ix[lo:hi][::-1]
    return ORIG_V["decode_paged"](q, kpages, vpages, page_indptr, ix, seq_lens, idx, logg, b,
                                  scale, use_gates)


def _sigmoid_jacobian_flipped(da, s_row, n, phi):
    out = ORIG_V["dscores_row_phi"](da, s_row, n, phi)
    if phi == "sigmoid":
        s = np.asarray(s_row[:n], np.float64)
        for m, a in da.items():
            out[m] = a / (1.0 + np.exp(-s[m]))  # sigma(s) where 1 - sigma(s) belongs
    return out


def _sigmoid_log_gate_sign(s_row, n, phi):
    if phi == "sigmoid":
        return -np.logaddexp(0.0, np.asarray(s_row[:n], np.float64))
    return ORIG_V["log_gates_row_phi"](s_row, n, phi)


def _outer_da_without_gate(q, k, v, dO, idx, gates, bi, kvh, j, b, scale=0.0, operands=None):
    r = ORIG_V["attn_bwd_outer_block"](q, k, v, dO, idx, gates, bi, kvh, j, b, scale, operands)
    r["da"] = {m: a / float(gates[bi, kvh, j, m]) for m, a in r["da"].items()}
    return r


def _current_block_gated(j, b, T, sel_row, gates_row):
    w = ORIG_V["_col_gates"](j, b, T, sel_row, gates_row)
    ncur = min(T, (j + 1) * b) - j * b
    w[len(w) - ncur:] = 0.5
    return w


ORIG_S = O.block_summaries


def _summaries_summed(x, b):
    """Block summaries as sums instead of means."""
    return ORIG_S(x, b) * b


def _pin(fn, *args):
    def run():
        fn(*args)
    run.__name__ = fn.__name__ + "".join(f"[{a}]" for a in args)
    return run


MUTANTS = {
    "dropped 1/sqrt(d)": ("_default_scale", _no_scale,
                          [P.test_golden_scale, P.test_fwd_reduces_to_dense_causal]),
    "dropped log-gate bias": ("_key_set", _key_set_no_bias,
                              [P.test_golden_zero_query_gated,
                               P.test_fwd_gates_on_all_selected_is_block_masked_sdpa]),
    "flipped Jacobian sign": ("dscores_row", _dscores_sign,
                              [P.test_bwd_finite_differences, P.test_dscores_rows_sum_to_zero]),
    "off-by-one causal mask": ("_block_logits", _mask_strict,
                               [P.test_fwd_reduces_to_dense_causal, P.test_golden_zero_query_gated]),
    "ties to higher index": ("topk_row", _topk_high_ties,
                             [P.test_golden_topk_ties, P.test_topk_all_equal_rows]),
    "history length + 1": ("log_gates_row", _lse_one_more,
                           [P.test_golden_gate_softmax, P.test_gates_sum_to_one_and_positive]),
    "lse without the sum": ("_lse_rows", _lse_max_only,
                            [P.test_fwd_reduces_to_dense_causal, P.test_golden_scale]),
    "sigmoid Jacobian uses sigma(s)": ("dscores_row_phi", _sigmoid_jacobian_flipped,
                                       [_pin(V.test_inner_gating_finite_differences, "sigmoid")]),
    "sigmoid log gate of -s": ("log_gates_row_phi", _sigmoid_log_gate_sign,
                               [V.test_sigmoid_gates_are_the_logistic_function]),
    "outer da without g_m": ("attn_bwd_outer_block", _outer_da_without_gate,
                             [V.test_eq5_outer_gate_gradient,
                              _pin(V.test_outer_gating_finite_differences, "softmax")]),
    "outer gate on the current block": ("_col_gates", _current_block_gated,
                                        [V.test_outer_with_unit_gates_is_ungated_sparse_attention,
                                         V.test_outer_backward_matches_autograd]),
    "selector: summed instead of mean-pooled": ("block_summaries", _summaries_summed,
                                                [SEL.test_scores_equal_mean_of_pair_logits,
                                                 SEL.test_constant_and_partial_blocks]),
    "paged: pages in reverse order": ("decode_paged", _paged_pages_reversed,
                                      [PG.test_uniform_lengths_equal_contiguous_decode,
                                       PG.test_full_selection_is_attention_of_the_last_token]),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn, pins = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for pin in pins:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the mutant '{name}'"
