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
