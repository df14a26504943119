"""Plant plausible mistakes in the oracle (on the CPU) and check the pins catch each.

Every mutant replaces one oracle function inside ``oracle.ffn`` for the length
of one test; the pins from ``test_oracle_pins`` must then fail.
"""
import numpy as np
import pytest

import oracle
import oracle.ffn as F
from tests import test_oracle_pins as P


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def m_swap_gate_up(act, Wg, Wu, bias, x, idx):
    X = F._tokens(x)
    idx = np.asarray(idx, dtype=np.int64)
    if act == "reglu":
        pre = X @ _f64(Wu)[idx].T + _f64(bias)[idx][None, :]
        return np.maximum(pre, 0.0) * (X @ _f64(Wg)[idx].T)
    return np.maximum(X @ _f64(Wu)[idx].T + _f64(bias)[idx][None, :], 0.0)


def m_drop_bias(act, Wg, Wu, bias, x, idx):
    return F_orig_activations(act, Wg, Wu, np.zeros_like(_f64(bias)), x, idx)


def m_bias_on_up(act, Wg, Wu, bias, x, idx):
    X = F._tokens(x)
    idx = np.asarray(idx, dtype=np.int64)
    b = _f64(bias)[idx][None, :]
    if act == "reglu":
        return np.maximum(X @ _f64(Wg)[idx].T, 0.0) * (X @ _f64(Wu)[idx].T + b)
    return np.maximum(X @ _f64(Wu)[idx].T + b, 0.0)


def m_transposed_down(act, Wg, Wu, WdT, bias, x, idx):
    idx = np.asarray(idx, dtype=np.int64)
    X = F._tokens(x)
    W = _f64(WdT)
    if W.shape[0] != W.shape[1]:
        pytest.skip("mutant only defined for square layers")
    a = F.activations(act, Wg, Wu, bias, X, idx)
    return a @ W.T[idx]


def m_logit_sign(tau):
    return -F_orig_logit(tau)


def m_no_hidden_relu(W1, b1, x):
    return F._tokens(x) @ _f64(W1).T + _f64(b1)[None, :]


def m_intersection(mask):
    m = np.asarray(mask, dtype=bool)
    if m.ndim == 2:
        m = m.all(axis=0)
    return np.flatnonzero(m).astype(np.int32)


def m_ascending(counts):
    return np.argsort(np.asarray(counts), kind="stable").astype(np.int32)


def m_unstable(counts):
    c = np.asarray(counts)
    return np.lexsort((-np.arange(c.size), -c)).astype(np.int32)


def m_count_ge(post_act):
    a = np.asarray(post_act).reshape(-1, np.asarray(post_act).shape[-1])
    return (a >= 0).sum(axis=0).astype(np.int64)


F_orig_activations = F.activations
F_orig_logit = F.logit

MUTANTS = [
    ("activations", m_swap_gate_up, [P.test_hand_worked_example_reglu,
                                     lambda: P.test_saturated_positive_bias_is_linear_algebra("reglu")]),
    ("activations", m_drop_bias, [P.test_hand_worked_example_relu,
                                  lambda: P.test_saturated_negative_bias_gives_exact_zero("relu")]),
    ("activations", m_bias_on_up, [P.test_hand_worked_example_reglu,
                                   lambda: P.test_saturated_positive_bias_is_linear_algebra("reglu")]),
    ("sparse_ffn", m_transposed_down, [P.test_hand_worked_example_relu]),
    ("logit", m_logit_sign, [P.test_predictor_identity_construction,
                             lambda: P.test_threshold_matches_scalar_sigmoid(0.3)]),
    ("predictor_hidden", m_no_hidden_relu, [P.test_predictor_hidden_relu_and_bias,
                                            P.test_predictor_identity_construction]),
    ("compact", m_intersection, [P.test_compact_matches_library_and_union]),
    ("hot_permutation", m_ascending, [P.test_hot_permutation_is_stable_descending_argsort,
                                      P.test_guide_harness_profile_golden]),
    ("hot_permutation", m_unstable, [P.test_hot_permutation_is_stable_descending_argsort]),
    ("record_activations", m_count_ge, [P.test_record_activations_matches_library]),
]


@pytest.mark.parametrize("name,mutant,pins", MUTANTS,
                         ids=[f"{m[0]}-{m[1].__name__}" for m in MUTANTS])
def test_pins_catch_mutant(monkeypatch, name, mutant, pins):
    monkeypatch.setattr(F, name, mutant)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, mutant)
    for pin in pins:
        with pytest.raises((AssertionError, ValueError, IndexError)):
            pin()
