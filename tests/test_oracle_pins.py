"""Pins for the CPU oracle: checks against facts outside the oracle itself.

Each test targets a plausible mistake (a dropped bias, a swapped gate/up, a
transposed W_down, a wrong threshold direction, an unstable or ascending sort)
and checks the oracle against a closed form, an identity of the FFN, a hand
computation, a library routine or brute force.  No GPU is used.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ffn(rng, act, d, n, bias_scale=0.5):
    Wg = rng.standard_normal((n, d)) / math.sqrt(d) if act == "reglu" else None
    Wu = rng.standard_normal((n, d)) / math.sqrt(d)
    WdT = rng.standard_normal((n, d)) / math.sqrt(n)
    bias = bias_scale * rng.standard_normal(n)
    return Wg, Wu, WdT, bias


ACTS = ["reglu", "relu"]


# ----------------------------------------------------------------- FFN pins --
def test_hand_worked_example_reglu():
    # d = 2, n = 2, worked by hand:
    #   gate pre = [1*1 + 0*2 + 0.5, 0*1 - 1*2 + 0] = [1.5, -2] -> ReLU [1.5, 0]
    #   up       = [0*1 + 1*2, 1*1 + 1*2]           = [2, 3]
    #   a = [3, 0];  y = 3 * WdT[0] + 0 * WdT[1] = [3, 6]
    # Swapping gate and up would give ReLU([2.5, 3]) * [1, -2] -> y = [-15.5, -19].
    x = np.array([1.0, 2.0])
    Wg = np.array([[1.0, 0.0], [0.0, -1.0]])
    Wu = np.array([[0.0, 1.0], [1.0, 1.0]])
    WdT = np.array([[1.0, 2.0], [3.0, 4.0]])
    b = np.array([0.5, 0.0])
    y = O.dense_ffn("reglu", Wg, Wu, WdT, b, x)
    np.testing.assert_array_equal(y, [[3.0, 6.0]])
    np.testing.assert_array_equal(O.sparse_ffn("reglu", Wg, Wu, WdT, b, x, [1]), [[0.0, 0.0]])


def test_hand_worked_example_relu():
    # up pre = [0*1 + 1*2 - 3, 1*1 + 1*2 + 0] = [-1, 3] -> a = [0, 3]
    # y = 3 * WdT[1] = [9, 12]; a transposed W_down would give 3 * [2, 4] = [6, 12].
    x = np.array([1.0, 2.0])
    Wu = np.array([[0.0, 1.0], [1.0, 1.0]])
    WdT = np.array([[1.0, 2.0], [3.0, 4.0]])
    b = np.array([-3.0, 0.0])
    np.testing.assert_array_equal(O.dense_ffn("relu", None, Wu, WdT, b, x), [[9.0, 12.0]])


@pytest.mark.parametrize("act", ACTS)
def test_saturated_positive_bias_is_linear_algebra(act):
    # With every ReLU input positive the ReLU is the identity, so the FFN
    # reduces to plain matrix products with W_down = WdT^T.
    rng = np.random.default_rng(1)
    d, n, B = 24, 40, 3
    Wg, Wu, WdT, _ = _ffn(rng, act, d, n)
    b = np.full(n, 50.0)
    X = rng.standard_normal((B, d))
    assert (O.relu_input(act, Wg, Wu, b, X) > 0).all()
    y = O.dense_ffn(act, Wg, Wu, WdT, b, X)
    Wdown = WdT.T
    for t in range(B):
        if act == "reglu":
            ref = Wdown @ ((Wg @ X[t] + b) * (Wu @ X[t]))
        else:
            ref = Wdown @ (Wu @ X[t] + b)
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


@pytest.mark.parametrize("act", ACTS)
def test_saturated_negative_bias_gives_exact_zero(act):
    rng = np.random.default_rng(2)
    Wg, Wu, WdT, _ = _ffn(rng, act, 16, 30)
    y = O.dense_ffn(act, Wg, Wu, WdT, np.full(30, -50.0), rng.standard_normal((2, 16)))
    assert np.array_equal(y, np.zeros_like(y))


@pytest.mark.parametrize("act", ACTS)
def test_odd_even_identity(act):
    # Zero bias.  ReLU(v) - ReLU(-v) = v and ReLU(v) + ... give closed forms:
    #   plain ReLU FFN:  y(x) - y(-x) = W_down W_up x
    #   ReGLU:           y(x) + y(-x) = W_down ((W_gate x) * (W_up x))
    rng = np.random.default_rng(3)
    d, n = 20, 33
    Wg, Wu, WdT, _ = _ffn(rng, act, d, n)
    b = np.zeros(n)
    x = rng.standard_normal(d)
    yp = O.dense_ffn(act, Wg, Wu, WdT, b, x)[0]
    ym = O.dense_ffn(act, Wg, Wu, WdT, b, -x)[0]
    if act == "relu":
        np.testing.assert_allclose(yp - ym, WdT.T @ (Wu @ x), rtol=1e-11, atol=1e-13)
    else:
        np.testing.assert_allclose(yp + ym, WdT.T @ ((Wg @ x) * (Wu @ x)), rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("act,degree", [("relu", 1), ("reglu", 2)])
def test_positive_homogeneity(act, degree):
    rng = np.random.default_rng(4)
    Wg, Wu, WdT, _ = _ffn(rng, act, 12, 25)
    b = np.zeros(25)
    x = rng.standard_normal(12)
    y1 = O.dense_ffn(act, Wg, Wu, WdT, b, x)
    y2 = O.dense_ffn(act, Wg, Wu, WdT, b, 2.0 * x)
    np.testing.assert_allclose(y2, (2.0 ** degree) * y1, rtol=1e-14, atol=0)


@pytest.mark.parametrize("act", ACTS)
def test_sparse_on_true_set_equals_dense(act):
    rng = np.random.default_rng(5)
    d, n = 48, 200
    Wg, Wu, WdT, _ = _ffn(rng, act, d, n)
    b = -1.0 * np.ones(n)            # about 16% of neurons active
    for t in range(4):
        x = rng.standard_normal(d)
        T = np.flatnonzero(O.true_active(act, Wg, Wu, b, x)[0])
        assert 0 < T.size < n
        yd = O.dense_ffn(act, Wg, Wu, WdT, b, x)
        ys = O.sparse_ffn(act, Wg, Wu, WdT, b, x, T)
        np.testing.assert_allclose(ys, yd, rtol=0, atol=1e-13 * np.abs(yd).max())
        # any superset of T gives the same output
        extra = rng.choice(n, size=n // 3, replace=False)
        sup = np.union1d(T, extra)
        np.testing.assert_allclose(O.sparse_ffn(act, Wg, Wu, WdT, b, x, sup), yd,
                                   rtol=0, atol=1e-13 * np.abs(yd).max())
        # inactive neurons contribute exactly zero
        comp = np.setdiff1d(np.arange(n), T)
        assert np.array_equal(O.sparse_ffn(act, Wg, Wu, WdT, b, x, comp), np.zeros((1, d)))


@pytest.mark.parametrize("act", ACTS)
def test_all_neurons_equals_dense(act):
    rng = np.random.default_rng(6)
    Wg, Wu, WdT, b = _ffn(rng, act, 16, 40)
    x = rng.standard_normal((3, 16))
    np.testing.assert_array_equal(O.sparse_ffn(act, Wg, Wu, WdT, b, x, np.arange(40)),
                                  O.dense_ffn(act, Wg, Wu, WdT, b, x))


@pytest.mark.parametrize("act", ACTS)
def test_bruteforce_all_masks_tiny(act):
    # d = 8, n = 10: every one of the 1024 index sets.  The output must be the sum
    # of single-neuron outputs (linearity in the index set), the true set must
    # reproduce the dense output, and empty sets give zero.
    rng = np.random.default_rng(7)
    d, n = 8, 10
    Wg, Wu, WdT, b = _ffn(rng, act, d, n)
    x = rng.standard_normal(d)
    single = [O.sparse_ffn(act, Wg, Wu, WdT, b, x, [k])[0] for k in range(n)]
    yd = O.dense_ffn(act, Wg, Wu, WdT, b, x)[0]
    T = set(np.flatnonzero(O.true_active(act, Wg, Wu, b, x)[0]).tolist())
    for bits in itertools.product([0, 1], repeat=n):
        idx = [k for k in range(n) if bits[k]]
        y = O.sparse_ffn(act, Wg, Wu, WdT, b, x, idx)[0]
        ref = np.zeros(d)
        for k in idx:
            ref = ref + single[k]
        np.testing.assert_allclose(y, ref, rtol=0, atol=1e-14)
        if set(idx) >= T:
            np.testing.assert_allclose(y, yd, rtol=0, atol=1e-14)
        if not (set(idx) & T):
            assert np.array_equal(y, np.zeros(d))


def test_batch_rows_are_independent_tokens():
    rng = np.random.default_rng(8)
    Wg, Wu, WdT, b = _ffn(rng, "reglu", 10, 20)
    X = rng.standard_normal((4, 10))
    idx = np.array([1, 3, 4, 9, 15])
    Y = O.sparse_ffn("reglu", Wg, Wu, WdT, b, X, idx)
    for t in range(4):
        np.testing.assert_allclose(Y[t], O.sparse_ffn("reglu", Wg, Wu, WdT, b, X[t], idx)[0],
                                   rtol=0, atol=1e-15)


# ----------------------------------------------------------- predictor pins --
def test_predictor_identity_construction():
    # d = r = n = 4, W1 = I, b1 = 0, W2 = permutation (W2[k, P[k]] = 1):
    # z_k = max(x[P[k]], 0) + b2_k.  Worked by hand for x, P, b2 below:
    #   x = [0.5, -1.0, 2.0, 0.25], P = [2, 0, 3, 1], b2 = [-1, -0.4, 0, 0.1]
    #   z = [2-1, 0.5-0.4, 0.25+0, 0+0.1] = [1.0, 0.1, 0.25, 0.1]
    # tau = 0.5 (threshold 0): all four active.  tau = sigmoid(0.2) (threshold 0.2):
    # only neurons 0 and 2.  A transposed W2 would give z = [0.5-1, ...] = [-0.5, ...].
    x = np.array([0.5, -1.0, 2.0, 0.25])
    P = [2, 0, 3, 1]
    W2 = np.zeros((4, 4))
    for k, j in enumerate(P):
        W2[k, j] = 1.0
    b2 = np.array([-1.0, -0.4, 0.0, 0.1])
    z = O.predictor_logits(np.eye(4), np.zeros(4), W2, b2, x)
    np.testing.assert_allclose(z, [[1.0, 0.1, 0.25, 0.1]], rtol=0, atol=1e-15)
    idx, _ = O.predict(np.eye(4), np.zeros(4), W2, b2, x, 0.5)
    assert idx.tolist() == [0, 1, 2, 3]
    tau = 1.0 / (1.0 + math.exp(-0.2))
    idx, _ = O.predict(np.eye(4), np.zeros(4), W2, b2, x, tau)
    assert idx.tolist() == [0, 2]


def test_predictor_hidden_relu_and_bias():
    # h = ReLU(W1 x + b1): with W1 = I, b1 = [1, -3, 0]: x = [-2, 2, 5] -> [0, 0, 5]
    h = O.predictor_hidden(np.eye(3), np.array([1.0, -3.0, 0.0]), np.array([-2.0, 2.0, 5.0]))
    np.testing.assert_array_equal(h, [[0.0, 0.0, 5.0]])


def _rand_pred(rng, d, r, n):
    W1 = rng.standard_normal((r, d)) / math.sqrt(d)
    b1 = 0.1 * rng.standard_normal(r)
    W2 = rng.standard_normal((n, r)) / math.sqrt(r)
    b2 = rng.standard_normal(n)
    return W1, b1, W2, b2


@pytest.mark.parametrize("tau", [0.05, 0.3, 0.45, 0.5, 0.62, 0.9])
def test_threshold_matches_scalar_sigmoid(tau):
    rng = np.random.default_rng(9)
    W1, b1, W2, b2 = _rand_pred(rng, 16, 12, 300)
    X = rng.standard_normal((5, 16))
    z = O.predictor_logits(W1, b1, W2, b2, X)
    m = O.predictor_mask(W1, b1, W2, b2, X, tau)
    thr = math.log(tau / (1 - tau))
    checked = 0
    for t in range(5):
        for k in range(300):
            if abs(z[t, k] - thr) < 1e-9:
                continue
            assert m[t, k] == (1.0 / (1.0 + math.exp(-z[t, k])) > tau)
            checked += 1
    assert checked > 1400


def test_tau_half_is_sign_and_extremes():
    rng = np.random.default_rng(10)
    W1, b1, W2, b2 = _rand_pred(rng, 8, 8, 100)
    X = rng.standard_normal((3, 8))
    z = O.predictor_logits(W1, b1, W2, b2, X)
    assert np.array_equal(O.predictor_mask(W1, b1, W2, b2, X, 0.5), z > 0)
    assert O.predictor_mask(W1, b1, W2, b2, X, 1e-300).all()
    assert not O.predictor_mask(W1, b1, W2, b2, X, 1.0 - 2.0 ** -52).any()
    with pytest.raises(ValueError):
        O.logit(0.0)
    with pytest.raises(ValueError):
        O.logit(1.0)


def test_mask_monotone_in_tau():
    rng = np.random.default_rng(11)
    W1, b1, W2, b2 = _rand_pred(rng, 8, 8, 200)
    X = rng.standard_normal((2, 8))
    prev = None
    for tau in [0.1, 0.2, 0.4, 0.5, 0.7, 0.95]:
        m = O.predictor_mask(W1, b1, W2, b2, X, tau)
        if prev is not None:
            assert not (m & ~prev).any()
        prev = m


def test_compact_matches_library_and_union():
    rng = np.random.default_rng(12)
    for n in [1, 31, 32, 33, 1000, 1376]:
        m = rng.random(n) < 0.1
        np.testing.assert_array_equal(O.compact(m), np.flatnonzero(m).astype(np.int32))
        M = rng.random((5, n)) < 0.1
        np.testing.assert_array_equal(O.compact(M), np.flatnonzero(M.any(axis=0)))
    assert O.compact(np.zeros(10, bool)).size == 0
    np.testing.assert_array_equal(O.compact(np.ones(7, bool)), np.arange(7))
    assert O.compact(np.zeros(10, bool)).dtype == np.int32


def test_union_prediction_properties():
    rng = np.random.default_rng(13)
    W1, b1, W2, b2 = _rand_pred(rng, 8, 16, 120)
    X = rng.standard_normal((6, 8))
    idx, masks = O.predict(W1, b1, W2, b2, X, 0.5)
    assert np.all(np.diff(idx) > 0)
    for t in range(6):
        single, _ = O.predict(W1, b1, W2, b2, X[t], 0.5)
        assert set(single.tolist()) <= set(idx.tolist())
        np.testing.assert_array_equal(single, np.flatnonzero(masks[t]))
    same, _ = O.predict(W1, b1, W2, b2, np.stack([X[0]] * 4), 0.5)
    np.testing.assert_array_equal(same, O.predict(W1, b1, W2, b2, X[0], 0.5)[0])


# ------------------------------------------------------------ profiler pins --
def test_guide_harness_profile_golden():
    g = json.load(open(os.path.join(GOLDEN, "guide_harness_profile.json")))
    n, T = g["intermediate_size"], g["calib_tokens"]
    rng = np.random.default_rng(2024)
    acts = np.zeros((T, n))
    hb = g["heavy_block"]
    acts[:, :hb] = rng.random((T, hb)) > 1.0 - g["p_heavy"]
    acts[:, hb:] = rng.random((T, n - hb)) > 1.0 - g["p_light"]
    counts = O.record_activations(acts)
    hot, cold, share = O.partition(counts, g["gpu_budget_ratio"])
    assert hot.size == g["k_hot"] and cold.size == n - g["k_hot"]
    assert abs(share - g["hot_share_expected"]) < g["hot_share_tolerance"]
    assert set(range(hb)) <= set(hot.tolist())
    mask = np.zeros(n, dtype=bool)
    mask[hot[:g["mask_hot_active"]]] = True
    mask[cold[:g["mask_cold_active"]]] = True
    idx = O.compact(mask)
    assert idx.size == g["active_count"]
    assert f"{idx.size / n * 100:.2f}" == g["active_percent_2dp"]


def test_record_activations_matches_library():
    rng = np.random.default_rng(14)
    a = np.maximum(rng.standard_normal((2, 7, 50)), 0) * (rng.random((2, 7, 50)) < 0.3)
    np.testing.assert_array_equal(O.record_activations(a), (a.reshape(-1, 50) > 0).sum(axis=0))


def test_hot_permutation_is_stable_descending_argsort():
    rng = np.random.default_rng(15)
    for n in [1, 2, 17, 500, 4096]:
        counts = rng.integers(0, 6, size=n)          # many ties
        perm = O.hot_permutation(counts)
        np.testing.assert_array_equal(perm, np.argsort(-counts, kind="stable"))
        assert sorted(perm.tolist()) == list(range(n))
    # hand case: ties resolved to the lower id
    assert O.hot_permutation([3, 5, 3, 9, 5]).tolist() == [3, 1, 4, 0, 2]
    # inverse of a 3-cycle: perm [1, 2, 0] sends storage 0 -> id 1, so inv[1] = 0
    assert O.inverse_permutation([1, 2, 0]).tolist() == [2, 0, 1]


@pytest.mark.parametrize("act", ACTS)
def test_profile_counts_match_true_active_sum(act):
    rng = np.random.default_rng(16)
    Wg, Wu, WdT, _ = _ffn(rng, act, 32, 64)
    b = -0.5 * np.ones(64)
    X = rng.standard_normal((40, 32))
    c = O.profile_counts(act, Wg, Wu, b, X)
    pre = (Wg if act == "reglu" else Wu) @ X.T + b[:, None]
    np.testing.assert_array_equal(c, (pre > 0).sum(axis=1))


@pytest.mark.parametrize("act", ACTS)
def test_permutation_equivariance(act):
    rng = np.random.default_rng(17)
    d, n = 24, 90
    Wg, Wu, WdT, b = _ffn(rng, act, d, n)
    W1, b1, W2, b2 = _rand_pred(rng, d, 16, n)
    X = rng.standard_normal((3, d))
    perm = rng.permutation(n).astype(np.int32)
    P = lambda M: None if M is None else O.permute_rows(M, perm)
    idx, _ = O.predict(W1, b1, W2, b2, X, 0.5)
    idx_p, _ = O.predict(W1, b1, P(W2), P(b2), X, 0.5)
    inv = O.inverse_permutation(perm)
    # same neurons, expressed in storage order of the permuted layout
    assert set(idx_p.tolist()) == set(inv[idx].tolist())
    assert np.all(np.diff(idx_p) > 0)
    y = O.sparse_ffn(act, Wg, Wu, WdT, b, X, idx)
    y_p = O.sparse_ffn(act, P(Wg), P(Wu), P(WdT), P(b), X, idx_p)
    np.testing.assert_allclose(y_p, y, rtol=0, atol=1e-13 * max(1.0, np.abs(y).max()))


# ---------------------------------------------------------------- band pins --
def _dot32_sequential(w, v):
    acc = np.float32(0.0)
    for a, c in zip(w.astype(np.float32), v.astype(np.float32)):
        acc = np.float32(acc + np.float32(a * c))
    return acc


def test_predictor_band_covers_binary32_evaluations():
    rng = np.random.default_rng(18)
    d, r, n = 64, 32, 80
    W1 = (rng.standard_normal((r, d)) / 8).astype(np.float16)
    W2 = (rng.standard_normal((n, r)) / 6).astype(np.float16)
    b1 = (0.1 * rng.standard_normal(r)).astype(np.float32)
    b2 = rng.standard_normal(n).astype(np.float32)
    X = rng.standard_normal((3, d)).astype(np.float16)
    z64 = O.predictor_logits(W1, b1, W2, b2, X)
    band = O.predictor_band(W1, b1, W2, b2, X, 0.5)
    for t in range(3):
        # two binary32 evaluations in different orders
        h32a = np.maximum(W1.astype(np.float32) @ X[t].astype(np.float32) + b1, 0)
        za = W2.astype(np.float32) @ h32a + b2
        h32b = np.array([max(np.float32(_dot32_sequential(W1[j][::-1], X[t][::-1]) + b1[j]), 0)
                         for j in range(r)], dtype=np.float32)
        zb = np.array([np.float32(_dot32_sequential(W2[k], h32b) + b2[k]) for k in range(n)])
        assert np.all(np.abs(za - z64[t]) <= band[t])
        assert np.all(np.abs(zb - z64[t]) <= band[t])
    # the band is a small fraction of the spread of z, so decisions are mostly unique
    assert np.median(band) < 0.01 * z64.std()


def test_relu_input_band_covers_binary32_evaluations():
    rng = np.random.default_rng(19)
    d, n = 128, 60
    W = (rng.standard_normal((n, d)) / 11).astype(np.float16)
    b = (0.3 * rng.standard_normal(n)).astype(np.float32)
    X = rng.standard_normal((2, d)).astype(np.float16)
    pre = O.relu_input("relu", None, W, b, X)
    band = O.relu_input_band("relu", None, W, b, X)
    for t in range(2):
        p32 = np.array([np.float32(_dot32_sequential(W[k], X[t]) + b[k]) for k in range(n)])
        assert np.all(np.abs(p32 - pre[t]) <= band[t])
