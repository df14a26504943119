"""CPU oracle for the activation-sparse FFN decode path (float64).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module; only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm may use it.  It shares no code with the CUDA path.

Every function takes the exact stored values (fp16 or fp32 arrays) and computes
in float64, step by step as the pages state it, with plain NumPy matrix
products as the only library primitive.  Sources:

* "PowerInfer Guide: Exploiting Activation Sparsity for LLM AI" (aifetchly),
  section "The Hidden Inefficiency": the gated FFN equation
  FFN(x) = W_down (sigma(W_gate x) * (W_up x)), with neurons that evaluate to
  exactly zero after sigma counted as inactive.
* same page, section 3 "Adaptive Online Neuron Predictors": the predictor
  equation  a_hat = sigma(x W_pred) > tau, and the Step 2 predictor module
  (linear layer with bias, sigmoid, strict ">" against the threshold).
* "PowerInfer_x64" (zingnex forum), "Prediction and Caching": the predictor is
  a 2-layer MLP, read here as d -> r (ReLU) -> d_ffn (sigmoid).
* PowerInfer Guide, Step 3 sparse FFN module: the plain ReLU FFN (up, ReLU,
  down) computed only over the active neurons.
* PowerInfer Guide, Step 1 profiler: counts of (post-activation > 0) per
  neuron over calibration tokens, then a descending sort of the counts; the
  first floor(beta * d_ffn) neurons are "hot".

Readings where the pages are silent (all listed in the design notes too):
bias of the FFN lives on the ReLU input (gate for ReGLU, up for ReLU); the
threshold test sigmoid(z) > tau is evaluated as z > logit(tau); for several
tokens the active set is the union of the per-token sets and every token is
computed over that union; index lists are ascending storage indices; ties in
the hot ordering go to the lower neuron id.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

U32 = 2.0 ** -24   # unit roundoff of IEEE binary32


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def _tokens(x) -> np.ndarray:
    x = _f64(x)
    return x[None, :] if x.ndim == 1 else x


# --------------------------------------------------------------------------- #
# predictor                                                                    #
# --------------------------------------------------------------------------- #
def logit(tau: float) -> float:
    """Inverse of the logistic sigmoid: sigmoid(z) > tau  <=>  z > logit(tau)."""
    if not (0.0 < tau < 1.0):
        raise ValueError("tau must lie strictly between 0 and 1")
    return math.log(tau / (1.0 - tau))


def predictor_hidden(W1, b1, x) -> np.ndarray:
    """First predictor layer: h = ReLU(W1 x + b1), shape [B, r]."""
    X = _tokens(x)
    pre = X @ _f64(W1).T + _f64(b1)[None, :]
    return np.maximum(pre, 0.0)


def predictor_logits(W1, b1, W2, b2, x) -> np.ndarray:
    """Second predictor layer: z = W2 h + b2, shape [B, n] (pre-sigmoid)."""
    h = predictor_hidden(W1, b1, x)
    return h @ _f64(W2).T + _f64(b2)[None, :]


def predictor_mask(W1, b1, W2, b2, x, tau: float) -> np.ndarray:
    """Per-token binary activation mask: sigmoid(z) > tau, strict, shape [B, n]."""
    return predictor_logits(W1, b1, W2, b2, x) > logit(tau)


def compact(mask) -> np.ndarray:
    """Ascending int32 indices of the set bits of a mask.

    A [B, n] mask is first reduced to the union over its B tokens.
    """
    m = np.asarray(mask, dtype=bool)
    if m.ndim == 2:
        union = np.zeros(m.shape[1], dtype=bool)
        for t in range(m.shape[0]):
            union |= m[t]
        m = union
    out = []
    for k in range(m.shape[0]):
        if m[k]:
            out.append(k)
    return np.array(out, dtype=np.int32)


def predict(W1, b1, W2, b2, x, tau: float) -> Tuple[np.ndarray, np.ndarray]:
    """predict(x) -> (ascending index list of the union of predicted sets, masks)."""
    mask = predictor_mask(W1, b1, W2, b2, x, tau)
    return compact(mask), mask


# --------------------------------------------------------------------------- #
# FFN                                                                          #
# --------------------------------------------------------------------------- #
def relu_input(act: str, Wg, Wu, bias, x, idx=None) -> np.ndarray:
    """Argument of the ReLU for the listed neurons, shape [B, count].

    ReGLU: W_gate[k] . x + b_k;  plain ReLU FFN: W_up[k] . x + b_k.
    """
    X = _tokens(x)
    W = np.asarray(Wg if act == "reglu" else Wu)
    b = np.asarray(bias)
    if idx is not None:
        idx = np.asarray(idx, dtype=np.int64)
        W = W[idx]
        b = b[idx]
    return X @ _f64(W).T + _f64(b)[None, :]


def activations(act: str, Wg, Wu, bias, x, idx) -> np.ndarray:
    """Post-activation value a_k of each listed neuron, shape [B, count].

    ReGLU: a_k = max(W_gate[k].x + b_k, 0) * (W_up[k].x)
    ReLU : a_k = max(W_up[k].x + b_k, 0)
    """
    X = _tokens(x)
    idx = np.asarray(idx, dtype=np.int64)
    pre = relu_input(act, Wg, Wu, bias, X, idx)
    if act == "reglu":
        up = X @ _f64(np.asarray(Wu)[idx]).T
        return np.maximum(pre, 0.0) * up
    if act == "relu":
        return np.maximum(pre, 0.0)
    raise ValueError("act must be 'reglu' or 'relu'")


def sparse_ffn(act: str, Wg, Wu, WdT, bias, x, idx) -> np.ndarray:
    """y = sum over listed k of a_k * W_down[:, k]  (W_down stored as WdT[k] rows).

    Every token is computed over the same index list.  Shape [B, d].
    """
    idx = np.asarray(idx, dtype=np.int64)
    X = _tokens(x)
    if idx.size == 0:
        return np.zeros((X.shape[0], np.asarray(WdT).shape[1]), dtype=np.float64)
    a = activations(act, Wg, Wu, bias, X, idx)
    return a @ _f64(np.asarray(WdT)[idx])


def dense_ffn(act: str, Wg, Wu, WdT, bias, x) -> np.ndarray:
    """The unsparsified FFN: every one of the n neurons is evaluated."""
    n = np.asarray(Wu).shape[0]
    return sparse_ffn(act, Wg, Wu, WdT, bias, x, np.arange(n))


def true_active(act: str, Wg, Wu, bias, x) -> np.ndarray:
    """T(x): neurons whose activation output is nonzero, i.e. ReLU input > 0. [B, n]"""
    return relu_input(act, Wg, Wu, bias, x) > 0.0


# --------------------------------------------------------------------------- #
# offline profiler and hot-neuron permutation                                  #
# --------------------------------------------------------------------------- #
def record_activations(post_act) -> np.ndarray:
    """Per-neuron count of tokens whose post-activation value is > 0 (int64 [n])."""
    a = np.asarray(post_act)
    a = a.reshape(-1, a.shape[-1])
    counts = np.zeros(a.shape[1], dtype=np.int64)
    for t in range(a.shape[0]):
        counts += (a[t] > 0).astype(np.int64)
    return counts


def profile_counts(act: str, Wg, Wu, bias, x_calib) -> np.ndarray:
    """Activation counts over calibration tokens: #tokens with ReLU input > 0."""
    return record_activations(true_active(act, Wg, Wu, bias, x_calib))


def hot_permutation(counts) -> np.ndarray:
    """Neuron ids ordered by descending count; equal counts keep ascending id."""
    c = [int(v) for v in np.asarray(counts).ravel()]
    order = sorted(range(len(c)), key=lambda k: (-c[k], k))
    return np.array(order, dtype=np.int32)


def partition(counts, ratio: float = 0.20):
    """Hot ids (first floor(ratio*n) of the descending order), cold ids, hot share."""
    c = np.asarray(counts, dtype=np.int64)
    k_hot = int(c.shape[0] * ratio)
    order = hot_permutation(c)
    hot, cold = order[:k_hot], order[k_hot:]
    share = float(c[hot].sum()) / max(1, int(c.sum()))
    return hot, cold, share


def permute_rows(M, perm) -> np.ndarray:
    """Row i of the result is row perm[i] of M."""
    M = np.asarray(M)
    return M[np.asarray(perm, dtype=np.int64)]


def inverse_permutation(perm) -> np.ndarray:
    """inv[perm[i]] = i: maps an original neuron id to its storage index."""
    perm = np.asarray(perm, dtype=np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.shape[0])
    return inv.astype(np.int32)


# --------------------------------------------------------------------------- #
# rounding bands for decisions taken in binary32 by an implementation          #
# --------------------------------------------------------------------------- #
def _gamma(m: int) -> float:
    """Worst-case relative error factor of an m-term binary32 sum/dot (m u / (1 - m u))."""
    return m * U32 / (1.0 - m * U32)


def predictor_band(W1, b1, W2, b2, x, tau: float) -> np.ndarray:
    """Bound on |z_fp32 - z| plus threshold rounding, per token and neuron [B, n].

    Assumes an implementation that forms h and z with binary32 products and
    sums in any order (fp16 or fp32 operands), then compares with the binary32
    value of logit(tau).  A decision taken outside this band is unique.
    """
    X = _tokens(x)
    W1a, W2a = np.abs(_f64(W1)), np.abs(_f64(W2))
    d = W1a.shape[1]
    r = W1a.shape[0]
    s1 = np.abs(X) @ W1a.T + np.abs(_f64(b1))[None, :]
    dh = _gamma(d + 1) * s1
    h = predictor_hidden(W1, b1, X)
    s2 = (h + dh) @ W2a.T + np.abs(_f64(b2))[None, :]
    thr = logit(tau)
    return _gamma(r + 1) * s2 + dh @ W2a.T + U32 * abs(thr) + 2.0 ** -60


def relu_input_band(act: str, Wg, Wu, bias, x) -> np.ndarray:
    """Bound on |pre_fp32 - pre| for the ReLU input of every neuron [B, n]."""
    X = _tokens(x)
    W = np.abs(_f64(Wg if act == "reglu" else Wu))
    s = np.abs(X) @ W.T + np.abs(_f64(bias))[None, :]
    return _gamma(W.shape[1] + 1) * s + 2.0 ** -60
