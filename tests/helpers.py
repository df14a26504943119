"""Test-side helpers built on the oracle (test infrastructure, not product code)."""
from __future__ import annotations

import numpy as np

import oracle as O


def condition_b2(W1, b1, W2, b2, X, tau: float, safety: float = 2.0) -> np.ndarray:
    """Shift predictor biases so no token's logit falls inside the rounding band.

    For neuron k and token t the decision z_kt > logit(tau) is unique when
    |z_kt - logit(tau)| exceeds the binary32 error bound delta_kt (oracle
    ``predictor_band``).  Changing b2_k moves every z_kt by the same amount, so
    each token forbids one open interval of b2_k values.  The new b2_k is the
    binary32 value closest to the old one outside every forbidden interval
    (widened by ``safety``).  Returns float32 biases.
    """
    b2 = np.asarray(b2, dtype=np.float32).copy()
    z = O.predictor_logits(W1, b1, W2, b2, X)                      # [B, n]
    band = safety * O.predictor_band(W1, b1, W2, b2, X, tau)       # [B, n]
    thr = O.logit(tau)
    base = z - b2.astype(np.float64)[None, :]                      # z without b2
    for k in range(b2.shape[0]):
        centre = thr - base[:, k]
        lo, hi = centre - band[:, k], centre + band[:, k]

        def clear(v: float) -> bool:
            return not np.any((v >= lo) & (v <= hi))

        if clear(float(b2[k])):
            continue
        cands = np.concatenate([lo, hi])
        cands = cands[np.argsort(np.abs(cands - float(b2[k])), kind="stable")]
        for c in cands:
            v_up = v_dn = np.float32(c)
            hit = None
            for _ in range(8):            # step outward a few binary32 ulps
                if clear(float(v_up)):
                    hit = v_up
                    break
                if clear(float(v_dn)):
                    hit = v_dn
                    break
                v_up = np.nextafter(v_up, np.float32(np.inf))
                v_dn = np.nextafter(v_dn, np.float32(-np.inf))
            if hit is not None:
                b2[k] = hit
                break
    return b2


def band_violations(W1, b1, W2, b2, X, tau: float) -> int:
    """Number of (token, neuron) decisions that lie inside the rounding band."""
    z = O.predictor_logits(W1, b1, W2, b2, X)
    band = O.predictor_band(W1, b1, W2, b2, X, tau)
    return int((np.abs(z - O.logit(tau)) <= band).sum())


def relu_band_ambiguous(act, Wg, Wu, bias, X) -> np.ndarray:
    """Mask [B, n] of ReLU-input signs that a binary32 evaluation may decide either way."""
    pre = O.relu_input(act, Wg, Wu, bias, X)
    return np.abs(pre) <= O.relu_input_band(act, Wg, Wu, bias, X)


def rel_err(y, ref) -> float:
    """max |y - ref| / max |ref| (with a floor of 1e-30 on the scale)."""
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(y - ref).max() / max(1e-30, np.abs(ref).max())) if ref.size else 0.0


# output tolerances relative to ||y_ref||_inf: fp16 weights with fp32
# accumulation, and the all-fp32 layer
TOL = {"f16": 2e-3, "f32": 1e-5}
