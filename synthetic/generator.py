"""Seeded synthetic weights and inputs for the sparse FFN and its predictor.

This module only draws random numbers and sets biases so that the activation
statistics match the pages' description; it contains none of the FFN or
predictor arithmetic.  Both the CUDA path and the CPU oracle are fed from it.

Recipe (one layer ``l`` of a config; every draw is seeded by (seed, l, tag)):

* x_{l,t} ~ N(0, I_d), rounded to the storage dtype.
* W_gate, W_up ~ N(0, std=1/sqrt(d)), W_down ~ N(0, std=1/sqrt(n)) stored
  transposed as WdT[n][d]; W1 ~ N(0, 1/sqrt(d)) of shape [r][d]; W2 ~ N(0,
  1/sqrt(r)) of shape [n][r]; all rounded to the storage dtype.
* Activation frequency follows a power law over neuron rank (PowerInfer Guide,
  "Empirical Power-Law Distribution and Skewness": P(k) ~ k^-gamma):
  p_rank(k) = min(0.99, c k^-gamma), with c found by bisection so that the
  mean of p equals the config's mean active fraction.  Ranks map to neuron ids
  through a seeded random permutation, so frequent neurons are scattered.
* Per-neuron bias of the ReLU input (gate for ReGLU, up for ReLU): for
  x ~ N(0, I) and a stored row w, P(w.x + b > 0) = Phi(b / ||w||_2), so
  b_k = ||w_k|| Phi^-1(p_k) makes neuron k active with probability p_k.
* Predictor biases: b1 = 0.  With h_j = ReLU(W1_j . x), E h_j = ||W1_j||/sqrt(2 pi)
  and Var h_j = ||W1_j||^2 (1/2 - 1/(2 pi)); a central-limit approximation of
  z_k = W2_k . h + b2_k then gives b2_k = logit(tau) - mu_k + sigma_k Phi^-1(p_k),
  so predicted sets have about the same sparsity and power-law profile.  The
  predictor is random: it does not reproduce the true active sets.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from statistics import NormalDist
from typing import Optional

import numpy as np
import torch

from .configs import FFNConfig

_TAGS = {"Wg": 1, "Wu": 2, "WdT": 3, "W1": 4, "W2": 5, "perm": 6,
         "x_eval": 7, "x_calib": 8, "x_extra": 9}

TORCH_DTYPE = {"f32": torch.float32, "f16": torch.float16}


def seed_for(cfg: FFNConfig, layer: int, tag: str) -> int:
    """Deterministic 63-bit seed for one tensor of one layer of a config."""
    return (cfg.seed * 1_000_003 + layer * 10_007 + _TAGS[tag] * 101 + 12345) & ((1 << 63) - 1)


def zipf_rank_profile(n: int, gamma: float, frac: float, cap: float = 0.99) -> np.ndarray:
    """p_rank(k) = min(cap, c k^-gamma), k = 1..n, with mean(p) = frac (bisection on c)."""
    if not (0.0 < frac < cap):
        raise ValueError("mean active fraction must be in (0, cap)")
    k = np.arange(1, n + 1, dtype=np.float64)

    def mean_p(c: float) -> float:
        return float(np.minimum(cap, c * k ** (-gamma)).mean())

    lo, hi = 0.0, 1.0
    while mean_p(hi) < frac:
        hi *= 2.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if mean_p(mid) < frac:
            lo = mid
        else:
            hi = mid
    return np.minimum(cap, hi * k ** (-gamma))


def rank_to_neuron(cfg: FFNConfig, layer: int) -> np.ndarray:
    """Seeded permutation: pi[rank-1] = neuron id holding that frequency rank."""
    g = torch.Generator(device="cpu").manual_seed(seed_for(cfg, layer, "perm"))
    return torch.randperm(cfg.n, generator=g).numpy().astype(np.int64)


def activity_profile(cfg: FFNConfig, layer: int) -> np.ndarray:
    """Target activation probability of every neuron id (float64, length n)."""
    p_rank = zipf_rank_profile(cfg.n, cfg.gamma, cfg.frac)
    pi = rank_to_neuron(cfg, layer)
    p = np.empty(cfg.n, dtype=np.float64)
    p[pi] = p_rank
    return p


def _probit(p: np.ndarray) -> np.ndarray:
    nd = NormalDist()
    return np.array([nd.inv_cdf(float(v)) for v in p], dtype=np.float64)


def _gen(device, seed: int) -> torch.Generator:
    dev = torch.device(device)
    return torch.Generator(device=dev).manual_seed(seed)


def gaussian(shape, std: float, dtype: str, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) draws in fp32, rounded once to the storage dtype."""
    g = _gen(device, seed)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(TORCH_DTYPE[dtype])


def _row_norms(w: torch.Tensor) -> np.ndarray:
    """Euclidean norm of each stored row, accumulated in float64 on the host."""
    out = np.empty(w.shape[0], dtype=np.float64)
    step = max(1, (1 << 24) // max(1, w.shape[1]))
    for s in range(0, w.shape[0], step):
        blk = w[s:s + step].to(torch.float64)
        out[s:s + step] = torch.sqrt((blk * blk).sum(dim=1)).cpu().numpy()
    return out


@dataclass
class LayerWeights:
    """One FFN layer plus its predictor, in storage order (row k = neuron k)."""
    act: str
    dtype: str
    Wg: Optional[torch.Tensor]   # [n, d] (ReGLU only)
    Wu: torch.Tensor             # [n, d]
    WdT: torch.Tensor            # [n, d]  (W_down transposed)
    bias: torch.Tensor           # [n] fp32: gate bias (ReGLU) or up bias (ReLU)
    W1: torch.Tensor             # [r, d]
    b1: torch.Tensor             # [r] fp32
    W2: torch.Tensor             # [n, r]
    b2: torch.Tensor             # [n] fp32
    p: np.ndarray                # target activation probability per neuron

    @property
    def d(self) -> int:
        return self.Wu.shape[1]

    @property
    def n(self) -> int:
        return self.Wu.shape[0]

    @property
    def r(self) -> int:
        return self.W1.shape[0]

    def to(self, device) -> "LayerWeights":
        mv = lambda t: None if t is None else t.to(device)
        return LayerWeights(self.act, self.dtype, mv(self.Wg), mv(self.Wu), mv(self.WdT),
                            mv(self.bias), mv(self.W1), mv(self.b1), mv(self.W2),
                            mv(self.b2), self.p)

    def numpy(self) -> dict:
        """Host copies (exact stored values) keyed by name."""
        cv = lambda t: None if t is None else t.detach().cpu().numpy()
        return {"act": self.act, "Wg": cv(self.Wg), "Wu": cv(self.Wu), "WdT": cv(self.WdT),
                "bias": cv(self.bias), "W1": cv(self.W1), "b1": cv(self.b1),
                "W2": cv(self.W2), "b2": cv(self.b2)}

    def permuted(self, perm: torch.Tensor) -> "LayerWeights":
        """Rows of every per-neuron tensor reordered: new row i = old row perm[i]."""
        pi = perm.to(self.Wu.device, torch.int64)
        g = lambda t: None if t is None else t.index_select(0, pi).contiguous()
        return LayerWeights(self.act, self.dtype, g(self.Wg), g(self.Wu), g(self.WdT),
                            g(self.bias), self.W1, self.b1, g(self.W2), g(self.b2),
                            self.p[perm.cpu().numpy()])


def layer_weights(cfg: FFNConfig, layer: int, device="cpu") -> LayerWeights:
    """Draw one layer's FFN and predictor weights and set the calibrated biases."""
    d, n, r, dt = cfg.d, cfg.n, cfg.r, cfg.dtype
    p = activity_profile(cfg, layer)
    Wg = gaussian((n, d), 1.0 / math.sqrt(d), dt, seed_for(cfg, layer, "Wg"), device) \
        if cfg.act == "reglu" else None
    Wu = gaussian((n, d), 1.0 / math.sqrt(d), dt, seed_for(cfg, layer, "Wu"), device)
    WdT = gaussian((n, d), 1.0 / math.sqrt(n), dt, seed_for(cfg, layer, "WdT"), device)
    W1 = gaussian((r, d), 1.0 / math.sqrt(d), dt, seed_for(cfg, layer, "W1"), device)
    W2 = gaussian((n, r), 1.0 / math.sqrt(r), dt, seed_for(cfg, layer, "W2"), device)

    probit = _probit(p)
    gated = Wg if cfg.act == "reglu" else Wu
    bias = _row_norms(gated) * probit

    # predictor output calibration (central-limit moments of z_k = W2_k . h)
    nrm1 = _row_norms(W1)
    mean_h = nrm1 / math.sqrt(2.0 * math.pi)
    var_h = nrm1 ** 2 * (0.5 - 1.0 / (2.0 * math.pi))
    w2 = W2.to(torch.float64).cpu().numpy() if n * r <= (1 << 26) else None
    if w2 is not None:
        mu = w2 @ mean_h
        sig = np.sqrt((w2 * w2) @ var_h)
    else:
        mu = np.empty(n)
        sig = np.empty(n)
        step = 4096
        for s in range(0, n, step):
            blk = W2[s:s + step].to(torch.float64).cpu().numpy()
            mu[s:s + step] = blk @ mean_h
            sig[s:s + step] = np.sqrt((blk * blk) @ var_h)
    thr = math.log(cfg.tau / (1.0 - cfg.tau))
    b2 = thr - mu + sig * probit

    f32 = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float32)).to(device)
    return LayerWeights(cfg.act, dt, Wg, Wu, WdT, f32(bias), W1, f32(np.zeros(r)), W2,
                        f32(b2), p)


def layer_tokens(cfg: FFNConfig, layer: int, count: int, device="cpu",
                 kind: str = "x_eval") -> torch.Tensor:
    """``count`` input vectors x ~ N(0, I_d) for one layer, rounded to the dtype."""
    return gaussian((count, cfg.d), 1.0, cfg.dtype, seed_for(cfg, layer, kind), device)
