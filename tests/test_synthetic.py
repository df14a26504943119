"""The seeded input recipe reproduces the activation statistics it promises.

Closed forms: the power-law profile has the requested mean and saturation;
for x ~ N(0, I) the bias b_k = ||w_k|| Phi^-1(p_k) makes neuron k fire with
probability exactly p_k, which the oracle's true active sets must show within
binomial error.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S


@pytest.mark.parametrize("name,sat", [("tiny_reglu_f32", 39), ("llama2_7b_reglu", 313),
                                      ("falcon_40b_relu", 933), ("llama70b_reglu", 1132),
                                      ("opt175b_relu", 929)])
def test_zipf_profile_mean_saturation_and_hot_share(name, sat):
    cfg = S.get(name)
    p = S.zipf_rank_profile(cfg.n, cfg.gamma, cfg.frac)
    assert abs(p.mean() - cfg.frac) < 1e-12
    assert int((p >= 0.99).sum()) == sat
    assert np.all(np.diff(p) <= 0)
    share = p[: int(0.2 * cfg.n)].sum() / p.sum()
    assert 0.72 < share < 0.75


def test_seeds_are_deterministic_and_distinct():
    cfg = S.get("tiny_reglu_f32")
    a = S.layer_weights(cfg, 0)
    b = S.layer_weights(cfg, 0)
    c = S.layer_weights(cfg.with_(seed=9), 0)
    assert torch.equal(a.Wg, b.Wg) and torch.equal(a.b2, b.b2)
    assert not torch.equal(a.Wg, c.Wg)
    x0 = S.layer_tokens(cfg, 0, 4)
    assert torch.equal(x0, S.layer_tokens(cfg, 0, 4))
    assert not torch.equal(x0, S.layer_tokens(cfg, 0, 4, kind="x_calib"))
    p = S.activity_profile(cfg, 0)
    assert sorted(np.round(np.sort(p)[::-1], 12).tolist()) == \
        sorted(np.round(S.zipf_rank_profile(cfg.n, cfg.gamma, cfg.frac), 12).tolist())


@pytest.mark.parametrize("name,shape", [
    ("tiny_reglu_f32", dict()),
    ("llama2_7b_reglu", dict(d=512, n=1024, r=128)),
    ("falcon_40b_relu", dict(d=512, n=2048, r=128)),
])
def test_realised_activity_matches_profile(name, shape):
    cfg = S.get(name).with_(**shape)
    w = S.layer_weights(cfg, 0).numpy()
    X = S.layer_tokens(cfg, 0, 1536, kind="x_calib").numpy()
    act = O.true_active(cfg.act, w["Wg"], w["Wu"], w["bias"], X)
    p = S.activity_profile(cfg, 0)
    rate = act.mean(axis=0)
    T = X.shape[0]
    sd = np.sqrt(p * (1 - p) / T)
    z = (rate - p) / sd
    assert np.abs(z).max() < 5.5
    assert abs(z.mean()) < 0.5   # no systematic bias in the calibration
    assert abs(rate.mean() - cfg.frac) < 0.01
    # the predictor is calibrated to the same mean sparsity (central-limit approximation)
    m = O.predictor_mask(w["W1"], w["b1"], w["W2"], w["b2"], X[:256], cfg.tau)
    assert abs(m.mean() - cfg.frac) < 0.03


def test_permuted_layer_moves_rows_together():
    cfg = S.get("tiny_reglu_f32")
    w = S.layer_weights(cfg, 0)
    perm = torch.randperm(cfg.n, generator=torch.Generator().manual_seed(3))
    wp = w.permuted(perm)
    for name in ["Wg", "Wu", "WdT", "bias", "W2", "b2"]:
        assert torch.equal(getattr(wp, name), getattr(w, name)[perm])
    assert torch.equal(wp.W1, w.W1)


def test_conditioning_clears_every_rounding_band():
    from tests.helpers import band_violations, condition_b2
    cfg = S.get("llama2_7b_reglu").with_(d=256, n=600, r=64)
    w = S.layer_weights(cfg, 1).numpy()
    X = S.layer_tokens(cfg, 1, 16).numpy()
    b2 = condition_b2(w["W1"], w["b1"], w["W2"], w["b2"], X, cfg.tau)
    assert b2.dtype == np.float32
    assert band_violations(w["W1"], w["b1"], w["W2"], b2, X, cfg.tau) == 0
    moved = np.flatnonzero(b2 != w["b2"])
    # only a few biases move, by a small amount
    assert moved.size < 0.2 * cfg.n
    assert np.abs(b2 - w["b2"]).max() < 0.5
