"""The many-token path (fp16 weights, B > 4): gate/up on the tensor cores in
launches of 16 tokens, the down projection on the CUDA cores, against the
oracle: list lengths across the ownership-chunk (32) and MMA-tile (128)
boundaries, empty lists, ragged d and n, one and two token launches (B <= 16
and B <= 32), and the predictor's index lists at those batch sizes bit-exact
on conditioned inputs."""
import numpy as np
import pytest
import torch

import synthetic as S
from tests.gpu_util import Layer, ensure_built
from tests.helpers import TOL, rel_err

pytestmark = pytest.mark.gpu

SHAPES = {
    # d 1096 = 17 K-stages of 64 + 8, 3 down ranges (2 x 512 + 72); n 3000
    "reglu_f16_ragged": S.get("llama2_7b_reglu").with_(d=1096, n=3000, r=136),
    # plain ReLU (up + down), d 1352, n 2085, r 72 (two K-stages, the second ragged)
    "relu_f16_ragged": S.get("falcon_40b_relu").with_(d=1352, n=2085, r=72),
}


@pytest.fixture(scope="module", params=list(SHAPES))
def layer(request):
    ensure_built()
    return Layer(SHAPES[request.param], n_tokens=40)


@pytest.mark.parametrize("B", [5, 8, 9, 16, 17, 24, 32])
@pytest.mark.parametrize("count", [0, 1, 31, 32, 33, 127, 128, 129, 700])
def test_tc_sparse_ffn_list_lengths(layer, B, count):
    rng = np.random.default_rng(count * 100 + B)
    ids = np.sort(rng.choice(layer.cfg.n, size=count, replace=False)).astype(np.int32)
    rows = slice(3, 3 + B)
    y = layer.sparse(rows, ids)
    ref = layer.oracle_y(rows, ids)
    if count == 0:
        assert (y == 0).all()
    else:
        assert rel_err(y, ref) <= TOL[layer.cfg.dtype]
    assert layer.error() == 0


@pytest.mark.parametrize("B", [5, 12, 32])
def test_tc_dense_matches_oracle(layer, B):
    rows = slice(0, B)
    y = layer.dense(rows)
    ref = layer.oracle_y(rows, np.arange(layer.cfg.n))
    assert rel_err(y, ref) <= TOL[layer.cfg.dtype]
    assert layer.error() == 0


@pytest.mark.parametrize("B", [9, 16, 17, 32])
def test_tc_predictor_lists_bit_exact(layer, B):
    rows = slice(2, 2 + B)
    got, full, c = layer.predict(rows)
    ref = layer.oracle_idx(rows)
    np.testing.assert_array_equal(got, ref)
    assert (full[c:] == -7).all()          # entries past count untouched
    assert layer.error() == 0


@pytest.mark.parametrize("B", [5, 16, 32])
def test_tc_results_are_deterministic(layer, B):
    ids = np.arange(0, layer.cfg.n, 3, dtype=np.int32)
    rows = slice(0, B)
    y0 = layer.sparse(rows, ids)
    y1 = layer.sparse(rows, ids)
    np.testing.assert_array_equal(y0, y1)
