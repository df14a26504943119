"""Layer 1 of the predictor on rows longer than 8 KB (d >= 8192 in fp16, d >
2048 in fp32), where the CTA's W1 slice is staged in shared memory by bulk
copies issued before the dependency wait: index lists bit-exact against the
oracle on conditioned inputs for batches of 1 to 32 (one and several token
groups over the same staged slice), slices of 7 rows and a ragged last CTA,
and the combined one-layer call (list and output) at batch 1."""
import numpy as np
import pytest
import torch

import synthetic as S
from tests.gpu_util import Layer, ensure_built
from tests.helpers import TOL, rel_err

import activation_sparse_ffn_predict_b200 as A

pytestmark = pytest.mark.gpu

SHAPES = {
    # the 70B shape's predictor (d 8192, r 1024: 7 rows per CTA), a short FFN
    "d8192_r1024_f16": S.get("llama70b_reglu").with_(n=3000),
    # the OPT-175B shape's row length (24 KB), r 304: 3 rows per CTA, the last of 102 CTAs 1 row
    "d12288_r304_f16": S.get("opt175b_relu").with_(n=2085, r=304),
    # fp32 rows of 12 KB, r 64: one row per CTA
    "d3072_r64_f32": S.get("tiny_reglu_f32").with_(d=3072),
}


@pytest.fixture(scope="module", params=list(SHAPES))
def layer(request):
    ensure_built()
    return Layer(SHAPES[request.param], n_tokens=40)


@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8, 9, 16, 32])
def test_wide_predictor_lists_bit_exact(layer, B):
    rows = slice(1, 1 + B)
    got, full, c = layer.predict(rows)
    ref = layer.oracle_idx(rows)
    np.testing.assert_array_equal(got, ref)
    assert layer.error() == 0


def test_wide_combined_call(layer):
    rows = slice(7, 8)
    x = layer.Xd[rows].contiguous()
    n, d = layer.cfg.n, layer.cfg.d
    idx = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    y = torch.full((1, d), float("nan"), dtype=torch.float32, device="cuda")
    A.asf_predict_sparse_ffn(layer.pred, layer.ffn, x, layer.cfg.tau, idx, cnt, y, layer.ws)
    torch.cuda.synchronize()
    c = int(cnt.item())
    ref_idx = layer.oracle_idx(rows)
    np.testing.assert_array_equal(idx[:c].cpu().numpy(), ref_idx)
    assert rel_err(y.cpu().numpy(), layer.oracle_y(rows, ref_idx)) <= TOL[layer.cfg.dtype]
    assert layer.error() == 0
