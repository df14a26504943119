"""Failure detection on the GPU without a GPU fault: the test hook makes one
CTA of the one-kernel sparse FFN withhold its row copies, so that CTA's bounded
wait (200 ms) runs out.  The kernel must record ASF_ERR_TIMEOUT in the
workspace error word and return -- no hang, no fault, the context stays usable
-- and the next call on the same workspace must run normally and match the
oracle."""
import numpy as np
import pytest
import torch

import synthetic as S
from tests.gpu_util import Layer, ensure_built
from tests.helpers import TOL, rel_err

import activation_sparse_ffn_predict_b200 as A
from activation_sparse_ffn_predict_b200 import _lib as L

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer():
    ensure_built()
    return Layer(S.get("llama2_7b_reglu").with_(d=1096, n=3000, r=136), n_tokens=8)


@pytest.mark.parametrize("call", ["sparse", "combined"])
def test_withheld_copies_time_out_and_the_next_call_recovers(layer, call):
    cfg = layer.cfg
    B = 1
    rows = slice(0, B)
    x = layer.Xd[rows].contiguous()
    ref_idx = layer.oracle_idx(rows)
    assert ref_idx.size > 0
    idx = torch.zeros(cfg.n, dtype=torch.int32, device="cuda")
    idx[:ref_idx.size] = torch.from_numpy(ref_idx).cuda()
    cnt = torch.tensor([ref_idx.size], dtype=torch.int32, device="cuda")

    def run():
        y = torch.full((B, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
        if call == "sparse":
            A.asf_sparse_ffn(layer.ffn, x, idx, cnt, y, layer.ws)
        else:
            A.asf_predict_sparse_ffn(layer.pred, layer.ffn, x, cfg.tau, idx, cnt, y, layer.ws)
        return y

    assert layer.error() == 0
    A.asf_set_fault_injection(L.ASF_INJECT_WITHHOLD_FFN_COPIES)
    try:
        y_bad = run()
        torch.cuda.synchronize()           # returns: the wait is bounded
    finally:
        A.asf_set_fault_injection(L.ASF_INJECT_NONE)
    assert layer.error() == L.ASF_ERR_TIMEOUT
    assert layer.error() == 0              # read and cleared
    assert torch.isfinite(y_bad).all()     # CTA 0's share is missing, nothing is garbage
    y = run()
    torch.cuda.synchronize()
    assert layer.error() == 0
    assert rel_err(y.cpu().numpy(), layer.oracle_y(rows, ref_idx)) <= TOL[cfg.dtype]
