"""Neuron-sharded layer on one GPU: the ranks' shards run one after another
(no collective here: their partial outputs are summed in rank order), and the
recombined index list and output match the oracle (lists bit-exact on
conditioned inputs) and the unsharded one-call layer."""
import numpy as np
import pytest
import torch

import synthetic as S
from tests.gpu_util import Layer, ensure_built
from tests.helpers import TOL, rel_err

import activation_sparse_ffn_predict_b200 as A
from activation_sparse_ffn_predict_b200 import shard as SH

pytestmark = pytest.mark.gpu

SHAPES = {
    "reglu_f16_ragged": S.get("llama2_7b_reglu").with_(d=1096, n=3000, r=136),
    "relu_f16_ragged": S.get("falcon_40b_relu").with_(d=1352, n=2085, r=72),
    "llama2_7b_shape": S.get("llama2_7b_reglu"),
}


@pytest.fixture(scope="module", params=list(SHAPES))
def layer(request):
    ensure_built()
    return Layer(SHAPES[request.param], n_tokens=8, device_gen=True)


@pytest.mark.parametrize("world", [2, 3, 8])
@pytest.mark.parametrize("B", [1, 4])
def test_shards_recombine_to_the_layer(layer, world, B):
    cfg = layer.cfg
    rows = slice(1, 1 + B)
    x = layer.Xd[rows].contiguous()
    y_sum = torch.zeros(B, cfg.d, dtype=torch.float32, device="cuda")
    lists = []
    for g in range(world):
        sh = SH.NeuronShard(layer.w, g, world)
        ws = sh.workspace(B)
        idx = torch.full((sh.n_local,), -3, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
        y = torch.full((B, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
        SH.sharded_layer(sh, x, cfg.tau, idx, cnt, y, ws)       # no process group: no collective
        torch.cuda.synchronize()
        c = int(cnt.item())
        lists.append(sh.global_ids(idx, c).cpu().numpy())
        y_sum += y
        assert A.asf_read_error(ws) == 0
    ref_idx = layer.oracle_idx(rows)
    np.testing.assert_array_equal(SH.merge_lists(lists), ref_idx)
    ref_y = layer.oracle_y(rows, ref_idx)
    assert rel_err(y_sum.cpu().numpy(), ref_y) <= TOL[cfg.dtype]
    # against the unsharded one-call layer: the same terms, summed in another order
    idx1 = torch.zeros(cfg.n, dtype=torch.int32, device="cuda")
    cnt1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    y1 = torch.zeros(B, cfg.d, dtype=torch.float32, device="cuda")
    A.asf_predict_sparse_ffn(layer.pred, layer.ffn, x, cfg.tau, idx1, cnt1, y1, layer.ws)
    torch.cuda.synchronize()
    assert rel_err(y_sum.cpu().numpy(), y1.cpu().numpy()) <= TOL[cfg.dtype]


def test_sharded_layer_orders_the_combine_on_the_callers_stream(layer, monkeypatch):
    """With a non-default stream, the layer's kernels and the combine step (the
    all-reduce under a process group) are enqueued on that stream, so the
    collective cannot read y before the layer has written it."""
    cfg = layer.cfg
    B = 2
    x = layer.Xd[:B].contiguous()
    sh = SH.NeuronShard(layer.w, 0, 2)
    ws = sh.workspace(B)
    idx = torch.zeros(sh.n_local, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    seen = []
    real = SH.combine_partials

    def spy(y, group=None):
        seen.append(torch.cuda.current_stream())
        return real(y, group)

    monkeypatch.setattr(SH, "combine_partials", spy)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    for stream_arg in (side, side.cuda_stream):          # torch stream and raw handle
        y = torch.full((B, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
        SH.sharded_layer(sh, x, cfg.tau, idx, cnt, y, ws, stream=stream_arg)
        assert seen[-1].cuda_stream == side.cuda_stream
        side.synchronize()
        assert torch.isfinite(y).all()
    # without a stream, the combine runs on the current stream
    y = torch.zeros(B, cfg.d, dtype=torch.float32, device="cuda")
    SH.sharded_layer(sh, x, cfg.tau, idx, cnt, y, ws)
    assert seen[-1].cuda_stream == torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    assert A.asf_read_error(ws) == 0
