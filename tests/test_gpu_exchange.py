"""The peer exchange of the neuron-sharded layer on one GPU.

Several GPUs are not available here, so every rank of a group is held by one
process and the ranks' exchange runs as one cooperative launch (all blocks
resident while they wait on one another).  Checks: y equals the sum over
ranks and partials (float64 reference), is the same on every rank bit for bit,
stays right over consecutive calls (the publication buffer alternates halves),
and a peer that never publishes makes the wait give up with ASF_ERR_TIMEOUT
instead of hanging.  The one-rank layer call with the exchange equals the
plain layer call bit for bit."""
import numpy as np
import pytest
import torch

import synthetic as S
from tests.gpu_util import Layer, ensure_built
from tests.helpers import rel_err

import activation_sparse_ffn_predict_b200 as A
from activation_sparse_ffn_predict_b200 import _lib as L
from activation_sparse_ffn_predict_b200 import shard as SH

pytestmark = pytest.mark.gpu


def _ws():
    return A.Workspace(None, A.FFN("relu", None, torch.zeros(1, 8, dtype=torch.float16, device="cuda"),
                                   torch.zeros(1, 8, dtype=torch.float16, device="cuda"),
                                   torch.zeros(1, dtype=torch.float32, device="cuda")), 1)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
# blocks of all ranks must be resident at once: (d/32) * B * world within the GPU
@pytest.mark.parametrize("G,B,d", [(148, 1, 2048), (5, 2, 1096), (1, 2, 40)])
def test_emulated_exchange_sums_every_rank(world, G, B, d):
    ensure_built()
    grp = SH.EmulatedGroup(world, d, max_batch=4)
    ws = _ws()
    gen = torch.Generator(device="cuda").manual_seed(world * 1000 + G)
    for call in range(3):                          # consecutive calls alternate the halves
        part = torch.randn(world, G, B, d, device="cuda", generator=gen)
        y = torch.full((world, B, d), float("nan"), device="cuda")
        A.asf_reduce_exchange(part, grp.desc, y, ws)
        torch.cuda.synchronize()
        ref = part.double().sum(dim=(0, 1)).cpu().numpy()
        for r in range(world):
            assert torch.equal(y[r], y[0])          # every rank the same, bit for bit
        assert rel_err(y[0].cpu().numpy(), ref) <= 1e-5
    assert A.asf_read_error(ws) == 0


def test_missing_peer_times_out():
    """Rank 0 of a two-rank group runs alone: rank 1's flag is never set, so
    the bounded wait gives up, records ASF_ERR_TIMEOUT, and y holds rank 0's
    own sum; the context stays usable."""
    ensure_built()
    d, B, G = 256, 1, 4
    grp = SH.EmulatedGroup(2, d, max_batch=1)
    ws = _ws()
    part = torch.randn(G, B, d, device="cuda")
    y = torch.zeros(B, d, device="cuda")
    A.asf_reduce_exchange(part, grp.desc, y, ws)
    torch.cuda.synchronize()
    assert A.asf_read_error(ws) == L.ASF_ERR_TIMEOUT
    assert rel_err(y.cpu().numpy(), part.double().sum(dim=0).cpu().numpy()) <= 1e-5
    # the device still works
    grp1 = SH.EmulatedGroup(1, d, max_batch=1)
    A.asf_reduce_exchange(part, grp1.desc, y, ws)
    torch.cuda.synchronize()
    assert A.asf_read_error(ws) == 0


@pytest.mark.parametrize("B", [1, 4, 9])
def test_one_rank_layer_with_exchange_is_the_layer(B):
    ensure_built()
    lay = Layer(S.get("llama2_7b_reglu").with_(d=1096, n=3000, r=136), n_tokens=16)
    x = lay.Xd[:B].contiguous()
    grp = SH.EmulatedGroup(1, lay.cfg.d, max_batch=16)
    outs = []
    for exchange in (False, True):
        idx = torch.zeros(lay.cfg.n, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
        y = torch.full((B, lay.cfg.d), float("nan"), device="cuda")
        if exchange:
            A.asf_predict_sparse_ffn_exchange(lay.pred, lay.ffn, x, lay.cfg.tau, idx, cnt, y, lay.ws, grp.desc)
        else:
            A.asf_predict_sparse_ffn(lay.pred, lay.ffn, x, lay.cfg.tau, idx, cnt, y, lay.ws)
        torch.cuda.synchronize()
        outs.append((idx.cpu().numpy(), int(cnt.item()), y))
    assert outs[0][1] == outs[1][1]
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][2], outs[1][2])
    assert lay.error() == 0
