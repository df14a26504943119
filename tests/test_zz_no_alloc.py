"""asf_sparse_ffn_noalloc: the sparse FFN for callers that cannot allocate.

Some callers cannot allocate device memory where they run the FFN (a plugin
whose host framework owns every device allocation, or a latency-critical path
that cannot afford cudaMalloc's implicit synchronisation).  The no-alloc entry
point takes its scratch from a static device array inside the library.  This
test calls it through the C ABI twice in a row, on different inputs, and
checks each result against asf_sparse_ffn with a caller workspace.  Both run
the same kernels with the same fixed-order reductions, so y must agree bit for
bit; the tolerance of the other parity tests is reported if it does not.  It
is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic as S
from tests.gpu_util import ensure_built
from tests.helpers import TOL, rel_err

import activation_sparse_ffn_predict_b200 as A
from activation_sparse_ffn_predict_b200 import _lib as L

pytestmark = pytest.mark.gpu

CASES = [
    ("reglu_f16_ragged", S.get("llama2_7b_reglu").with_(d=1096, n=3000, r=136), 1),
    ("reglu_f16_batch4", S.get("llama2_7b_reglu").with_(d=1096, n=3000, r=136), 4),
    ("llama2_7b_layer", S.get("llama2_7b_reglu"), 1),
    ("relu_f32_tiny", S.get("tiny_reglu_f32").with_(act="relu"), 2),
]


def _idx(n, rng, frac=0.1):
    k = max(1, int(n * frac))
    return np.sort(rng.choice(n, size=k, replace=False)).astype(np.int32)


@pytest.mark.parametrize("name,cfg,B", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_path_on_two_calls(name, cfg, B):
    ensure_built()
    w = S.layer_weights(cfg, 0, device="cuda")
    ffn = A.FFN(w.act, w.Wg, w.Wu, w.WdT, w.bias)
    ws = A.Workspace(None, ffn, B)
    X = S.layer_tokens(cfg, 0, 2 * B, device="cuda")
    rng = np.random.default_rng(7)
    fault = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    lib = L.load()
    for call in range(2):                      # two calls in a row, different inputs
        x = X[call * B:(call + 1) * B].contiguous()
        ids = _idx(cfg.n, rng)
        idx = torch.zeros(cfg.n, dtype=torch.int32, device="cuda")
        idx[:ids.size] = torch.from_numpy(ids).cuda()
        cnt = torch.tensor([ids.size], dtype=torch.int32, device="cuda")
        y_ref = torch.zeros(B, cfg.d, dtype=torch.float32, device="cuda")
        A.asf_sparse_ffn(ffn, x, idx, cnt, y_ref, ws)
        y = torch.full((B, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.asf_sparse_ffn_noalloc(ctypes.byref(ffn.desc), ctypes.c_void_p(x.data_ptr()), B,
                                        ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()),
                                        ctypes.c_void_p(y.data_ptr()), ctypes.c_void_p(fault.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == L.ASF_OK, A.asf_status_string(st)
        torch.cuda.synchronize()
        assert int(fault.item()) == 0
        yr = y_ref.cpu().numpy()
        assert np.isfinite(y.cpu().numpy()).all()
        assert torch.equal(y, y_ref), (
            f"call {call}: not bitwise equal to the workspace path (rel err "
            f"{rel_err(y.cpu().numpy(), yr):.3e}, parity tolerance {TOL[cfg.dtype]:.0e})")
    assert A.asf_read_error(ws) == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    ensure_built()
    lib = L.load()
    fake = 1 << 20          # never dereferenced: the size check fails first
    # 262144 neurons x 32 tokens of fp32 activations alone are 33.5 MB > 32 MiB
    big = L.asf_ffn(4096, 262144, L.ASF_F16, L.ASF_ACT_RELU, 0, fake, fake, fake)
    st = lib.asf_sparse_ffn_noalloc(ctypes.byref(big), fake, 32, fake, fake, fake, None, None)
    assert st == L.ASF_ERR_UNSUPPORTED
