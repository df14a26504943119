"""Host-side logic of the layer stack (no GPU): the launch count it claims
follows the library's dispatch rules.  On a GPU, tests/test_gpu_stack.py
checks the same count against the kernel nodes of the captured graph."""
import pytest
import torch

from activation_sparse_ffn_predict_b200 import stack as ST


@pytest.mark.parametrize("d,dtype,B,fused", [
    (4096, torch.float16, 1, True), (4096, torch.float16, 4, True), (4096, torch.float16, 5, False),
    (8192, torch.float16, 2, True), (8192, torch.float16, 4, False),
    (12288, torch.float16, 1, True), (12288, torch.float16, 2, False),
    (512, torch.float32, 4, True), (1096, torch.float16, 3, True), (2048 + 8, torch.float16, 4, True),
    (4096 + 8, torch.float16, 4, False), (4096 + 8, torch.float16, 2, True),
])
def test_fused_sparse_ffn_rule(d, dtype, B, fused):
    # at most 64 fp32 accumulators per lane: chunks of 16 bytes per lane
    # (rounded up to 1, 2, 4 or 6) x elements per chunk x token group
    assert ST._fused_sparse_ffn(d, dtype, B) is fused


class _Stub:
    def __init__(self, d, dtype, B, L, mode, combined):
        self.d, self.dtype, self.B, self.L, self.mode, self.combined = d, dtype, B, L, mode, combined


@pytest.mark.parametrize("B,mode,combined,per_layer", [
    (1, "predict", True, 4),    # layer 1, layer 2 ring, sparse FFN ranking the mask, reduction
    (1, "predict", False, 5),   # + the compaction kernel between the two calls
    (4, "predict", True, 4),
    (6, "predict", True, 5),    # ring layer 2 + compaction, two-kernel FFN
    (12, "predict", True, 4),   # register layer 2 compacts itself, two-kernel FFN
    (1, "sparse", True, 2), (32, "dense", True, 2),
])
def test_launches_per_step(B, mode, combined, per_layer):
    st = _Stub(4096, torch.float16, B, 32, mode, combined)
    assert ST.LayerStack.launches_per_step(st) == 32 * per_layer
