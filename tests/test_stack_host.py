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


@pytest.mark.parametrize("B,dtype,mode,combined,per_layer", [
    (1, torch.float16, "predict", True, 4),    # layer 1, layer 2 ring, sparse FFN ranking the mask, reduction
    (1, torch.float16, "predict", False, 5),   # + the compaction kernel between the two calls
    (4, torch.float16, "predict", True, 4),
    (6, torch.float16, "predict", True, 6),    # ring + compaction, tensor-core gate/up, down, reduction
    (12, torch.float16, "predict", True, 7),   # two ring groups of tokens
    (16, torch.float16, "predict", True, 7),
    (17, torch.float16, "predict", True, 9),   # three ring groups, two gate/up launches
    (32, torch.float16, "predict", True, 10),  # four ring groups, two gate/up launches
    (12, torch.float32, "predict", True, 6),   # fp32: CUDA-core gate/up + down
    (1, torch.float16, "sparse", True, 2), (32, torch.float16, "dense", True, 4),
    (32, torch.float32, "dense", True, 2),
])
def test_launches_per_step(B, dtype, mode, combined, per_layer):
    st = _Stub(4096 if dtype == torch.float16 else 512, dtype, B, 32, mode, combined)
    assert ST.LayerStack.launches_per_step(st) == 32 * per_layer


@pytest.mark.parametrize("d,B,per_layer", [
    (8192, 1, 4),    # the one-kernel FFN holds one token at d = 8192
    (8192, 2, 4),
    (8192, 4, 5),    # too many accumulators: compaction + CUDA-core gate/up and down
    (12288, 2, 5),
    (12288, 6, 6),   # tensor-core gate/up, down, reduction
])
def test_launches_per_step_wide_layers(d, B, per_layer):
    st = _Stub(d, torch.float16, B, 80, "predict", True)
    assert ST.LayerStack.launches_per_step(st) == 80 * per_layer
