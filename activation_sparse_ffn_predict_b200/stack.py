"""A decode step over a stack of FFN layers: predictor then sparse FFN per layer.

One step takes the B tokens' FFN inputs for every layer (``x[l]``), runs the
predictor and the sparse FFN (one asf_predict_sparse_ffn call) for
l = 0..L-1 in order on one stream, and leaves y[l], idx[l], count[l] on the
device.  The launch sequence is captured
once into a CUDA graph; kernels inside it overlap through programmatic
dependent launch (each waits for its predecessor before reading its inputs).
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from .api import (FFN, Predictor, Workspace, asf_dense_ffn, asf_predict, asf_predict_sparse_ffn,
                  asf_sparse_ffn)


class LayerStack:
    def __init__(self, preds: Sequence[Optional[Predictor]], ffns: Sequence[FFN], batch: int,
                 tau: float = 0.5, mode: str = "predict", device=None, combined: bool = True):
        """mode: "predict" (predictor + sparse FFN), "sparse" (sparse FFN over
        caller-filled idx/count), or "dense" (all neurons).  combined: in
        predict mode, one asf_predict_sparse_ffn call per layer instead of
        asf_predict followed by asf_sparse_ffn (same results)."""
        if mode not in ("predict", "sparse", "dense"):
            raise ValueError("mode must be predict, sparse or dense")
        self.preds = list(preds)
        self.ffns = list(ffns)
        self.L = len(self.ffns)
        self.B = int(batch)
        self.tau = float(tau)
        self.mode = mode
        self.combined = bool(combined)
        f0 = self.ffns[0]
        dev = device if device is not None else f0.tensors[1].device
        self.d, self.n, self.dtype = f0.d, f0.n, f0.dtype
        self.x = torch.zeros(self.L, self.B, self.d, dtype=self.dtype, device=dev)
        self.y = torch.zeros(self.L, self.B, self.d, dtype=torch.float32, device=dev)
        self.idx = torch.zeros(self.L, self.n, dtype=torch.int32, device=dev)
        self.count = torch.zeros(self.L, dtype=torch.int32, device=dev)
        p0 = self.preds[0] if (self.preds and mode == "predict") else None
        self.ws = Workspace(p0, f0, self.B, device=dev)
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    def launches_per_step(self) -> int:
        """Kernels this library launches per step, following its dispatch.
        Predictor: the layer-1 kernel, the layer-2 ring kernel once per group
        of up to 8 tokens (all groups OR into one union mask), and the
        compaction kernel -- except in the combined call when the one-kernel
        sparse FFN (batches up to 4 whose per-lane accumulators fit) ranks the
        mask itself.  FFN: the one-kernel FFN and its reduction when it holds
        the batch; otherwise, for 5-32 tokens with fp16 weights, the
        tensor-core gate/up kernel once per 16 tokens, the tensor-core down
        projection and the reduction of its splits; else gate/up and down on
        the CUDA cores."""
        fused = _fused_sparse_ffn(self.d, self.dtype, self.B)
        if fused:
            ffn = 2
        elif self.dtype == torch.float16 and self.B > 4:
            ffn = -(-self.B // 16) + 2
        else:
            ffn = 2
        if self.mode != "predict":
            return self.L * ffn
        pred = 1 + -(-self.B // 8)
        compact = 0 if (self.combined and fused) else 1
        return self.L * (pred + compact + ffn)

    def enqueue(self, stream=None) -> None:
        for l in range(self.L):
            x, y = self.x[l], self.y[l]
            if self.mode == "dense":
                asf_dense_ffn(self.ffns[l], x, y, self.ws, stream)
                continue
            cnt = self.count[l:l + 1]
            if self.mode == "predict" and self.combined:
                asf_predict_sparse_ffn(self.preds[l], self.ffns[l], x, self.tau, self.idx[l], cnt, y, self.ws,
                                       stream)
                continue
            if self.mode == "predict":
                asf_predict(self.preds[l], x, self.tau, self.idx[l], cnt, self.ws, stream)
            asf_sparse_ffn(self.ffns[l], x, self.idx[l], cnt, y, self.ws, stream)

    def capture(self, warmup: int = 2) -> None:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(warmup):
                self.enqueue()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph(keep_graph=True)     # keeps the node list readable
        with torch.cuda.graph(g):
            self.enqueue()
        g.instantiate()
        torch.cuda.synchronize()
        self.graph = g

    def kernel_nodes(self) -> Optional[int]:
        """Kernel launches recorded in the captured graph (None if the CUDA
        runtime bindings cannot read it): the measured counterpart of
        launches_per_step()."""
        if self.graph is None:
            return None
        try:
            from cuda.bindings import runtime as rt
            graph = rt.cudaGraph_t(init_value=self.graph.raw_cuda_graph())
            err, _, num = rt.cudaGraphGetNodes(graph, 0)
            if err != rt.cudaError_t.cudaSuccess:
                return None
            err, nodes, num = rt.cudaGraphGetNodes(graph, num)
            if err != rt.cudaError_t.cudaSuccess:
                return None
            kernels = 0
            for nd in nodes[:num]:
                err, kind = rt.cudaGraphNodeGetType(nd)
                if err == rt.cudaError_t.cudaSuccess and kind == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                    kernels += 1
            return kernels
        except Exception:
            return None

    def step(self) -> None:
        if self.graph is None:
            self.enqueue()
        else:
            self.graph.replay()

    def release(self) -> None:
        self.graph = None


def _fused_sparse_ffn(d: int, dtype, B: int) -> bool:
    """Whether the library runs the one-kernel sparse FFN for this shape: up to
    4 tokens, and at most 64 fp32 accumulators per lane (d / (8 warps x 32
    lanes x elements per 16 bytes), rounded up to 1, 2, 4 or 6 chunks, times
    elements per chunk times the token group)."""
    if B > 4:
        return False
    v = 8 if dtype == torch.float16 else 4
    q = -(-(d // v) // 256)
    q = next((c for c in (1, 2, 4, 6) if q <= c), None)
    nb = next(c for c in (1, 2, 4) if B <= c)
    return q is not None and q * v * nb <= 64


def build_layers(weights: List, device, hot_rows: Optional[Sequence[int]] = None,
                 l2_next: bool = False) -> tuple:
    """Predictor and FFN descriptors for a list of ``synthetic.LayerWeights`` on ``device``.

    hot_rows[l] (optional) is the number of leading rows of layer l that the
    offline profile found active for most tokens (the prefetch hint).  With
    l2_next, layer l's sparse FFN prefetches the predictor weights of layer
    l+1 (of layer 0 after the last layer: the next token's first layer) into
    L2; off by default, since the benchmark stack measured faster without it."""
    preds, ffns = [], []
    for l, w in enumerate(weights):
        preds.append(Predictor(w.W1, w.b1, w.W2, w.b2))
        ffns.append(FFN(w.act, w.Wg, w.Wu, w.WdT, w.bias, hot_rows=(hot_rows[l] if hot_rows else 0)))
    if l2_next:
        link_l2_next(preds, ffns)
    return preds, ffns


def link_l2_next(preds: Sequence[Predictor], ffns: Sequence[FFN]) -> None:
    """Point each layer's L2 hint at the next layer's predictor weights (cyclic)."""
    L = len(ffns)
    for l in range(L):
        nxt = preds[(l + 1) % L]
        ffns[l].set_l2_next(nxt.tensors[0], nxt.tensors[2])
