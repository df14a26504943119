"""Shared set-up for the GPU parity tests (inputs from ``synthetic``, references
from ``oracle``; the CUDA path is reached only through the C ABI binding)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import synthetic as S
from tests.helpers import condition_b2

import activation_sparse_ffn_predict_b200 as A


def ensure_built():
    from activation_sparse_ffn_predict_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


class Layer:
    """One layer: host (numpy) copy for the oracle, device tensors for the kernels."""

    def __init__(self, cfg: S.FFNConfig, layer: int = 0, n_tokens: int = 8, condition: bool = True,
                 device_gen: bool = False, extra_tokens=None):
        self.cfg = cfg
        dev = torch.device("cuda")
        w = S.layer_weights(cfg, layer, device=dev if device_gen else "cpu")
        X = S.layer_tokens(cfg, layer, n_tokens, device=dev if device_gen else "cpu")
        self.h = w.numpy()
        self.X = X.cpu().numpy()
        if condition:
            self.h["b2"] = condition_b2(self.h["W1"], self.h["b1"], self.h["W2"], self.h["b2"], self.X,
                                        cfg.tau)
            w.b2 = torch.from_numpy(self.h["b2"])
        self.w = w.to(dev)
        self.Xd = X.to(dev)
        self.pred = A.Predictor(self.w.W1, self.w.b1, self.w.W2, self.w.b2)
        self.ffn = A.FFN(self.w.act, self.w.Wg, self.w.Wu, self.w.WdT, self.w.bias)
        self.ws = A.Workspace(self.pred, self.ffn, 32)

    # ---------------------------------------------------------------- oracle --
    def oracle_idx(self, rows) -> np.ndarray:
        h = self.h
        return O.predict(h["W1"], h["b1"], h["W2"], h["b2"], self.X[rows], self.cfg.tau)[0]

    def oracle_y(self, rows, idx) -> np.ndarray:
        h = self.h
        return O.sparse_ffn(h["act"], h["Wg"], h["Wu"], h["WdT"], h["bias"], self.X[rows], idx)

    # --------------------------------------------------------------- device --
    def predict(self, rows):
        x = self.Xd[rows].contiguous()
        idx = torch.full((self.cfg.n,), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        A.asf_predict(self.pred, x, self.cfg.tau, idx, cnt, self.ws)
        torch.cuda.synchronize()
        c = int(cnt.item())
        return idx[:c].cpu().numpy(), idx.cpu().numpy(), c

    def sparse(self, rows, idx_np, count=None):
        x = self.Xd[rows].contiguous()
        idx = torch.zeros(self.cfg.n, dtype=torch.int32, device="cuda")
        k = len(idx_np)
        if k:
            idx[:k] = torch.from_numpy(np.asarray(idx_np, dtype=np.int32)).cuda()
        cnt = torch.tensor([k if count is None else count], dtype=torch.int32, device="cuda")
        y = torch.full((x.shape[0], self.cfg.d), float("nan"), dtype=torch.float32, device="cuda")
        A.asf_sparse_ffn(self.ffn, x, idx, cnt, y, self.ws)
        torch.cuda.synchronize()
        return y.cpu().numpy()

    def dense(self, rows):
        x = self.Xd[rows].contiguous()
        y = torch.full((x.shape[0], self.cfg.d), float("nan"), dtype=torch.float32, device="cuda")
        A.asf_dense_ffn(self.ffn, x, y, self.ws)
        torch.cuda.synchronize()
        return y.cpu().numpy()

    def error(self) -> int:
        return A.asf_read_error(self.ws)
