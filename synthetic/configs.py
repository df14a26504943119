"""Workload shapes for the decode-time sparse FFN.

Each entry is a seeded synthetic stand-in for one of the model shapes the
activation-sparsity pages discuss (Llama-2, Falcon-40B, a 70B ReGLU model,
OPT-175B, plus a tiny fp32 layer).  No dataset or trained checkpoint is used:
weights and inputs are drawn from the recipe in ``synthetic.generator``.

Notation (PowerInfer Guide, "The Hidden Inefficiency" FFN equation):
  d      hidden size (length of x)
  n      intermediate size d_ffn (number of FFN neurons)
  r      hidden width of the two-layer predictor MLP (PowerInfer_x64 page,
         "Prediction and Caching": a 2-layer MLP predictor)
  act    "reglu": FFN(x) = W_down (ReLU(W_gate x + b) * (W_up x))
         "relu" : FFN(x) = W_down  ReLU(W_up x + b)      (up + down, no gate)
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Tuple


@dataclass(frozen=True)
class FFNConfig:
    name: str
    act: str                 # "reglu" or "relu"
    d: int
    n: int
    r: int
    layers: int
    dtype: str               # "f32" or "f16": weight and x storage type
    tokens: int              # evaluation tokens per batch size
    batches: Tuple[int, ...] = (1,)
    gamma: float = 1.2       # Zipf exponent of per-neuron activation frequency
    frac: float = 0.10       # mean active fraction per token
    seed: int = 0
    hot_perm: bool = False   # store the hot rows first (offline permutation)
    tau: float = 0.5         # predictor threshold on sigmoid output
    hot_ratio: float = 0.20  # fraction of neurons called "hot"
    calib_tokens: int = 512  # tokens used by the offline activation profiler

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def mats(self) -> int:
        """Weight rows touched per active neuron (gate+up+down or up+down)."""
        return 3 if self.act == "reglu" else 2

    def with_(self, **kw) -> "FFNConfig":
        return replace(self, **kw)


CONFIGS = {
    # Tiny ReGLU layer in fp32; L2-resident, reported as time per token.
    "tiny_reglu_f32": FFNConfig(
        name="tiny_reglu_f32", act="reglu", d=512, n=1376, r=64, layers=1,
        dtype="f32", tokens=64, gamma=1.2, frac=0.10, seed=0),
    # Llama2-7B-shaped ReGLU stack (ProSparse-like ~90% sparsity), hot rows first.
    "llama2_7b_reglu": FFNConfig(
        name="llama2_7b_reglu", act="reglu", d=4096, n=11008, r=1024, layers=32,
        dtype="f16", tokens=256, gamma=1.2, frac=0.10, seed=1, hot_perm=True),
    # Falcon-40B-shaped plain ReLU FFN (up + down).
    "falcon_40b_relu": FFNConfig(
        name="falcon_40b_relu", act="relu", d=8192, n=32768, r=1024, layers=60,
        dtype="f16", tokens=128, gamma=1.2, frac=0.10, seed=2),
    # 70B-shaped ReGLU, batched decode over the union of per-token active sets.
    "llama70b_reglu": FFNConfig(
        name="llama70b_reglu", act="reglu", d=8192, n=28672, r=1024, layers=80,
        dtype="f16", tokens=64, batches=(1, 4, 16, 32), gamma=1.3, frac=0.12, seed=3),
    # OPT-175B-shaped ReLU FFN with a heavier cold tail; permutation on/off and
    # a dense GEMV reference at the same shapes.
    "opt175b_relu": FFNConfig(
        name="opt175b_relu", act="relu", d=12288, n=49152, r=1024, layers=8,
        dtype="f16", tokens=64, batches=(1, 4, 16), gamma=1.1, frac=0.08, seed=4,
        hot_perm=True),
}

CONFIG_ORDER = ["tiny_reglu_f32", "llama2_7b_reglu", "falcon_40b_relu",
                "llama70b_reglu", "opt175b_relu"]


def get(name: str) -> FFNConfig:
    return CONFIGS[name]
