"""Activation-sparse FFN decode path for B200 (sm_100a).

PowerInfer-style neuron-level sparsity on one GPU: a two-layer predictor turns
the FFN input into an ascending list of active neurons, and a neuron-aware
sparse operator gathers only those rows of W_gate / W_up and W_down^T.  All
arithmetic runs in the CUDA kernels of ``libasffn.so`` behind the C ABI of
``include/asffn.h``; this package is the thin Python binding to it (torch is
used for device memory and streams only).  There is no CPU fallback: calls
fail loudly if the library is not built or a tensor is not on the GPU.
"""
from . import _lib  # noqa: F401
from .api import (FFN, AsfError, Predictor, Workspace, asf_activation_counts,  # noqa: F401
                  asf_dense_ffn, asf_gather_rows, asf_hot_permutation, asf_permute_rows, asf_predict,
                  asf_predict_sparse_ffn, asf_predict_sparse_ffn_begin, asf_predict_sparse_ffn_end,
                  asf_predict_sparse_ffn_exchange, asf_read_error, asf_reduce_exchange, asf_set_fault_injection, asf_sparse_ffn, asf_sparse_ffn_noalloc,
                  asf_status_string, asf_version, asf_workspace_bytes, asf_workspace_init, pack_layer)
from .stack import LayerStack  # noqa: F401
