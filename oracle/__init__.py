"""CPU oracle (float64) for the activation-sparse FFN decode path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference arm, never by the product path.
"""
from .ffn import (activations, compact, dense_ffn, hot_permutation,  # noqa: F401
                  inverse_permutation, logit, partition, permute_rows, predict,
                  predictor_band, predictor_hidden, predictor_logits, predictor_mask,
                  profile_counts, record_activations, relu_input, relu_input_band,
                  sparse_ffn, true_active)
