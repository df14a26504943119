"""Seeded synthetic workloads shared by the CUDA path's tests/bench and the oracle.

Holds random draws and bias calibration only; no FFN or predictor arithmetic.
"""
from .configs import CONFIGS, CONFIG_ORDER, FFNConfig, get  # noqa: F401
from .generator import (LayerWeights, activity_profile, layer_tokens,  # noqa: F401
                        layer_weights, rank_to_neuron, seed_for, zipf_rank_profile)
