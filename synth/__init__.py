"""Seeded synthetic inputs for the predictor-gated sparse FFN.

This package only *draws* data: Gaussian weights, a Zipf firing profile, a
predictor built from the true activation, Q4_0 packing and input tokens.  It
computes none of the steps the sparse FFN itself performs (no predictor
evaluation, no mask, no gathered up/down projection); both the CUDA library
and the fp64 oracle receive its tensors as plain inputs.
"""
from .configs import CONFIGS, Config, get_config
from .layers import (
    LayerData,
    make_layer,
    make_tokens,
    with_mode,
    zipf_profile,
    quantize_q4_0,
    q4_0_row_bytes,
)

__all__ = [
    "CONFIGS",
    "Config",
    "get_config",
    "LayerData",
    "make_layer",
    "make_tokens",
    "with_mode",
    "zipf_profile",
    "quantize_q4_0",
    "q4_0_row_bytes",
]
