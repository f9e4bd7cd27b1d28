"""B200-native predictor-gated sparse FFN (PowerInfer's neuron-aware FFN).

The compute lives in libpi.so (CUDA, sm_100a); this package is its ctypes
binding.  See include/pi.h for the C ABI.
"""
from .binding import (  # noqa: F401
    ACTS,
    DTYPES,
    EXPORTS,
    PI_BF16,
    PI_F16,
    PI_Q4_0,
    PI_REGLU,
    PI_RELU,
    PI_SQRELU,
    PiError,
    PiLayer,
    PiPredictor,
    layer_array,
    layer_desc,
    layer_from_tensors,
    lib,
    pi_compact,
    pi_device_error,
    pi_ffn_stack,
    pi_ffn_stack_timed,
    pi_last_error,
    pi_launch_count,
    pi_permute_layer,
    pi_predict,
    pi_sparse_ffn,
    pi_sparse_ffn_static,
    pi_status_string,
    pi_workspace_size,
    predictor_desc,
)
