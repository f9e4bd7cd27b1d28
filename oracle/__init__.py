"""fp64 CPU oracle of the predictor-gated sparse FFN (test infrastructure).

The oracle is the plain, single-threaded C++ program in pi_oracle.cpp; this
package exposes it to the tests, the smoke check and the benchmark's CPU legs
through ctypes (cpp.py).  numpy_xcheck.py is an independent numpy restatement
kept only as a cross-check pin.  Nothing here is used by the CUDA library.
"""
from .cpp import (  # noqa: F401
    RMS_EPS,
    CppOracle,
    band,
    default,
    dense_ffn,
    dequant_q4_0,
    ffn_stack,
    masked_ffn,
    neuron_outputs,
    predict,
    rms_cast,
    round16,
    round_bf16,
    round_f16,
    sparse_ffn_layer,
    true_support,
    union_index,
    widen,
    widen_bf16,
    widen_f16,
)
from .layer import OracleLayer  # noqa: F401
