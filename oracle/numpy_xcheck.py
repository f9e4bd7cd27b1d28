"""numpy cross-check of the C++ fp64 oracle (test infrastructure).

The oracle the CUDA library is checked against is the plain single-threaded
C++ program in oracle/pi_oracle.cpp.  This module restates the same steps with
numpy matrix products and serves one purpose: a pin that the two independent
restatements agree.  Only the test suite imports it; it shares no code with
the CUDA path or with the C++ oracle.

What it computes, and where the pages state it:

* Per token and layer, an activation predictor scores every FFN neuron and
  only neurons predicted active are processed; the rest are skipped
  (PowerInfer, unite.ai page, section "Adaptive Sparsity-Prädiktoren"; the
  machine-heart page, Figure 8: the prediction decides, a neuron labelled
  "hot" offline but predicted inactive, neuron 7, is skipped).
* The active neurons are kept in a table that maps each neuron to its original
  row of the weight matrix (unite.ai page, section "Neuronen-Platzierung und
  -Verwaltung").
* The neuron-aware operator computes the active neurons' individual row and
  column vectors directly, without converting to a sparse format (unite.ai
  page, section "Neuronenbewusster Operator").
* Models use ReLU, ReGLU or Squared-ReLU activations (GeekNews page, summary
  and limitations list); weights may be INT4 Q4_0 (GeekNews page,
  "Quantization and compatibility").

The pages give no formulas.  The readings used here are the plain ones:

* predictor: a = relu(W1 x + b1), s = W2 a + b2, neuron i predicted active iff
  s_i > tau (a tie is inactive);
* batch: the active set is the union of the tokens' predicted sets, in
  ascending neuron order, and every token is computed on the whole union;
* ReLU neuron:  h_i = max(W_up[i] . x + b_up[i], 0);
  ReGLU neuron: h_i = max(W_gate[i] . x + b_gate[i], 0) * (W_up[i] . x);
  Squared-ReLU neuron: h_i = max(W_up[i] . x + b_up[i], 0)^2 (the pages name
  the family only; squaring the ReLU output is its definition);
* output: y = sum over active i of h_i W_down^T[i] (no down bias);
* stack: pre-norm residual chain, x_l = round16(x_resid / rms(x_resid)),
  x_resid <- x_resid + FFN_l(x_l), where rms is sqrt(mean(x^2) + 1e-6) and
  round16 is round-to-nearest-even to the layer's 16-bit activation type;
* Q4_0: per 32-element block an fp16 scale and 16 bytes, byte j holding
  element j (low nibble) and j+16 (high nibble); value = (q - 8) * scale.

Every weight is widened exactly to fp64; all arithmetic is fp64.
"""
from typing import Iterable, Optional

import numpy as np

from .layer import OracleLayer

RMS_EPS = 1e-6


# --------------------------------------------------------------------------
# exact widening of stored weights
# --------------------------------------------------------------------------
def widen_f16(bits: np.ndarray) -> np.ndarray:
    """IEEE binary16 values (raw uint16 bits or np.float16) -> fp64."""
    a = np.asarray(bits)
    if a.dtype == np.float16:
        return a.astype(np.float64)
    return a.astype(np.uint16).view(np.float16).astype(np.float64)


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bfloat16 values given as raw uint16 bits -> fp64 (the bits are the top
    half of an IEEE binary32)."""
    u = np.asarray(bits).astype(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def dequant_q4_0(rows: np.ndarray, d_model: int) -> np.ndarray:
    """Q4_0 rows [n x d/32*18] (uint8) -> fp64 [n x d]."""
    rows = np.asarray(rows, dtype=np.uint8)
    n = rows.shape[0]
    nb = d_model // 32
    blk = rows.reshape(n, nb, 18)
    scale = blk[:, :, 0:2].copy().view(np.uint16).reshape(n, nb)
    scale = widen_f16(scale)
    qs = blk[:, :, 2:18].astype(np.int64)
    lo = (qs & 0x0F) - 8          # elements 0..15 of the block
    hi = (qs >> 4) - 8            # elements 16..31 of the block
    q = np.concatenate([lo, hi], axis=2).astype(np.float64)
    return (q * scale[:, :, None]).reshape(n, d_model)


def widen(a: np.ndarray, dtype: str, d_model: Optional[int] = None) -> np.ndarray:
    if dtype == "f16":
        return widen_f16(a)
    if dtype == "bf16":
        return widen_bf16(a)
    if dtype == "q4_0":
        if d_model is None:
            raise ValueError("Q4_0 widening needs d_model")
        return dequant_q4_0(a, d_model)
    raise ValueError(f"unknown dtype {dtype!r}")


# --------------------------------------------------------------------------
# rounding to the 16-bit activation types
# --------------------------------------------------------------------------
def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bfloat16 (8 significant bits), nearest-even, in one
    step.  Values are assumed to lie in the normal bf16 range or be zero."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2^e, 0.5 <= |m| < 1
    q = np.rint(np.ldexp(m, 8))             # 8 significant bits, ties to even
    out = np.ldexp(q, e - 8)
    tiny = (x != 0) & (np.abs(x) < 2.0**-126)
    if np.any(tiny):
        raise ValueError("round_bf16: subnormal inputs are outside this oracle's range")
    return out


def round_f16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to IEEE binary16, nearest-even (numpy's direct
    double-to-half conversion)."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def round16(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f16":
        return round_f16(x)
    if dtype == "bf16":
        return round_bf16(x)
    raise ValueError(f"activations are f16 or bf16, not {dtype!r}")


# --------------------------------------------------------------------------
# a layer's rows, widened on use
# --------------------------------------------------------------------------
def rows(layer: OracleLayer, name: str, idx: np.ndarray) -> np.ndarray:
    """fp64 copies of the given neuron rows of one FFN matrix."""
    m = getattr(layer, name)
    return widen(np.asarray(m)[np.asarray(idx, dtype=np.int64)], layer.wdtype, layer.d_model)


# --------------------------------------------------------------------------
# the hot path, step by step
# --------------------------------------------------------------------------
def predict(layer: OracleLayer, x: np.ndarray):
    """Activation predictor for tokens x [B x d] (fp64 values).

    Returns (a [B x r], s [B x F], mask [B x F] bool).  a = relu(W1 x + b1),
    s = W2 a + b2, mask = s > threshold.
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    w1 = widen(layer.w1, layer.pdtype)
    w2 = widen(layer.w2, layer.pdtype)
    z = x @ w1.T
    if layer.b1 is not None:
        z = z + np.asarray(layer.b1, dtype=np.float64)
    a = np.maximum(z, 0.0)
    s = a @ w2.T + np.asarray(layer.b2, dtype=np.float64)
    return a, s, s > layer.threshold


def union_index(mask: np.ndarray) -> np.ndarray:
    """Ascending list of neurons predicted active for at least one token."""
    mask = np.atleast_2d(np.asarray(mask, dtype=bool))
    return np.flatnonzero(mask.any(axis=0)).astype(np.int64)


def band(s: np.ndarray, threshold: float, width: float = 1e-3) -> np.ndarray:
    """Neurons whose logit lies within `width` of the threshold; near the
    threshold either decision is acceptable for a rounding-level difference."""
    return np.abs(np.asarray(s, dtype=np.float64) - threshold) < width


def neuron_outputs(layer: OracleLayer, x: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """h [B x K]: activation of each listed neuron for each token."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    idx = np.asarray(idx, dtype=np.int64)
    up = rows(layer, "w_up", idx)
    if layer.act in ("relu", "sqrelu"):
        pre = x @ up.T
        if layer.b_up is not None:
            pre = pre + np.asarray(layer.b_up, dtype=np.float64)[idx]
        r = np.maximum(pre, 0.0)
        return r if layer.act == "relu" else r * r
    if layer.act == "reglu":
        gate = rows(layer, "w_gate", idx)
        g = x @ gate.T
        if layer.b_gate is not None:
            g = g + np.asarray(layer.b_gate, dtype=np.float64)[idx]
        return np.maximum(g, 0.0) * (x @ up.T)
    raise ValueError(f"unknown activation {layer.act!r}")


def masked_ffn(layer: OracleLayer, x: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """y [B x d] = sum over the listed neurons i of h_i * W_down^T[i]."""
    idx = np.asarray(idx, dtype=np.int64)
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    if idx.size == 0:
        return np.zeros((x.shape[0], layer.d_model))
    h = neuron_outputs(layer, x, idx)
    down = rows(layer, "w_down_t", idx)
    return h @ down


def dense_ffn(layer: OracleLayer, x: np.ndarray) -> np.ndarray:
    """Every neuron computed: the dense-inference result."""
    return masked_ffn(layer, x, np.arange(layer.d_ff))


def true_support(layer: OracleLayer, x: np.ndarray) -> np.ndarray:
    """[B x F] bool: neurons whose activation is nonzero (ReLU and Squared-ReLU:
    pre-activation > 0; ReGLU: gate pre-activation > 0 and up projection
    nonzero)."""
    return neuron_outputs(layer, x, np.arange(layer.d_ff)) != 0.0


def sparse_ffn_layer(layer: OracleLayer, x: np.ndarray):
    """Predict, take the union, compute the masked FFN.

    Returns (y [B x d], idx, s [B x F]).
    """
    _, s, mask = predict(layer, x)
    idx = union_index(mask)
    return masked_ffn(layer, x, idx), idx, s


def rms_cast(x_resid: np.ndarray, adtype: str) -> np.ndarray:
    """Layer input: each token divided by its RMS, rounded to the 16-bit type."""
    x = np.atleast_2d(np.asarray(x_resid, dtype=np.float64))
    rms = np.sqrt(np.mean(x * x, axis=1, keepdims=True) + RMS_EPS)
    return round16(x / rms, adtype)


def ffn_stack(layers: Iterable[OracleLayer], x_resid: np.ndarray, adtype: str):
    """Run the layer stack on the residual stream x_resid [B x d].

    Returns (x_resid_out, per-layer list of (idx, s, x_l)).
    """
    x = np.atleast_2d(np.asarray(x_resid, dtype=np.float64)).copy()
    trace = []
    for layer in layers:
        xl = rms_cast(x, adtype)
        y, idx, s = sparse_ffn_layer(layer, xl)
        trace.append((idx, s, xl))
        x = x + y
    return x, trace
