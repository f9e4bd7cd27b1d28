"""Python face of the C++ fp64 oracle (oracle/pi_oracle.cpp): marshalling only.

Test infrastructure: only the test suite, the package smoke check and the
benchmark's CPU legs use it.  Every function converts numpy inputs to the
contiguous host arrays the C entry points take, calls one of them and wraps the
result; no arithmetic of the method happens here.

`CppOracle(path)` binds one build of the library, so a test can load a copy of
the oracle compiled from a deliberately altered source; the module-level
functions use the default build (oracle/libpi_oracle.so, compiled on first use).
"""
import ctypes
from ctypes import POINTER, c_double, c_int32, c_int64, c_uint16, c_void_p

import numpy as np

from . import build as _build
from .layer import OracleLayer

RMS_EPS = 1e-6
ACT = {"relu": 0, "reglu": 1, "sqrelu": 2}
DT = {"f16": 0, "bf16": 1, "q4_0": 2}


class _PoLayer(ctypes.Structure):
    _fields_ = [
        ("d_model", c_int32), ("d_ff", c_int32), ("rank", c_int32),
        ("act", c_int32), ("wdtype", c_int32), ("pdtype", c_int32),
        ("w1", c_void_p), ("b1", c_void_p), ("w2", c_void_p), ("b2", c_void_p),
        ("threshold", c_double),
        ("w_up", c_void_p), ("w_gate", c_void_p), ("w_down_t", c_void_p),
        ("b_up", c_void_p), ("b_gate", c_void_p),
    ]


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _bits(a, dtype):
    """Stored weights as the contiguous array the C side reads: uint16 bit
    patterns for 16-bit types, uint8 bytes for Q4_0."""
    a = np.asarray(a)
    if dtype == "q4_0":
        return np.ascontiguousarray(a, dtype=np.uint8)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    return np.ascontiguousarray(a.astype(np.uint16, copy=False))


def _p(a):
    return None if a is None else a.ctypes.data_as(c_void_p)


class CppOracle:
    """One loaded build of the C++ oracle."""

    def __init__(self, path=None):
        self.path = path or _build.build()
        L = ctypes.CDLL(self.path)
        L.po_widen_f16.restype = c_double
        L.po_widen_f16.argtypes = [c_uint16]
        L.po_widen_bf16.restype = c_double
        L.po_widen_bf16.argtypes = [c_uint16]
        for n in ("po_widen_f16_n", "po_widen_bf16_n"):
            getattr(L, n).restype = None
            getattr(L, n).argtypes = [c_void_p, c_int64, c_void_p]
        L.po_dequant_q4_0.restype = None
        L.po_dequant_q4_0.argtypes = [c_void_p, c_int64, c_int32, c_void_p]
        for n in ("po_round_f16_n", "po_round_bf16_n"):
            getattr(L, n).restype = None
            getattr(L, n).argtypes = [c_void_p, c_int64, c_void_p]
        L.po_rms_cast.restype = None
        L.po_rms_cast.argtypes = [c_void_p, c_int32, c_int32, c_int32, c_void_p]
        L.po_predict.restype = None
        L.po_predict.argtypes = [POINTER(_PoLayer), c_void_p, c_int32, c_void_p, c_void_p,
                                 c_void_p]
        L.po_union_index.restype = c_int64
        L.po_union_index.argtypes = [c_void_p, c_int32, c_int32, c_void_p]
        L.po_band.restype = None
        L.po_band.argtypes = [c_void_p, c_int64, c_double, c_double, c_void_p]
        for n in ("po_neuron_outputs", "po_masked_ffn"):
            getattr(L, n).restype = c_int32
            getattr(L, n).argtypes = [POINTER(_PoLayer), c_void_p, c_int32, c_void_p, c_int64,
                                      c_void_p]
        L.po_sparse_ffn_layer.restype = c_int64
        L.po_sparse_ffn_layer.argtypes = [POINTER(_PoLayer), c_void_p, c_int32, c_void_p,
                                          c_void_p, c_void_p]
        self.lib = L

    # ------------------------------------------------------------ marshalling
    def _layer(self, layer: OracleLayer):
        """(C descriptor, list of arrays it points into, kept alive by the caller)."""
        keep = []

        def hold(a):
            if a is not None:
                keep.append(a)
            return _p(a)

        w1 = _bits(layer.w1, layer.pdtype)
        w2 = _bits(layer.w2, layer.pdtype)
        desc = _PoLayer(
            int(layer.d_model), int(layer.d_ff), int(w1.shape[0]),
            ACT[layer.act], DT[layer.wdtype], DT[layer.pdtype],
            hold(w1), hold(None if layer.b1 is None else _f64(layer.b1)),
            hold(w2), hold(_f64(layer.b2)), float(layer.threshold),
            hold(_bits(layer.w_up, layer.wdtype)),
            hold(None if layer.w_gate is None else _bits(layer.w_gate, layer.wdtype)),
            hold(_bits(layer.w_down_t, layer.wdtype)),
            hold(None if layer.b_up is None else _f64(layer.b_up)),
            hold(None if layer.b_gate is None else _f64(layer.b_gate)),
        )
        return desc, keep

    # ------------------------------------------------------------ widening
    def widen_f16(self, bits):
        a = np.asarray(bits)
        if a.dtype == np.float16:
            a = a.view(np.uint16)
        a = np.ascontiguousarray(a, dtype=np.uint16)
        out = np.empty(a.shape, dtype=np.float64)
        self.lib.po_widen_f16_n(_p(a), a.size, _p(out))
        return out

    def widen_bf16(self, bits):
        a = np.ascontiguousarray(np.asarray(bits), dtype=np.uint16)
        out = np.empty(a.shape, dtype=np.float64)
        self.lib.po_widen_bf16_n(_p(a), a.size, _p(out))
        return out

    def dequant_q4_0(self, rows, d_model):
        r = np.ascontiguousarray(np.asarray(rows), dtype=np.uint8)
        n = r.shape[0]
        if r.size != n * (d_model // 32) * 18:
            raise ValueError("Q4_0 rows have d_model/32 * 18 bytes each")
        out = np.empty((n, d_model), dtype=np.float64)
        self.lib.po_dequant_q4_0(_p(r), n, int(d_model), _p(out))
        return out

    def widen(self, a, dtype, d_model=None):
        if dtype == "f16":
            return self.widen_f16(a)
        if dtype == "bf16":
            return self.widen_bf16(a)
        if dtype == "q4_0":
            if d_model is None:
                raise ValueError("Q4_0 widening needs d_model")
            return self.dequant_q4_0(a, d_model)
        raise ValueError(f"unknown dtype {dtype!r}")

    # ------------------------------------------------------------ rounding
    def round_f16(self, x):
        x = _f64(x)
        out = np.empty_like(x)
        self.lib.po_round_f16_n(_p(x), x.size, _p(out))
        return out

    def round_bf16(self, x):
        x = _f64(x)
        out = np.empty_like(x)
        self.lib.po_round_bf16_n(_p(x), x.size, _p(out))
        return out

    def round16(self, x, dtype):
        if dtype == "f16":
            return self.round_f16(x)
        if dtype == "bf16":
            return self.round_bf16(x)
        raise ValueError(f"activations are f16 or bf16, not {dtype!r}")

    def rms_cast(self, x_resid, adtype):
        x = np.ascontiguousarray(np.atleast_2d(_f64(x_resid)))
        if adtype not in ("f16", "bf16"):
            raise ValueError(f"activations are f16 or bf16, not {adtype!r}")
        out = np.empty_like(x)
        self.lib.po_rms_cast(_p(x), x.shape[0], x.shape[1], DT[adtype], _p(out))
        return out

    # ------------------------------------------------------------ the path
    def predict(self, layer, x):
        """(a [B x r], s [B x F], mask [B x F] bool) for tokens x [B x d]."""
        x = np.ascontiguousarray(np.atleast_2d(_f64(x)))
        desc, keep = self._layer(layer)
        B = x.shape[0]
        a = np.empty((B, desc.rank), dtype=np.float64)
        s = np.empty((B, layer.d_ff), dtype=np.float64)
        m = np.empty((B, layer.d_ff), dtype=np.uint8)
        self.lib.po_predict(ctypes.byref(desc), _p(x), B, _p(a), _p(s), _p(m))
        del keep
        return a, s, m.astype(bool)

    def union_index(self, mask):
        m = np.ascontiguousarray(np.atleast_2d(np.asarray(mask, dtype=bool)).astype(np.uint8))
        B, F = m.shape
        idx = np.empty(F, dtype=np.int64)
        K = self.lib.po_union_index(_p(m), B, F, _p(idx))
        return idx[:K].copy()

    def band(self, s, threshold, width=1e-3):
        s = _f64(s)
        out = np.empty(s.shape, dtype=np.uint8)
        self.lib.po_band(_p(s), s.size, float(threshold), float(width), _p(out))
        return out.astype(bool)

    def _idx(self, idx):
        return np.ascontiguousarray(np.asarray(idx, dtype=np.int64).reshape(-1))

    def neuron_outputs(self, layer, x, idx):
        x = np.ascontiguousarray(np.atleast_2d(_f64(x)))
        idx = self._idx(idx)
        desc, keep = self._layer(layer)
        h = np.empty((x.shape[0], idx.size), dtype=np.float64)
        if self.lib.po_neuron_outputs(ctypes.byref(desc), _p(x), x.shape[0], _p(idx), idx.size,
                                      _p(h)):
            raise ValueError("neuron id outside [0, d_ff)")
        del keep
        return h

    def masked_ffn(self, layer, x, idx):
        x = np.ascontiguousarray(np.atleast_2d(_f64(x)))
        idx = self._idx(idx)
        desc, keep = self._layer(layer)
        y = np.empty((x.shape[0], layer.d_model), dtype=np.float64)
        if self.lib.po_masked_ffn(ctypes.byref(desc), _p(x), x.shape[0], _p(idx), idx.size,
                                  _p(y)):
            raise ValueError("neuron id outside [0, d_ff)")
        del keep
        return y

    def dense_ffn(self, layer, x):
        return self.masked_ffn(layer, x, np.arange(layer.d_ff))

    def true_support(self, layer, x):
        return self.neuron_outputs(layer, x, np.arange(layer.d_ff)) != 0.0

    def sparse_ffn_layer(self, layer, x):
        """(y [B x d], idx, s [B x F]): predict, union, masked FFN."""
        x = np.ascontiguousarray(np.atleast_2d(_f64(x)))
        desc, keep = self._layer(layer)
        B = x.shape[0]
        y = np.empty((B, layer.d_model), dtype=np.float64)
        idx = np.empty(layer.d_ff, dtype=np.int64)
        s = np.empty((B, layer.d_ff), dtype=np.float64)
        K = self.lib.po_sparse_ffn_layer(ctypes.byref(desc), _p(x), B, _p(y), _p(idx), _p(s))
        del keep
        return y, idx[:K].copy(), s

    def ffn_stack(self, layers, x_resid, adtype):
        """Pre-norm residual chain; returns (x_resid_out, [(idx, s, x_l)] per layer)."""
        x = np.atleast_2d(_f64(x_resid)).copy()
        trace = []
        for layer in layers:
            xl = self.rms_cast(x, adtype)
            y, idx, s = self.sparse_ffn_layer(layer, xl)
            trace.append((idx, s, xl))
            x = x + y
        return x, trace


_DEFAULT = None


def default() -> CppOracle:
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = CppOracle()
    return _DEFAULT


def _delegate(name):
    def f(*a, **k):
        return getattr(default(), name)(*a, **k)
    f.__name__ = name
    f.__doc__ = getattr(CppOracle, name).__doc__
    return f


widen_f16 = _delegate("widen_f16")
widen_bf16 = _delegate("widen_bf16")
dequant_q4_0 = _delegate("dequant_q4_0")
widen = _delegate("widen")
round_f16 = _delegate("round_f16")
round_bf16 = _delegate("round_bf16")
round16 = _delegate("round16")
rms_cast = _delegate("rms_cast")
predict = _delegate("predict")
union_index = _delegate("union_index")
band = _delegate("band")
neuron_outputs = _delegate("neuron_outputs")
masked_ffn = _delegate("masked_ffn")
dense_ffn = _delegate("dense_ffn")
true_support = _delegate("true_support")
sparse_ffn_layer = _delegate("sparse_ffn_layer")
ffn_stack = _delegate("ffn_stack")

API = ("widen_f16", "widen_bf16", "dequant_q4_0", "widen", "round_f16", "round_bf16", "round16",
       "rms_cast", "predict", "union_index", "band", "neuron_outputs", "masked_ffn", "dense_ffn",
       "true_support", "sparse_ffn_layer", "ffn_stack")
