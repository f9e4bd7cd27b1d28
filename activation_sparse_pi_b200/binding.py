"""Thin ctypes binding of libpi (include/pi.h): argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors (device memory) or None where the C call takes a pointer, and raises
PiError when the call returns a non-zero status.  All computation happens in
the library's CUDA kernels; there is no fallback.
"""
import ctypes
import os
from ctypes import c_float, c_int32, c_size_t, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpi.so")

PI_OK, PI_ERR_INVALID_ARG, PI_ERR_UNSUPPORTED, PI_ERR_WORKSPACE, PI_ERR_CUDA = range(5)
PI_STATIC_SCRATCH_BYTES = 16 << 20  # fixed scratch of pi_sparse_ffn_static
PI_F16, PI_BF16, PI_Q4_0 = 0, 1, 2
PI_RELU, PI_REGLU, PI_SQRELU = 0, 1, 2
DTYPES = {"f16": PI_F16, "bf16": PI_BF16, "q4_0": PI_Q4_0}
ACTS = {"relu": PI_RELU, "reglu": PI_REGLU, "sqrelu": PI_SQRELU}

EXPORTS = (
    "pi_status_string", "pi_last_error", "pi_device_error", "pi_launch_count", "pi_workspace_size",
    "pi_predict", "pi_compact", "pi_sparse_ffn", "pi_ffn_stack", "pi_ffn_stack_timed",
    "pi_sparse_ffn_static", "pi_permute_layer",
)


class PiError(RuntimeError):
    def __init__(self, status, where, detail):
        super().__init__(f"{where}: status {status}: {detail}")
        self.status = status


class PiPredictor(ctypes.Structure):
    _fields_ = [
        ("d_model", c_int32), ("rank", c_int32), ("d_ff", c_int32), ("dtype", c_int32),
        ("w1", c_void_p), ("b1", c_void_p), ("w2", c_void_p), ("b2", c_void_p),
        ("threshold", c_float), ("reserved", c_int32),
    ]


class PiLayer(ctypes.Structure):
    _fields_ = [
        ("d_model", c_int32), ("d_ff", c_int32), ("wdtype", c_int32), ("adtype", c_int32),
        ("act", c_int32), ("reserved", c_int32),
        ("w_up", c_void_p), ("w_gate", c_void_p), ("w_down_t", c_void_p),
        ("b_up", c_void_p), ("b_gate", c_void_p),
        ("pred", PiPredictor),
    ]


_lib = None


def lib():
    """The loaded library; raises if libpi.so has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m activation_sparse_pi_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.pi_status_string.restype = ctypes.c_char_p
        L.pi_status_string.argtypes = [c_int32]
        L.pi_last_error.restype = ctypes.c_char_p
        L.pi_last_error.argtypes = []
        L.pi_device_error.restype = c_int32
        L.pi_device_error.argtypes = [ctypes.POINTER(c_int32)]
        L.pi_launch_count.restype = ctypes.c_uint64
        L.pi_launch_count.argtypes = []
        L.pi_workspace_size.restype = c_size_t
        L.pi_workspace_size.argtypes = [ctypes.POINTER(PiLayer), c_int32, c_int32]
        L.pi_predict.restype = c_int32
        L.pi_predict.argtypes = [ctypes.POINTER(PiPredictor), c_void_p, c_int32, c_void_p,
                                 c_void_p, c_void_p, c_size_t, c_void_p]
        L.pi_compact.restype = c_int32
        L.pi_compact.argtypes = [c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                 c_size_t, c_void_p]
        L.pi_sparse_ffn.restype = c_int32
        L.pi_sparse_ffn.argtypes = [ctypes.POINTER(PiLayer), c_void_p, c_int32, c_void_p,
                                    c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]
        L.pi_sparse_ffn_static.restype = c_int32
        L.pi_sparse_ffn_static.argtypes = [ctypes.POINTER(PiLayer), c_void_p, c_int32, c_void_p,
                                           c_void_p, c_void_p, c_void_p]
        L.pi_ffn_stack.restype = c_int32
        L.pi_ffn_stack.argtypes = [ctypes.POINTER(PiLayer), c_int32, c_void_p, c_int32,
                                   c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]
        L.pi_ffn_stack_timed.restype = c_int32
        L.pi_ffn_stack_timed.argtypes = [ctypes.POINTER(PiLayer), c_int32, c_void_p, c_int32,
                                         c_void_p, c_void_p, c_void_p, c_size_t, c_void_p,
                                         ctypes.POINTER(c_void_p)]
        L.pi_permute_layer.restype = c_int32
        L.pi_permute_layer.argtypes = [ctypes.POINTER(PiLayer), c_void_p, ctypes.POINTER(PiLayer),
                                       c_void_p]
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        if not torch.cuda.is_available():
            return None  # the legacy default stream; host-side validation still runs
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status, where):
    if status != PI_OK:
        detail = lib().pi_last_error().decode(errors="replace")
        raise PiError(status, where, detail)


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


# ---------------------------------------------------------------- descriptors
def predictor_desc(d_model, rank, d_ff, dtype, w1, b1, w2, b2, threshold=0.0):
    return PiPredictor(d_model, rank, d_ff, DTYPES.get(dtype, dtype), _ptr(w1), _ptr(b1),
                       _ptr(w2), _ptr(b2), float(threshold), 0)


def layer_desc(d_model, d_ff, wdtype, adtype, act, w_up, w_gate, w_down_t, b_up, b_gate,
               pred: PiPredictor):
    return PiLayer(d_model, d_ff, DTYPES.get(wdtype, wdtype), DTYPES.get(adtype, adtype),
                   ACTS.get(act, act), 0, _ptr(w_up), _ptr(w_gate), _ptr(w_down_t), _ptr(b_up),
                   _ptr(b_gate), pred)


def layer_from_tensors(*, d_model, d_ff, rank, wdtype, adtype, act, w1, b1, w2, b2, threshold,
                       w_up, w_gate, w_down_t, b_up, b_gate):
    """A pi_layer descriptor over device tensors (the caller keeps them alive)."""
    pred = predictor_desc(d_model, rank, d_ff, adtype, w1, b1, w2, b2, threshold)
    return layer_desc(d_model, d_ff, wdtype, adtype, act, w_up, w_gate, w_down_t, b_up, b_gate,
                      pred)


def layer_array(descs):
    arr = (PiLayer * len(descs))()
    for i, d in enumerate(descs):
        arr[i] = d
    return arr


# ---------------------------------------------------------------- entry points
def pi_status_string(status):
    return lib().pi_status_string(status).decode()


def pi_last_error():
    return lib().pi_last_error().decode(errors="replace")


def pi_device_error():
    v = c_int32(0)
    _check(lib().pi_device_error(ctypes.byref(v)), "pi_device_error")
    return v.value


def pi_launch_count():
    return int(lib().pi_launch_count())


def pi_workspace_size(layers, batch):
    arr = layers if isinstance(layers, ctypes.Array) else layer_array(list(layers))
    return int(lib().pi_workspace_size(arr, len(arr), int(batch)))


def pi_predict(pred, x, batch, mask_bits, logits, workspace, stream=None):
    _check(lib().pi_predict(ctypes.byref(pred), _ptr(x), int(batch), _ptr(mask_bits),
                            _ptr(logits), _ptr(workspace), _nbytes(workspace),
                            _stream(stream)), "pi_predict")


def pi_compact(mask_bits, batch, d_ff, idx, count, workspace=None, stream=None):
    _check(lib().pi_compact(_ptr(mask_bits), int(batch), int(d_ff), _ptr(idx), _ptr(count),
                            _ptr(workspace), _nbytes(workspace), _stream(stream)), "pi_compact")


def pi_sparse_ffn(layer, x, batch, idx, count, y, workspace, stream=None):
    _check(lib().pi_sparse_ffn(ctypes.byref(layer), _ptr(x), int(batch), _ptr(idx), _ptr(count),
                               _ptr(y), _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "pi_sparse_ffn")


def pi_sparse_ffn_static(layer, x, batch, idx, count, y, stream=None):
    _check(lib().pi_sparse_ffn_static(ctypes.byref(layer), _ptr(x), int(batch), _ptr(idx),
                                      _ptr(count), _ptr(y), _stream(stream)),
           "pi_sparse_ffn_static")


def pi_ffn_stack(layers, x_resid, batch, idx_out, count_out, workspace, stream=None):
    arr = layers if isinstance(layers, ctypes.Array) else layer_array(list(layers))
    _check(lib().pi_ffn_stack(arr, len(arr), _ptr(x_resid), int(batch), _ptr(idx_out),
                              _ptr(count_out), _ptr(workspace), _nbytes(workspace),
                              _stream(stream)), "pi_ffn_stack")


def pi_ffn_stack_timed(layers, x_resid, batch, idx_out, count_out, workspace, ffn_events,
                       stream=None):
    """ffn_events: sequence of 2 * n_layers torch.cuda.Event (enable_timing=True)."""
    arr = layers if isinstance(layers, ctypes.Array) else layer_array(list(layers))
    if ffn_events is None:
        ev = None
    else:
        ev = (c_void_p * len(ffn_events))(*[e.cuda_event if hasattr(e, "cuda_event") else e
                                            for e in ffn_events])
    _check(lib().pi_ffn_stack_timed(arr, len(arr), _ptr(x_resid), int(batch), _ptr(idx_out),
                                    _ptr(count_out), _ptr(workspace), _nbytes(workspace),
                                    _stream(stream), ev), "pi_ffn_stack_timed")


def pi_permute_layer(src, perm, dst, stream=None):
    """src, dst: PiLayer descriptors; perm: int32 device tensor [d_ff]."""
    _check(lib().pi_permute_layer(ctypes.byref(src), _ptr(perm), ctypes.byref(dst),
                                  _stream(stream)), "pi_permute_layer")
