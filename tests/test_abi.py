"""Host-side checks of the C-ABI library (no GPU needed).

The library must load and export every entry point declared in
include/pi.h, and argument validation happens on the host before anything is
enqueued, so invalid calls return their error code without a device.
"""
import ctypes
import os
import re

import pytest

import activation_sparse_pi_b200 as pi
from activation_sparse_pi_b200 import build as pibuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    pibuild.build()
    return pi.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "pi.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pi_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(pi.EXPORTS), names
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_struct_layout_matches_header():
    # pi_predictor: 4 x int32, 4 pointers, float, int32 -> 56 bytes
    assert ctypes.sizeof(pi.PiPredictor) == 56
    assert pi.PiPredictor.w1.offset == 16 and pi.PiPredictor.threshold.offset == 48
    # pi_layer: 6 x int32, 5 pointers, pi_predictor -> 120 bytes
    assert ctypes.sizeof(pi.PiLayer) == 120
    assert pi.PiLayer.w_up.offset == 24 and pi.PiLayer.pred.offset == 64


def test_status_strings(lib):
    assert pi.pi_status_string(0) == "success"
    for s in range(1, 5):
        assert pi.pi_status_string(s) not in ("success", "unknown status")
    assert pi.pi_status_string(99) == "unknown status"


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced here


def _pred(**kw):
    a = dict(d_model=512, rank=128, d_ff=2048, dtype="f16", w1=FAKE, b1=None, w2=FAKE, b2=FAKE,
             threshold=0.0)
    a.update(kw)
    return pi.predictor_desc(**a)


def _layer(**kw):
    pred = kw.pop("pred", _pred())
    a = dict(d_model=512, d_ff=2048, wdtype="f16", adtype="f16", act="relu", w_up=FAKE,
             w_gate=None, w_down_t=FAKE, b_up=FAKE, b_gate=None)
    a.update(kw)
    return pi.layer_desc(pred=pred, **a)


def _status(fn, *args):
    try:
        fn(*args)
    except pi.PiError as e:
        return e.status
    return 0


@pytest.mark.parametrize("kw,expect", [
    (dict(d_model=500), pi.binding.PI_ERR_UNSUPPORTED),
    (dict(d_model=16384), pi.binding.PI_ERR_UNSUPPORTED),
    (dict(d_ff=100), pi.binding.PI_ERR_UNSUPPORTED),
    (dict(rank=4), pi.binding.PI_ERR_UNSUPPORTED),
    (dict(dtype="q4_0"), pi.binding.PI_ERR_UNSUPPORTED),
    (dict(w1=None), pi.binding.PI_ERR_INVALID_ARG),
    (dict(b2=None), pi.binding.PI_ERR_INVALID_ARG),
    (dict(w2=FAKE + 8), pi.binding.PI_ERR_INVALID_ARG),
])
def test_predict_rejects_bad_predictor(lib, kw, expect):
    st = _status(pi.pi_predict, _pred(**kw), FAKE, 1, FAKE, None, None, 0)
    assert st == expect, pi.pi_last_error()


def test_predict_rejects_batch_and_workspace(lib):
    assert _status(pi.pi_predict, _pred(), FAKE, 0, FAKE, None, None, 0) == pi.binding.PI_ERR_UNSUPPORTED
    assert _status(pi.pi_predict, _pred(), FAKE, 65, FAKE, None, None, 0) == pi.binding.PI_ERR_UNSUPPORTED
    assert _status(pi.pi_predict, _pred(), FAKE, 1, FAKE, None, None, 0) == pi.binding.PI_ERR_WORKSPACE
    assert "workspace" in pi.pi_last_error()
    assert _status(pi.pi_predict, _pred(), None, 1, FAKE, None, None, 0) == pi.binding.PI_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,expect", [
    (dict(act="reglu"), pi.binding.PI_ERR_INVALID_ARG),              # no w_gate
    (dict(w_gate=FAKE), pi.binding.PI_ERR_INVALID_ARG),              # gate for ReLU
    (dict(wdtype="bf16"), pi.binding.PI_ERR_UNSUPPORTED),            # weights != activations
    (dict(wdtype="q4_0", d_model=512), 0),                           # allowed (d % 256 == 0)
    (dict(act="sqrelu"), 0),                                         # Squared-ReLU: like ReLU
    (dict(act="sqrelu", w_gate=FAKE), pi.binding.PI_ERR_INVALID_ARG),  # no gate
    (dict(act="sqrelu", b_gate=FAKE), pi.binding.PI_ERR_INVALID_ARG),
    (dict(wdtype="q4_0", d_model=480, pred=_pred(d_model=480)), pi.binding.PI_ERR_UNSUPPORTED),
    (dict(adtype="bf16"), pi.binding.PI_ERR_UNSUPPORTED),            # != predictor dtype
    (dict(d_ff=1024), pi.binding.PI_ERR_INVALID_ARG),                # != predictor d_ff
    (dict(w_down_t=None), pi.binding.PI_ERR_INVALID_ARG),
    (dict(act="reglu", w_gate=FAKE, b_up=FAKE), pi.binding.PI_ERR_INVALID_ARG),
])
def test_layer_validation(lib, kw, expect):
    L = _layer(**kw)
    size = pi.pi_workspace_size([L], 1)
    if expect == 0:
        assert size > 0
    else:
        assert size == 0
        st = _status(pi.pi_sparse_ffn, L, FAKE, 1, FAKE, FAKE, FAKE, None)
        assert st == expect, pi.pi_last_error()


def test_workspace_size_grows_with_batch(lib):
    L = _layer()
    s1, s8 = pi.pi_workspace_size([L], 1), pi.pi_workspace_size([L], 8)
    assert 0 < s1 < s8
    assert pi.pi_workspace_size([L], 0) == 0
    assert pi.pi_workspace_size([L], 65) == 0


def test_compact_and_stack_validation(lib):
    assert _status(pi.pi_compact, FAKE, 1, 100, FAKE, FAKE) == pi.binding.PI_ERR_UNSUPPORTED
    assert _status(pi.pi_compact, None, 1, 128, FAKE, FAKE) == pi.binding.PI_ERR_INVALID_ARG
    assert _status(pi.pi_compact, FAKE, 1, 128, FAKE + 4, FAKE) == pi.binding.PI_ERR_INVALID_ARG
    L1, L2 = _layer(), _layer(d_model=1024, pred=_pred(d_model=1024))
    st = _status(pi.pi_ffn_stack, [L1, L2], FAKE, 1, None, None, None)
    assert st == pi.binding.PI_ERR_INVALID_ARG  # mixed d_model
    st = _status(pi.pi_ffn_stack, [L1], FAKE, 1, None, None, None)
    assert st == pi.binding.PI_ERR_WORKSPACE


@pytest.mark.parametrize("d,B", [(4096, 8), (2048, 8), (8192, 64), (512, 64)])
def test_static_scratch_rejects_oversized_shapes(lib, d, B):
    # each shape needs more than the fixed scratch holds; the call must refuse
    # before touching the device (only refused shapes may use fake pointers)
    L = _layer(d_model=d, pred=_pred(d_model=d))
    st = _status(pi.pi_sparse_ffn_static, L, FAKE, B, FAKE, FAKE, FAKE)
    assert st == pi.binding.PI_ERR_WORKSPACE, pi.pi_last_error()
    msg = pi.pi_last_error()
    assert "needs" in msg and str(pi.binding.PI_STATIC_SCRATCH_BYTES) in msg, msg


def test_static_scratch_validates_arguments(lib):
    L = _layer()
    st = _status(pi.pi_sparse_ffn_static, L, None, 1, FAKE, FAKE, FAKE)
    assert st == pi.binding.PI_ERR_INVALID_ARG
    st = _status(pi.pi_sparse_ffn_static, L, FAKE + 8, 1, FAKE, FAKE, FAKE)
    assert st == pi.binding.PI_ERR_INVALID_ARG
    st = _status(pi.pi_sparse_ffn_static, L, FAKE, 65, FAKE, FAKE, FAKE)
    assert st == pi.binding.PI_ERR_UNSUPPORTED
    st = _status(pi.pi_sparse_ffn_static, _layer(w_down_t=None), FAKE, 1, FAKE, FAKE, FAKE)
    assert st == pi.binding.PI_ERR_INVALID_ARG


def test_permute_layer_validation(lib):
    """pi_permute_layer rejects mismatched layers, a missing perm and a dst
    tensor that overlaps its src, before touching the device."""
    E = 1 << 40  # another fake region, far from FAKE
    src = _layer()
    dst = _layer(w_up=E, w_down_t=E + (8 << 20), b_up=E + (16 << 20),
                 pred=_pred(w2=E + (24 << 20), b2=E + (32 << 20)))
    perm = FAKE
    assert _status(pi.pi_permute_layer, src, None, dst) == pi.binding.PI_ERR_INVALID_ARG
    # shapes must match
    other = _layer(d_model=1024, pred=_pred(d_model=1024), w_up=E, w_down_t=E + (8 << 20),
                   b_up=E + (16 << 20))
    assert _status(pi.pi_permute_layer, src, perm, other) == pi.binding.PI_ERR_INVALID_ARG
    # a bias present on one side only
    nob = _layer(w_up=E, w_down_t=E + (8 << 20), b_up=None,
                 pred=_pred(w2=E + (24 << 20), b2=E + (32 << 20)))
    assert _status(pi.pi_permute_layer, src, perm, nob) == pi.binding.PI_ERR_INVALID_ARG
    # dst W_up overlapping src W_up (2048 rows of 1 KB from FAKE)
    ov = _layer(w_up=FAKE + 4096, w_down_t=E + (8 << 20), b_up=E + (16 << 20),
                pred=_pred(w2=E + (24 << 20), b2=E + (32 << 20)))
    assert _status(pi.pi_permute_layer, src, perm, ov) == pi.binding.PI_ERR_INVALID_ARG
    # in place
    assert _status(pi.pi_permute_layer, src, perm, src) == pi.binding.PI_ERR_INVALID_ARG
