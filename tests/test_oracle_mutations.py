"""The pins must catch plausible mistakes in the oracle.

Each case swaps one oracle function for a copy with a planted mistake (on the
CPU, in this process only) and checks that at least one pin then fails.
"""
import numpy as np
import pytest

import oracle
import oracle.pi_oracle as po
from tests import test_oracle_pins as pins


def _predict_no_relu(layer, x):
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    w1 = po.widen(layer.w1, layer.pdtype)
    w2 = po.widen(layer.w2, layer.pdtype)
    a = x @ w1.T + (0 if layer.b1 is None else layer.b1)
    s = a @ w2.T + layer.b2
    return a, s, s > layer.threshold


def _predict_no_b2(layer, x):
    a, s, _ = _ORIG["predict"](layer, x)
    s = s - np.asarray(layer.b2)
    return a, s, s > layer.threshold


def _predict_tie_active(layer, x):
    a, s, _ = _ORIG["predict"](layer, x)
    return a, s, s >= layer.threshold


def _masked_wrong_row(layer, x, idx):
    idx = np.asarray(idx, dtype=np.int64)
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    if idx.size == 0:
        return np.zeros((x.shape[0], layer.d_model))
    h = po.neuron_outputs(layer, x, idx)
    down = layer.rows("w_down_t", np.arange(idx.size))   # position, not neuron id
    return h @ down


def _outputs_reglu_swapped(layer, x, idx):
    if layer.act != "reglu":
        return _ORIG["neuron_outputs"](layer, x, idx)
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    up = layer.rows("w_up", idx)
    gate = layer.rows("w_gate", idx)
    g = x @ up.T
    if layer.b_gate is not None:
        g = g + np.asarray(layer.b_gate)[idx]
    return np.maximum(g, 0.0) * (x @ gate.T)


def _outputs_sqrelu_unsquared(layer, x, idx):
    if layer.act != "sqrelu":
        return _ORIG["neuron_outputs"](layer, x, idx)
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    pre = x @ layer.rows("w_up", idx).T
    if layer.b_up is not None:
        pre = pre + np.asarray(layer.b_up)[idx]
    return np.maximum(pre, 0.0)


def _outputs_drop_bias(layer, x, idx):
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    up = layer.rows("w_up", idx)
    if layer.act == "relu":
        return np.maximum(x @ up.T, 0.0)
    if layer.act == "sqrelu":
        return np.maximum(x @ up.T, 0.0) ** 2
    gate = layer.rows("w_gate", idx)
    return np.maximum(x @ gate.T, 0.0) * (x @ up.T)


def _dequant_nibbles_swapped(rows, d_model):
    rows = np.asarray(rows, dtype=np.uint8)
    n = rows.shape[0]
    nb = d_model // 32
    blk = rows.reshape(n, nb, 18)
    scale = po.widen_f16(blk[:, :, 0:2].copy().view(np.uint16).reshape(n, nb))
    qs = blk[:, :, 2:18].astype(np.int64)
    q = np.concatenate([(qs >> 4) - 8, (qs & 0x0F) - 8], axis=2).astype(np.float64)
    return (q * scale[:, :, None]).reshape(n, d_model)


def _dequant_offset7(rows, d_model):
    return _ORIG["dequant_q4_0"](rows, d_model) + _scale_rows(rows, d_model)


def _scale_rows(rows, d_model):
    n = rows.shape[0]
    nb = d_model // 32
    blk = np.asarray(rows, dtype=np.uint8).reshape(n, nb, 18)
    scale = po.widen_f16(blk[:, :, 0:2].copy().view(np.uint16).reshape(n, nb))
    return np.repeat(scale, 32, axis=1)


def _union_intersection(mask):
    mask = np.atleast_2d(np.asarray(mask, dtype=bool))
    return np.flatnonzero(mask.all(axis=0)).astype(np.int64)


def _rms_no_eps(x_resid, adtype):
    x = np.atleast_2d(np.asarray(x_resid, dtype=np.float64))
    with np.errstate(invalid="ignore", divide="ignore"):
        return po.round16(x / np.sqrt(np.mean(x * x, axis=1, keepdims=True)), adtype)


def _round_bf16_truncate(x):
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.trunc(np.ldexp(m, 8)), e - 8)


_ORIG = {k: getattr(po, k) for k in
         ("predict", "masked_ffn", "neuron_outputs", "dequant_q4_0", "union_index",
          "rms_cast", "round_bf16")}

MUTANTS = [
    ("predict", _predict_no_relu),
    ("predict", _predict_no_b2),
    ("predict", _predict_tie_active),
    ("masked_ffn", _masked_wrong_row),
    ("neuron_outputs", _outputs_reglu_swapped),
    ("neuron_outputs", _outputs_drop_bias),
    ("neuron_outputs", _outputs_sqrelu_unsquared),
    ("dequant_q4_0", _dequant_nibbles_swapped),
    ("dequant_q4_0", _dequant_offset7),
    ("union_index", _union_intersection),
    ("rms_cast", _rms_no_eps),
    ("round_bf16", _round_bf16_truncate),
]

PIN_CASES = [
    (pins.test_predict_and_ffn_brute_force, dict(act="relu", shape=(16, 8, 4))),
    (pins.test_predict_and_ffn_brute_force, dict(act="reglu", shape=(48, 16, 6))),
    (pins.test_every_subset_closed_form, dict(act="relu")),
    (pins.test_every_subset_closed_form, dict(act="reglu")),
    (pins.test_predict_and_ffn_brute_force, dict(act="sqrelu", shape=(16, 8, 4))),
    (pins.test_tie_is_inactive, {}),
    (pins.test_fig8_worked_example, {}),
    (pins.test_union_index_brute_force, {}),
    (pins.test_predictor_closed_form_pm_construction, {}),
    (pins.test_measured_sparsity_matches_profile, {}),
    (pins.test_q4_0_golden_block, {}),
    (pins.test_round_bf16_ties_and_library, {}),
    (pins.test_rms_cast_special_cases, {}),
    (pins.test_stack_brute_force, {}),
]


@pytest.mark.parametrize("name,fn", MUTANTS, ids=[f"{n}:{f.__name__}" for n, f in MUTANTS])
def test_planted_mistake_fails_a_pin(monkeypatch, name, fn):
    monkeypatch.setattr(po, name, fn)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, fn)
    caught = []
    for case, kw in PIN_CASES:
        try:
            case(**kw)
        except (AssertionError, ValueError, FloatingPointError) as e:  # noqa: PERF203
            caught.append(case.__name__)
    assert caught, f"no pin caught the planted mistake {fn.__name__}"
