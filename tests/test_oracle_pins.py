"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test compares the oracle with something other than itself: pure-Python
brute force on tiny shapes, closed forms, the worked example of the pages'
Figure 8, hand-derived Q4_0 values, library rounding routines, and
distributional properties of the generated data.
"""
import itertools
import json
import math
import os
import struct

import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import oracle_layer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# pure-Python brute force (lists of Python floats, explicit loops)
# ---------------------------------------------------------------------------
def bf_dot(u, v):
    t = 0.0
    for a, b in zip(u, v):
        t += a * b
    return t


def bf_predict(W1, b1, W2, b2, x, tau):
    a = [max(bf_dot(W1[j], x) + b1[j], 0.0) for j in range(len(W1))]
    s = [bf_dot(W2[n], a) + b2[n] for n in range(len(W2))]
    return a, s, [v > tau for v in s]


def bf_h(act, Wup, Wgate, bup, bgate, x, i):
    if act == "relu":
        return max(bf_dot(Wup[i], x) + (bup[i] if bup is not None else 0.0), 0.0)
    if act == "sqrelu":
        r = max(bf_dot(Wup[i], x) + (bup[i] if bup is not None else 0.0), 0.0)
        return r * r
    g = max(bf_dot(Wgate[i], x) + (bgate[i] if bgate is not None else 0.0), 0.0)
    return g * bf_dot(Wup[i], x)


def bf_y(act, Wup, Wgate, Wdt, bup, bgate, x, idx):
    d = len(Wdt[0])
    y = [0.0] * d
    for i in idx:
        h = bf_h(act, Wup, Wgate, bup, bgate, x, i)
        for j in range(d):
            y[j] += h * Wdt[i][j]
    return y


def f16_round_py(v):
    """Round a Python float to binary16 with the struct module's packer."""
    return struct.unpack("<e", struct.pack("<e", v))[0]


# ---------------------------------------------------------------------------
# stored-weight decoding in plain Python (struct), independent of the oracle
# ---------------------------------------------------------------------------
def f16_py(bits):
    return struct.unpack("<e", int(bits).to_bytes(2, "little"))[0]


def bf16_py(bits):
    """bfloat16 bits are the top half of an IEEE binary32."""
    return struct.unpack("<f", (int(bits) << 16).to_bytes(4, "little"))[0]


def q4_0_row_py(row, d):
    """One Q4_0 row (d/32 blocks of 18 bytes) decoded byte by byte."""
    out = []
    for blk in range(d // 32):
        b = bytes(row[18 * blk: 18 * blk + 18])
        scale = struct.unpack("<e", b[0:2])[0]
        lo = [((b[2 + j] & 15) - 8) * scale for j in range(16)]
        hi = [((b[2 + j] >> 4) - 8) * scale for j in range(16)]
        out += lo + hi
    return out


def decode_py(bits, dtype, d=None):
    bits = np.asarray(bits)
    if dtype == "q4_0":
        return [q4_0_row_py(r.tolist(), d) for r in bits]
    f = f16_py if dtype == "f16" else bf16_py
    return [[f(v) for v in row] for row in bits.tolist()]


def bf16_bits(x):
    """float32 values -> bfloat16 bit patterns (library round-to-nearest-even)."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def q4_0_pack(rng, F, d, std):
    """Random Q4_0 rows: random nibbles and positive/negative fp16 scales."""
    nb = d // 32
    rows = np.zeros((F, nb * 18), dtype=np.uint8)
    for i in range(F):
        for blk in range(nb):
            scale = np.float16(std / 8 * rng.uniform(0.5, 1.5) * rng.choice([-1, 1]))
            q = rng.integers(0, 16, 32)
            b = bytearray(np.array([scale]).view(np.uint8).tobytes())
            b += bytes(int(q[j]) | (int(q[j + 16]) << 4) for j in range(16))
            rows[i, 18 * blk: 18 * blk + 18] = np.frombuffer(bytes(b), dtype=np.uint8)
    return rows


# ---------------------------------------------------------------------------
# a tiny random layer with weights exact in their stored type
# ---------------------------------------------------------------------------
def tiny_layer(rng, d, F, r, act, tau=0.0, bias=True, wdtype="f16", pdtype=None):
    pdtype = pdtype or ("bf16" if wdtype == "bf16" else "f16")

    def store(shape, std, dt):
        x = rng.standard_normal(shape) * std
        if dt == "f16":
            return x.astype(np.float16).view(np.uint16)
        if dt == "bf16":
            return bf16_bits(x)
        return q4_0_pack(rng, shape[0], shape[1], std)

    W1 = store((r, d), 0.4, pdtype)
    W2 = store((F, r), 0.4, pdtype)
    Wup = store((F, d), 0.3, wdtype)
    Wgate = store((F, d), 0.3, wdtype) if act == "reglu" else None
    Wdt = store((F, d), 0.3, wdtype)
    b1 = rng.standard_normal(r).astype(np.float32)
    b2 = rng.standard_normal(F).astype(np.float32)
    bact = (rng.standard_normal(F) * 0.5).astype(np.float32) if bias else None
    L = oracle.OracleLayer(
        d_model=d, d_ff=F, act=act, wdtype=wdtype, pdtype=pdtype,
        w1=W1, b1=b1, w2=W2, b2=b2, threshold=tau,
        w_up=Wup, w_gate=Wgate, w_down_t=Wdt,
        b_up=bact if act != "reglu" else None, b_gate=bact if act == "reglu" else None,
    )
    lists = dict(
        W1=decode_py(W1, pdtype), W2=decode_py(W2, pdtype),
        Wup=decode_py(Wup, wdtype, d),
        Wgate=None if Wgate is None else decode_py(Wgate, wdtype, d),
        Wdt=decode_py(Wdt, wdtype, d), b1=b1.astype(float).tolist(),
        b2=b2.astype(float).tolist(),
        bup=bact.astype(float).tolist() if (bias and act != "reglu") else None,
        bgate=bact.astype(float).tolist() if (bias and act == "reglu") else None,
    )
    return L, lists


def tokens16(rng, B, d, adtype="f16"):
    x = rng.standard_normal((B, d))
    if adtype == "bf16":
        return np.array(decode_py(bf16_bits(x), "bf16"))
    return x.astype(np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# masked FFN and predictor against brute force
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("act", ["relu", "reglu", "sqrelu"])
@pytest.mark.parametrize("shape", [(16, 8, 4), (48, 16, 6), (64, 12, 8)])
@pytest.mark.parametrize("wdtype", ["f16", "bf16", "q4_0"])
def test_predict_and_ffn_brute_force(act, shape, wdtype):
    d, F, r = shape
    if wdtype == "q4_0":
        d = 32 * ((d + 31) // 32)
    rng = np.random.default_rng(11 + d + F)
    L, P = tiny_layer(rng, d, F, r, act, tau=0.3, wdtype=wdtype)
    x = tokens16(rng, 3, d, L.pdtype)
    a, s, m = oracle.predict(L, x)
    for b in range(3):
        ab, sb, mb = bf_predict(P["W1"], P["b1"], P["W2"], P["b2"], x[b].tolist(), 0.3)
        np.testing.assert_allclose(a[b], ab, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(s[b], sb, rtol=1e-12, atol=1e-12)
        assert list(m[b]) == mb
    idx = oracle.union_index(m)
    assert 0 < idx.size < F
    y = oracle.masked_ffn(L, x, idx)
    yd = oracle.dense_ffn(L, x)
    for b in range(3):
        yb = bf_y(act, P["Wup"], P["Wgate"], P["Wdt"], P["bup"], P["bgate"], x[b].tolist(),
                  idx.tolist())
        np.testing.assert_allclose(y[b], yb, rtol=1e-12, atol=1e-12)
        ybd = bf_y(act, P["Wup"], P["Wgate"], P["Wdt"], P["bup"], P["bgate"], x[b].tolist(),
                   range(F))
        np.testing.assert_allclose(yd[b], ybd, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("act", ["relu", "reglu", "sqrelu"])
@pytest.mark.parametrize("wdtype", ["f16", "bf16"])
def test_every_subset_closed_form(act, wdtype):
    """Every index set I of an F = 8 layer: y(I) = y_dense - sum over
    support-minus-I of h_i W_down^T[i]."""
    d, F, r = 24, 8, 4
    for seed in range(100):  # first seed whose token has both zero and nonzero h
        rng = np.random.default_rng(seed)
        L, P = tiny_layer(rng, d, F, r, act, wdtype=wdtype)
        x = tokens16(rng, 1, d, L.pdtype)[0]
        xl = x.tolist()
        h = [bf_h(act, P["Wup"], P["Wgate"], P["bup"], P["bgate"], xl, i) for i in range(F)]
        if 2 <= sum(v != 0.0 for v in h) <= F - 2:
            break
    yd = bf_y(act, P["Wup"], P["Wgate"], P["Wdt"], P["bup"], P["bgate"], xl, range(F))
    assert any(v == 0.0 for v in h) and any(v != 0.0 for v in h)
    for k in range(F + 1):
        for I in itertools.combinations(range(F), k):
            expect = list(yd)
            for i in range(F):
                if h[i] != 0.0 and i not in I:
                    for j in range(d):
                        expect[j] -= h[i] * P["Wdt"][i][j]
            got = oracle.masked_ffn(L, x, np.array(I, dtype=np.int64))[0]
            np.testing.assert_allclose(got, expect, rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("act", ["relu", "reglu", "sqrelu"])
def test_superset_of_support_equals_dense(act):
    rng = np.random.default_rng(7)
    L, _ = tiny_layer(rng, 32, 16, 4, act)
    x = tokens16(rng, 4, 32)
    supp = oracle.true_support(L, x)
    assert 0 < supp.sum() < supp.size
    idx = oracle.union_index(supp)
    np.testing.assert_allclose(oracle.masked_ffn(L, x, idx), oracle.dense_ffn(L, x),
                               rtol=1e-12, atol=1e-14)
    extra = np.union1d(idx, rng.choice(16, 5, replace=False))
    np.testing.assert_allclose(oracle.masked_ffn(L, x, extra), oracle.dense_ffn(L, x),
                               rtol=1e-12, atol=1e-14)


def test_all_ones_mask_and_empty_index():
    rng = np.random.default_rng(9)
    L, _ = tiny_layer(rng, 32, 16, 4, "relu", tau=-1e30)
    x = tokens16(rng, 2, 32)
    _, _, m = oracle.predict(L, x)
    assert m.all()
    y, idx, _ = oracle.sparse_ffn_layer(L, x)
    assert list(idx) == list(range(16))
    np.testing.assert_allclose(y, oracle.dense_ffn(L, x), rtol=1e-14, atol=0)
    L.threshold = 1e30
    y, idx, _ = oracle.sparse_ffn_layer(L, x)
    assert idx.size == 0 and np.all(y == 0.0)


def test_tie_is_inactive():
    rng = np.random.default_rng(1)
    L, _ = tiny_layer(rng, 16, 8, 4, "relu")
    L.w2 = np.zeros_like(L.w2)
    L.b2 = np.array([0.0, 1.0, -1.0, 0.0, 2.0, 0.0, 0.0, 0.5])
    _, s, m = oracle.predict(L, tokens16(rng, 1, 16))
    assert list(np.flatnonzero(m[0])) == [1, 4, 7]


def test_fig8_worked_example():
    """The pages' Figure 8: hot neurons 3, 5, 7; predictor flags 3, 4, 5; 7 is
    skipped although it is hot."""
    g = json.load(open(os.path.join(GOLDEN, "fig8_worked_example.json")))
    F, d = g["d_ff"], 4
    rng = np.random.default_rng(8)
    W1 = np.eye(d, dtype=np.float16)
    W2 = np.zeros((F, d), dtype=np.float16)
    b2 = np.array([1.0 if i in g["predicted_active"] else -1.0 for i in range(F)])
    Wup = (rng.standard_normal((F, d)) * 0.1).astype(np.float16)
    Wdt = (rng.standard_normal((F, d)) * 0.5).astype(np.float16)
    # hot neurons carry large positive biases (they fire for most inputs)
    bup = np.array([2.0 if i in g["hot"] else 0.25 for i in range(F)])
    L = oracle.OracleLayer(d, F, "relu", "f16", "f16", W1.view(np.uint16), np.zeros(d),
                           W2.view(np.uint16), b2, 0.0, Wup.view(np.uint16), None,
                           Wdt.view(np.uint16), b_up=bup)
    x = np.ones((1, d))
    y, idx, _ = oracle.sparse_ffn_layer(L, x)
    assert list(idx) == g["computed"]
    for n in g["skipped_hot"]:
        assert n not in idx
        assert oracle.neuron_outputs(L, x, np.array([n]))[0, 0] > 0  # it would fire
    P = dict(Wup=Wup.astype(float).tolist(), Wdt=Wdt.astype(float).tolist())
    expect = bf_y("relu", P["Wup"], None, P["Wdt"], bup.tolist(), None, [1.0] * d,
                  g["computed"])
    np.testing.assert_allclose(y[0], expect, rtol=1e-12)
    with_7 = bf_y("relu", P["Wup"], None, P["Wdt"], bup.tolist(), None, [1.0] * d,
                  g["computed"] + g["skipped_hot"])
    assert np.abs(np.array(with_7) - y[0]).max() > 1e-3


# ---------------------------------------------------------------------------
# compaction
# ---------------------------------------------------------------------------
def test_union_index_brute_force():
    rng = np.random.default_rng(3)
    for _ in range(200):
        B = int(rng.integers(1, 9))
        F = int(rng.integers(1, 130))
        m = rng.random((B, F)) < rng.random()
        sets = [{i for i in range(F) if m[b, i]} for b in range(B)]
        expect = sorted(set().union(*sets))
        got = oracle.union_index(m)
        assert got.tolist() == expect
        assert np.all(np.diff(got) > 0)
        for sb in sets:
            assert sb <= set(got.tolist())
    assert oracle.union_index(np.zeros((2, 64), bool)).size == 0
    assert oracle.union_index(np.ones((1, 64), bool)).tolist() == list(range(64))


def test_band():
    s = np.array([-2e-3, -9.9e-4, 0.0, 5e-4, 1.5e-3])
    assert oracle.band(s, 0.0).tolist() == [False, True, True, True, False]
    assert oracle.band(s + 1.0, 1.0).tolist() == [False, True, True, True, False]


# ---------------------------------------------------------------------------
# predictor: the +/- construction's closed form
# ---------------------------------------------------------------------------
def test_predictor_closed_form_pm_construction():
    """With W1 = [G; -G], b1 = 0 and W2 = [M, -M], relu(g) - relu(-g) = g gives
    s = M G x + b2 exactly."""
    cfg = synth.get_config("toy")
    Ld = synth.make_layer(cfg, 0, "cpu", "R")
    L = oracle_layer(Ld)
    r2 = cfg.rank // 2
    G = oracle.widen_f16(L.w1[:r2])
    M = oracle.widen_f16(L.w2[:, :r2])
    assert np.array_equal(oracle.widen_f16(L.w1[r2:]), -G)
    assert np.array_equal(oracle.widen_f16(L.w2[:, r2:]), -M)
    x = synth.make_tokens(cfg, 8).double().numpy()
    _, s, m = oracle.predict(L, x)
    closed = (M @ (G @ x.T)).T + L.b2
    np.testing.assert_allclose(s, closed, rtol=1e-10, atol=1e-10)
    assert np.array_equal(m, closed > 0.0) or np.abs(closed[m != (closed > 0)]).max() < 1e-9


# ---------------------------------------------------------------------------
# sparsity of the generated layers, measured through the oracle
# ---------------------------------------------------------------------------
def test_measured_sparsity_matches_profile():
    cfg = synth.get_config("toy")
    Ld = synth.make_layer(cfg, 0, "cpu", "R")
    L = oracle_layer(Ld)
    N = 2000
    x = synth.make_tokens(cfg, N, seed_offset=17).double().numpy()
    supp = oracle.true_support(L, x)
    p = Ld.p
    frac = supp.mean()
    sigma = math.sqrt((p * (1 - p)).sum() * N) / (N * cfg.d_ff)
    assert abs(frac - p.mean()) < 4 * sigma, (frac, p.mean(), sigma)
    rate = supp.mean(axis=0)
    # per-neuron rates track the profile (Spearman rank correlation)
    rr = np.argsort(np.argsort(rate)); rp = np.argsort(np.argsort(p))
    rho = np.corrcoef(rr, rp)[0, 1]
    assert rho > 0.9, rho
    hot = p > 0.99
    assert hot.sum() > 10 and rate[hot].mean() > 0.97
    # predictor quality matches the generator's closed-form expectation
    _, _, m = oracle.predict(L, x)
    recall = (m & supp).sum() / supp.sum()
    assert abs(recall - Ld.expected_recall) < 0.02
    assert abs(m.mean() - Ld.expected_pred_frac) < 0.02


# ---------------------------------------------------------------------------
# Q4_0
# ---------------------------------------------------------------------------
def test_q4_0_golden_block():
    g = json.load(open(os.path.join(GOLDEN, "q4_0_block.json")))
    raw = np.frombuffer(bytes.fromhex(g["bytes_hex"]), dtype=np.uint8).reshape(1, 18)
    assert int.from_bytes(bytes(raw[0, :2]), "little") == int(g["scale_fp16_bits"], 16)
    got = oracle.dequant_q4_0(raw, 32)[0]
    assert got.tolist() == g["values"]
    # two blocks in a row: the second block's values follow the first's
    two = np.concatenate([raw, raw], axis=1)
    assert oracle.dequant_q4_0(two, 64)[0].tolist() == g["values"] * 2


def test_q4_0_roundtrip_bound_and_zero_block():
    torch.manual_seed(0)
    w = torch.randn(64, 256) * 0.015
    w[3, 32:64] = 0.0
    q = synth.quantize_q4_0(w)
    assert q.shape == (64, synth.q4_0_row_bytes(256))
    deq = oracle.dequant_q4_0(q.numpy(), 256)
    assert np.all(deq[3, 32:64] == 0.0)
    blk = q.numpy().reshape(64, 8, 18)
    scale = np.abs(oracle.widen_f16(blk[:, :, 0:2].copy().view(np.uint16).reshape(64, 8)))
    err = np.abs(deq - w.double().numpy()).reshape(64, 8, 32)
    # half a step, plus one step where the top code 16 clamps to 15, plus the
    # fp16 rounding of the scale itself (relative 2^-11 of up to 8 steps)
    bound = scale[:, :, None] * (0.5 + 8 * 2.0**-11) + 1e-12
    clamped = err > bound
    assert np.all(err <= scale[:, :, None] * (1.0 + 8 * 2.0**-11) + 1e-12)
    assert clamped.mean() < 0.01


# ---------------------------------------------------------------------------
# rounding and the stack
# ---------------------------------------------------------------------------
def test_round_f16_ties_and_library():
    v = np.array([1 + 2**-11, 1 + 3 * 2**-11, 2049.0, 2051.0, -1 - 2**-11, 2.0**-25])
    assert oracle.round_f16(v).tolist() == [1.0, 1 + 2**-9, 2048.0, 2052.0, -1.0, 0.0]
    rng = np.random.default_rng(0)
    x = rng.standard_normal(2000) * 3
    assert oracle.round_f16(x).tolist() == [f16_round_py(t) for t in x.tolist()]


def test_round_bf16_ties_and_library():
    v = np.array([1 + 2**-8, 1 + 3 * 2**-8, 257.0, 259.0, -(1 + 2**-8)])
    assert oracle.round_bf16(v).tolist() == [1.0, 1 + 2**-6, 256.0, 260.0, -1.0]
    rng = np.random.default_rng(1)
    x32 = (rng.standard_normal(5000) * 10).astype(np.float32)
    lib = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.round_bf16(x32.astype(np.float64)), lib)


def test_rms_cast_special_cases():
    for c in (0.37, 5.0, 1e3):
        x = c * np.array([[1.0, -1.0] * 64])
        assert np.all(np.abs(oracle.rms_cast(x, "f16")) == 1.0)
        assert np.all(np.abs(oracle.rms_cast(x, "bf16")) == 1.0)
    x = np.array([[3.0, 4.0] * 32 + [0.0] * 64])   # mean square 12.5/2 = 6.25
    got = oracle.rms_cast(x, "f16")[0]
    assert got[0] == f16_round_py(3.0 / math.sqrt(6.25 + 1e-6))
    assert got[1] == f16_round_py(4.0 / math.sqrt(6.25 + 1e-6))
    assert np.all(oracle.rms_cast(np.zeros((1, 64)), "f16") == 0.0)


def test_stack_brute_force():
    """Two-layer stack against a pure-Python pre-norm residual chain."""
    d, F, r = 16, 8, 4
    rng = np.random.default_rng(21)
    layers = [tiny_layer(rng, d, F, r, "relu", tau=0.2) for _ in range(2)]
    x0 = rng.standard_normal((1, d)) * 2.0
    out, trace = oracle.ffn_stack([L for L, _ in layers], x0, "f16")
    x = x0[0].tolist()
    for li, (L, P) in enumerate(layers):
        ms = sum(v * v for v in x) / d
        xl = [f16_round_py(v / math.sqrt(ms + 1e-6)) for v in x]
        assert trace[li][2][0].tolist() == xl
        _, _, m = bf_predict(P["W1"], P["b1"], P["W2"], P["b2"], xl, 0.2)
        idx = [i for i in range(F) if m[i]]
        assert trace[li][0].tolist() == idx
        y = bf_y("relu", P["Wup"], None, P["Wdt"], P["bup"], None, xl, idx)
        x = [a + b for a, b in zip(x, y)]
    np.testing.assert_allclose(out[0], x, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# widening of stored 16-bit weights, from hand-written bit patterns
# ---------------------------------------------------------------------------
def _same(a, b):
    """Equal as numbers and in sign (so -0.0 differs from 0.0)."""
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


def test_widen_bf16_hand_patterns():
    """bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits."""
    cases = {
        0x0000: 0.0, 0x8000: -0.0,
        0x3F80: 1.0, 0xBF80: -1.0, 0x4000: 2.0, 0x3FC0: 1.5, 0x3F81: 1.0 + 2.0**-7,
        0xC2F7: -123.5,                        # -(1 + 119/128) * 2^6
        0x7F7F: (2.0 - 2.0**-7) * 2.0**127,    # largest finite
        0xFF7F: -(2.0 - 2.0**-7) * 2.0**127,
        0x0080: 2.0**-126,                     # smallest normal
        0x0001: 2.0**-133,                     # smallest subnormal
        0x007F: 127 * 2.0**-133,               # largest subnormal
        0x7F80: math.inf, 0xFF80: -math.inf,
    }
    got = oracle.widen_bf16(np.array(list(cases), dtype=np.uint16))
    for (bits, want), g in zip(cases.items(), got.tolist()):
        assert _same(g, want), (hex(bits), g, want)
    assert np.isnan(oracle.widen_bf16(np.array([0x7FC0], dtype=np.uint16)))[0]


def test_widen_f16_hand_patterns():
    """IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits."""
    cases = {
        0x0000: 0.0, 0x8000: -0.0, 0x3C00: 1.0, 0xC000: -2.0, 0x3E00: 1.5,
        0x3C01: 1.0 + 2.0**-10, 0x7BFF: 65504.0, 0xFBFF: -65504.0,
        0x0400: 2.0**-14, 0x0001: 2.0**-24, 0x03FF: 1023 * 2.0**-24,
        0x7C00: math.inf, 0xFC00: -math.inf,
    }
    got = oracle.widen_f16(np.array(list(cases), dtype=np.uint16))
    for (bits, want), g in zip(cases.items(), got.tolist()):
        assert _same(g, want), (hex(bits), g, want)


def test_widen_every_pattern_against_struct():
    """All 65536 patterns of both types against the struct module's decoders."""
    bits = np.arange(65536, dtype=np.uint32)
    f16 = oracle.widen_f16(bits.astype(np.uint16))
    bf = oracle.widen_bf16(bits.astype(np.uint16))
    with np.errstate(invalid="ignore"):  # signalling NaN patterns
        ref16 = np.frombuffer(bits.astype("<u2").tobytes(), dtype="<f2").astype(np.float64)
        refbf = np.frombuffer((bits << 16).astype("<u4").tobytes(), dtype="<f4").astype(np.float64)
    for got, ref in ((f16, ref16), (bf, refbf)):
        nan = np.isnan(ref)
        assert np.array_equal(np.isnan(got), nan)
        assert np.array_equal(got[~nan], ref[~nan])
        assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))
    for b in (0x1234, 0x8001, 0xBEEF, 0x3555):
        assert f16[b] == f16_py(b) and bf[b] == bf16_py(b)


def test_widen_then_round_is_identity():
    """Every finite pattern survives widening followed by rounding back."""
    bits = np.arange(65536, dtype=np.uint16)
    bf = oracle.widen_bf16(bits)
    f16 = oracle.widen_f16(bits)
    for v, rnd in ((bf, oracle.round_bf16), (f16, oracle.round_f16)):
        fin = np.isfinite(v)
        back = rnd(v[fin])
        assert np.array_equal(back, v[fin])
        assert np.array_equal(np.signbit(back), np.signbit(v[fin]))


# ---------------------------------------------------------------------------
# rounding at the edges of the formats
# ---------------------------------------------------------------------------
def test_round_overflow_and_subnormal_ties():
    f16 = oracle.round_f16(np.array([
        65504.0, 65519.99, 65520.0, -70000.0,     # largest finite, below / at the tie to inf
        2.0**-25, 3 * 2.0**-25, 1.4 * 2.0**-24,   # subnormal ties to even, nearest
        2.0**-14 - 2.0**-25,                      # rounds up into the normal range
    ]))
    assert f16.tolist() == [65504.0, 65504.0, math.inf, -math.inf,
                            0.0, 2.0**-23, 2.0**-24, 2.0**-14]
    big = (2.0 - 2.0**-8) * 2.0**127
    bf = oracle.round_bf16(np.array([
        big * (1 - 2.0**-30), big, 2.0**-134, 3 * 2.0**-134, 2.0**-126 * (1 + 2.0**-8),
    ]))
    assert bf.tolist() == [(2.0 - 2.0**-7) * 2.0**127, math.inf, 0.0, 2.0**-132, 2.0**-126]


# ---------------------------------------------------------------------------
# cross-check: an independent numpy restatement agrees with the C++ oracle
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("act", ["relu", "reglu", "sqrelu"])
@pytest.mark.parametrize("wdtype", ["f16", "bf16", "q4_0"])
def test_numpy_restatement_agrees(act, wdtype):
    import oracle.numpy_xcheck as nx
    rng = np.random.default_rng(40 + len(act) + len(wdtype))
    d, F, r = 64, 40, 16
    L, _ = tiny_layer(rng, d, F, r, act, tau=0.1, wdtype=wdtype)
    x = tokens16(rng, 5, d, L.pdtype)
    a1, s1, m1 = oracle.predict(L, x)
    a2, s2, m2 = nx.predict(L, x)
    np.testing.assert_allclose(a1, a2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s1, s2, rtol=1e-12, atol=1e-13)
    assert np.array_equal(m1, m2)
    assert np.array_equal(oracle.union_index(m1), nx.union_index(m2))
    I = oracle.union_index(m1)
    np.testing.assert_allclose(oracle.masked_ffn(L, x, I), nx.masked_ffn(L, x, I),
                               rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(oracle.rms_cast(x * 3.0, L.pdtype), nx.rms_cast(x * 3.0, L.pdtype))
    assert np.array_equal(oracle.widen(L.w_up, wdtype, d), nx.widen(L.w_up, wdtype, d))
