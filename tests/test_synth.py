"""Properties of the synthetic workloads that the benchmarks and parity tests rely on."""
import numpy as np
import pytest

import synth
from synth.configs import Config


def test_adaptive_rank_profile():
    """Per-layer predictor sizing (unite.ai page, "Adaptive Sparsity-Prädiktoren"):
    the skew rises across the stack and the rank falls with it, within
    [rank / 2, 2 rank], in multiples of 16 (even for the +/- construction and
    a multiple of 8 for the library)."""
    c = synth.get_config("opt-6.7b-adaptive")
    s = [c.layer_zipf(l) for l in range(c.n_layers)]
    r = [c.layer_rank(l) for l in range(c.n_layers)]
    assert s[0] == pytest.approx(c.zipf_s - c.skew_spread)
    assert s[-1] == pytest.approx(c.zipf_s + c.skew_spread)
    assert all(b > a for a, b in zip(s, s[1:]))
    assert all(b <= a for a, b in zip(r, r[1:])) and r[0] > r[-1]
    assert all(x % 16 == 0 and c.rank // 2 <= x <= 2 * c.rank for x in r)
    plain = synth.get_config("opt-6.7b")
    assert {plain.layer_rank(l) for l in range(plain.n_layers)} == {plain.rank}


def test_adaptive_layers_follow_the_profile():
    c = Config(19, "t-adaptive-rank", 4, 1024, 4096, "relu", "f16", "f16", 0.02, 1.1, 0.15, 256,
               skew_spread=0.3, adaptive_rank=True)
    tops = []
    for l in range(c.n_layers):
        L = synth.make_layer(c, l, "cpu", "R")
        assert L.w1.shape == (c.layer_rank(l), c.d_model)
        assert L.w2.shape == (c.d_ff, c.layer_rank(l))
        assert abs(L.p.mean() - c.mean_active) < 1e-6
        top = np.sort(L.p)[::-1][: c.d_ff // 100].sum() / L.p.sum()
        tops.append(top)
    # a more skewed layer concentrates more of its firing in its hottest 1%
    assert all(b > a for a, b in zip(tops, tops[1:])), tops
