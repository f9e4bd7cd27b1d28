"""GPU checks of pi_sparse_ffn_static, the gathered FFN over a fixed device scratch.

It must give what pi_sparse_ffn gives on the same inputs (within the FFN
tolerance of the parity tests, and in fact bit for bit, since both run the
same kernels in the same order), on calls made back to back so that the second
finds the scratch dirty from the first; and both must match the fp64 oracle's
masked FFN on the same neuron list.  This file stands alone (run it by itself
or after the rest of the suite) and is collected last.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth.configs import Config
from tests._util import device_layer, oracle_layer, rel_l2, to16

pytestmark = pytest.mark.gpu

# (config, batches): fused 16-bit and Q4_0 paths at batch 1-4, the batched
# path at batch 3, 5 and 6 (the largest batch the scratch covers everywhere)
CASES = {
    "toy": (synth.get_config("toy"), [1, 2, 4, 6]),
    "reglu-bf16": (Config(11, "t-reglu-bf16", 3, 512, 2048, "reglu", "bf16", "bf16",
                          0.02, 1.2, 0.12, 128), [1, 3]),
    "q4-reglu": (Config(13, "t-q4-reglu", 3, 512, 1536, "reglu", "q4_0", "f16",
                        0.015, 1.1, 0.1, 128), [1, 2, 5]),
    "relu-f16-8192": (Config(15, "t-relu-f16-8192", 2, 8192, 1024, "relu", "f16", "f16",
                             0.015, 1.0, 0.08, 512), [1, 4, 6]),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from activation_sparse_pi_b200 import build
    build.build()
    import activation_sparse_pi_b200 as pi
    pi.lib()
    yield
    assert pi.pi_device_error() == 0, "a kernel flagged a device-side error"


def _inputs(cfg, B, seed):
    L = synth.make_layer(cfg, 0, "cpu", "R")
    Ld, desc = device_layer(L)
    xf = synth.make_tokens(cfg, B, seed_offset=seed)
    x = to16(xf, cfg.adtype).cuda()
    rng = np.random.default_rng(cfg.d_ff * 7 + B)
    n = max(1, cfg.d_ff // 5)
    I = rng.permutation(cfg.d_ff)[:n].astype(np.int32)
    idx = torch.zeros(cfg.d_ff, dtype=torch.int32, device="cuda")
    idx[:n] = torch.from_numpy(I).cuda()
    cnt = torch.tensor([n], dtype=torch.int32, device="cuda")
    # what the oracle says these inputs give
    expect = oracle.masked_ffn(oracle_layer(L), xf.double().numpy(), I)
    return (Ld, expect), desc, x, idx, cnt


def _reference(desc, x, B, idx, cnt, d):
    import activation_sparse_pi_b200 as pi
    ws = torch.empty(pi.pi_workspace_size([desc], B), dtype=torch.uint8, device="cuda")
    y = torch.full((B, d), float("nan"), dtype=torch.float32, device="cuda")
    pi.pi_sparse_ffn(desc, x, B, idx, cnt, y, ws)
    torch.cuda.synchronize()
    return y.cpu().double().numpy()


def _static(desc, x, B, idx, cnt, d):
    import activation_sparse_pi_b200 as pi
    y = torch.full((B, d), float("nan"), dtype=torch.float32, device="cuda")
    pi.pi_sparse_ffn_static(desc, x, B, idx, cnt, y)
    return y


@pytest.mark.parametrize("name", list(CASES))
def test_static_scratch_matches_workspace_call(name):
    cfg, batches = CASES[name]
    tol = 2e-3 if cfg.wdtype == "q4_0" else 1e-3
    for B in batches:
        (keep, expect), desc, x, idx, cnt = _inputs(cfg, B, seed=B)
        want = _reference(desc, x, B, idx, cnt, cfg.d_model)
        assert rel_l2(want, expect) <= tol, (B, rel_l2(want, expect))
        # two calls in a row on one stream, no synchronisation between them
        y1 = _static(desc, x, B, idx, cnt, cfg.d_model)
        y2 = _static(desc, x, B, idx, cnt, cfg.d_model)
        torch.cuda.synchronize()
        for y in (y1, y2):
            got = y.cpu().double().numpy()
            assert np.isfinite(got).all()
            assert rel_l2(got, expect) <= tol, (B, rel_l2(got, expect))
            assert rel_l2(got, want) <= tol, (B, rel_l2(got, want))
            assert np.array_equal(got, want), f"batch {B}: not bit-identical to pi_sparse_ffn"


def test_static_scratch_reused_across_shapes():
    # a large shape leaves the scratch full of its partials; a small shape
    # after it must not see them
    big_cfg, _ = CASES["relu-f16-8192"]
    small_cfg, _ = CASES["toy"]
    (kb, eb), db, xb, ib, cb = _inputs(big_cfg, 4, seed=1)
    (ks, es), ds, xs, is_, cs = _inputs(small_cfg, 2, seed=2)
    want_b = _reference(db, xb, 4, ib, cb, big_cfg.d_model)
    want_s = _reference(ds, xs, 2, is_, cs, small_cfg.d_model)
    outs = []
    for _ in range(2):
        outs.append(("b", _static(db, xb, 4, ib, cb, big_cfg.d_model)))
        outs.append(("s", _static(ds, xs, 2, is_, cs, small_cfg.d_model)))
    torch.cuda.synchronize()
    for which, y in outs:
        want = want_b if which == "b" else want_s
        got = y.cpu().double().numpy()
        assert np.array_equal(got, want), which
        assert rel_l2(got, eb if which == "b" else es) <= 1e-3, which
