"""GPU checks of pi_permute_layer (hot-row ordering).

The permuted layer's tensors are the source rows gathered by the permutation,
bit for bit; the permuted layer predicts the same neurons (renumbered) and
computes the same FFN output, checked against the fp64 oracle on the original
layer.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth.configs import Config
from tests._util import device_layer, oracle_layer, rel_l2

pytestmark = pytest.mark.gpu

CFGS = [
    synth.get_config("toy"),
    Config(11, "t-reglu-bf16", 3, 512, 2048, "reglu", "bf16", "bf16", 0.02, 1.2, 0.12, 128),
    Config(13, "t-q4-reglu", 3, 512, 1536, "reglu", "q4_0", "f16", 0.015, 1.1, 0.1, 128),
]
NEURON_TENSORS = ("w_up", "w_gate", "w_down_t", "w2", "b2", "b_up", "b_gate")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from activation_sparse_pi_b200 import build
    build.build()
    import activation_sparse_pi_b200 as pi
    pi.lib()
    yield
    assert pi.pi_device_error() == 0


def permuted_copy(L, Ld, desc, perm):
    """(permuted LayerData on the device, its descriptor) via pi_permute_layer."""
    import activation_sparse_pi_b200 as pi
    kw = dict(Ld.__dict__)
    for k in NEURON_TENSORS:
        v = getattr(Ld, k)
        kw[k] = None if v is None else torch.empty_like(v)
    P = synth.LayerData(**kw)
    c = L.cfg
    pdesc = pi.layer_from_tensors(
        d_model=c.d_model, d_ff=c.d_ff, rank=P.w1.shape[0], wdtype=c.wdtype, adtype=c.adtype,
        act=c.act, w1=P.w1, b1=P.b1, w2=P.w2, b2=P.b2, threshold=P.threshold, w_up=P.w_up,
        w_gate=P.w_gate, w_down_t=P.w_down_t, b_up=P.b_up, b_gate=P.b_gate)
    pt = torch.from_numpy(perm.astype(np.int32)).cuda()
    pi.pi_permute_layer(desc, pt, pdesc)
    torch.cuda.synchronize()
    return P, pdesc


def one_layer(desc, x0, F):
    import activation_sparse_pi_b200 as pi
    ws = torch.empty(pi.pi_workspace_size([desc], x0.shape[0]), dtype=torch.uint8, device="cuda")
    xr = x0.clone().cuda()
    idx = torch.zeros(1, F, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    pi.pi_ffn_stack(pi.layer_array([desc]), xr, x0.shape[0], idx, cnt, ws)
    torch.cuda.synchronize()
    return xr.cpu().double().numpy(), idx[0, : int(cnt.item())].cpu().numpy()


@pytest.mark.parametrize("cfg", CFGS, ids=[c.name for c in CFGS])
@pytest.mark.parametrize("order", ["hot_first", "random"])
def test_permuted_layer(cfg, order):
    L = synth.make_layer(cfg, 0, "cpu", "R")
    Ld, desc = device_layer(L)
    F = cfg.d_ff
    if order == "hot_first":
        perm = np.argsort(-L.p, kind="stable")
    else:
        perm = np.random.default_rng(F).permutation(F)
    P, pdesc = permuted_copy(L, Ld, desc, perm)
    # every neuron-indexed tensor: the source rows in the new order, bit for bit
    for k in NEURON_TENSORS:
        v = getattr(L, k)
        if v is not None:
            assert torch.equal(getattr(P, k).cpu(), v[torch.from_numpy(perm)]), k
    assert torch.equal(P.w1.cpu(), L.w1)
    # same function, renumbered neurons
    B = 2
    x0 = synth.make_tokens(cfg, B, seed_offset=3)
    y_src, idx_src = one_layer(desc, x0, F)
    y_dst, idx_dst = one_layer(pdesc, x0, F)
    assert np.array_equal(np.sort(perm[idx_dst]), idx_src)
    tol = 2e-3 if cfg.wdtype == "q4_0" else 1e-3
    xd = x0.double().numpy()
    xl = oracle.rms_cast(xd, cfg.adtype)
    OL = oracle_layer(L)
    expect = xd + oracle.masked_ffn(OL, xl, idx_src)
    assert rel_l2(y_dst - xd, expect - xd) <= tol
    assert rel_l2(y_dst - xd, y_src - xd) <= 1e-5


def test_bad_perm_entry_is_flagged():
    import activation_sparse_pi_b200 as pi
    cfg = CFGS[0]
    L = synth.make_layer(cfg, 0, "cpu", "R")
    Ld, desc = device_layer(L)
    perm = np.arange(cfg.d_ff)
    perm[5] = cfg.d_ff + 3
    permuted_copy(L, Ld, desc, perm)
    assert pi.pi_device_error() == 2
