"""Test helpers: hand generator tensors to the oracle, and compare results."""
import numpy as np
import torch

import oracle


def raw(t):
    """A torch tensor as the numpy array the oracle widens (uint16 bits for
    16-bit floats, uint8 for Q4_0 bytes, float64 for f32 vectors)."""
    if t is None:
        return None
    t = t.detach().cpu()
    if t.dtype in (torch.float16, torch.bfloat16):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.uint8:
        return t.numpy()
    return t.double().numpy()


def oracle_layer(L):
    """synth.LayerData -> oracle.OracleLayer (weights copied to the host)."""
    c = L.cfg
    return oracle.OracleLayer(
        d_model=c.d_model, d_ff=c.d_ff, act=c.act, wdtype=c.wdtype, pdtype=c.adtype,
        w1=raw(L.w1), b1=raw(L.b1), w2=raw(L.w2), b2=raw(L.b2), threshold=float(L.threshold),
        w_up=raw(L.w_up), w_gate=raw(L.w_gate), w_down_t=raw(L.w_down_t),
        b_up=raw(L.b_up), b_gate=raw(L.b_gate),
    )


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    if den == 0:
        return float(np.linalg.norm(a))
    return float(np.linalg.norm(a - b) / den)
