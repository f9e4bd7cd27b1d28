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


def device_layer(L, device="cuda"):
    """(LayerData on `device`, pi_layer descriptor over its tensors)."""
    import activation_sparse_pi_b200 as pi
    Ld = L.to(device)
    c = Ld.cfg
    desc = pi.layer_from_tensors(
        d_model=c.d_model, d_ff=c.d_ff, rank=Ld.w1.shape[0], wdtype=c.wdtype, adtype=c.adtype, act=c.act,
        w1=Ld.w1, b1=Ld.b1, w2=Ld.w2, b2=Ld.b2, threshold=Ld.threshold,
        w_up=Ld.w_up, w_gate=Ld.w_gate, w_down_t=Ld.w_down_t, b_up=Ld.b_up, b_gate=Ld.b_gate)
    return Ld, desc


ADT = {"f16": torch.float16, "bf16": torch.bfloat16}


def to16(x, adtype):
    """f32 tensor holding 16-bit-exact values -> the 16-bit tensor."""
    return x.to(ADT[adtype]).contiguous()


def bits_to_bool(mask_words, F):
    """[B x F/32] int32/uint32 words -> [B x F] bool (bit n%32 of word n/32)."""
    m = np.asarray(mask_words).astype(np.uint32)
    B = m.shape[0]
    bits = (m[:, :, None] >> np.arange(32, dtype=np.uint32)[None, None, :]) & 1
    return bits.reshape(B, F).astype(bool)
