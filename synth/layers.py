"""Seeded layer and token generators.

Every tensor is drawn from a torch.Generator keyed by (config seed, layer,
tensor id) on the requested device, so one call yields the same values each
time; small configs are drawn on the CPU and copied, so CPU and GPU tests see
identical data.

Recipe (one layer, d = d_model, F = d_ff, r = predictor rank):

* FFN matrices W_up, W_gate (ReGLU only) and W_down^T, each [F x d] with one
  neuron per row, i.i.d. N(0, sigma_w^2) rounded to the 16-bit type, or packed
  to Q4_0 (blocks of 32 values with one fp16 scale) for the INT4 config.
* Firing profile: a seeded permutation pi of the neurons and
  p_pi(k) = min(1, c k^-s), c bisected so the mean equals the target, clipped to
  [1e-6, 1 - 1e-6] (the GeekNews page and the unite.ai page describe a
  power-law activation distribution with a few "hot" neurons).
* Bias of the activation row (b_up for ReLU, b_gate for ReGLU): layer inputs
  have unit RMS, so the pre-activation w_i . x + b_i is close to
  N(b_i, |w_i|^2) and b_i = |w_i| Phi^-1(p_i) gives firing probability p_i.
* Predictor built from the true activation ("+/-" construction): G ~
  N(0, sigma_p^2) [r/2 x d], W1 = [G; -G], b1 = 0; M = W_act G^T (G G^T)^-1,
  W2 = [M, -M].  Since relu(g) - relu(-g) = g, the predictor logit is
  s = M G x + b2, the projection of the true pre-activation onto G's row
  space.  b2 = b + delta with one delta per layer:
    - mode "R": delta so that the expected recall equals the config target
      (0.9);
    - mode "F": delta so that the expected predicted fraction equals the
      mean firing probability.
  Both expectations are closed forms over x ~ N(0, I): (u_i, s_i) is a
  bivariate normal, and its orthant probability comes from Owen's T function.
* Tokens: x ~ N(0, 1) rounded to the activation dtype.
"""
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch
from scipy.special import ndtr, ndtri, owens_t

from .configs import Config

_DT = {"f16": torch.float16, "bf16": torch.bfloat16}

# tensor ids for the per-tensor seeds
_T_UP, _T_GATE, _T_DOWN, _T_G, _T_PERM = 1, 2, 3, 4, 5


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) % (2**63 - 1))
    return g


def _sub_seed(base: int, layer: int, tensor: int) -> int:
    return base * 1_000_003 + layer * 1009 + tensor


def _randn(shape, seed, device, std=1.0) -> torch.Tensor:
    t = torch.randn(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def q4_0_row_bytes(d_model: int) -> int:
    """Bytes of one Q4_0 row: d/32 blocks of (2-byte fp16 scale + 16 nibble bytes)."""
    if d_model % 32:
        raise ValueError("Q4_0 rows need d_model % 32 == 0")
    return d_model // 32 * 18


def quantize_q4_0(w: torch.Tensor) -> torch.Tensor:
    """Pack float rows [F x d] into Q4_0 rows [F x d/32*18] (uint8).

    Block layout (the ggml Q4_0 block that PowerInfer's INT4 models use):
    bytes 0-1 hold the fp16 scale (little endian); byte 2+j holds element j in
    its low nibble and element j+16 in its high nibble (j = 0..15).  A value
    decodes as (q - 8) * scale.  The quantiser takes scale = m / -8 with m the
    signed element of largest magnitude and q = clamp(round(x / scale) + 8, 0,
    15); it only shapes the data, both the oracle and the kernels decode the
    packed bytes.
    """
    F, d = w.shape
    nb = d // 32
    blocks = w.float().reshape(F, nb, 32)
    amax_idx = blocks.abs().argmax(dim=-1, keepdim=True)
    m = torch.gather(blocks, -1, amax_idx).squeeze(-1)
    scale = (m / -8.0).to(torch.float16)
    sf = scale.float()
    inv = torch.where(sf != 0, 1.0 / torch.where(sf != 0, sf, torch.ones_like(sf)),
                      torch.zeros_like(sf))
    q = torch.clamp(torch.round(blocks * inv.unsqueeze(-1)) + 8, 0, 15).to(torch.uint8)
    packed = q[..., :16] | (q[..., 16:] << 4)
    sbytes = scale.view(torch.int16).view(torch.uint8).reshape(F, nb, 2)
    return torch.cat([sbytes, packed], dim=-1).reshape(F, nb * 18).contiguous()


def zipf_profile(F: int, s: float, mean: float, seed: int) -> np.ndarray:
    """Per-neuron firing probabilities: Zipf(s) over a seeded permutation."""
    perm = torch.randperm(F, generator=_gen(seed, "cpu")).numpy()
    k = np.arange(1, F + 1, dtype=np.float64)
    base = k ** (-s)
    lo, hi = 0.0, 1.0
    while np.minimum(1.0, hi * base).mean() < mean:
        hi *= 2.0
    for _ in range(200):
        c = 0.5 * (lo + hi)
        if np.minimum(1.0, c * base).mean() < mean:
            lo = c
        else:
            hi = c
    p_rank = np.clip(np.minimum(1.0, 0.5 * (lo + hi) * base), 1e-6, 1.0 - 1e-6)
    p = np.empty(F)
    p[perm] = p_rank
    return p


def _bvn_cdf(h, k, rho):
    """P(X <= h, Y <= k) for a standard bivariate normal with correlation rho
    (Owen's T-function form)."""
    h = np.where(h == 0, 1e-12, h)
    k = np.where(k == 0, 1e-12, k)
    rho = np.clip(rho, -1 + 1e-12, 1 - 1e-12)
    sq = np.sqrt(1.0 - rho * rho)
    ah = (k - rho * h) / (h * sq)
    ak = (h - rho * k) / (k * sq)
    beta = np.where(h * k > 0, 0.0, 0.5)
    return 0.5 * (ndtr(h) + ndtr(k)) - owens_t(h, ah) - owens_t(k, ak) - beta


def _bisect(f, target, lo, hi, iters=60):
    """Root of the increasing function f(x) = target on [lo, hi]."""
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if f(mid) < target:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


@dataclass
class LayerData:
    """One synthetic layer: every tensor the library's layer descriptor names."""
    cfg: Config
    layer: int
    mode: str
    w1: torch.Tensor             # [r x d] 16-bit
    b1: torch.Tensor             # [r] f32
    w2: torch.Tensor             # [F x r] 16-bit
    b2: torch.Tensor             # [F] f32
    threshold: float
    w_up: torch.Tensor           # [F x d] 16-bit, or uint8 [F x d/32*18] (Q4_0)
    w_gate: Optional[torch.Tensor]
    w_down_t: torch.Tensor
    b_up: Optional[torch.Tensor]   # [F] f32 (ReLU only)
    b_gate: Optional[torch.Tensor] # [F] f32 (ReGLU only)
    p: np.ndarray                # [F] firing profile
    delta: float
    expected_pred_frac: float
    expected_recall: float
    bias64: Optional[np.ndarray] = None   # [F] activation-row bias before rounding
    deltas: Optional[dict] = None         # {"R": delta_R, "F": delta_F}
    stats: Optional[dict] = None          # expected fraction / recall per mode

    def tensors(self):
        return {k: getattr(self, k) for k in
                ("w1", "b1", "w2", "b2", "w_up", "w_gate", "w_down_t", "b_up", "b_gate")}

    def to(self, device) -> "LayerData":
        kw = dict(self.__dict__)
        for k, v in self.tensors().items():
            kw[k] = None if v is None else v.to(device)
        return LayerData(**kw)

    def nbytes(self) -> int:
        return sum(v.numel() * v.element_size() for v in self.tensors().values() if v is not None)


def make_layer(cfg: Config, layer: int, device="cpu", mode: str = "R") -> LayerData:
    if mode not in ("R", "F"):
        raise ValueError("mode must be 'R' (recall target) or 'F' (fraction target)")
    d, F, r = cfg.d_model, cfg.d_ff, cfg.layer_rank(layer)
    if r % 2:
        raise ValueError("predictor rank must be even for the +/- construction")
    S = cfg.seed_weights
    adt = _DT[cfg.adtype]

    def draw_matrix(tid):
        w = _randn((F, d), _sub_seed(S, layer, tid), device, cfg.sigma_w)
        if cfg.wdtype == "q4_0":
            return quantize_q4_0(w), w
        wq = w.to(_DT[cfg.wdtype])
        return wq, None

    w_up, up_f = draw_matrix(_T_UP)
    w_gate, gate_f = (draw_matrix(_T_GATE) if cfg.act == "reglu" else (None, None))
    w_down_t, _ = draw_matrix(_T_DOWN)
    # the row whose pre-activation carries the firing profile
    act_q, act_f = (w_gate, gate_f) if cfg.act == "reglu" else (w_up, up_f)
    w_act = act_f if act_f is not None else act_q  # unquantised floats for Q4_0
    del up_f, gate_f

    # predictor first layer
    g = _randn((r // 2, d), _sub_seed(S, layer, _T_G), device, cfg.sigma_p).to(adt)
    w1 = torch.cat([g, -g], dim=0).contiguous()
    b1 = torch.zeros(r, dtype=torch.float32, device=device)
    gf = g.float()
    gram = (gf.double() @ gf.double().T)
    chol = torch.linalg.cholesky(gram)

    # M = W_act G^T (G G^T)^-1, its rounded copy, and the closed-form moments of
    # the (true, predicted) pre-activation pair, in row chunks.
    rows = 4096
    m_parts, su, sv, cuv = [], [], [], []
    for i0 in range(0, F, rows):
        wa = w_act[i0:i0 + rows].float()
        wg = (wa @ gf.T).double()
        m = torch.cholesky_solve(wg.T, chol).T
        mh = m.to(adt)
        v = mh.float() @ gf
        m_parts.append(mh)
        su.append(wa.double().norm(dim=1))
        sv.append(v.double().norm(dim=1))
        cuv.append((wa.double() * v.double()).sum(dim=1))
        del wa, wg, m, v
    mh = torch.cat(m_parts, dim=0)
    w2 = torch.cat([mh, -mh], dim=1).contiguous()
    del m_parts, mh
    su = torch.cat(su).cpu().numpy()
    sv = torch.cat(sv).cpu().numpy()
    cuv = torch.cat(cuv).cpu().numpy()
    sv = np.maximum(sv, 1e-30)
    rho = cuv / (su * sv)

    p = zipf_profile(F, cfg.layer_zipf(layer), cfg.mean_active, _sub_seed(S, layer, _T_PERM))
    b = su * ndtri(p)

    def frac(delta):
        return float(ndtr((b + delta) / sv).mean())

    def recall(delta):
        return float(_bvn_cdf(b / su, (b + delta) / sv, rho).sum() / p.sum())

    span = 20.0 * float(su.max() + sv.max())
    deltas = {"F": _bisect(frac, float(p.mean()), -span, span),
              "R": _bisect(recall, cfg.recall, -span, span)}
    stats = {m: {"pred_frac": frac(dl), "recall": recall(dl)} for m, dl in deltas.items()}
    delta = deltas[mode]

    bias = torch.tensor(b, dtype=torch.float32, device=device)
    b2 = torch.tensor(b + delta, dtype=torch.float32, device=device)
    return LayerData(
        cfg=cfg, layer=layer, mode=mode,
        w1=w1, b1=b1, w2=w2, b2=b2, threshold=0.0,
        w_up=w_up, w_gate=w_gate, w_down_t=w_down_t,
        b_up=None if cfg.act == "reglu" else bias,
        b_gate=bias if cfg.act == "reglu" else None,
        p=p, delta=delta,
        expected_pred_frac=stats[mode]["pred_frac"], expected_recall=stats[mode]["recall"],
        bias64=b, deltas=deltas, stats=stats,
    )


def with_mode(L: LayerData, mode: str) -> LayerData:
    """The same layer with the predictor bias of the other calibration mode."""
    kw = dict(L.__dict__)
    kw["mode"] = mode
    kw["delta"] = L.deltas[mode]
    kw["b2"] = torch.tensor(L.bias64 + L.deltas[mode], dtype=torch.float32, device=L.b2.device)
    kw["expected_pred_frac"] = L.stats[mode]["pred_frac"]
    kw["expected_recall"] = L.stats[mode]["recall"]
    return LayerData(**kw)


def make_tokens(cfg: Config, n: int, device="cpu", seed_offset: int = 0) -> torch.Tensor:
    """n tokens x ~ N(0, 1) rounded to the activation dtype, returned as f32."""
    x = _randn((n, cfg.d_model), cfg.seed_tokens * 7919 + seed_offset, device)
    return x.to(_DT[cfg.adtype]).float()
