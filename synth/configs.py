"""The five synthetic layer-stack workloads.

Shapes follow the models the PowerInfer pages evaluate (OPT-6.7B,
ReLU-Llama-2-13B, Falcon(ReLU)-40B, LLaMA(ReGLU)-70B; the machine-heart page,
experiments section, and the PyTorchKR page, "Model Weights" tables) plus one
toy layer.  Activation fractions follow the machine-heart page's discussion of
Figure 10 (about 20% of neurons active per token for OPT-30B).
"""
from dataclasses import dataclass, field
from typing import Tuple


@dataclass(frozen=True)
class Config:
    index: int            # 0-based position in CONFIGS (seeds derive from it)
    name: str
    n_layers: int
    d_model: int
    d_ff: int
    act: str              # "relu", "reglu" or "sqrelu"
    wdtype: str           # "f16", "bf16" or "q4_0" (FFN matrices)
    adtype: str           # 16-bit activation / predictor dtype: "f16" or "bf16"
    sigma_w: float        # std of the FFN weights
    zipf_s: float         # Zipf exponent of the per-neuron firing profile
    mean_active: float    # target mean firing probability
    rank: int             # predictor hidden width r
    sigma_p: float = 0.05 # std of the predictor's first layer
    recall: float = 0.9   # predictor recall target (mode "R")
    batches: Tuple[int, ...] = (1,)
    n_tokens: int = 128
    prompt_tokens: int = 0
    # adaptive predictor sizing (unite.ai page, "Adaptive Sparsity-Prädiktoren":
    # each layer's predictor is sized from that layer's sparsity and skew):
    # the Zipf exponent runs linearly over [zipf_s - skew_spread, zipf_s +
    # skew_spread] across the layers, and with adaptive_rank the predictor
    # rank shrinks where the firing profile is more skewed
    skew_spread: float = 0.0
    adaptive_rank: bool = False

    def layer_zipf(self, layer: int) -> float:
        if self.n_layers <= 1 or self.skew_spread == 0.0:
            return self.zipf_s
        return self.zipf_s + self.skew_spread * (2.0 * layer / (self.n_layers - 1) - 1.0)

    def layer_rank(self, layer: int) -> int:
        """Predictor rank of one layer: the config's rank scaled by
        (zipf_s / s_layer)^2, a multiple of 16 within [rank / 2, 2 rank]."""
        if not self.adaptive_rank:
            return self.rank
        r = self.rank * (self.zipf_s / self.layer_zipf(layer)) ** 2
        r = int(round(r / 16.0)) * 16
        return max(self.rank // 2, min(2 * self.rank, r))

    @property
    def seed_weights(self) -> int:
        return 1000 + self.index

    @property
    def seed_tokens(self) -> int:
        return 2000 + self.index


CONFIGS = {
    c.name: c
    for c in [
        Config(0, "toy", 1, 512, 2048, "relu", "f16", "f16", 0.02, 1.1, 0.10, 128,
               n_tokens=64),
        Config(1, "opt-6.7b", 32, 4096, 16384, "relu", "f16", "f16", 0.02, 1.1, 0.20, 1024,
               n_tokens=128),
        Config(2, "relu-llama2-13b", 40, 5120, 13824, "reglu", "bf16", "bf16", 0.02, 1.2,
               0.12, 1024, batches=(1, 8), n_tokens=128),
        Config(3, "falcon-40b", 60, 8192, 32768, "relu", "f16", "f16", 0.015, 1.0, 0.08, 1024,
               n_tokens=128, prompt_tokens=64),
        Config(4, "llama2-70b-q4", 80, 8192, 28672, "reglu", "q4_0", "f16", 0.015, 1.1, 0.10,
               1536, batches=(1, 8, 32), n_tokens=128),
        # the OPT-6.7B shapes with Squared-ReLU neurons (GeekNews page, limitations
        # list: ReLU, ReGLU and Squared-ReLU models)
        Config(5, "opt-6.7b-sqrelu", 32, 4096, 16384, "sqrelu", "f16", "f16", 0.02, 1.1, 0.20,
               1024, n_tokens=128),
        # the OPT-6.7B shapes with a per-layer skew profile (Zipf 0.8 .. 1.4) and
        # predictors sized per layer (ranks 624 .. 1936)
        Config(6, "opt-6.7b-adaptive", 32, 4096, 16384, "relu", "f16", "f16", 0.02, 1.1, 0.20,
               1024, n_tokens=128, skew_spread=0.3, adaptive_rank=True),
    ]
}


def get_config(name: str) -> Config:
    if name not in CONFIGS:
        raise KeyError(f"unknown config {name!r}; known: {sorted(CONFIGS)}")
    return CONFIGS[name]
