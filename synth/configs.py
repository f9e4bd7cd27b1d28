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
    ]
}


def get_config(name: str) -> Config:
    if name not in CONFIGS:
        raise KeyError(f"unknown config {name!r}; known: {sorted(CONFIGS)}")
    return CONFIGS[name]
