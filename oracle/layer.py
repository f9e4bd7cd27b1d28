"""The oracle's layer record: stored weights exactly as the GPU reads them.

Test infrastructure (see oracle/pi_oracle.cpp).  This module holds data only;
the arithmetic is in the C++ oracle (and, as a cross-check, in numpy_xcheck).
"""
from dataclasses import dataclass
from typing import Optional

import numpy as np


@dataclass
class OracleLayer:
    d_model: int
    d_ff: int
    act: str                     # "relu" | "reglu" | "sqrelu"
    wdtype: str                  # FFN matrices: "f16" | "bf16" | "q4_0"
    pdtype: str                  # predictor matrices: "f16" | "bf16"
    w1: np.ndarray               # stored [r x d] (uint16 bits)
    b1: Optional[np.ndarray]     # [r] or None
    w2: np.ndarray               # stored [F x r] (uint16 bits)
    b2: np.ndarray               # [F]
    threshold: float
    w_up: np.ndarray             # stored rows [F x ...] (uint16 bits, or uint8 Q4_0 bytes)
    w_gate: Optional[np.ndarray]
    w_down_t: np.ndarray
    b_up: Optional[np.ndarray] = None
    b_gate: Optional[np.ndarray] = None

    @property
    def rank(self) -> int:
        return self.w1.shape[0]
