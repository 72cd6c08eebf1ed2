"""Call parameters of the estimator, mirrored on the CPU side.

sigma is an fp32 quantity in the library's interface; the oracle takes its
exact fp32 value (``sigma32``) so both sides perturb by the same amount.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Params:
    T: int
    d: int
    V: int
    K: int
    S: int = 0                 # <= 0: full vocabulary
    sigma: float = 1e-2
    seed: int = 0
    token_offset: int = 0
    draw_offset: int = 0
    subset_a: int = 0          # 0: default multiplier
    stream_id: int = 0         # mixed into Philox counter word 3 (layer id)
    d_ff: int = 0
    literal_target_scale: bool = False

    @property
    def sigma32(self) -> float:
        return float(np.float32(self.sigma))

    @property
    def full_vocab(self) -> bool:
        return self.S <= 0
