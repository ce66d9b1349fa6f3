"""Guidance weights and time steps of the flow-matching sampler (host side).

Ideogram 4 deep dive, section 4-4: the guidance weight gw may change from step to step; the
V4_QUALITY_48 preset guides hard with gw = 7 for its first 45 steps and with gw = 3 for the
last 3.  Section 4-6: the latent is integrated from t = 1 to t = 0 by Euler steps
z <- z + v (s - t), where s is the next, smaller time.  The pages describe the noise schedule
only as logit-normal and adjusted to the resolution, without its formula, so the time grid is
an argument of the sampler; ``uniform_dts`` gives the plain uniform grid.
"""
from __future__ import annotations

from typing import Callable, Dict, List

import numpy as np

# Depth of the DiT: the Ideogram 4.0 announcement thread describes a 34-layer single-stream DiT.
DIT_LAYERS = 34


def v4_quality_48() -> List[float]:
    """Per-step guidance of the V4_QUALITY_48 preset: 45 steps at 7, then 3 at 3."""
    return [7.0] * 45 + [3.0] * 3


PRESETS: Dict[str, Callable[[], List[float]]] = {"V4_QUALITY_48": v4_quality_48}


def guidance(preset: str) -> List[float]:
    """Guidance weights of a named preset, one per step."""
    return PRESETS[preset]()


def uniform_dts(n_steps: int) -> List[float]:
    """dt = s - t of each step on the uniform grid t_k = 1 - k / n_steps (all equal to -1/n), in fp32."""
    t = 1.0 - np.arange(n_steps + 1, dtype=np.float64) / n_steps
    return [float(np.float32(t[k + 1] - t[k])) for k in range(n_steps)]
