"""Error metrics used by the parity tests (TEST INFRASTRUCTURE).

max-abs = max_i |x_i - y_i|; relative RMS = ||x - y||_2 / ||y||_2 over the
whole tensor, y being the oracle (the readings of the tolerances' metrics).
"""

from __future__ import annotations

import numpy as np


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def max_abs(x, ref) -> float:
    x, ref = _f64(x), _f64(ref)
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


def rel_rms(x, ref) -> float:
    x, ref = _f64(x), _f64(ref)
    den = float(np.sqrt(np.sum(ref * ref)))
    num = float(np.sqrt(np.sum((x - ref) ** 2)))
    return num / den if den > 0 else num
