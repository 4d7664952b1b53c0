"""Oracle: rotary position embedding with per-document positions, half-split form.
TEST INFRASTRUCTURE ONLY.

Source: MindSpeed pull request #3820, "feat: kvallgather cp thd load balance",
section "Does this PR introduce any user-facing change?": positions restart with every
EOD-delimited document.  The pages name no rotary variant; reading: the half-split
form, pairing dimension i with i + R/2 (R = rotary width), angle pos * base^(-2i/R),
dimensions R .. D-1 unchanged.
"""
from __future__ import annotations

import numpy as np


def rope(x, pos, rot_dim: int, base: float = 10000.0) -> np.ndarray:
    """x [T, H, D] (upcast to float64), pos [T] -> rotated copy, float64."""
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    half = rot_dim // 2
    out = x.copy()
    for i in range(half):
        ang = pos * base ** (-2.0 * i / rot_dim)            # [T]
        c = np.cos(ang)[:, None]
        s = np.sin(ang)[:, None]
        a = x[:, :, i]
        b = x[:, :, i + half]
        out[:, :, i] = a * c - b * s
        out[:, :, i + half] = b * c + a * s
    return out
