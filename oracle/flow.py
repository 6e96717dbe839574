"""Flow-matching Euler step, fp64.

papernotes note, 损失函数: the velocity model regresses x1 - x0.  Reading: x1
is noise at t = 1, x0 is data at t = 0, x_t = (1 - t) x0 + t x1, so
dx/dt = x1 - x0 = v and one Euler step from t_i to t_{i+1} < t_i is
x_{t_{i+1}} = x_{t_i} + (t_{i+1} - t_i) v.
"""
from __future__ import annotations

import numpy as np


def euler_step(x, v, t_from: float, t_to: float):
    return np.asarray(x, np.float64) + (float(t_to) - float(t_from)) * np.asarray(v, np.float64)
