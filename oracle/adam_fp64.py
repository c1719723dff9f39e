"""Textbook Adam in float64 (Kingma & Ba, "Adam: A Method for Stochastic
Optimization", Algorithm 1), used only to bound the fp32 oracle's rounding
error.  Test infrastructure.

The concept page "ZeRO", section "为什么需要它", names the state mixed-precision
Adam keeps (low-precision parameters, fp32 master weight, first and second
moments); the update itself is the textbook one, written here in its original
form with explicit bias-corrected moments:
    m_t = b1 m + (1-b1) g,   v_t = b2 v + (1-b2) g^2,
    mhat = m_t / (1-b1^t),   vhat = v_t / (1-b2^t),
    w_t = w - lr * mhat / (sqrt(vhat) + eps).
"""
import numpy as np


def adam_fp64(g, w, m, v, lr, beta1, beta2, eps, t):
    """All inputs float64 arrays (or floats); returns new (w, m, v)."""
    g = np.asarray(g, dtype=np.float64)
    b1 = float(beta1)
    b2 = float(beta2)
    m_t = b1 * m + (1.0 - b1) * g
    v_t = b2 * v + (1.0 - b2) * g * g
    mhat = m_t / (1.0 - b1 ** t)
    vhat = v_t / (1.0 - b2 ** t)
    w_t = w - float(lr) * mhat / (np.sqrt(vhat) + float(eps))
    return w_t, m_t, v_t
