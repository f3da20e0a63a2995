"""Input preprocessing of the KDA operator, fp64 numpy -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may
import this module; it shares nothing with the CUDA library.

The pages give the per-channel decay as the output of an "alpha projection"
with every alpha between 0 and 1 ("22580倍参数量级" article,
tahou.com/article/213680821660188677, sections on Gated DeltaNet and on the
Kimi Linear architecture), and the learning rate beta between 0 and 1
("我终于看懂了 KDA" explainer, pwwt.cn/news/3787313, section 六).  They do not
fix how raw projections are mapped into those ranges.  This library reads it as
the usual parametrisation:

* keys and queries are divided by their L2 norm over d_k (an all-zero vector
  stays zero), so that every ``I - beta k k^T`` has spectral norm at most 1;
* log alpha = -softplus(a) = -log(1 + e^a) for a raw gate logit a;
* beta = sigmoid(b) = 1 / (1 + e^-b) for a raw logit b.

Each function is the definition written out with numpy primitives.
"""
from __future__ import annotations

import numpy as np

QK_L2NORM, GATE_SOFTPLUS, BETA_SIGMOID = 1, 2, 4


def l2_normalize(x):
    """x / ||x||_2 over the last axis; rows that are all zero stay zero."""
    x = np.asarray(x, dtype=np.float64)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return np.divide(x, n, out=np.zeros_like(x), where=n > 0)


def log_alpha_from_gate(a):
    """log alpha = -softplus(a) = -log(e^0 + e^a)."""
    return -np.logaddexp(0.0, np.asarray(a, dtype=np.float64))


def beta_from_logit(b):
    """beta = 1 / (1 + e^-b)."""
    b = np.asarray(b, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-b))


def preprocess(q, k, gate, beta, flags: int):
    """Apply the preprocessing selected by ``flags`` (QK_L2NORM | GATE_SOFTPLUS |
    BETA_SIGMOID); unselected inputs pass through unchanged.  Returns fp64
    ``(q, k, log_alpha, beta)``."""
    q, k, gate, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, gate, beta))
    if flags & QK_L2NORM:
        q, k = l2_normalize(q), l2_normalize(k)
    if flags & GATE_SOFTPLUS:
        gate = log_alpha_from_gate(gate)
    if flags & BETA_SIGMOID:
        beta = beta_from_logit(beta)
    return q, k, gate, beta
