"""Softmax attention, float64.  (Oracle: test infrastructure only.)

The textbook definition, written out: s = (q . k) * scale for every key,
p = exp(s - max s) / sum exp(s - max s), o = sum_k p_k v_k. The log-sum-exp of
the scaled scores is returned too (natural log).
"""

import numpy as np


def softmax_attention(q, k, v, scale, mask=None):
    """q [n, D], k [m, D], v [m, Dv] -> (o [n, Dv], lse [n]), all float64.

    ``mask`` (optional, bool [n, m]) marks the keys each query may see.
    """
    s = (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T) * scale
    if mask is not None:
        s = np.where(mask, s, -np.inf)
    smax = s.max(axis=1, keepdims=True)
    e = np.exp(s - smax)
    denom = e.sum(axis=1, keepdims=True)
    o = (e @ np.asarray(v, np.float64)) / denom
    lse = (smax + np.log(denom))[:, 0]
    return o, lse
