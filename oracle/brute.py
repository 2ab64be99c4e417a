"""NumPy brute-force attention over contiguous (unpaged) K/V -- test infrastructure.

Used only on tiny inputs, as an independent check of the paged oracle's gather:
the test builds each sequence's K/V as plain contiguous arrays first, pages them
into a pool itself, and compares this function's result on the contiguous
arrays with the C oracle's result on the paged pool.
"""
from __future__ import annotations

import numpy as np


def attention_contiguous(q, k, v, scale, group):
    """Causal-tail attention for one sequence.

    q: [Q, H, D] query rows (the sequence's last Q tokens), k/v: [L, Hk, D].
    Row t sees keys 0 .. L - Q + t.  Head h reads KV head h // group.
    Returns float64 [Q, H, D].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    nq, nh, _ = q.shape
    L = k.shape[0]
    out = np.zeros_like(q)
    for t in range(nq):
        n = L - nq + t + 1
        if L == 0 or n <= 0:
            continue
        for h in range(nh):
            kv = h // group
            s = (k[:n, kv, :] @ q[t, h, :]) * scale
            w = np.exp(s - s.max())
            out[t, h, :] = (w[:, None] * v[:n, kv, :]).sum(axis=0) / w.sum()
    return out
