"""Independent NumPy brute force used to pin the C oracle.  Test infrastructure.

It works on UNPAGED per-sequence K/V (the arrays the paged cache was filled
from), so it shares neither the gather nor the loops of ``pa_oracle.c``: a
mistake in the oracle's block-table walk, head mapping or softmax shows up as
a disagreement.  Attention as defined on lqnn.cn/news/235768 section 1.2:
softmax(Q K^T / sqrt(d)) V, one query row per head.
"""
import numpy as np


def dense_attention(q, K, V, scale, group):
    """q [H_q][d]; K, V [L][H_kv][d] (any float dtype); returns [H_q][d] fp64.

    Query head h uses KV head h // group.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    Hq, d = q.shape
    out = np.zeros((Hq, d))
    if K.shape[0] == 0:
        return out
    for h in range(Hq):
        g = h // group
        s = (K[:, g, :] @ q[h]) * scale
        w = np.exp(s - s.max())
        out[h] = (w / w.sum()) @ V[:, g, :]
    return out
