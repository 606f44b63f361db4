"""A second, literal restatement of the cluster-attention forward in NumPy.

TEST INFRASTRUCTURE ONLY (see the package docstring).  It exists to catch
indexing or memory mistakes in oracle.c on tiny inputs: it loops in Python,
measures distances in the direct form |Q_i - mu_k|^2 (the model card
"Hooshaai/distilbert-sst2-cluster-attention", section 1) rather than the
expanded one, and keeps every value in float64.  Being a restatement of the
same steps, it is a cross-check, not a pin.
"""

from __future__ import annotations

import numpy as np


def kmeans_direct(q: np.ndarray, K: int, iters: int, mu_f32: bool = True):
    L, d = q.shape
    mu = np.stack([q[(k * L) // K] for k in range(K)]).astype(np.float64)
    c = np.zeros(L, dtype=np.int64)
    for _ in range(iters):
        for i in range(L):
            best, best_d = 0, None
            for k in range(K):
                diff = q[i] - mu[k]
                dk = float(np.sum(diff * diff))
                if best_d is None or dk < best_d:
                    best, best_d = k, dk
            c[i] = best
        new = np.zeros_like(mu)
        for k in range(K):
            members = q[c == k]
            m = members.sum(axis=0) / max(1, members.shape[0])
            new[k] = m.astype(np.float32).astype(np.float64) if mu_f32 else m
        mu = new
    return c, mu


def _softmax_rows(z: np.ndarray) -> np.ndarray:
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def forward_head(q, k, v, K: int, iters: int, W: int, alpha: float, mu_f32: bool = True):
    L, d = q.shape
    c, mu = kmeans_direct(q, K, iters, mu_f32)
    s = 1.0 / np.sqrt(d)
    vcent = _softmax_rows(mu @ k.T * s) @ v
    r = W // 2
    local = np.empty_like(q)
    for i in range(L):
        lo, hi = max(0, i - r), min(L - 1, i + r)
        p = _softmax_rows((k[lo:hi + 1] @ q[i]) * s)
        local[i] = p @ v[lo:hi + 1]
    out = (1.0 - alpha) * vcent[c] + alpha * local
    return out, c, mu
