"""Seeded synthetic workloads for the cluster-attention forward pass.

This module only draws random numbers and lays them out as [B, H, L, d]
row-major arrays.  It holds none of the method's arithmetic, so both the CUDA
path (through the binding) and the fp64 oracle can consume the same inputs.

Workloads follow the shapes of the model cards "Hooshaai/distilbert-sst2-
cluster-attention" (benchmark table: B=32, L=128, H=12, d=64, K=16, W=32) and
"Hooshaai/svd-sst2-roberta-cluster" (section 2.1, the same method), extended
to long sequences.  No dataset is involved: the cards' SST-2 evaluations need
text data and trained weights, and these synthetic tensors stand in for the
query/key/value activations of such a model.

Recipe (every workload uses ``numpy.random.default_rng(seed)``, seed 0):

* draw order: mixture means, mixture labels, query noise, K, V, then the
  duplicate positions;
* fp32 workloads draw float64 and cast once to float32;
* bf16 workloads draw float32 and round once to bf16 (round to nearest even);
  the bf16 arrays are returned as raw uint16 bit patterns plus their exact
  float64 values;
* ``gmm`` queries: per (b, h) ``C`` means ~ N(0, 4 I) (std 2 per coordinate),
  i.i.d. uniform labels over the C components, Q_i = m_label + s * N(0, I);
* ``dup`` workloads copy 10% of the token positions of each head (Q, K and V
  rows together) from other positions.  The copied-to set always contains
  every position floor(k L / K) with k odd, each copying position
  floor((k-1) L / K): two strided starting centroids are then bitwise equal,
  which forces exact distance ties and an empty cluster.  The remaining
  destinations copy a uniformly drawn position outside the destination set.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "make_inputs",
    "bf16_round_bits",
    "bf16_bits_to_f64",
    "bf16_bits_to_f32",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int
    K: int
    iters: int
    W: int
    alpha: float
    dtype: str  # "f32" or "bf16"
    q_kind: str  # "normal" or "gmm"
    gmm_components: int = 0
    gmm_std: float = 0.0
    dup_frac: float = 0.0

    @property
    def heads(self) -> int:
        return self.B * self.H

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.L

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a small fp32 case, the model card's benchmark shape with
# well-separated queries, and three bf16 long-sequence cases.
WORKLOADS: Dict[str, Workload] = {
    "small_f32": Workload("small_f32", 2, 12, 128, 64, 16, 3, 32, 0.5, "f32", "normal"),
    "card_gmm_f32": Workload("card_gmm_f32", 32, 12, 128, 64, 16, 3, 32, 0.5, "f32", "gmm",
                             gmm_components=16, gmm_std=0.1),
    "l512_bf16": Workload("l512_bf16", 64, 12, 512, 64, 16, 3, 32, 0.5, "bf16", "normal"),
    "l4k_gmm_bf16": Workload("l4k_gmm_bf16", 8, 12, 4096, 64, 32, 3, 64, 0.3, "bf16", "gmm",
                             gmm_components=32, gmm_std=0.5),
    "l32k_dup_bf16": Workload("l32k_dup_bf16", 1, 16, 32768, 64, 64, 5, 128, 0.5, "bf16",
                              "normal", dup_frac=0.1),
}
WORKLOAD_ORDER = ["small_f32", "card_gmm_f32", "l512_bf16", "l4k_gmm_bf16", "l32k_dup_bf16"]


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


def _draw(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return rng.standard_normal(shape, dtype=np.float64)
    return rng.standard_normal(shape, dtype=np.float32)


def make_inputs(w: Workload, seed: int = 0, heads: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw Q, K, V for workload ``w``.

    Returns a dict with ``q``, ``k``, ``v`` in storage form (float32 arrays, or
    uint16 bf16 bit patterns) and ``q64``, ``k64``, ``v64``: the exact float64
    values of the stored elements.  ``heads`` (optional) draws only the first
    ``heads`` heads of a B=1 layout, for bounded samples of a large workload;
    the result then has shape [1, heads, L, d] and its own random stream.
    """
    B, H, L, d = w.B, w.H, w.L, w.d
    if heads is not None:
        B, H = 1, heads
    rng = np.random.default_rng(seed)
    shape = (B, H, L, d)
    f = np.float64 if w.dtype == "f32" else np.float32

    if w.q_kind == "gmm":
        C = w.gmm_components
        means = (2.0 * _draw(rng, (B, H, C, d), w.dtype)).astype(f)
        labels = rng.integers(0, C, size=(B, H, L))
        noise = _draw(rng, shape, w.dtype).astype(f)
        picked = np.take_along_axis(means, labels[..., None].repeat(d, axis=-1), axis=2)
        q = (picked + f(w.gmm_std) * noise).astype(f)
    elif w.q_kind == "normal":
        q = _draw(rng, shape, w.dtype).astype(f)
    else:
        raise ValueError(f"unknown q_kind {w.q_kind!r}")
    k = _draw(rng, shape, w.dtype).astype(f)
    v = _draw(rng, shape, w.dtype).astype(f)

    if w.dup_frac > 0.0:
        n_dup = int(np.floor(w.dup_frac * L))
        forced_dst = np.array([(kk * L) // w.K for kk in range(1, w.K, 2)], dtype=np.int64)
        forced_src = np.array([((kk - 1) * L) // w.K for kk in range(1, w.K, 2)], dtype=np.int64)
        for b in range(B):
            for h in range(H):
                free = np.setdiff1d(np.arange(L), np.concatenate([forced_dst, forced_src]))
                extra = rng.choice(free, size=max(0, n_dup - forced_dst.size), replace=False)
                dst_all = np.concatenate([forced_dst, np.sort(extra)])
                pool = np.setdiff1d(np.arange(L), dst_all)
                src_extra = rng.choice(pool, size=extra.size, replace=True)
                src_all = np.concatenate([forced_src, src_extra])
                for arr in (q, k, v):
                    arr[b, h, dst_all, :] = arr[b, h, src_all, :]

    out: Dict[str, np.ndarray] = {}
    for name, arr in (("q", q), ("k", k), ("v", v)):
        if w.dtype == "f32":
            s = np.ascontiguousarray(arr.astype(np.float32))
            out[name] = s
            out[name + "64"] = s.astype(np.float64)
        else:
            bits = bf16_round_bits(arr)
            out[name] = bits
            out[name + "64"] = bf16_bits_to_f64(bits)
    return out
