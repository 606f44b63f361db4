"""fp64 CPU oracle for the cluster-attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
product path never imports, links or calls anything here, and the oracle
never imports the product package (it shares no code with it).

``oracle.c`` is the plain C implementation (IEEE double, index-order sums,
threads over heads only).  This module compiles it with gcc on first use and
wraps it with ctypes; ``oracle_np`` holds a small NumPy restatement used to
cross-check the C code on tiny inputs.

Pins (tests/test_oracle_pins.py) tie it to facts outside itself: the dense
attention limit K = L of "Hooshaai/svd-sst2-roberta-cluster" section 2.3
(against torch's scaled_dot_product_attention), alpha = 1 against band-masked
scaled_dot_product_attention, K = 1 against softmax(mean(Q) K^T / sqrt(d)) V,
the Lloyd objective's monotonicity, scikit-learn's Lloyd k-means, scipy's
cdist, Theorem 1 of both model cards, W = 0 (each token attends to itself
only), and hand-derived worked examples under tests/golden/.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain gcc, IEEE semantics)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-o", tmp, _SRC, "-lpthread", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            ci, cd = ctypes.c_int, ctypes.c_double
            lib.oracle_forward.argtypes = [dp, dp, dp, ci, ci, ci, ci, ci, ci, ci, cd, ci, dp, ip, dp, ip, ci]
            lib.oracle_forward_at.argtypes = [dp, dp, dp, ci, ci, ci, ci, ci, ci, ci, cd, ci, ip, dp, dp, ci]
            u8p = ctypes.POINTER(ctypes.c_uint8)
            lib.oracle_forward_ex.argtypes = [dp, dp, dp, ci, ci, ci, ci, ci, ci, ci, cd, ci, ci, ci, ci, ci,
                                              u8p, ci, dp, ip, dp, ip, ci]
            lib.oracle_kmeans.argtypes = [dp, ci, ci, ci, ci, ci, ip, dp, ip]
            lib.oracle_update.argtypes = [dp, ip, ci, ci, ci, ci, dp]
            lib.oracle_distances.argtypes = [dp, dp, ci, ci, ci, dp]
            lib.oracle_centroid_attention.argtypes = [dp, dp, dp, ci, ci, ci, dp]
            lib.oracle_window_attention.argtypes = [dp, dp, dp, ci, ci, ci, dp]
            for f in (lib.oracle_forward, lib.oracle_forward_at, lib.oracle_forward_ex, lib.oracle_kmeans, lib.oracle_update,
                      lib.oracle_distances, lib.oracle_centroid_attention, lib.oracle_window_attention):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _dp(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _check(st: int, what: str) -> None:
    if st != 0:
        raise ValueError(f"oracle {what} failed with status {st}")


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def forward(q, k, v, K: int, iters: int, W: int, alpha: float, mu_f32: bool = True,
            hist: bool = False, nthreads: Optional[int] = None):
    """Full forward on [B,H,L,d] float64 inputs.

    Returns (out [B,H,L,d] f64, assign [B,H,L] i32, centroids [B,H,K,d] f64,
    hist [B,H,iters,L] i32 or None).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, L, d = q.shape
    out = np.empty_like(q)
    assign = np.empty((B, H, L), dtype=np.int32)
    cent = np.empty((B, H, K, d), dtype=np.float64)
    hh = np.empty((B, H, iters, L), dtype=np.int32) if hist else None
    lib = _load()
    st = lib.oracle_forward(_dp(q), _dp(k), _dp(v), B, H, L, d, K, iters, W, float(alpha),
                            int(bool(mu_f32)), _dp(out), _ip(assign), _dp(cent), _ip(hh),
                            nthreads or default_threads())
    _check(st, "forward")
    return out, assign, cent, hh


def forward_ex(q, k, v, K: int, iters: int, W: int, alpha: float, mu_f32: bool = True,
               window_module: bool = False, empty_keep: bool = False, init_stride: bool = False,
               soft_gather: bool = False, key_valid=None, H_kv: int = 0, hist: bool = False,
               nthreads: Optional[int] = None):
    """The forward with the variants of the card's module ([P2] section 5):
    window_module (band |i-j| <= W; no local branch when W == 0 or W >= L),
    empty_keep, init_stride (k * max(1, L // K)), soft_gather, key_valid
    ([B, L] bool/uint8 or None) and grouped key/value heads (k, v of shape
    [B, H_kv, L, d]).  Returns (out, assign, centroids, hist)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, L, d = q.shape
    out = np.empty_like(q)
    assign = np.empty((B, H, L), dtype=np.int32)
    cent = np.empty((B, H, K, d), dtype=np.float64)
    hh = np.empty((B, H, iters, L), dtype=np.int32) if hist else None
    kv = None
    if key_valid is not None:
        kv = np.ascontiguousarray(key_valid, dtype=np.uint8).reshape(B, L)
    kvp = None if kv is None else kv.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
    st = _load().oracle_forward_ex(_dp(q), _dp(k), _dp(v), B, H, L, d, K, iters, W, float(alpha),
                                   int(bool(mu_f32)), int(bool(window_module)), int(bool(empty_keep)),
                                   int(bool(init_stride)), int(bool(soft_gather)), kvp, int(H_kv),
                                   _dp(out), _ip(assign), _dp(cent), _ip(hh),
                                   nthreads or default_threads())
    _check(st, "forward_ex")
    return out, assign, cent, hh


def forward_at(q, k, v, assign, K: int, iters: int, W: int, alpha: float, mu_f32: bool = True,
               nthreads: Optional[int] = None):
    """The forward evaluated at given final assignments: returns (out, centroids)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, L, d = q.shape
    a = _i32(assign).reshape(B, H, L)
    out = np.empty_like(q)
    cent = np.empty((B, H, K, d), dtype=np.float64)
    st = _load().oracle_forward_at(_dp(q), _dp(k), _dp(v), B, H, L, d, K, iters, W, float(alpha),
                                   int(bool(mu_f32)), _ip(a), _dp(out), _dp(cent),
                                   nthreads or default_threads())
    _check(st, "forward_at")
    return out, cent


def kmeans(q_head, K: int, iters: int, mu_f32: bool = True):
    """One head's k-means: returns (c [L], mu [K,d], hist [iters,L])."""
    q = _f64(q_head)
    L, d = q.shape
    c = np.empty(L, dtype=np.int32)
    mu = np.empty((K, d), dtype=np.float64)
    hist = np.empty((iters, L), dtype=np.int32)
    _check(_load().oracle_kmeans(_dp(q), L, d, K, iters, int(bool(mu_f32)), _ip(c), _dp(mu), _ip(hist)),
           "kmeans")
    return c, mu, hist


def update(q_head, c, K: int, mu_f32: bool = True):
    q = _f64(q_head)
    L, d = q.shape
    cc = _i32(c)
    mu = np.empty((K, d), dtype=np.float64)
    _check(_load().oracle_update(_dp(q), _ip(cc), L, d, K, int(bool(mu_f32)), _dp(mu)), "update")
    return mu


def distances(q_head, mu):
    q, m = _f64(q_head), _f64(mu)
    L, d = q.shape
    K = m.shape[0]
    D = np.empty((L, K), dtype=np.float64)
    _check(_load().oracle_distances(_dp(q), _dp(m), L, d, K, _dp(D)), "distances")
    return D


def centroid_attention(mu, k_head, v_head):
    m, k, v = _f64(mu), _f64(k_head), _f64(v_head)
    K, d = m.shape
    L = k.shape[0]
    out = np.empty((K, d), dtype=np.float64)
    _check(_load().oracle_centroid_attention(_dp(m), _dp(k), _dp(v), L, d, K, _dp(out)),
           "centroid_attention")
    return out


def window_attention(q_head, k_head, v_head, W: int):
    q, k, v = _f64(q_head), _f64(k_head), _f64(v_head)
    L, d = q.shape
    out = np.empty((L, d), dtype=np.float64)
    _check(_load().oracle_window_attention(_dp(q), _dp(k), _dp(v), L, d, W, _dp(out)),
           "window_attention")
    return out
