"""Pins for the fp64 oracle: facts fixed by the model cards and by mathematics.

Each test ties the oracle to something other than itself: a library routine
(torch scaled_dot_product_attention, scipy cdist, scikit-learn's Lloyd
k-means, numpy mean), a closed form, an invariant of the method, or a worked
example derived by hand (tests/golden/worked_examples.json).  The comments say
which plausible mistake each one catches.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import oracle_np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _sdpa(q, k, v, mask=None):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    out = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=None if mask is None else torch.from_numpy(mask))
    return out.numpy()


# --------------------------------------------------------------------------
# Dense-attention limit: with K = L every token is its own cluster and the
# centroid branch is full softmax attention ("Hooshaai/svd-sst2-roberta-
# cluster", section 2.3).  Catches a wrong scale, softmax axis, swapped K/V,
# wrong gather index or wrong V_cent row.
@pytest.mark.parametrize("mu_f32", [True, False])
@pytest.mark.parametrize("L,iters", [(1, 1), (5, 1), (24, 3), (33, 2)])
def test_dense_limit_k_equals_l(mu_f32, L, iters):
    B, H, d = 1, 2, 64
    q, k, v = (_f32(_rand((B, H, L, d), s)) for s in (1, 2, 3))
    out, assign, cent, _ = oracle.forward(q, k, v, K=L, iters=iters, W=8, alpha=0.0, mu_f32=mu_f32)
    ref = _sdpa(q, k, v)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    if iters > 0:
        assert (assign == np.arange(L)[None, None, :]).all()
    np.testing.assert_array_equal(cent, q)


# --------------------------------------------------------------------------
# alpha = 1 leaves only the local branch, which must equal dense attention
# with a band mask |i - j| <= floor(W/2).  Catches off-by-one window edges,
# radius W instead of W/2, and wrong clipping at both ends.
@pytest.mark.parametrize("W", [0, 1, 2, 3, 7, 32, 100])
def test_alpha_one_is_band_attention(W):
    B, H, L, d = 1, 2, 37, 64
    q, k, v = (_rand((B, H, L, d), s) for s in (4, 5, 6))
    out, *_ = oracle.forward(q, k, v, K=4, iters=2, W=W, alpha=1.0)
    idx = np.arange(L)
    band = np.abs(idx[:, None] - idx[None, :]) <= W // 2
    ref = _sdpa(q, k, v, mask=band)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# W = 0 (and W = 1) leaves each token only itself: softmax over one key is 1,
# so the local output is exactly V_i.
@pytest.mark.parametrize("W", [0, 1])
def test_window_self_only(W):
    q, k, v = (_rand((1, 1, 9, 64), s) for s in (7, 8, 9))
    out, *_ = oracle.forward(q, k, v, K=3, iters=1, W=W, alpha=1.0)
    np.testing.assert_allclose(out, v, rtol=0, atol=1e-14)


# W >= 2(L-1) covers every key: the local branch is full dense attention.
def test_full_window_is_dense():
    L = 21
    q, k, v = (_rand((1, 3, L, 64), s) for s in (10, 11, 12))
    out, *_ = oracle.forward(q, k, v, K=5, iters=2, W=2 * (L - 1), alpha=1.0)
    np.testing.assert_allclose(out, _sdpa(q, k, v), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# K = 1: the single centroid is the mean of all queries after one iteration,
# so every token gets softmax(mean(Q) K^T / sqrt(d)) V.  Catches a wrong
# update rule (sum instead of mean, wrong count) and centroid-branch errors.
@pytest.mark.parametrize("iters", [1, 3])
def test_single_cluster_mean(iters):
    B, H, L, d = 2, 2, 19, 64
    q, k, v = (_rand((B, H, L, d), s) for s in (13, 14, 15))
    out, assign, cent, _ = oracle.forward(q, k, v, K=1, iters=iters, W=4, alpha=0.0, mu_f32=False)
    mean = q.mean(axis=2, keepdims=True)
    ref = _sdpa(np.broadcast_to(mean, q.shape).copy(), k, v)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(cent[:, :, 0, :], mean[:, :, 0, :], rtol=0, atol=1e-14)
    assert (assign == 0).all()


# In the default mode the stored centroid is the fp32 rounding of the mean.
def test_centroids_rounded_to_fp32():
    q = _f32(_rand((1, 1, 40, 64), 16))
    _, _, cent, _ = oracle.forward(q, q, q, K=1, iters=2, W=4, alpha=0.5, mu_f32=True)
    ref = q[0, 0].mean(axis=0).astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(cent[0, 0, 0], ref)


# --------------------------------------------------------------------------
# The expanded distance |Q|^2 + |mu|^2 - 2 Q.mu equals scipy's squared
# Euclidean distance.  Catches a sign error in the cross term or a missing
# square.
def test_distance_matches_scipy():
    from scipy.spatial.distance import cdist
    q = _rand((50, 64), 17)
    mu = _rand((9, 64), 18)
    D = oracle.distances(q, mu)
    np.testing.assert_allclose(D, cdist(q, mu, "sqeuclidean"), rtol=1e-12, atol=1e-10)


# --------------------------------------------------------------------------
# Lloyd's objective never increases: J(t) = sum_i |Q_i - mu^(t)_{c_i^(t)}|^2
# and the assignment step cannot raise it either.  Catches argmax instead of
# argmin and any update that is not the member mean.
def test_lloyd_objective_monotone():
    q = _rand((300, 64), 19)
    T, K = 8, 12
    J_prev = None
    mu_prev = np.stack([q[(k * 300) // K] for k in range(K)])
    for t in range(1, T + 1):
        c, mu, hist = oracle.kmeans(q, K, t, mu_f32=False)
        J_assign = float(np.sum((q - mu_prev[c]) ** 2))
        J = float(np.sum((q - mu[c]) ** 2))
        assert J <= J_assign + 1e-9
        if J_prev is not None:
            assert J_assign <= J_prev + 1e-9
        J_prev, mu_prev = J, mu


# --------------------------------------------------------------------------
# scikit-learn's Lloyd k-means from the same starting centroids: its centres
# after I iterations are mu^(I); its labels are taken against those centres,
# i.e. our assignment of iteration I+1.  Well-separated data keeps every
# cluster non-empty (scikit-learn relocates empty clusters, the cards zero
# them).
@pytest.mark.parametrize("iters", [1, 2, 4])
def test_matches_sklearn_lloyd(iters):
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(20)
    K, L, d = 6, 240, 64
    means = rng.standard_normal((K, d)) * 4.0
    lab = np.arange(L) % K
    rng.shuffle(lab)
    q = means[lab] + 0.3 * rng.standard_normal((L, d))
    init = np.stack([q[(k * L) // K] for k in range(K)])
    c, mu, hist = oracle.kmeans(q, K, iters + 1, mu_f32=False)
    c_i, mu_i, _ = oracle.kmeans(q, K, iters, mu_f32=False)
    for t in range(iters + 1):
        assert np.bincount(hist[t], minlength=K).min() > 0
    km = KMeans(n_clusters=K, init=init, n_init=1, max_iter=iters, tol=0.0, algorithm="lloyd")
    km.fit(q)
    np.testing.assert_allclose(mu_i, km.cluster_centers_, rtol=0, atol=1e-10)
    np.testing.assert_array_equal(hist[iters], km.labels_)


# --------------------------------------------------------------------------
# Theorem 1 of both cards: |A_dense(Q_i) - V_cent[c_i]| <= 2 kappa nu / sqrt(d)
# |Q_i - mu_{c_i}|, with kappa, nu the largest key and value norms.
@pytest.mark.parametrize("K", [1, 4, 16])
def test_theorem1_bound(K):
    B, H, L, d = 1, 2, 64, 64
    q, k, v = (_rand((B, H, L, d), s, 0.5) for s in (21, 22, 23))
    out, assign, cent, _ = oracle.forward(q, k, v, K=K, iters=3, W=4, alpha=0.0, mu_f32=False)
    dense = _sdpa(q, k, v)
    for h in range(H):
        kappa = np.linalg.norm(k[0, h], axis=1).max()
        nu = np.linalg.norm(v[0, h], axis=1).max()
        err = np.linalg.norm(dense[0, h] - out[0, h], axis=1)
        gap = np.linalg.norm(q[0, h] - cent[0, h][assign[0, h]], axis=1)
        assert (err <= 2 * kappa * nu / math.sqrt(d) * gap + 1e-12).all()


# --------------------------------------------------------------------------
# Softmax shift invariance: adding one vector to every key adds a per-query
# constant to every logit of that row, which the softmax ignores, in both
# branches.  Catches logits that depend on anything but Q.K (e.g. |K|^2).
def test_key_shift_invariance():
    q, k, v = (_rand((1, 2, 30, 64), s) for s in (24, 25, 26))
    shift = _rand((1, 1, 1, 64), 27)
    a, *_ = oracle.forward(q, k, v, K=5, iters=2, W=6, alpha=0.4)
    b, *_ = oracle.forward(q, k + shift, v, K=5, iters=2, W=6, alpha=0.4)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


# Linearity in V (assignments depend on Q only): catches V entering a
# non-linear step or being mixed with K.
def test_linear_in_v():
    q, k, v1, v2 = (_rand((1, 2, 30, 64), s) for s in (28, 29, 30, 31))
    a, *_ = oracle.forward(q, k, v1, K=5, iters=2, W=6, alpha=0.3)
    b, *_ = oracle.forward(q, k, v2, K=5, iters=2, W=6, alpha=0.3)
    c, *_ = oracle.forward(q, k, 2.0 * v1 - 3.0 * v2, K=5, iters=2, W=6, alpha=0.3)
    np.testing.assert_allclose(c, 2.0 * a - 3.0 * b, rtol=0, atol=1e-11)


# Convex fusion is affine in alpha: O(a) = (1-a) O(0) + a O(1).
def test_affine_in_alpha():
    q, k, v = (_rand((1, 2, 30, 64), s) for s in (32, 33, 34))
    o0, *_ = oracle.forward(q, k, v, K=5, iters=2, W=6, alpha=0.0)
    o1, *_ = oracle.forward(q, k, v, K=5, iters=2, W=6, alpha=1.0)
    for a in (0.25, 0.5, 0.7):
        oa, *_ = oracle.forward(q, k, v, K=5, iters=2, W=6, alpha=a)
        np.testing.assert_allclose(oa, (1 - a) * o0 + a * o1, rtol=0, atol=1e-12)


# At alpha = 0 tokens of one cluster get the identical output row.
def test_rows_equal_within_cluster():
    q, k, v = (_rand((1, 1, 40, 64), s) for s in (35, 36, 37))
    out, assign, *_ = oracle.forward(q, k, v, K=4, iters=3, W=6, alpha=0.0)
    for c in np.unique(assign):
        rows = out[0, 0][assign[0, 0] == c]
        assert (rows == rows[0]).all()


# iters = 0: every token is in cluster 0 and the centroids stay at init.
def test_zero_iterations():
    q, k, v = (_f32(_rand((1, 1, 12, 64), s)) for s in (38, 39, 40))
    out, assign, cent, _ = oracle.forward(q, k, v, K=3, iters=0, W=4, alpha=0.0)
    assert (assign == 0).all()
    np.testing.assert_array_equal(cent[0, 0], q[0, 0][[0, 4, 8]])
    ref = _sdpa(np.broadcast_to(q[:, :, :1], q.shape).copy(), k, v)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# Init index floor(k L / K) when K does not divide L.
def test_init_index_non_dividing():
    L, K = 10, 4  # floor(k*10/4) = 0, 2, 5, 7
    q = _f32(_rand((1, 1, L, 64), 41))
    _, _, cent, _ = oracle.forward(q, q, q, K=K, iters=0, W=2, alpha=0.5)
    np.testing.assert_array_equal(cent[0, 0], q[0, 0][[0, 2, 5, 7]])


# --------------------------------------------------------------------------
# Hand-derived worked examples.
def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _pad64(a):
    a = np.asarray(a, dtype=np.float64)
    out = np.zeros(a.shape[:-1] + (64,))
    out[..., : a.shape[-1]] = a
    return out


def test_golden_kmeans_two_blobs():
    g = _golden()["kmeans_two_blobs"]
    q = np.asarray(g["Q"], dtype=np.float64)
    c, mu, _ = oracle.kmeans(q, g["K"], g["iters"], mu_f32=False)
    np.testing.assert_array_equal(c, g["assign"])
    np.testing.assert_allclose(mu, np.asarray(g["centroids_num"]) / g["centroids_den"], rtol=0, atol=1e-15)
    c32, mu32, _ = oracle.kmeans(q, g["K"], g["iters"], mu_f32=True)
    np.testing.assert_array_equal(mu32, (np.asarray(g["centroids_num"]) / g["centroids_den"]).astype(np.float32))


def test_golden_tie_and_empty():
    g = _golden()["kmeans_tie_and_empty"]
    q = np.asarray(g["Q"], dtype=np.float64)
    c, mu, _ = oracle.kmeans(q, g["K"], g["iters"])
    np.testing.assert_array_equal(c, g["assign"])
    np.testing.assert_array_equal(mu, np.asarray(g["centroids"], dtype=np.float64))


def test_golden_centroid_attention():
    g = _golden()
    e = g["centroid_attention_equal_keys"]
    out = oracle.centroid_attention(_pad64(e["mu"]), _pad64(e["Kmat"]), _pad64(e["V"]))
    np.testing.assert_allclose(out, _pad64(e["vcent"]), rtol=0, atol=1e-14)
    t = g["centroid_attention_two_keys"]
    mu = np.array([[2.0 * math.log(3.0), 0, 0, 0]])
    out = oracle.centroid_attention(mu, np.asarray(t["Kmat"], float), np.asarray(t["V"], float))
    np.testing.assert_allclose(out, np.asarray(t["vcent"], float), rtol=0, atol=1e-13)


def test_golden_window_uniform():
    g = _golden()["window_uniform"]
    L = g["L"]
    v = _pad64(g["V"])
    q = np.zeros((L, 64))
    k = _rand((L, 64), 42)
    out = oracle.window_attention(q, k, v, g["W"])
    np.testing.assert_allclose(out, _pad64(g["out"]), rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# Cross-check of the C code against the literal NumPy restatement on tiny
# inputs, every K from 1 to L (a check of the C indexing, not a pin).
@pytest.mark.parametrize("L", [1, 2, 3, 7, 12])
def test_c_matches_literal_numpy(L):
    d = 64
    for K in range(1, L + 1):
        q, k, v = (_f32(_rand((1, 1, L, d), 100 + L * 17 + K + s)) for s in (0, 1, 2))
        out, assign, cent, _ = oracle.forward(q, k, v, K=K, iters=3, W=3, alpha=0.6)
        o2, c2, mu2 = oracle_np.forward_head(q[0, 0], k[0, 0], v[0, 0], K, 3, 3, 0.6)
        np.testing.assert_array_equal(assign[0, 0], c2)
        np.testing.assert_array_equal(cent[0, 0], mu2)
        np.testing.assert_allclose(out[0, 0], o2, rtol=0, atol=1e-12)


# forward_at with the oracle's own assignments reproduces the forward.
def test_forward_at_consistent():
    q, k, v = (_f32(_rand((2, 2, 50, 64), s)) for s in (43, 44, 45))
    out, assign, cent, _ = oracle.forward(q, k, v, K=7, iters=3, W=10, alpha=0.35)
    o2, c2 = oracle.forward_at(q, k, v, assign, K=7, iters=3, W=10, alpha=0.35)
    np.testing.assert_array_equal(out, o2)
    np.testing.assert_array_equal(cent, c2)


def test_invalid_arguments_rejected():
    q = np.zeros((1, 1, 4, 64))
    with pytest.raises(ValueError):
        oracle.forward(q, q, q, K=5, iters=1, W=2, alpha=0.5)  # K > L
    with pytest.raises(ValueError):
        oracle.forward(q, q, q, K=2, iters=1, W=2, alpha=1.5)


# --------------------------------------------------------------------------
# Variants of the card's module ([P2] section 5).

# With everything off, the extended form is the plain forward.
def test_ex_defaults_equal_plain():
    q, k, v = (_f32(_rand((2, 3, 40, 64), s)) for s in (50, 51, 52))
    a = oracle.forward(q, k, v, K=6, iters=3, W=10, alpha=0.4, hist=True)
    b = oracle.forward_ex(q, k, v, K=6, iters=3, W=10, alpha=0.4, hist=True)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# The module's window is the radius W; at alpha = 1 it is band-masked SDPA
# with |i - j| <= W.  With W == 0 or W >= L it drops the local branch, so
# the output is the gathered global context at any alpha.
@pytest.mark.parametrize("W", [1, 5, 17])
def test_ex_module_window_radius(W):
    L = 30
    q, k, v = (_rand((1, 2, L, 64), s) for s in (53, 54, 55))
    out, *_ = oracle.forward_ex(q, k, v, K=4, iters=2, W=W, alpha=1.0, window_module=True)
    idx = np.arange(L)
    ref = _sdpa(q, k, v, mask=np.abs(idx[:, None] - idx[None, :]) <= W)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("W", [0, 30, 64])
def test_ex_module_window_skipped(W):
    q, k, v = (_rand((1, 2, 30, 64), s) for s in (56, 57, 58))
    out, *_ = oracle.forward_ex(q, k, v, K=4, iters=2, W=W, alpha=0.7, window_module=True)
    g, *_ = oracle.forward_ex(q, k, v, K=4, iters=2, W=3, alpha=0.0, window_module=True)
    np.testing.assert_allclose(out, g, rtol=0, atol=1e-14)


# The module's stride init: rows k * (L // K) (L=10, K=4 -> 0, 2, 4, 6).
def test_ex_init_stride():
    q = _f32(_rand((1, 1, 10, 64), 59))
    _, _, cent, _ = oracle.forward_ex(q, q, q, K=4, iters=0, W=2, alpha=0.5, init_stride=True)
    np.testing.assert_array_equal(cent[0, 0], q[0, 0][[0, 2, 4, 6]])


# Empty cluster keeps its previous centroid (worked example: the tie case of
# tests/golden, where cluster 1 is empty after one step and keeps (1, 0)).
def test_ex_empty_keep_golden():
    g = _golden()["kmeans_tie_and_empty"]
    q = _pad64(np.asarray(g["Q"], dtype=np.float64))[None, None]
    _, assign, cent, _ = oracle.forward_ex(q, q, q, K=2, iters=1, W=2, alpha=0.5, empty_keep=True)
    np.testing.assert_array_equal(assign[0, 0], g["assign"])
    np.testing.assert_array_equal(cent[0, 0, 0, :2], g["centroids"][0])
    np.testing.assert_array_equal(cent[0, 0, 1, :2], [1.0, 0.0])


# Soft gather: g_i = softmax(Q_i mu^T / sqrt(d)) V_cent and V_cent =
# softmax(mu K^T / sqrt(d)) V, i.e. two nested SDPA calls on the oracle's
# own centroids.
def test_ex_soft_gather_is_nested_sdpa():
    q, k, v = (_f32(_rand((1, 2, 36, 64), s)) for s in (60, 61, 62))
    out, assign, cent, _ = oracle.forward_ex(q, k, v, K=5, iters=3, W=6, alpha=0.0, soft_gather=True)
    vcent = _sdpa(cent, k, v)
    ref = _sdpa(q, cent, vcent)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# Key-padding mask: invalid keys take no weight in either branch and rows of
# invalid queries are zero.  At alpha = 1 the valid rows equal band-masked
# SDPA restricted to valid keys; at alpha = 0 with K = L they equal dense
# SDPA restricted to valid keys.
def test_ex_key_padding_mask():
    B, H, L = 2, 2, 24
    q, k, v = (_f32(_rand((B, H, L, 64), s)) for s in (63, 64, 65))
    valid = np.ones((B, L), dtype=bool)
    valid[0, 17:] = False
    valid[1, [0, 5, 6, 23]] = False
    idx = np.arange(L)
    band = np.abs(idx[:, None] - idx[None, :]) <= 4
    out1, *_ = oracle.forward_ex(q, k, v, K=3, iters=2, W=8, alpha=1.0, key_valid=valid)
    out0, *_ = oracle.forward_ex(q, k, v, K=L, iters=2, W=8, alpha=0.0, key_valid=valid)
    for b in range(B):
        m1 = band & valid[b][None, :]
        m0 = np.broadcast_to(valid[b][None, :], (L, L))
        r1 = _sdpa(q[b:b + 1], k[b:b + 1], v[b:b + 1], mask=np.ascontiguousarray(m1))
        r0 = _sdpa(q[b:b + 1], k[b:b + 1], v[b:b + 1], mask=np.ascontiguousarray(m0))
        rows = valid[b]
        np.testing.assert_allclose(out1[b][:, rows], r1[0][:, rows], rtol=0, atol=1e-12)
        np.testing.assert_allclose(out0[b][:, rows], r0[0][:, rows], rtol=0, atol=1e-12)
        assert (out1[b][:, ~rows] == 0).all() and (out0[b][:, ~rows] == 0).all()


# Grouped key/value heads equal the plain forward on K, V repeated per group
# (torch repeat_interleave along the head axis).
def test_ex_grouped_kv_heads():
    B, H, Hkv, L = 2, 6, 2, 20
    q = _f32(_rand((B, H, L, 64), 66))
    k, v = (_f32(_rand((B, Hkv, L, 64), s)) for s in (67, 68))
    out, assign, cent, _ = oracle.forward_ex(q, k, v, K=4, iters=2, W=6, alpha=0.5, H_kv=Hkv)
    kr = torch.from_numpy(k).repeat_interleave(H // Hkv, dim=1).numpy()
    vr = torch.from_numpy(v).repeat_interleave(H // Hkv, dim=1).numpy()
    ref, ref_a, ref_c, _ = oracle.forward(q, kr, vr, K=4, iters=2, W=6, alpha=0.5)
    np.testing.assert_array_equal(out, ref)
    np.testing.assert_array_equal(assign, ref_a)


@pytest.mark.parametrize("name", ["card_gmm_f32", "l4k_gmm_bf16"])
def test_fp32_stored_centroids_decide_like_plain_fp64(name):
    """Reading of the precision of the decision: the oracle stores each
    centroid rounded once to fp32 (as the module of "Hooshaai/svd-sst2-
    roberta-cluster" section 5 casts its centroids to float before measuring
    distances).  On the well-separated Gaussian-mixture workloads, where the
    assignments must match bit for bit, that rounding must not change a single
    assignment at any Lloyd iteration compared with the pages' plain fp64
    formulas (Mathematical Formulation section 1 of "Hooshaai/distilbert-
    sst2-cluster-attention"), so bit-exactness there rests on the pages and
    not on this reading."""
    from means_cluster_attention_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS[name]
    x = make_inputs(w)
    a32 = oracle.forward(x["q64"], x["k64"], x["v64"], K=w.K, iters=w.iters, W=w.W, alpha=w.alpha,
                         mu_f32=True, hist=True)
    a64 = oracle.forward(x["q64"], x["k64"], x["v64"], K=w.K, iters=w.iters, W=w.W, alpha=w.alpha,
                         mu_f32=False, hist=True)
    np.testing.assert_array_equal(a32[3], a64[3])
    np.testing.assert_array_equal(a32[1], a64[1])
    # the stored centroids differ from the fp64 ones only by that one rounding
    np.testing.assert_allclose(a32[2], a64[2], rtol=2 ** -24, atol=0)
