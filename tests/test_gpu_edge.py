"""GPU edge cases against the oracle: ragged and tiny sequence lengths, K at
1, at L and at its maximum, zero iterations, zero and very wide windows,
alpha at both ends, both dtypes; plus determinism, the host-buffer entry
point, and device status after a clean run."""

import numpy as np
import pytest

import oracle
from means_cluster_attention_b200.inputs import Workload, make_inputs
from helpers import TOL, run_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # L, K, iters, W, alpha, B, H
    (1, 1, 3, 32, 0.5, 1, 2),
    (2, 2, 1, 0, 0.5, 1, 1),
    (63, 7, 4, 1, 0.25, 2, 3),
    (65, 65, 2, 33, 0.0, 1, 2),
    (100, 1, 3, 400, 1.0, 2, 1),
    (129, 128, 3, 16, 0.7, 1, 1),
    (1000, 13, 0, 32, 0.5, 1, 2),
    (1025, 100, 2, 64, 0.3, 1, 2),
    (2049, 32, 3, 129, 0.6, 1, 1),
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L,K,iters,W,alpha,B,H", CASES)
def test_edge_case_parity(dtype, L, K, iters, W, alpha, B, H):
    w = Workload("edge", B, H, L, 64, K, iters, W, alpha, dtype, "normal")
    x = make_inputs(w, seed=L * 31 + K)
    g = run_gpu(x, dtype, K, iters, W, alpha, hist=iters > 0)
    ref_out, ref_assign, ref_cent, ref_hist = oracle.forward(
        x["q64"], x["k64"], x["v64"], K=K, iters=iters, W=W, alpha=alpha, hist=True)
    np.testing.assert_array_equal(g["assign"], ref_assign)
    if iters > 0:
        np.testing.assert_array_equal(g["hist"], ref_hist)
    np.testing.assert_array_equal(g["cent"], ref_cent)
    err = float(np.abs(g["out"] - ref_out).max())
    assert err <= TOL[dtype], err


def test_gmm_with_tiny_clusters_and_exact_ties():
    # Mixture data with more clusters than components: duplicated centroids,
    # empty clusters and zero centroids all appear.
    w = Workload("gmm_edge", 2, 4, 300, 64, 40, 4, 32, 0.5, "bf16", "gmm", gmm_components=8,
                 gmm_std=0.05)
    x = make_inputs(w, seed=5)
    g = run_gpu(x, "bf16", w.K, w.iters, w.W, w.alpha, hist=True)
    _, ref_assign, ref_cent, ref_hist = oracle.forward(x["q64"], x["k64"], x["v64"], K=w.K,
                                                      iters=w.iters, W=w.W, alpha=w.alpha, hist=True)
    np.testing.assert_array_equal(g["hist"], ref_hist)
    np.testing.assert_array_equal(g["cent"], ref_cent)


@pytest.mark.parametrize("L,K,profile_kernel", [(512, 64, "fused_forward"), (1500, 64, "tiled_assign")])
def test_three_distinct_queries(L, K, profile_kernel):
    # Every query is one of three rows: all but three strided starting centroids
    # are bitwise copies of a lower one, most clusters end empty (zero
    # centroids, themselves copies of each other) and all distances tie.
    from means_cluster_attention_b200 import _lib
    w = Workload("three_rows", 1, 2, L, 64, K, 3, 32, 0.5, "bf16", "normal")
    x = make_inputs(w, seed=L + K)
    src = np.random.default_rng(L).integers(0, 3, size=L)
    for key in ("q", "q64"):
        x[key] = np.ascontiguousarray(x[key][:, :, src, :])
    _lib.profile_start(profile_kernel)
    g = run_gpu(x, "bf16", K, w.iters, w.W, w.alpha, hist=True)
    stat = _lib.profile_stop()
    assert stat.launches > 0, f"{profile_kernel} did not run"
    ref_out, ref_assign, ref_cent, ref_hist = oracle.forward(x["q64"], x["k64"], x["v64"], K=K, iters=w.iters,
                                                             W=w.W, alpha=w.alpha, hist=True)
    np.testing.assert_array_equal(g["hist"], ref_hist)
    np.testing.assert_array_equal(g["cent"], ref_cent)
    assert float(np.abs(g["out"] - ref_out).max()) <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_deterministic(dtype):
    import torch
    import means_cluster_attention_b200 as ca
    from helpers import to_device
    w = Workload("det", 2, 4, 3000, 64, 24, 3, 40, 0.5, dtype, "normal")
    x = make_inputs(w, seed=11)
    q, k, v = to_device(x, dtype)
    o1, a1, c1 = ca.forward(q, k, v, w.K, w.iters, w.W, w.alpha)
    o2, a2, c2 = ca.forward(q, k, v, w.K, w.iters, w.W, w.alpha)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(a1, a2) and torch.equal(c1, c2)
    ca.sync_status()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_host_entry_point_matches_device_path(dtype):
    import torch
    import means_cluster_attention_b200 as ca
    from helpers import to_device
    w = Workload("host", 2, 3, 777, 64, 16, 3, 32, 0.5, dtype, "normal")
    x = make_inputs(w, seed=3)
    q, k, v = to_device(x, dtype)
    o_dev, a_dev, c_dev = ca.forward(q, k, v, w.K, w.iters, w.W, w.alpha, sync_check=True)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    o_h = torch.empty_like(qh).pin_memory()
    a_h = torch.empty((2, 3, 777), dtype=torch.int32).pin_memory()
    c_h = torch.empty((2, 3, 16, 64), dtype=torch.float32).pin_memory()
    ca.forward_host(qh, kh, vh, w.K, w.iters, w.W, w.alpha, out=o_h, assign=a_h, centroids=c_h)
    assert torch.equal(o_h, o_dev.cpu())
    assert torch.equal(a_h, a_dev.cpu())
    assert torch.equal(c_h, c_dev.cpu())


@pytest.mark.parametrize("dtype,B,H,L,K,W", [
    ("bf16", 10, 13, 512, 16, 32),   # fused kernel, 130 heads in uneven chunks
    ("bf16", 2, 8, 4096, 32, 64),    # tiled path, two heads per chunk
    ("f32", 8, 8, 512, 16, 32),      # general path
])
def test_host_entry_point_in_chunks_matches_device_path(dtype, B, H, L, K, W):
    # Large enough (>= 32 MB of q, k, v, out) for the host entry point to copy
    # in, compute and copy back in chunks of whole heads on three streams.
    import torch
    import means_cluster_attention_b200 as ca
    from helpers import to_device
    w = Workload("host_chunks", B, H, L, 64, K, 3, W, 0.5, dtype, "normal")
    x = make_inputs(w, seed=11)
    q, k, v = to_device(x, dtype)
    o_dev, a_dev, c_dev = ca.forward(q, k, v, w.K, w.iters, w.W, w.alpha, sync_check=True)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    o_h = torch.empty_like(qh).pin_memory()
    a_h = torch.empty((B, H, L), dtype=torch.int32).pin_memory()
    c_h = torch.empty((B, H, K, 64), dtype=torch.float32).pin_memory()
    ca.forward_host(qh, kh, vh, w.K, w.iters, w.W, w.alpha, out=o_h, assign=a_h, centroids=c_h)
    ca.sync_status()
    assert torch.equal(o_h, o_dev.cpu())
    assert torch.equal(a_h, a_dev.cpu())
    assert torch.equal(c_h, c_dev.cpu())


def test_invalid_call_launches_nothing_and_status_stays_clean():
    import torch
    import means_cluster_attention_b200 as ca
    q = torch.zeros((1, 1, 8, 64), device="cuda")
    with pytest.raises(ca.ClusterAttnError):
        ca.forward(q, q, q, 4, -1, 4, 0.5)
    ca.sync_status()


# Shapes served by the fused one-CTA-per-head kernel (bf16, L <= 512, K <= 64,
# floor(W/2) <= 16): ragged lengths, K at the 16/32/64 padding boundaries,
# windows at the radius limit.
FUSED_CASES = [
    # L, K, iters, W, alpha, B, H
    (1, 1, 2, 32, 0.5, 1, 3),
    (17, 5, 3, 33, 0.4, 2, 2),
    (64, 16, 0, 2, 0.5, 1, 2),
    (100, 17, 5, 31, 0.9, 1, 2),
    (255, 33, 3, 32, 0.5, 2, 1),
    (256, 64, 3, 16, 0.1, 1, 2),
    (300, 48, 2, 1, 0.5, 1, 2),
    (511, 16, 4, 32, 0.5, 2, 2),
    (512, 64, 5, 33, 0.5, 1, 3),
]


@pytest.mark.parametrize("L,K,iters,W,alpha,B,H", FUSED_CASES)
def test_fused_path_parity(L, K, iters, W, alpha, B, H):
    from means_cluster_attention_b200 import _lib
    w = Workload("fused", B, H, L, 64, K, iters, W, alpha, "bf16", "normal")
    x = make_inputs(w, seed=L * 7 + K)
    _lib.profile_start("fused_forward")
    g = run_gpu(x, "bf16", K, iters, W, alpha, hist=iters > 0)
    stat = _lib.profile_stop()
    assert stat.launches == 1, "the fused kernel did not run"
    ref_out, ref_assign, ref_cent, ref_hist = oracle.forward(
        x["q64"], x["k64"], x["v64"], K=K, iters=iters, W=W, alpha=alpha, hist=True)
    if iters > 0:
        np.testing.assert_array_equal(g["hist"], ref_hist)
    np.testing.assert_array_equal(g["assign"], ref_assign)
    np.testing.assert_array_equal(g["cent"], ref_cent)
    err = float(np.abs(g["out"] - ref_out).max())
    assert err <= TOL["bf16"], err


def test_fused_gmm_forced_ties():
    # Mixture data plus duplicated rows at the strided start positions: exact
    # ties, empty and zero centroids inside the fused kernel.
    from means_cluster_attention_b200 import _lib
    w = Workload("fused_dup", 2, 3, 400, 64, 40, 4, 32, 0.5, "bf16", "gmm", gmm_components=6,
                 gmm_std=0.05, dup_frac=0.1)
    x = make_inputs(w, seed=9)
    _lib.profile_start("fused_forward")
    g = run_gpu(x, "bf16", w.K, w.iters, w.W, w.alpha, hist=True)
    assert _lib.profile_stop().launches == 1
    _, ref_assign, ref_cent, ref_hist = oracle.forward(x["q64"], x["k64"], x["v64"], K=w.K,
                                                      iters=w.iters, W=w.W, alpha=w.alpha, hist=True)
    np.testing.assert_array_equal(g["hist"], ref_hist)
    np.testing.assert_array_equal(g["cent"], ref_cent)


# Shapes served by the tiled bf16 path (L > 512 or floor(W/2) > 16, K <= 64,
# floor(W/2) <= 128): tile and chunk tails, K at the padding boundaries,
# windows wider than a tile.
TILED_CASES = [
    # L, K, iters, W, alpha, B, H
    (513, 1, 2, 32, 0.5, 1, 2),
    (1000, 17, 3, 0, 0.4, 1, 2),
    (1537, 33, 1, 65, 0.3, 1, 1),
    (2048, 64, 4, 129, 0.6, 1, 1),
    (300, 16, 3, 100, 0.5, 2, 1),
    (4095, 32, 0, 256, 0.5, 1, 1),
]


@pytest.mark.parametrize("L,K,iters,W,alpha,B,H", TILED_CASES)
def test_tiled_path_parity(L, K, iters, W, alpha, B, H):
    from means_cluster_attention_b200 import _lib
    w = Workload("tiled", B, H, L, 64, K, iters, W, alpha, "bf16", "normal")
    x = make_inputs(w, seed=L + 3 * K)
    _lib.profile_start("tiled_window")
    g = run_gpu(x, "bf16", K, iters, W, alpha, hist=iters > 0)
    assert _lib.profile_stop().launches == 1, "the tiled path did not run"
    ref_out, ref_assign, ref_cent, ref_hist = oracle.forward(
        x["q64"], x["k64"], x["v64"], K=K, iters=iters, W=W, alpha=alpha, hist=True)
    if iters > 0:
        np.testing.assert_array_equal(g["hist"], ref_hist)
    np.testing.assert_array_equal(g["assign"], ref_assign)
    np.testing.assert_array_equal(g["cent"], ref_cent)
    err = float(np.abs(g["out"] - ref_out).max())
    assert err <= TOL["bf16"], err


def test_tiled_forced_ties_across_tiles():
    from means_cluster_attention_b200 import _lib
    w = Workload("tiled_dup", 1, 2, 2500, 64, 48, 4, 64, 0.5, "bf16", "gmm", gmm_components=10,
                 gmm_std=0.05, dup_frac=0.1)
    x = make_inputs(w, seed=21)
    _lib.profile_start("tiled_assign")
    g = run_gpu(x, "bf16", w.K, w.iters, w.W, w.alpha, hist=True)
    assert _lib.profile_stop().launches == w.iters
    _, ref_assign, ref_cent, ref_hist = oracle.forward(x["q64"], x["k64"], x["v64"], K=w.K,
                                                      iters=w.iters, W=w.W, alpha=w.alpha, hist=True)
    np.testing.assert_array_equal(g["hist"], ref_hist)
    np.testing.assert_array_equal(g["cent"], ref_cent)


# Window radii around the tensor-core window kernel's key windows (radius
# <= 32 and <= 64) and the mma.sync kernel beyond, with a ragged last block;
# alpha = 1 leaves only the window branch in the output.
@pytest.mark.parametrize("W", [2, 62, 63, 64, 66, 127, 128, 129, 130])
def test_tiled_window_radius_boundaries(W):
    w = Workload("tiled_win", 1, 2, 700, 64, 8, 1, W, 1.0, "bf16", "normal")
    x = make_inputs(w, seed=W)
    g = run_gpu(x, "bf16", w.K, w.iters, w.W, w.alpha)
    ref_out, _, _, _ = oracle.forward(x["q64"], x["k64"], x["v64"], K=w.K, iters=w.iters, W=w.W, alpha=w.alpha)
    err = float(np.abs(g["out"] - ref_out).max())
    assert err <= TOL["bf16"], f"W={W}: {err}"


def test_tiled_exact_ties_between_distinct_centroids():
    """Strided starting centroids e1, -e1, 3e3, -3e3 and tokens e2 or 0:
    every token is exactly equidistant from the first two centroids, so the
    exact decision cannot be certified from rounded distances and must fall
    back to the index-order comparison, where the lower index wins."""
    from means_cluster_attention_b200.inputs import bf16_bits_to_f64, bf16_round_bits
    L, K = 600, 4
    q = np.zeros((1, 1, L, 64), dtype=np.float32)
    q[0, 0, 1::2, 1] = 1.0                      # e2 on odd positions, 0 on even ones
    rows = [(k * L) // K for k in range(K)]
    for r_, (dim, val) in zip(rows, [(0, 1.0), (0, -1.0), (2, 3.0), (2, -3.0)]):
        q[0, 0, r_, :] = 0.0
        q[0, 0, r_, dim] = val
    rng = np.random.default_rng(5)
    x = {}
    for name, a in (("q", q), ("k", rng.standard_normal(q.shape, dtype=np.float32)),
                    ("v", rng.standard_normal(q.shape, dtype=np.float32))):
        x[name] = bf16_round_bits(a)
        x[name + "64"] = bf16_bits_to_f64(x[name])
    g = run_gpu(x, "bf16", K, 1, 8, 0.5, hist=True)
    _, ref_assign, ref_cent, ref_hist = oracle.forward(x["q64"], x["k64"], x["v64"], K=K, iters=1, W=8,
                                                      alpha=0.5, hist=True)
    np.testing.assert_array_equal(g["hist"], ref_hist)
    np.testing.assert_array_equal(g["assign"], ref_assign)
    np.testing.assert_array_equal(g["cent"], ref_cent)
    tokens = [i for i in range(L) if i not in rows]
    assert (ref_assign[0, 0, tokens] == 0).all()


def test_tiled_many_movers_two_batches():
    """More than 256 tokens of one 512-query tile change cluster in one
    iteration, so the tile's running-sum update runs in two batches of signed
    entries.  Rows 0 and 512 (the strided starting centroids for K = 2) are
    the same near-zero row: centroid 1 starts as a copy and takes nothing, so
    the first update leaves it empty (the zero vector) while centroid 0 moves
    to the mean of all rows; in the second iteration the 300 near-zero rows
    of the first tile move to centroid 1."""
    from means_cluster_attention_b200 import _lib
    from means_cluster_attention_b200.inputs import bf16_bits_to_f64, bf16_round_bits
    L, K, iters = 1024, 2, 3
    rng = np.random.default_rng(11)
    q = np.zeros((1, 1, L, 64), dtype=np.float32)
    q[0, 0, :300] = 0.01 * rng.standard_normal((300, 64), dtype=np.float32)
    q[0, 0, 300:] = 0.1 * rng.standard_normal((L - 300, 64), dtype=np.float32)
    q[0, 0, 300:, 0] += 10.0
    q[0, 0, 512] = q[0, 0, 0]
    x = {}
    for name, a in (("q", q), ("k", rng.standard_normal(q.shape, dtype=np.float32)),
                    ("v", rng.standard_normal(q.shape, dtype=np.float32))):
        x[name] = bf16_round_bits(a)
        x[name + "64"] = bf16_bits_to_f64(x[name])
    _lib.profile_start("tiled_assign")
    g = run_gpu(x, "bf16", K, iters, 8, 0.5, hist=True)
    assert _lib.profile_stop().launches == iters
    ref_out, ref_assign, ref_cent, ref_hist = oracle.forward(x["q64"], x["k64"], x["v64"], K=K, iters=iters,
                                                             W=8, alpha=0.5, hist=True)
    moved_in_tile0 = int((ref_hist[0, 0, 1, :512] != ref_hist[0, 0, 0, :512]).sum())
    assert moved_in_tile0 > 256, moved_in_tile0
    np.testing.assert_array_equal(g["hist"], ref_hist)
    np.testing.assert_array_equal(g["assign"], ref_assign)
    np.testing.assert_array_equal(g["cent"], ref_cent)
    assert float(np.abs(g["out"] - ref_out).max()) <= TOL["bf16"]
