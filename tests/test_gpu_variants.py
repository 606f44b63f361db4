"""GPU parity for the variants of the card's module (ca_forward_ex):
radius-W window with the skipped local branch, empty clusters keeping their
centroid, stride init, soft gather, key-padding masks and grouped key/value
heads — each against the oracle's extended forward on the same inputs."""

import numpy as np
import pytest

import oracle
from means_cluster_attention_b200.inputs import Workload, make_inputs
from helpers import TOL, out_to_f64, to_device

pytestmark = pytest.mark.gpu


def _case(dtype, B, H, L, K, iters, W, alpha, seed, H_kv=None, gmm=False):
    H_kv = H_kv or H
    wq = Workload("v", B, H, L, 64, K, iters, W, alpha, dtype, "gmm" if gmm else "normal",
                  gmm_components=5 if gmm else 0, gmm_std=0.05 if gmm else 0.0)
    xq = make_inputs(wq, seed=seed)
    wk = Workload("vkv", B, H_kv, L, 64, K, iters, W, alpha, dtype, "normal")
    xk = make_inputs(wk, seed=seed + 1000)
    return xq, xk


def _run(dtype, xq, xk, K, iters, W, alpha, key_valid=None, **modes):
    import torch
    import means_cluster_attention_b200 as ca
    q, _, _ = to_device(xq, dtype)
    _, k, v = to_device(xk, dtype)
    B, H, L, _ = q.shape
    hist = torch.full((B, H, max(iters, 1), L), -1, dtype=torch.int32, device="cuda")
    kv = None if key_valid is None else torch.from_numpy(key_valid.astype(np.uint8)).cuda()
    out, assign, cent = ca.forward_ex(q, k, v, K, iters, W, alpha, key_valid=kv, assign_hist=hist,
                                      sync_check=True, **modes)
    torch.cuda.synchronize()
    return (out_to_f64(out), assign.cpu().numpy(), cent.cpu().numpy().astype(np.float64),
            hist.cpu().numpy()[:, :, :iters])


def _check(dtype, xq, xk, K, iters, W, alpha, key_valid=None, H_kv=0, **modes):
    g_out, g_assign, g_cent, g_hist = _run(dtype, xq, xk, K, iters, W, alpha, key_valid=key_valid, **modes)
    ref_out, ref_assign, ref_cent, ref_hist = oracle.forward_ex(
        xq["q64"], xk["k64"], xk["v64"], K=K, iters=iters, W=W, alpha=alpha,
        window_module=bool(modes.get("window_mode")), empty_keep=bool(modes.get("empty_mode")),
        init_stride=bool(modes.get("init_mode")), soft_gather=bool(modes.get("gather_mode")),
        key_valid=key_valid, H_kv=H_kv, hist=True)
    if iters > 0:
        np.testing.assert_array_equal(g_hist, ref_hist)
    np.testing.assert_array_equal(g_assign, ref_assign)
    np.testing.assert_array_equal(g_cent, ref_cent)
    err = float(np.abs(g_out - ref_out).max())
    assert err <= TOL[dtype], err
    if key_valid is not None:
        B, H, L, _ = g_out.shape
        for b in range(B):
            assert (g_out[b][:, ~key_valid[b].astype(bool)] == 0).all()
    return err


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("W", [1, 7, 40, 300, 0])
def test_module_window(dtype, W):
    xq, xk = _case(dtype, 2, 2, 150, 9, 3, W, 0.6, seed=W + 1)
    _check(dtype, xq, xk, 9, 3, W, 0.6, window_mode=1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_empty_clusters_keep_centroid(dtype):
    # Mixture queries with more clusters than components leave clusters empty.
    xq, xk = _case(dtype, 2, 3, 200, 24, 4, 16, 0.5, seed=7, gmm=True)
    _check(dtype, xq, xk, 24, 4, 16, 0.5, empty_mode=1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L,K", [(100, 8), (97, 13), (64, 64)])
def test_stride_init(dtype, L, K):
    xq, xk = _case(dtype, 1, 2, L, K, 2, 10, 0.5, seed=L + K)
    _check(dtype, xq, xk, K, 2, 10, 0.5, init_mode=1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K", [1, 7, 32])
def test_soft_gather(dtype, K):
    xq, xk = _case(dtype, 2, 2, 130, K, 3, 20, 0.3, seed=K + 5)
    _check(dtype, xq, xk, K, 3, 20, 0.3, gather_mode=1)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_key_padding_mask(dtype):
    B, L = 3, 180
    xq, xk = _case(dtype, B, 2, L, 11, 3, 24, 0.5, seed=31)
    valid = np.ones((B, L), dtype=bool)
    valid[0, 150:] = False          # right padding
    valid[1, :37] = False           # left padding
    valid[2, ::5] = False           # scattered
    _check(dtype, xq, xk, 11, 3, 24, 0.5, key_valid=valid)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_grouped_kv_heads(dtype):
    xq, xk = _case(dtype, 2, 6, 120, 10, 3, 16, 0.5, seed=41, H_kv=2)
    _check(dtype, xq, xk, 10, 3, 16, 0.5, H_kv=2)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_all_variants_together(dtype):
    B, L = 2, 160
    xq, xk = _case(dtype, B, 4, L, 12, 3, 20, 0.4, seed=51, H_kv=2)
    valid = np.ones((B, L), dtype=bool)
    valid[1, 120:] = False
    _check(dtype, xq, xk, 12, 3, 20, 0.4, key_valid=valid, H_kv=2, window_mode=1, empty_mode=1,
           init_mode=1, gather_mode=1)


def test_default_options_take_the_fast_path():
    from means_cluster_attention_b200 import _lib
    xq, xk = _case("bf16", 1, 2, 256, 16, 3, 32, 0.5, seed=61)
    _lib.profile_start("fused_forward")
    _run("bf16", xq, xk, 16, 3, 32, 0.5)
    assert _lib.profile_stop().launches == 1


@pytest.mark.parametrize("modes,H_kv,W", [
    (dict(window_mode=1), 0, 60),                                # radius 60: tensor-core window
    (dict(window_mode=1), 0, 100),                               # radius 100: mma.sync window
    (dict(window_mode=1), 0, 5000),                              # W >= L: no local branch
    (dict(empty_mode=1), 0, 40),
    (dict(init_mode=1), 0, 40),
    ({}, 2, 40),                                                 # grouped key/value heads
    (dict(window_mode=1, empty_mode=1, init_mode=1), 2, 33),
])
def test_variants_on_the_tiled_kernels(modes, H_kv, W):
    # bf16 variants without key masks or the soft gather run the tiled
    # tensor-core kernels: several query tiles, key chunks and window blocks.
    from means_cluster_attention_b200 import _lib
    xq, xk = _case("bf16", 1, 4, 1500, 24, 3, W, 0.5, seed=71 + W, H_kv=H_kv or None,
                   gmm=bool(modes.get("empty_mode")))
    _lib.profile_start("tiled_assign")
    _check("bf16", xq, xk, 24, 3, W, 0.5, H_kv=H_kv, **modes)
    assert _lib.profile_stop().launches == 3, "the tiled path did not run"


@pytest.mark.parametrize("W,modes", [(40, {}), (128, {}), (30, dict(window_mode=1)), (5000, dict(window_mode=1))])
def test_key_padding_mask_on_the_tiled_kernels(W, modes):
    # Several key chunks and window blocks per head: right, left and scattered
    # padding, and one batch row with no valid key at all (every key then
    # weighs the same in both softmaxes, and every output row is zero).
    from means_cluster_attention_b200 import _lib
    B, L = 4, 1500
    xq, xk = _case("bf16", B, 2, L, 20, 3, W, 0.5, seed=91 + W)
    valid = np.ones((B, L), dtype=bool)
    valid[0, 1100:] = False
    valid[1, :613] = False
    valid[2, ::3] = False
    valid[3, :] = False
    _lib.profile_start("tiled_assign")
    _check("bf16", xq, xk, 20, 3, W, 0.5, key_valid=valid, **modes)
    assert _lib.profile_stop().launches == 3, "the tiled path did not run"


@pytest.mark.parametrize("K,W,modes,masked", [(64, 64, {}, False), (9, 40, {}, True), (33, 5000, dict(window_mode=1), False),
                                              (20, 30, dict(window_mode=1), True)])
def test_soft_gather_on_the_tiled_kernels(K, W, modes, masked):
    # The soft gather softmax(Q_i mu^T / sqrt(d)) V_cent inside the tensor-core
    # window kernel (radius <= 32 or no local branch), with and without masks.
    from means_cluster_attention_b200 import _lib
    B, L = 2, 1500
    xq, xk = _case("bf16", B, 3, L, K, 3, W, 0.4, seed=7 * K + W)
    valid = None
    if masked:
        valid = np.ones((B, L), dtype=bool)
        valid[0, 900:] = False
        valid[1, ::4] = False
    _lib.profile_start("tiled_assign")
    _check("bf16", xq, xk, K, 3, W, 0.4, key_valid=valid, gather_mode=1, **modes)
    assert _lib.profile_stop().launches == 3, "the tiled path did not run"


@pytest.mark.parametrize("masked,modes", [(False, {}), (True, {}), (True, dict(gather_mode=1))])
def test_long_centroid_chunks(masked, modes):
    # 80 heads of 2600 keys: the centroid attention takes 2048-key chunks
    # (80 x 2 CTAs fill a 148-multiprocessor device), the second one ragged
    # (552 keys); with a scattered and a trailing key mask.
    from means_cluster_attention_b200 import _lib
    B, H, L = 2, 40, 2600
    xq, xk = _case("bf16", B, H, L, 20, 2, 64, 0.5, seed=131 + len(modes) + masked)
    valid = None
    if masked:
        valid = np.ones((B, L), dtype=bool)
        valid[0, 2300:] = False
        valid[1, ::5] = False
    _lib.profile_start("tiled_centroid")
    _check("bf16", xq, xk, 20, 2, 64, 0.5, key_valid=valid, **modes)
    assert _lib.profile_stop().launches == 1, "the tiled path did not run"
