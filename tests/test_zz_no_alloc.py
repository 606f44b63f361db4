"""The allocation-free entry point, ca_forward_noalloc.

Callers that cannot let a library allocate device memory (runtimes that
reserve the whole GPU for their own allocator, serving loops that forbid
allocation calls on their hot path) use ca_forward_noalloc: it takes its
working memory from a fixed 16 MiB array inside the library instead of
allocating.  These tests call it through the C ABI and check it against the
regular entry points (ca_forward / ca_forward_bf16) and against the fp64
oracle on the same inputs, twice in a row, since the shared array keeps the
previous call's contents; and, in a fresh process, that repeated calls leave
the device's free memory unchanged.

This file is named so that pytest collects it last.
"""

import ctypes
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest

import oracle
from means_cluster_attention_b200.inputs import WORKLOADS, make_inputs
from helpers import TOL, out_to_f64, to_device

pytestmark = pytest.mark.gpu


def _run_pair(w, x):
    import torch
    from means_cluster_attention_b200 import _lib
    lib = _lib.load()
    q, k, v = to_device(x, w.dtype)
    B, H, L, d = q.shape
    stream = torch.cuda.current_stream().cuda_stream
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())

    ref_out = torch.empty_like(q)
    ref_assign = torch.empty((B, H, L), dtype=torch.int32, device="cuda")
    ref_cent = torch.empty((B, H, w.K, d), dtype=torch.float32, device="cuda")
    regular = lib.ca_forward if w.dtype == "f32" else lib.ca_forward_bf16
    st = regular(ptr(q), ptr(k), ptr(v), B, H, L, d, w.K, w.iters, w.W, w.alpha, ptr(ref_out),
                 ptr(ref_assign), ptr(ref_cent), stream)
    _lib.check(st)

    results = []
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        assign = torch.full((B, H, L), -1, dtype=torch.int32, device="cuda")
        cent = torch.full((B, H, w.K, d), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.ca_forward_noalloc(ptr(q), ptr(k), ptr(v), 0 if w.dtype == "f32" else 1, B, H, L, d,
                                    w.K, w.iters, w.W, w.alpha, ptr(out), ptr(assign), ptr(cent), stream)
        _lib.check(st)
        _lib.check(lib.ca_sync_status(stream))
        results.append((out_to_f64(out), assign.cpu().numpy(), cent.cpu().numpy()))
    return (out_to_f64(ref_out), ref_assign.cpu().numpy(), ref_cent.cpu().numpy()), results


@pytest.mark.parametrize("name,shrink", [("card_gmm_f32", None), ("l512_bf16", dict(B=8))])
def test_noalloc_matches_regular_entry_point_twice(name, shrink):
    w = WORKLOADS[name]
    if shrink:
        w = w.replace(**shrink)
    x = make_inputs(w)
    (ref_out, ref_assign, ref_cent), results = _run_pair(w, x)
    o_out, o_assign, o_cent, _ = oracle.forward(x["q64"], x["k64"], x["v64"], K=w.K, iters=w.iters, W=w.W,
                                                alpha=w.alpha)
    for out, assign, cent in results:
        np.testing.assert_array_equal(assign, ref_assign)
        np.testing.assert_array_equal(cent, ref_cent)
        err = float(np.abs(out - ref_out).max())
        assert err <= TOL[w.dtype], err
        # and against the oracle directly: exact assignments and centroids,
        # outputs within the stated tolerance
        np.testing.assert_array_equal(assign, o_assign)
        np.testing.assert_array_equal(cent.astype(np.float64), o_cent)
        err = float(np.abs(out - o_out).max())
        assert err <= TOL[w.dtype], err


def test_noalloc_rejects_problems_beyond_its_fixed_array():
    import torch
    from means_cluster_attention_b200 import _lib
    lib = _lib.load()
    w = WORKLOADS["l512_bf16"]  # 768 heads need more than 16 MiB of working memory
    q = torch.zeros((w.B, w.H, w.L, w.d), dtype=torch.bfloat16, device="cuda")
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.ca_forward_noalloc(ptr(q), ptr(q), ptr(q), 1, w.B, w.H, w.L, w.d, w.K, w.iters, w.W,
                                w.alpha, ptr(q), None, None, torch.cuda.current_stream().cuda_stream)
    assert st == 1
    msg = lib.ca_last_error().decode()
    assert "working memory" in msg and "16777216" in msg


_NO_ALLOC_PROBE = textwrap.dedent("""
    import ctypes, sys
    import torch
    sys.path.insert(0, sys.argv[1])
    from means_cluster_attention_b200 import _lib
    lib = _lib.load()
    B, H, L, d, K = 4, 12, 128, 64, 16
    q = torch.randn(B, H, L, d, device="cuda")
    out = torch.empty_like(q)
    assign = torch.empty(B, H, L, dtype=torch.int32, device="cuda")
    cent = torch.empty(B, H, K, d, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = torch.cuda.current_stream().cuda_stream

    def call():
        _lib.check(lib.ca_forward_noalloc(p(q), p(q), p(q), 0, B, H, L, d, K, 3, 32, 0.5, p(out), p(assign),
                                          p(cent), st))
        _lib.check(lib.ca_sync_status(st))

    call()  # first call: looks up the fixed array's address (module loaded)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(5):
        call()
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    print("FREE", free0, free1)
    sys.exit(0 if free0 == free1 else 3)
""")


def test_noalloc_calls_leave_free_device_memory_unchanged():
    """In a fresh process (so no earlier call has set up the library's memory
    pool), calls after the first one must not change the device's free
    memory: no allocation, no pool growth."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _NO_ALLOC_PROBE, root], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FREE" in r.stdout
