"""The bounds-checked build (compiled with -DCA_CHECKED, selected with the
environment variable CA_CHECKED=1): every computed index that addresses
memory is checked on the device, and a bad one records CA_ERR_DEVICE instead
of faulting.  Run in a fresh process (the library is chosen at load time) on
shapes that exercise the fused kernel, the tiled path with both window
kernels and forced ties, and the general path: no check may fire, and the
results must still match the oracle."""

import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_PROBE = textwrap.dedent("""
    import os, sys
    sys.path.insert(0, sys.argv[1]); sys.path.insert(0, os.path.join(sys.argv[1], "tests"))
    import numpy as np
    import oracle
    from means_cluster_attention_b200 import _lib
    from means_cluster_attention_b200.inputs import Workload, make_inputs
    from helpers import TOL, run_gpu
    assert _lib.load()._name.endswith("libclusterattn_checked.so")
    cases = [
        Workload("fused", 2, 3, 512, 64, 16, 3, 32, 0.5, "bf16", "normal"),
        Workload("tiled_tc", 1, 2, 2500, 64, 48, 3, 64, 0.5, "bf16", "gmm", gmm_components=10,
                 gmm_std=0.05, dup_frac=0.1),
        Workload("tiled_wide", 1, 1, 1300, 64, 33, 2, 200, 0.5, "bf16", "normal"),
        Workload("general", 1, 4, 300, 64, 16, 3, 32, 0.5, "f32", "normal"),
    ]
    for w in cases:
        x = make_inputs(w, seed=7)
        g = run_gpu(x, w.dtype, w.K, w.iters, w.W, w.alpha, hist=True)   # sync_check: raises on a recorded error
        r_out, r_assign, r_cent, r_hist = oracle.forward(x["q64"], x["k64"], x["v64"], K=w.K, iters=w.iters,
                                                         W=w.W, alpha=w.alpha, hist=True)
        assert np.array_equal(g["hist"], r_hist), w.name
        assert np.array_equal(g["cent"], r_cent), w.name
        err = float(np.abs(g["out"] - oracle.forward_at(x["q64"], x["k64"], x["v64"], g["assign"], K=w.K,
                                                        iters=w.iters, W=w.W, alpha=w.alpha)[0]).max())
        assert err <= TOL[w.dtype], (w.name, err)
        print(w.name, "ok", err)
    print("CHECKED OK")
""")


def test_checked_build_records_no_error_and_matches_oracle():
    from means_cluster_attention_b200 import build
    build.build(checked=True)
    r = subprocess.run([sys.executable, "-c", _PROBE, ROOT], capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, CA_CHECKED="1"))
    assert r.returncode == 0, r.stdout + r.stderr
    assert "CHECKED OK" in r.stdout
