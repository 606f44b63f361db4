"""Device-side error reporting through the C ABI, with no GPU fault.

A kernel that detects a problem records a status code in the library's
device error word (it never traps or faults); ca_sync_status reads the word
once, returns the code and clears it.  ca_debug_record_error launches a
one-thread kernel that records a code exactly as such a kernel would, so the
whole reporting path is exercised without breaking anything.
"""

import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _lib_and_stream():
    import torch
    from means_cluster_attention_b200 import _lib
    return _lib, _lib.load(), torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("code", [4, 5])
def test_recorded_device_error_is_reported_once_then_cleared(code):
    _lib, lib, stream = _lib_and_stream()
    assert lib.ca_sync_status(stream) == 0
    assert lib.ca_debug_record_error(code, stream) == 0
    assert lib.ca_sync_status(stream) == code
    assert "site 99" in lib.ca_last_error().decode()
    assert lib.ca_sync_status(stream) == 0


def test_debug_hook_rejects_other_codes():
    _lib, lib, stream = _lib_and_stream()
    for bad in (0, 1, 3, 6, -1):
        assert lib.ca_debug_record_error(bad, stream) == 1
    assert lib.ca_sync_status(stream) == 0


def test_forward_after_a_recorded_error_still_runs():
    """The error word is per device and shared by every stream: a recorded
    error is returned by the next status check whoever made it, and the
    context stays usable for the next forward."""
    import torch
    import means_cluster_attention_b200 as ca
    _lib, lib, stream = _lib_and_stream()
    assert lib.ca_debug_record_error(5, stream) == 0
    with pytest.raises(_lib.ClusterAttnError):
        ca.sync_status()
    q = torch.randn(1, 2, 64, 64, device="cuda")
    out, assign, cent = ca.forward(q, q, q, 4, 2, 8, 0.5, sync_check=True)
    assert torch.isfinite(out).all()
