"""ctypes binding of libclusterattn (argument marshalling only).

Every step of the forward pass runs in the library's CUDA kernels; this module
only checks tensor metadata and passes raw pointers.  There is no CPU
fallback: if the library cannot be loaded, every call raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libclusterattn.so")
# CA_CHECKED=1 selects the bounds-checked build (same ABI; index checks on the
# device report CA_ERR_DEVICE through ca_sync_status instead of faulting).
LIB_CHECKED_PATH = os.path.join(PKG, "libclusterattn_checked.so")

CA_OK = 0
STATUS_NAMES = {0: "CA_OK", 1: "CA_ERR_INVALID_ARG", 2: "CA_ERR_UNSUPPORTED", 3: "CA_ERR_CUDA",
                4: "CA_ERR_TIMEOUT", 5: "CA_ERR_DEVICE"}

# Every symbol include/clusterattn.h declares, with its ctypes signature.
_vp, _ci, _cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
SIGNATURES = {
    "ca_forward": ([_vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp, _vp], _ci),
    "ca_forward_bf16": ([_vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp, _vp], _ci),
    "ca_forward_trace": ([_vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp, _vp, _vp], _ci),
    "ca_forward_host": ([_vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp, _vp], _ci),
    "ca_forward_ex": ([_vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp, _vp, _vp, _vp], _ci),
    "ca_forward_noalloc": ([_vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _vp, _vp, _vp], _ci),
    "ca_sync_status": ([_vp], _ci),
    "ca_debug_record_error": ([_ci, _vp], _ci),
    "ca_status_string": ([_ci], ctypes.c_char_p),
    "ca_last_error": ([], ctypes.c_char_p),
    "ca_version": ([], ctypes.c_char_p),
    "ca_profile_start": ([ctypes.c_char_p], _ci),
    "ca_profile_stop": ([_vp], _ci),
    "ca_launch_count": ([], ctypes.c_longlong),
}


class Options(ctypes.Structure):
    """Mirror of ca_options (include/clusterattn.h)."""
    _fields_ = [("window_mode", ctypes.c_int), ("empty_mode", ctypes.c_int), ("init_mode", ctypes.c_int),
                ("gather_mode", ctypes.c_int), ("key_valid", ctypes.c_void_p), ("H_kv", ctypes.c_int)]


class KernelStat(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_longlong), ("total_ms", ctypes.c_double),
                ("algorithmic_bytes", ctypes.c_double)]

_lib = None


class ClusterAttnError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {detail}")


def load(path: Optional[str] = None):
    """Load libclusterattn.so (raises if it is missing: no fallback exists)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or (LIB_CHECKED_PATH if os.environ.get("CA_CHECKED") == "1" else LIB_PATH)
    if not os.path.exists(p):
        raise OSError(f"libclusterattn.so not found at {p}; build it with "
                      "`python -m means_cluster_attention_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (args, res) in SIGNATURES.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    if path is None:
        _lib = lib
    return lib


def check(status: int) -> None:
    if status != CA_OK:
        detail = load().ca_last_error()
        raise ClusterAttnError(status, detail.decode() if detail else "")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def forward(q, k, v, K: int, iters: int, W: int, alpha: float, out=None, assign=None,
            centroids=None, assign_hist=None, stream=None, sync_check: bool = False) -> Tuple:
    """Cluster-attention forward on CUDA tensors [B, H, L, d] (fp32 or bf16).

    Returns (out, assign, centroids).  ``K`` is clamped to L as the model
    card's module does (K = min(num_clusters, L)).  Outputs are allocated when
    not given.  The call is asynchronous on ``stream`` (default: torch's
    current stream); ``sync_check`` synchronizes and checks device status.
    """
    import torch
    if q.device.type != "cuda":
        raise ValueError("q, k, v must be CUDA tensors")
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("q, k, v must share dtype float32 or bfloat16")
    if q.shape != k.shape or q.shape != v.shape or q.dim() != 4:
        raise ValueError("q, k, v must have the same [B, H, L, d] shape")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    B, H, L, d = q.shape
    K = min(int(K), L)
    if out is None:
        out = torch.empty_like(q)
    if assign is None:
        assign = torch.empty((B, H, L), dtype=torch.int32, device=q.device)
    if centroids is None:
        centroids = torch.empty((B, H, K, d), dtype=torch.float32, device=q.device)
    lib = load()
    dtype = 0 if q.dtype == torch.float32 else 1
    st = lib.ca_forward_trace(_ptr(q), _ptr(k), _ptr(v), dtype, B, H, L, d, K, int(iters), int(W),
                              float(alpha), _ptr(out), _ptr(assign), _ptr(centroids),
                              _ptr(assign_hist), _stream_handle(stream))
    check(st)
    if sync_check:
        check(lib.ca_sync_status(_stream_handle(stream)))
    return out, assign, centroids


def forward_ex(q, k, v, K: int, iters: int, W: int, alpha: float, window_mode: int = 0,
               empty_mode: int = 0, init_mode: int = 0, gather_mode: int = 0, key_valid=None,
               out=None, assign=None, centroids=None, assign_hist=None, stream=None,
               sync_check: bool = False) -> Tuple:
    """The forward with the variants of the card's module (see ca_options):
    q is [B, H, L, d]; k and v are [B, H_kv, L, d] (grouped key/value heads);
    key_valid is a [B, L] bool/uint8 CUDA tensor or None."""
    import torch
    if q.device.type != "cuda":
        raise ValueError("q, k, v must be CUDA tensors")
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("q, k, v must share dtype float32 or bfloat16")
    if k.shape != v.shape or q.dim() != 4 or k.dim() != 4 or q.shape[0] != k.shape[0] or q.shape[2:] != k.shape[2:]:
        raise ValueError("q must be [B, H, L, d] and k, v [B, H_kv, L, d]")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    B, H, L, d = q.shape
    K = min(int(K), L)
    kv = None
    if key_valid is not None:
        kv = key_valid.to(device=q.device, dtype=torch.uint8).contiguous()
        if kv.numel() != B * L:
            raise ValueError("key_valid must have B * L elements")
    if out is None:
        out = torch.empty_like(q)
    if assign is None:
        assign = torch.empty((B, H, L), dtype=torch.int32, device=q.device)
    if centroids is None:
        centroids = torch.empty((B, H, K, d), dtype=torch.float32, device=q.device)
    opt = Options(int(window_mode), int(empty_mode), int(init_mode), int(gather_mode), _ptr(kv), int(k.shape[1]))
    lib = load()
    dtype = 0 if q.dtype == torch.float32 else 1
    st = lib.ca_forward_ex(_ptr(q), _ptr(k), _ptr(v), dtype, B, H, L, d, K, int(iters), int(W), float(alpha),
                           ctypes.byref(opt), _ptr(out), _ptr(assign), _ptr(centroids), _ptr(assign_hist),
                           _stream_handle(stream))
    check(st)
    if sync_check:
        check(lib.ca_sync_status(_stream_handle(stream)))
    return out, assign, centroids


def forward_host(q, k, v, K: int, iters: int, W: int, alpha: float, out=None, assign=None,
                 centroids=None, stream=None) -> Tuple:
    """End-to-end call on HOST tensors (ideally pinned): copies in, runs,
    copies out and synchronizes inside the library."""
    import torch
    if q.device.type != "cpu":
        raise ValueError("forward_host takes host tensors")
    B, H, L, d = q.shape
    K = min(int(K), L)
    if out is None:
        out = torch.empty_like(q)
    dtype = 0 if q.dtype == torch.float32 else 1
    st = load().ca_forward_host(_ptr(q), _ptr(k), _ptr(v), dtype, B, H, L, d, K, int(iters), int(W),
                                float(alpha), _ptr(out), _ptr(assign), _ptr(centroids),
                                _stream_handle(stream))
    check(st)
    return out, assign, centroids


def sync_status(stream=None) -> None:
    check(load().ca_sync_status(_stream_handle(stream)))


def profile_start(kernel_name: Optional[str]) -> None:
    check(load().ca_profile_start(kernel_name.encode() if kernel_name else None))


def profile_stop() -> KernelStat:
    st = KernelStat()
    check(load().ca_profile_stop(ctypes.byref(st)))
    return st


def launch_count() -> int:
    return int(load().ca_launch_count())
