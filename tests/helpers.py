"""Shared helpers for the GPU parity tests: move seeded host inputs to the
device, run the library through its binding, and compare with the oracle."""

from __future__ import annotations

import numpy as np

from means_cluster_attention_b200.inputs import bf16_bits_to_f64

# Output tolerances stated for this method: max abs error 2e-3 for fp32
# inputs and 2e-2 for bf16 inputs (fp32 accumulation, bf16 output rounding).
TOL = {"f32": 2e-3, "bf16": 2e-2}


def to_device(x: dict, dtype: str):
    import torch
    if dtype == "f32":
        conv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    else:
        conv = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return conv(x["q"]), conv(x["k"]), conv(x["v"])


def out_to_f64(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return bf16_bits_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.cpu().numpy().astype(np.float64)


def run_gpu(x: dict, dtype: str, K: int, iters: int, W: int, alpha: float, hist: bool = False):
    import torch
    import means_cluster_attention_b200 as ca
    q, k, v = to_device(x, dtype)
    B, H, L, d = q.shape
    h = torch.full((B, H, max(iters, 1), L), -1, dtype=torch.int32, device="cuda") if hist else None
    out, assign, cent = ca.forward(q, k, v, K, iters, W, alpha, assign_hist=h, sync_check=True)
    torch.cuda.synchronize()
    res = dict(out=out_to_f64(out), assign=assign.cpu().numpy(), cent=cent.cpu().numpy().astype(np.float64))
    if hist:
        res["hist"] = h.cpu().numpy()[:, :, :iters]
    return res


def select_heads(x: dict, heads) -> dict:
    """Restrict [B,H,L,d] inputs to a list of flat head indices as [1, n, L, d]."""
    out = {}
    for key, a in x.items():
        B, H = a.shape[:2]
        flat = a.reshape((B * H,) + a.shape[2:])
        out[key] = np.ascontiguousarray(flat[list(heads)])[None]
    return out
