"""Helpers for GPU-vs-oracle parity: device copies of seeded inputs, and the
tolerances (relative L2 over a whole tensor: <= 1e-4 for all-fp32 paths,
<= 2e-2 for paths with bf16 q/k/v, fp32 state and accumulation)."""
from __future__ import annotations

import numpy as np

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    if den == 0.0:
        return float(num)
    return float(num / den)


def tol_for(io_dtype: str) -> float:
    return TOL_F32 if io_dtype == "f32" else TOL_BF16


def to_device(x, dtype_name, device="cuda"):
    """Host array -> torch tensor on the device (bf16 from uint16 bit patterns)."""
    import torch
    if dtype_name == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(device)


def to_host(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def prefill_device_inputs(x, device="cuda"):
    """PrefillInputs -> dict of device tensors shaped [B, T, H, d] (packed: B = 1)."""
    import torch
    w = x.w
    if x.w.varlen or x.num_seqs != w.B or (x.total_tokens != w.B * w.T):
        B, T = 1, x.total_tokens
        cu = torch.from_numpy(x.cu_seqlens.astype(np.int32)).to(device)
    else:
        B, T = w.B, w.T
        cu = None
    io = w.io_dtype
    shp = lambda a: a.reshape((B, T) + a.shape[1:])
    d = dict(
        q=to_device(shp(x.q), io, device), k=to_device(shp(x.k), io, device),
        v=to_device(shp(x.v), io, device),
        g=to_device(shp(x.g), "f32", device), beta=to_device(shp(x.beta), "f32", device),
        initial_state=None if x.initial_state is None else to_device(x.initial_state, "f32", device),
        cu_seqlens=cu,
    )
    return d


def oracle_prefill(x, heads=None, threads=None):
    """Run the oracle on a PrefillInputs (optionally only the v-heads in ``heads``,
    each given its own copy of its q/k head).  Returns (o [Ttot, nh, d_v],
    final [N, nh, d_k, d_v])."""
    import oracle
    w = x.w
    s0 = x.initial_state
    if heads is None:
        return oracle.gated_delta(x.q32, x.k32, x.v32, x.g, x.beta, s0,
                                  x.cu_seqlens.astype(np.int64), threads=threads)
    group = w.H_v // w.H_qk
    hk = [h // group for h in heads]
    return oracle.gated_delta(
        x.q32[:, hk], x.k32[:, hk], x.v32[:, heads], x.g[:, heads], x.beta[:, heads],
        None if s0 is None else s0[:, heads], x.cu_seqlens.astype(np.int64), threads=threads)
