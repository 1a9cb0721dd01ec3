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


# Errors measured by the parity tests, printed in pytest's terminal summary
# (conftest.py) so that a GPU run's log records the margin to the bounds.
RECORDS: list = []

# A block whose reference norm is below this fraction of the median block norm
# is measured against that floor instead of its own norm, so that a
# near-zero block cannot turn rounding noise into a large relative error.
BLOCK_FLOOR = 1e-3


def _floored_rel(diff_norms, ref_norms):
    ref_norms = np.asarray(ref_norms, np.float64)
    floor = BLOCK_FLOOR * float(np.median(ref_norms)) if ref_norms.size else 0.0
    den = np.maximum(ref_norms, max(floor, 1e-300))
    return np.asarray(diff_norms, np.float64) / den


def token_block_errors(o, ro, cu_seqlens, block: int = 64):
    """Relative L2 error of o against ro ([tokens, H, d]) for every (v-head,
    64-token block of a sequence) and every (sequence, v-head).  A wrong chunk
    of one head shows up here even where the whole-tensor norm hides it.
    Returns (max over blocks, max over sequences)."""
    o = np.asarray(o, np.float64)
    ro = np.asarray(ro, np.float64)
    cu = np.asarray(cu_seqlens, np.int64)
    bd, br, sd, sr = [], [], [], []
    for n in range(len(cu) - 1):
        a, b = int(cu[n]), int(cu[n + 1])
        if b == a:
            continue
        sd.append(np.linalg.norm(o[a:b] - ro[a:b], axis=(0, 2)))
        sr.append(np.linalg.norm(ro[a:b], axis=(0, 2)))
        for s in range(a, b, block):
            e = min(s + block, b)
            bd.append(np.linalg.norm(o[s:e] - ro[s:e], axis=(0, 2)))
            br.append(np.linalg.norm(ro[s:e], axis=(0, 2)))
    if not bd:
        return 0.0, 0.0
    eb = _floored_rel(np.concatenate(bd), np.concatenate(br))
    es = _floored_rel(np.concatenate(sd), np.concatenate(sr))
    return float(eb.max()), float(es.max())


def state_errors(s, rs):
    """Max relative L2 error over the (sequence, head) states [N, H, d_k, d_v]."""
    s = np.asarray(s, np.float64)
    rs = np.asarray(rs, np.float64)
    if s.size == 0:
        return 0.0
    d = np.linalg.norm((s - rs).reshape(s.shape[0] * s.shape[1], -1), axis=1)
    r = np.linalg.norm(rs.reshape(s.shape[0] * s.shape[1], -1), axis=1)
    return float(_floored_rel(d, r).max())


def check_prefill_parity(label, o, ro, s, rs, cu_seqlens, tol, regress=None):
    """Whole-tensor, per-(head, 64-token block), per-(sequence, head) and
    per-state errors, each against the contract bound ``tol``; the
    whole-tensor errors also against ``regress`` (a bound near the measured
    error, so that a drift shows long before the contract bound is reached).
    Records the errors for the run's summary and returns them."""
    eo = rel_l2(o, ro)
    eblk, eseq = token_block_errors(o, ro, cu_seqlens)
    es = rel_l2(s, rs) if s is not None else 0.0
    esx = state_errors(s, rs) if s is not None else 0.0
    RECORDS.append((label, eo, eblk, eseq, es, esx, tol))
    assert np.isfinite(o).all(), f"{label}: non-finite output"
    if s is not None:
        assert np.isfinite(s).all(), f"{label}: non-finite final state"
    assert eo <= tol, f"{label}: output rel-L2 {eo:.3e} > {tol}"
    assert eblk <= tol, f"{label}: worst (head, chunk) block rel-L2 {eblk:.3e} > {tol}"
    assert eseq <= tol, f"{label}: worst (sequence, head) rel-L2 {eseq:.3e} > {tol}"
    assert es <= tol, f"{label}: final-state rel-L2 {es:.3e} > {tol}"
    assert esx <= tol, f"{label}: worst (sequence, head) state rel-L2 {esx:.3e} > {tol}"
    if regress is not None:
        assert eo <= regress and es <= regress, (
            f"{label}: errors {eo:.3e} / {es:.3e} above the regression bound {regress}")
    return eo, eblk, eseq, es, esx


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


def oracle_prefill(x, heads=None, threads=None, order="erase_then_decay"):
    """Run the oracle on a PrefillInputs (optionally only the v-heads in ``heads``,
    each given its own copy of its q/k head).  Returns (o [Ttot, nh, d_v],
    final [N, nh, d_k, d_v])."""
    import oracle
    w = x.w
    s0 = x.initial_state
    if heads is None:
        return oracle.gated_delta(x.q32, x.k32, x.v32, x.g, x.beta, s0,
                                  x.cu_seqlens.astype(np.int64), threads=threads, order=order)
    group = w.H_v // w.H_qk
    hk = [h // group for h in heads]
    return oracle.gated_delta(
        x.q32[:, hk], x.k32[:, hk], x.v32[:, heads], x.g[:, heads], x.beta[:, heads],
        None if s0 is None else s0[:, heads], x.cu_seqlens.astype(np.int64), threads=threads,
        order=order)
