"""Seeded synthetic inputs for the gated delta rule.

This module only draws and shapes random inputs; it holds none of the
recurrence's arithmetic.  The same bytes feed the CUDA path and the fp64
oracle.  Shapes and distributions follow the workloads stated for the method
(per-head d_k = d_v = 128, long prefill, packed variable-length prefill,
batched decode, long Gated DeltaNet prefill with shared q/k heads, and a
small all-fp32 Gated DeltaNet case).

Generation recipe.  Varlen lengths come first, from
``numpy.random.default_rng(seed).integers(lo, hi, n, endpoint=True)``.  Every
tensor is then drawn as standard normals in fp64, in blocks of whole rows along
its leading axis (about 2^22 elements per block); block b of tensor number
``tag`` (q = 1, k = 2, v = 3, gate = 4, beta = 5, initial state = 6) comes
from its own stream ``numpy.random.default_rng([seed, tag, b])``, so blocks
are drawn in parallel and the result does not depend on the thread count.

* q, k: standard normal in fp64, L2-normalised per (token, head) over d_k in
  fp64, then rounded to the io dtype (round to nearest even for bf16).
* v: standard normal, rounded to the io dtype.
* gate (log-decay, <= 0): ``-scale * softplus(N(0,1))`` in fp64, stored fp32;
  shape [T, H, d_k] for the per-channel gate, [T, H_v] for the scalar gate.
* beta: ``sigmoid(N(0,1))`` in fp64, stored fp32, shape [T, H_v].
* initial state: ``0.02 * N(0,1)`` fp32 of shape [N, H_v, d_k, d_v], or zeros.

Decode workloads draw every step's q, k, v, gate and beta as one
[steps, N, H, ...] array each (same order), then the initial state.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "PrefillInputs",
    "DecodeInputs",
    "make_prefill",
    "make_decode",
    "bf16_round",
    "bf16_bits_to_f32",
]


# --------------------------------------------------------------------------- #
# bf16 helpers (bit manipulation only)
# --------------------------------------------------------------------------- #
def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    rounding = 0x7FFF + ((b >> 16) & 1)
    return ((b + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------- #
# workload descriptions
# --------------------------------------------------------------------------- #
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                  # "prefill" or "decode"
    gate: str                  # "channel" (KDA) or "scalar" (Gated DeltaNet)
    io_dtype: str              # "bf16" or "f32"
    B: int = 1
    T: int = 0                 # tokens per sequence (dense) or total (varlen)
    H_qk: int = 1
    H_v: int = 1
    d_k: int = 128
    d_v: int = 128
    gate_scale: float = 0.1
    init_state: bool = False   # N(0, 0.02) initial state, else zeros
    varlen: int = 0            # number of packed sequences (0 = dense)
    varlen_range: tuple = (1024, 16384)
    N: int = 0                 # decode batch
    steps: int = 0             # decode steps
    description: str = ""

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "gdn_small_f32": Workload(
        name="gdn_small_f32", kind="prefill", gate="scalar", io_dtype="f32",
        B=1, T=128, H_qk=2, H_v=2, d_k=64, d_v=64, gate_scale=0.1,
        description="Gated DeltaNet B=1 H=2 T=128 d=64, all fp32, zero initial state"),
    "kda_prefill": Workload(
        name="kda_prefill", kind="prefill", gate="channel", io_dtype="bf16",
        B=1, T=4096, H_qk=32, H_v=32, d_k=128, d_v=128, gate_scale=0.1,
        init_state=True,
        description="KDA prefill B=1 H=32 T=4096 d=128, bf16 q/k/v, fp32 gate/beta/state"),
    "kda_varlen": Workload(
        name="kda_varlen", kind="prefill", gate="channel", io_dtype="bf16",
        B=1, H_qk=32, H_v=32, d_k=128, d_v=128, gate_scale=0.1, varlen=8,
        description="KDA packed prefill, 8 sequences of 1024..16384 tokens, H=32 d=128"),
    "kda_decode": Workload(
        name="kda_decode", kind="decode", gate="channel", io_dtype="bf16",
        N=256, H_qk=32, H_v=32, d_k=128, d_v=128, gate_scale=0.1, init_state=True,
        steps=64,
        description="KDA decode, 256 sequences x 32 heads, d=128, 64 consecutive steps"),
    "gdn_long": Workload(
        name="gdn_long", kind="prefill", gate="scalar", io_dtype="bf16",
        B=1, T=65536, H_qk=16, H_v=32, d_k=128, d_v=128, gate_scale=0.05,
        description="Gated DeltaNet prefill T=65536, 16 q/k heads shared by 32 v heads, d=128"),
}


# --------------------------------------------------------------------------- #
# containers
# --------------------------------------------------------------------------- #
@dataclasses.dataclass
class PrefillInputs:
    """Host arrays for one prefill call (layout [B*T, H, d], d contiguous).

    For bf16 workloads ``q``, ``k``, ``v`` hold uint16 bf16 bit patterns and
    ``q32``/``k32``/``v32`` their exact float32 values; for fp32 workloads
    both name the same float32 arrays.
    """
    w: Workload
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    g: np.ndarray                 # float32, [Ttot, H_v, d_k] or [Ttot, H_v]
    beta: np.ndarray              # float32, [Ttot, H_v]
    initial_state: Optional[np.ndarray]   # float32 [N, H_v, d_k, d_v] or None
    cu_seqlens: np.ndarray        # int32 [N+1] token offsets into the flat token axis
    q32: np.ndarray
    k32: np.ndarray
    v32: np.ndarray

    @property
    def num_seqs(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def total_tokens(self) -> int:
        return int(self.cu_seqlens[-1])


@dataclasses.dataclass
class DecodeInputs:
    """Host arrays for ``steps`` consecutive decode calls ([steps, N, H, d])."""
    w: Workload
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    g: np.ndarray
    beta: np.ndarray
    initial_state: np.ndarray
    q32: np.ndarray
    k32: np.ndarray
    v32: np.ndarray


# --------------------------------------------------------------------------- #
# generation
# --------------------------------------------------------------------------- #
_BLOCK_ELEMS = 1 << 22
_TAGS = {"q": 1, "k": 2, "v": 3, "gate": 4, "beta": 5, "state": 6}


def _pool():
    import concurrent.futures
    import os
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        n = os.cpu_count() or 1
    return concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(n, 32)))


def _blocked(seed: int, tag: str, shape: tuple, transform, out_dtypes):
    """Draw N(0,1) fp64 for ``shape`` block by block, map each block through
    ``transform`` (fp64 block -> tuple of arrays) and assemble the outputs."""
    shape = tuple(int(x) for x in shape)
    rows = shape[0]
    row_elems = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    per = max(1, _BLOCK_ELEMS // max(row_elems, 1))
    outs = [np.empty(shape, dtype=dt) for dt in out_dtypes]

    def work(b):
        r0, r1 = b * per, min(rows, (b + 1) * per)
        rng = np.random.default_rng([seed, _TAGS[tag], b])
        x = rng.standard_normal(size=(r1 - r0,) + shape[1:], dtype=np.float64)
        for o, y in zip(outs, transform(x)):
            o[r0:r1] = y

    nblk = (rows + per - 1) // per
    if nblk <= 1:
        for b in range(nblk):
            work(b)
    else:
        with _pool() as ex:
            list(ex.map(work, range(nblk)))
    return outs


def _unit_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.einsum("...i,...i->...", x, x))[..., None]
    return x / n


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.log1p(np.exp(-np.abs(x))) + np.maximum(x, 0.0)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def _io_transform(io_dtype: str, normalise: bool):
    def f(x):
        if normalise:
            x = _unit_rows(x)
        x32 = x.astype(np.float32)
        if io_dtype == "bf16":
            bits = bf16_round(x32)
            return bits, bf16_bits_to_f32(bits)
        if io_dtype == "f32":
            return x32, x32
        raise ValueError(f"unknown io dtype {io_dtype}")
    return f


def _io_dtypes(io_dtype: str):
    return (np.uint16, np.float32) if io_dtype == "bf16" else (np.float32, np.float32)


def _draw_block(seed, w: Workload, lead: tuple):
    """Draw q, k, v, gate, beta for token-axis shape ``lead``."""
    io_t = _io_dtypes(w.io_dtype)
    q, q32 = _blocked(seed, "q", lead + (w.H_qk, w.d_k), _io_transform(w.io_dtype, True), io_t)
    k, k32 = _blocked(seed, "k", lead + (w.H_qk, w.d_k), _io_transform(w.io_dtype, True), io_t)
    v, v32 = _blocked(seed, "v", lead + (w.H_v, w.d_v), _io_transform(w.io_dtype, False), io_t)
    if w.gate == "channel":
        gshape = lead + (w.H_v, w.d_k)
    elif w.gate == "scalar":
        gshape = lead + (w.H_v,)
    else:
        raise ValueError(w.gate)
    if q is q32:
        q32, k32, v32 = q, k, v
    (g,) = _blocked(seed, "gate", gshape,
                    lambda x: ((-w.gate_scale * _softplus(x)).astype(np.float32),), (np.float32,))
    (beta,) = _blocked(seed, "beta", lead + (w.H_v,),
                       lambda x: (_sigmoid(x).astype(np.float32),), (np.float32,))
    return (q, q32), (k, k32), (v, v32), g, beta


def _draw_state(seed, n, w: Workload):
    (s0,) = _blocked(seed, "state", (n, w.H_v, w.d_k, w.d_v),
                     lambda x: ((0.02 * x).astype(np.float32),), (np.float32,))
    return s0


def varlen_lengths(w: Workload, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    lo, hi = w.varlen_range
    return rng.integers(lo, hi, size=w.varlen, endpoint=True)


def make_prefill(w: Workload, seed: int = 0, lengths=None) -> PrefillInputs:
    """Generate one prefill problem.

    ``lengths`` overrides the varlen draw (a list of per-sequence lengths,
    zeros allowed); it implies a packed batch with B = 1.
    """
    if w.kind != "prefill":
        raise ValueError("not a prefill workload")
    if lengths is None and w.varlen:
        lengths = varlen_lengths(w, seed)
    if lengths is not None:
        lengths = np.asarray(lengths, dtype=np.int64)
        cu = np.zeros(len(lengths) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(lengths)
    else:
        cu = (np.arange(w.B + 1, dtype=np.int64) * w.T).astype(np.int32)
    total = int(cu[-1])
    n = len(cu) - 1
    (q, q32), (k, k32), (v, v32), g, beta = _draw_block(seed, w, (total,))
    s0 = _draw_state(seed, n, w) if w.init_state else None
    return PrefillInputs(w=w, q=q, k=k, v=v, g=g, beta=beta, initial_state=s0,
                         cu_seqlens=cu, q32=q32, k32=k32, v32=v32)


def make_decode(w: Workload, seed: int = 0) -> DecodeInputs:
    if w.kind != "decode":
        raise ValueError("not a decode workload")
    (q, q32), (k, k32), (v, v32), g, beta = _draw_block(seed, w, (w.steps, w.N))
    if w.init_state:
        s0 = _draw_state(seed, w.N, w)
    else:
        s0 = np.zeros((w.N, w.H_v, w.d_k, w.d_v), dtype=np.float32)
    return DecodeInputs(w=w, q=q, k=k, v=v, g=g, beta=beta, initial_state=s0,
                        q32=q32, k32=k32, v32=v32)
