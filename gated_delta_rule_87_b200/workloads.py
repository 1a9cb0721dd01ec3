"""Seeded synthetic inputs for the gated delta rule.

This module only draws and shapes random inputs; it holds none of the
recurrence's arithmetic.  The same bytes feed the CUDA path and the fp64
oracle.  Shapes and distributions follow the workloads stated for the method
(per-head d_k = d_v = 128, long prefill, packed variable-length prefill,
batched decode, long Gated DeltaNet prefill with shared q/k heads, and a
small all-fp32 Gated DeltaNet case).

Generation recipe (one ``numpy.random.default_rng(seed)`` stream per
workload, draws in this fixed order):

    [varlen lengths] -> q -> k -> v -> gate -> beta -> initial state

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
def _normal(rng, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float64)


def _unit_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / n


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.log1p(np.exp(-np.abs(x))) + np.maximum(x, 0.0)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def _store(x64: np.ndarray, io_dtype: str):
    """Return (stored array, exact float32 view of the stored values)."""
    if io_dtype == "bf16":
        bits = bf16_round(x64.astype(np.float32))
        return bits, bf16_bits_to_f32(bits)
    if io_dtype == "f32":
        f = x64.astype(np.float32)
        return f, f
    raise ValueError(f"unknown io dtype {io_dtype}")


def _draw_block(rng, w: Workload, lead: tuple):
    """Draw q, k, v, gate, beta for token-axis shape ``lead`` (in that order)."""
    q = _store(_unit_rows(_normal(rng, lead + (w.H_qk, w.d_k))), w.io_dtype)
    k = _store(_unit_rows(_normal(rng, lead + (w.H_qk, w.d_k))), w.io_dtype)
    v = _store(_normal(rng, lead + (w.H_v, w.d_v)), w.io_dtype)
    if w.gate == "channel":
        gshape = lead + (w.H_v, w.d_k)
    elif w.gate == "scalar":
        gshape = lead + (w.H_v,)
    else:
        raise ValueError(w.gate)
    g = (-w.gate_scale * _softplus(_normal(rng, gshape))).astype(np.float32)
    beta = _sigmoid(_normal(rng, lead + (w.H_v,))).astype(np.float32)
    return q, k, v, g, beta


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
    rng = np.random.default_rng(seed)
    if lengths is None and w.varlen:
        lo, hi = w.varlen_range
        lengths = rng.integers(lo, hi, size=w.varlen, endpoint=True)
    if lengths is not None:
        lengths = np.asarray(lengths, dtype=np.int64)
        cu = np.zeros(len(lengths) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(lengths)
    else:
        cu = (np.arange(w.B + 1, dtype=np.int64) * w.T).astype(np.int32)
    total = int(cu[-1])
    n = len(cu) - 1
    (q, q32), (k, k32), (v, v32), g, beta = _draw_block(rng, w, (total,))
    s0 = None
    if w.init_state:
        s0 = (0.02 * _normal(rng, (n, w.H_v, w.d_k, w.d_v))).astype(np.float32)
    return PrefillInputs(w=w, q=q, k=k, v=v, g=g, beta=beta, initial_state=s0,
                         cu_seqlens=cu, q32=q32, k32=k32, v32=v32)


def make_decode(w: Workload, seed: int = 0) -> DecodeInputs:
    if w.kind != "decode":
        raise ValueError("not a decode workload")
    rng = np.random.default_rng(seed)
    (q, q32), (k, k32), (v, v32), g, beta = _draw_block(rng, w, (w.steps, w.N))
    if w.init_state:
        s0 = (0.02 * _normal(rng, (w.N, w.H_v, w.d_k, w.d_v))).astype(np.float32)
    else:
        s0 = np.zeros((w.N, w.H_v, w.d_k, w.d_v), dtype=np.float32)
    return DecodeInputs(w=w, q=q, k=k, v=v, g=g, beta=beta, initial_state=s0,
                        q32=q32, k32=k32, v32=v32)
