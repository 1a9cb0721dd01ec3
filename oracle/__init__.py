"""fp64 CPU oracle of the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it and shares no code with it.

Two independent implementations live here:

* ``gated_delta`` -- the token-by-token recurrence in plain C (fp64), run over
  every (sequence, head) chain with POSIX threads
  (``gated_delta_oracle.c``);
* ``brute.transition_products`` -- a NumPy fp64 evaluation that forms every
  transition matrix explicitly and multiplies them out (tiny T only).

The update rules followed are the rows "Linear attention", "Delta rule",
"Gated DeltaNet" and "KDA" of the table "Everything, in one table" on the
thethings.ai page "The argument, in one page"; the readout o_t = S_t^T q_t
reads the state after the token's own update.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gated_delta_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

ORDERS = {"erase_then_decay": 0, "decay_then_erase": 1}
RULES = {"delta": 0, "linear": 1}
MUTATIONS = {
    "none": 0, "drop_erase": 1, "erase_sign": 2, "gate_late": 3, "read_before": 4,
    "read_transposed": 5, "write_no_beta": 6, "decay_write": 7, "read_with_key": 8,
    "gate_channel": 9,
}


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/_build/liboracle.so``."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
               "-pthread", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            lib = ctypes.CDLL(path)
            f = lib.oracle_gated_delta
            dp = ctypes.POINTER(ctypes.c_double)
            f.argtypes = [dp, dp, dp, dp, ctypes.c_int, dp, dp, dp, dp,
                          ctypes.POINTER(ctypes.c_int64), ctypes.c_int64,
                          ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
            f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x: Optional[np.ndarray]):
    if x is None:
        return None
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def gated_delta(q, k, v, g, beta, initial_state=None, offsets=None, *,
                order: str = "erase_then_decay", rule: str = "delta",
                mutation: str = "none", threads: Optional[int] = None
                ) -> Tuple[np.ndarray, np.ndarray]:
    """Token-by-token fp64 recurrence.

    q, k: [Ttot, H_qk, d_k]; v: [Ttot, H_v, d_v]; g: [Ttot, H_v, d_k] (per-channel
    gate) or [Ttot, H_v] (scalar gate), log-decay; beta: [Ttot, H_v];
    initial_state: [N, H_v, d_k, d_v] or None; offsets: [N+1] token offsets
    (None = one sequence of Ttot tokens).  Returns (o [Ttot, H_v, d_v],
    final_state [N, H_v, d_k, d_v]) in fp64.
    """
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    Ttot, H_qk, d_k = q.shape
    H_v, d_v = v.shape[1], v.shape[2]
    if k.shape != q.shape or v.shape[0] != Ttot:
        raise ValueError("shape mismatch between q, k, v")
    if g.ndim == 3:
        per_channel = 1
        if g.shape != (Ttot, H_v, d_k):
            raise ValueError("per-channel gate must be [Ttot, H_v, d_k]")
    else:
        per_channel = 0
        if g.shape != (Ttot, H_v):
            raise ValueError("scalar gate must be [Ttot, H_v]")
    if beta.shape != (Ttot, H_v):
        raise ValueError("beta must be [Ttot, H_v]")
    if offsets is None:
        offsets = np.array([0, Ttot], dtype=np.int64)
    offsets = np.ascontiguousarray(offsets, dtype=np.int64)
    N = offsets.shape[0] - 1
    if offsets[-1] != Ttot:
        raise ValueError("offsets[-1] must equal the token count")
    s0 = None
    if initial_state is not None:
        s0 = _f64(initial_state)
        if s0.shape != (N, H_v, d_k, d_v):
            raise ValueError("initial_state must be [N, H_v, d_k, d_v]")
    o = np.zeros((Ttot, H_v, d_v), dtype=np.float64)
    sT = np.zeros((N, H_v, d_k, d_v), dtype=np.float64)
    lib = _load()
    rc = lib.oracle_gated_delta(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), per_channel, _ptr(beta), _ptr(s0),
        _ptr(o), _ptr(sT), offsets.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        N, H_qk, H_v, d_k, d_v, ORDERS[order], RULES[rule], MUTATIONS[mutation],
        int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_gated_delta failed with status {rc}")
    return o, sT


def decode_steps(q, k, v, g, beta, state, **kw) -> Tuple[np.ndarray, np.ndarray]:
    """``steps`` consecutive one-token updates of N independent sequences.

    q, k: [steps, N, H_qk, d_k]; v: [steps, N, H_v, d_v]; g: [steps, N, H_v, d_k]
    or [steps, N, H_v]; beta: [steps, N, H_v]; state: [N, H_v, d_k, d_v].
    Returns (o [steps, N, H_v, d_v], final state).  Sequence n's tokens are
    its steps in order, so this is the same recurrence as a prefill of
    ``steps`` tokens per sequence.
    """
    steps, N = q.shape[0], q.shape[1]
    sw = lambda x: np.ascontiguousarray(np.swapaxes(x, 0, 1)).reshape((N * steps,) + x.shape[2:])
    offsets = np.arange(N + 1, dtype=np.int64) * steps
    o, sT = gated_delta(sw(np.asarray(q, np.float64)), sw(np.asarray(k, np.float64)),
                        sw(np.asarray(v, np.float64)), sw(np.asarray(g, np.float64)),
                        sw(np.asarray(beta, np.float64)), state, offsets, **kw)
    o = np.swapaxes(o.reshape((N, steps) + o.shape[1:]), 0, 1)
    return np.ascontiguousarray(o), sT
