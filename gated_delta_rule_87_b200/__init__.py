"""Gated delta rule (KDA / Gated DeltaNet) on B200: Python binding.

A thin ctypes layer over the C ABI in ``include/gated_delta.h``
(``libgated_delta.so``, built in-tree for sm_100a).  It only marshals
arguments: every step of the computation runs in the library's CUDA kernels.
PyTorch is used for device memory and streams.  There is no CPU path: if the
library is missing or no CUDA device is present the calls raise.

Operator (thethings.ai "The argument, in one page", table "Everything, in
one table", rows "KDA" and "Gated DeltaNet"; column-vector keys):

    S_t = Diag(exp(g_t)) (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
    o_t = S_t^T q_t
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading
from typing import Optional, Tuple

__all__ = [
    "lib", "library_path", "KdaError", "kda_chunk_fwd", "gdn_chunk_fwd", "kda_decode_step",
    "gdn_decode_step", "kda_recurrent_fwd", "gdn_recurrent_fwd", "state_gather", "state_scatter",
    "chunk_workspace_size", "check_device_status", "EXPORTED_SYMBOLS",
    "checked_library_path", "use_library", "bounds_checked", "bounds_violations",
    "kda_chunk_fwd_host",
    "trace_enable", "trace_read", "ERASE_THEN_DECAY", "DECAY_THEN_ERASE",
    "KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED", "KDA_ERR_CUDA",
    "KDA_ERR_DEVICE_CHECK", "KDA_ERR_WORKSPACE",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libgated_delta.so")
# the bounds-checked build of the same sources (see kda_bounds_checked)
checked_library_path = os.path.join(_PKG, "libgated_delta_checked.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_DEVICE_CHECK, \
    KDA_ERR_WORKSPACE = range(6)
KDA_F32, KDA_BF16 = 0, 1
# device codes in a workspace's status word (kda_check_device_status)
KDA_DEVICE_OK, KDA_DEVICE_BAD_CU_SEQLENS, KDA_DEVICE_TIMEOUT = 0, 1, 2
# decay order (KDA): the table's literal order, or the decay applied before the erase
ERASE_THEN_DECAY, DECAY_THEN_ERASE = "erase_then_decay", "decay_then_erase"
_ORDER = {ERASE_THEN_DECAY: 0, DECAY_THEN_ERASE: 1}

EXPORTED_SYMBOLS = (
    "kda_chunk_fwd", "kda_chunk_fwd_workspace_size", "gdn_chunk_fwd",
    "gdn_chunk_fwd_workspace_size", "kda_decode_step", "gdn_decode_step",
    "kda_check_device_status", "kda_status_string", "kda_last_error", "kda_abi_version",
    "kda_trace_enable", "kda_trace_read", "kda_chunk_fwd_noalloc", "kda_chunk_fwd_ex",
    "gdn_chunk_fwd_ex", "kda_recurrent_fwd", "gdn_recurrent_fwd", "kda_state_gather",
    "kda_state_scatter", "kda_selftest_wait_timeout", "kda_bounds_checked",
    "kda_bounds_violations", "kda_chunk_fwd_host", "kda_chunk_fwd_host_buffer_size",
)

_lock = threading.Lock()
_lib = None

_vp, _fp, _i32, _sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_i64, _int = ctypes.c_int64, ctypes.c_int
_SIGS = {
    "kda_chunk_fwd_ex": ([_vp] * 9 + [_i64, _vp] + [_i32] * 6 + [_int, _int, _vp, _sz, _vp], _int),
    "gdn_chunk_fwd_ex": ([_vp] * 9 + [_i64, _vp] + [_i32] * 7 + [_int, _vp, _sz, _vp], _int),
    "kda_recurrent_fwd": ([_vp] * 8 + [_i64] + [_i32] * 5 + [_int, _int, _vp], _int),
    "gdn_recurrent_fwd": ([_vp] * 8 + [_i64] + [_i32] * 6 + [_int, _vp], _int),
    "kda_state_gather": ([_vp, _vp, _i64, _vp] + [_i32] * 4 + [_vp], _int),
    "kda_state_scatter": ([_vp, _vp, _vp, _i64] + [_i32] * 4 + [_vp], _int),
    "kda_chunk_fwd": ([_vp] * 9 + [_i32] * 6 + [ctypes.c_int, _vp, _sz, _vp], ctypes.c_int),
    "gdn_chunk_fwd": ([_vp] * 9 + [_i32] * 7 + [ctypes.c_int, _vp, _sz, _vp], ctypes.c_int),
    "kda_chunk_fwd_workspace_size": ([_i32] * 6 + [ctypes.c_int], _sz),
    "gdn_chunk_fwd_workspace_size": ([_i32] * 7 + [ctypes.c_int], _sz),
    "kda_decode_step": ([_vp] * 7 + [_i32] * 4 + [ctypes.c_int, _vp], ctypes.c_int),
    "gdn_decode_step": ([_vp] * 7 + [_i32] * 5 + [ctypes.c_int, _vp], ctypes.c_int),
    "kda_check_device_status": ([_vp, _vp, ctypes.POINTER(_i32)], ctypes.c_int),
    "kda_selftest_wait_timeout": ([_vp, _i32, _vp], ctypes.c_int),
    "kda_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "kda_last_error": ([], ctypes.c_char_p),
    "kda_abi_version": ([], _i32),
    "kda_trace_enable": ([_i32], ctypes.c_int),
    "kda_chunk_fwd_noalloc": ([_vp] * 9 + [_i32] * 6 + [ctypes.c_int, _vp], ctypes.c_int),
    "kda_trace_read": ([ctypes.c_char_p, _i32, ctypes.POINTER(ctypes.c_float), _i32], _i32),
    "kda_bounds_checked": ([], _i32),
    "kda_chunk_fwd_host_buffer_size": ([_i32] * 5 + [ctypes.c_int, _i32], _sz),
    "kda_chunk_fwd_host": ([_vp] * 8 + [_i32] * 5 + [ctypes.c_int, _i32, _vp, _sz, _vp], ctypes.c_int),
    "kda_bounds_violations": ([_vp, ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
}


class KdaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{detail} (status {status})")


_libs = {}                   # path -> loaded CDLL
_active_path = library_path  # the library the calls below go through


def _load(path: str) -> ctypes.CDLL:
    with _lock:
        L = _libs.get(path)
        if L is None:
            if not os.path.exists(path):
                raise ImportError(
                    f"{path} is missing: build it with "
                    "`python -m gated_delta_rule_87_b200.build` (nvcc, sm_100a)")
            L = ctypes.CDLL(path)
            for name, (args, res) in _SIGS.items():
                f = getattr(L, name)
                f.argtypes = args
                f.restype = res
            _libs[path] = L
    return L


def lib() -> ctypes.CDLL:
    """Load ``libgated_delta.so`` (raises if it has not been built), or the
    library selected by :func:`use_library`."""
    global _lib
    L = _load(_active_path)
    if _active_path == library_path:
        _lib = L
    return L


@contextlib.contextmanager
def use_library(path: str):
    """Route every call of this module through the library at ``path`` (for
    instance :data:`checked_library_path`) inside the ``with`` block."""
    global _active_path
    prev = _active_path
    L = _load(path)
    _active_path = path
    try:
        yield L
    finally:
        _active_path = prev


def bounds_checked() -> bool:
    """True when the active library is the bounds-checked build."""
    return bool(lib().kda_bounds_checked())


def bounds_violations() -> int:
    """Waits for the current stream and returns the out-of-bounds accesses the
    active library's kernels caught (and skipped) since the last call."""
    n = ctypes.c_uint32(0)
    _check(lib().kda_bounds_violations(_stream_handle(None, None), ctypes.byref(n)),
           "kda_bounds_violations")
    return int(n.value)


def _check(status: int, what: str):
    if status != KDA_OK:
        L = lib()
        msg = L.kda_last_error().decode() or L.kda_status_string(status).decode()
        raise KdaError(status, f"{what}: {msg}")


# --------------------------------------------------------------------------- #
# torch plumbing
# --------------------------------------------------------------------------- #
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _host_ptr(t) -> Optional[int]:
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("tensors must live in host memory")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream_handle(stream, device) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _f32(t, name):
    torch = _torch()
    if t is not None and t.dtype != torch.float32:
        raise TypeError(f"{name} must be float32")
    return t


def chunk_workspace_size(B: int, T: int, H_qk: int, H_v: int, d_k: int, d_v: int,
                         num_seqs: int, io_dtype: int, gate: str = "channel") -> int:
    L = lib()
    if gate == "channel":
        return int(L.kda_chunk_fwd_workspace_size(B, T, H_v, d_k, d_v, num_seqs, io_dtype))
    return int(L.gdn_chunk_fwd_workspace_size(B, T, H_qk, H_v, d_k, d_v, num_seqs, io_dtype))


def _alloc_workspace(nbytes: int, device):
    torch = _torch()
    # 256-byte alignment: torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _order_code(order) -> int:
    if order not in _ORDER:
        raise ValueError(f"order must be one of {sorted(_ORDER)}, got {order!r}")
    return _ORDER[order]


def _slots(state_slots, state_pool, N):
    torch = _torch()
    if state_slots is None:
        if state_pool is not None:
            raise ValueError("state_pool needs state_slots")
        return None, 0
    if state_pool is None:
        raise ValueError("state_slots needs state_pool")
    if state_slots.dtype != torch.int32 or state_slots.numel() != N:
        raise ValueError(f"state_slots must be int32 with {N} entries")
    return state_slots, state_pool.shape[0]


def _chunk_fwd(gate, q, k, v, g, beta, initial_state, cu_seqlens, output_final_state,
               o, final_state, workspace, stream, order=ERASE_THEN_DECAY, state_pool=None,
               state_slots=None):
    torch = _torch()
    if q.dim() != 4:
        raise ValueError("q, k, v must be [B, T, H, d]")
    B, T, H_qk, d_k = q.shape
    H_v, d_v = v.shape[2], v.shape[3]
    io = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share a dtype")
    _f32(g, "g"), _f32(beta, "beta"), _f32(initial_state, "initial_state")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    dev = q.device
    if o is None:
        o = torch.empty((B, T, H_v, d_v), dtype=q.dtype, device=dev)
    slots, num_slots = _slots(state_slots, state_pool, N)
    if slots is not None:
        # pool mode: read and update pool[state_slots[n]] in place
        if initial_state is not None or final_state is not None:
            raise ValueError("with state_pool, pass neither initial_state nor final_state")
        _f32(state_pool, "state_pool")
        initial_state = final_state = state_pool
    elif final_state is None and output_final_state:
        final_state = torch.empty((N, H_v, d_k, d_v), dtype=torch.float32, device=dev)
    need = chunk_workspace_size(B, T, H_qk, H_v, d_k, d_v, N if cu_seqlens is not None else 0,
                                io, gate)
    if workspace is None or workspace.numel() < need:
        workspace = _alloc_workspace(need, dev)
    L = lib()
    args_common = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(o), _ptr(initial_state),
                   _ptr(final_state), _ptr(slots), num_slots, _ptr(cu_seqlens), N]
    sh = _stream_handle(stream, dev)
    if gate == "channel":
        st = L.kda_chunk_fwd_ex(*args_common, B, T, H_v, d_k, d_v, _order_code(order), io,
                                _ptr(workspace), workspace.numel(), sh)
        _check(st, "kda_chunk_fwd_ex")
    else:
        st = L.gdn_chunk_fwd_ex(*args_common, B, T, H_qk, H_v, d_k, d_v, io, _ptr(workspace),
                                workspace.numel(), sh)
        _check(st, "gdn_chunk_fwd_ex")
    return o, final_state, workspace


def kda_chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *,
                  output_final_state: bool = True, o=None, final_state=None, workspace=None,
                  stream=None, order: str = ERASE_THEN_DECAY, state_pool=None,
                  state_slots=None):
    """KDA prefill.  q, k [B,T,H,d_k]; v [B,T,H,d_v] (bf16 or fp32); g [B,T,H,d_k]
    fp32 log-decay; beta [B,T,H] fp32; initial_state [N,H,d_k,d_v] fp32 or None;
    cu_seqlens int32 [N+1] (device) for packed sequences with B = 1.
    ``order`` places the decay after (default) or before the erase.  With
    ``state_pool`` [num_slots,H,d_k,d_v] and ``state_slots`` int32 [N], sequence
    n starts from pool[state_slots[n]] and its final state is written back
    there (slots outside the pool: start from zeros, no final state).
    Returns (o, final_state, workspace); final_state is the pool in pool mode."""
    return _chunk_fwd("channel", q, k, v, g, beta, initial_state, cu_seqlens,
                      output_final_state, o, final_state, workspace, stream, order, state_pool,
                      state_slots)


def kda_chunk_fwd_host(q, k, v, g, beta, initial_state=None, *, o, final_state=None,
                       device_buffer=None, pieces: int = 4, stream=None, device=None):
    """KDA prefill from pinned HOST tensors (dense batch; layouts as
    kda_chunk_fwd), the copies overlapped with the kernels (see the C call).
    ``o`` (and ``final_state`` if given) are host tensors the results land in
    once the stream is synchronised.  ``device_buffer`` (uint8, on the device)
    is allocated when None.  Returns the device buffer (its first bytes hold
    the status word for check_device_status)."""
    torch = _torch()
    if q.is_cuda or o.is_cuda:
        raise ValueError("kda_chunk_fwd_host takes host tensors")
    B, T, H, d_k = q.shape
    d_v = v.shape[3]
    io = _dtype_code(q)
    _f32(g, "g"), _f32(beta, "beta"), _f32(initial_state, "initial_state")
    _f32(final_state, "final_state")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    L = lib()
    need = int(L.kda_chunk_fwd_host_buffer_size(B, T, H, d_k, d_v, io, pieces))
    if device_buffer is None or device_buffer.numel() < need:
        device_buffer = torch.empty(need, dtype=torch.uint8, device=dev)
    sh = _stream_handle(stream, dev)
    hp = _host_ptr
    _check(L.kda_chunk_fwd_host(hp(q), hp(k), hp(v), hp(g), hp(beta), hp(o),
                                hp(initial_state), hp(final_state), B, T, H, d_k, d_v, io,
                                pieces, _ptr(device_buffer), device_buffer.numel(), sh),
           "kda_chunk_fwd_host")
    return device_buffer


def gdn_chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *,
                  output_final_state: bool = True, o=None, final_state=None, workspace=None,
                  stream=None, state_pool=None, state_slots=None):
    """Gated DeltaNet prefill.  q, k [B,T,H_qk,d_k]; v [B,T,H_v,d_v]; g, beta
    [B,T,H_v] fp32 (scalar log-decay per head-token).  ``state_pool`` /
    ``state_slots`` as in kda_chunk_fwd.  Returns (o, final_state, workspace)."""
    return _chunk_fwd("scalar", q, k, v, g, beta, initial_state, cu_seqlens,
                      output_final_state, o, final_state, workspace, stream, ERASE_THEN_DECAY,
                      state_pool, state_slots)


def _decode(gate, q, k, v, g, beta, state, o, stream):
    torch = _torch()
    N, H_qk, d_k = q.shape
    H_v, d_v = v.shape[1], v.shape[2]
    io = _dtype_code(q)
    _f32(g, "g"), _f32(beta, "beta"), _f32(state, "state")
    if o is None:
        o = torch.empty((N, H_v, d_v), dtype=q.dtype, device=q.device)
    L = lib()
    sh = _stream_handle(stream, q.device)
    ptrs = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(o), _ptr(state)]
    if gate == "channel":
        _check(L.kda_decode_step(*ptrs, N, H_v, d_k, d_v, io, sh), "kda_decode_step")
    else:
        _check(L.gdn_decode_step(*ptrs, N, H_qk, H_v, d_k, d_v, io, sh), "gdn_decode_step")
    return o


def _recurrent(gate, q, k, v, g, beta, state, state_slots, order, o, stream):
    torch = _torch()
    if q.dim() != 4:
        raise ValueError("q, k, v must be [N, T, H, d]")
    N, T, H_qk, d_k = q.shape
    H_v, d_v = v.shape[2], v.shape[3]
    io = _dtype_code(q)
    _f32(g, "g"), _f32(beta, "beta"), _f32(state, "state")
    slots, num_slots = _slots(state_slots, state if state_slots is not None else None, N)
    if o is None:
        o = torch.empty((N, T, H_v, d_v), dtype=q.dtype, device=q.device)
    L = lib()
    sh = _stream_handle(stream, q.device)
    ptrs = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(o), _ptr(state), _ptr(slots)]
    if gate == "channel":
        _check(L.kda_recurrent_fwd(*ptrs, num_slots, N, T, H_v, d_k, d_v, _order_code(order), io,
                                   sh), "kda_recurrent_fwd")
    else:
        _check(L.gdn_recurrent_fwd(*ptrs, num_slots, N, T, H_qk, H_v, d_k, d_v, io, sh),
               "gdn_recurrent_fwd")
    return o


def kda_recurrent_fwd(q, k, v, g, beta, state, *, state_slots=None,
                      order: str = ERASE_THEN_DECAY, o=None, stream=None):
    """T tokens for each of N sequences, token by token, state updated in place
    (read once, written once).  q, k [N,T,H,d_k]; v [N,T,H,d_v]; g [N,T,H,d_k];
    beta [N,T,H].  ``state`` is [N,H,d_k,d_v], or a pool [num_slots,H,d_k,d_v]
    indexed by ``state_slots`` (int32 [N]; a slot outside the pool is a padding
    entry: zero output, no state).  Returns o [N,T,H,d_v]."""
    return _recurrent("channel", q, k, v, g, beta, state, state_slots, order, o, stream)


def gdn_recurrent_fwd(q, k, v, g, beta, state, *, state_slots=None, o=None, stream=None):
    """Gated DeltaNet form of kda_recurrent_fwd: q, k [N,T,H_qk,d_k]; v [N,T,H_v,d_v];
    g, beta [N,T,H_v].  Returns o [N,T,H_v,d_v]."""
    return _recurrent("scalar", q, k, v, g, beta, state, state_slots, ERASE_THEN_DECAY, o,
                      stream)


def state_gather(pool, state_slots, *, out=None, stream=None):
    """out[n] = pool[state_slots[n]] (zeros for a slot outside the pool)."""
    torch = _torch()
    _f32(pool, "pool")
    N = state_slots.numel()
    _slots(state_slots, pool, N)
    _, H, d_k, d_v = pool.shape
    if out is None:
        out = torch.empty((N, H, d_k, d_v), dtype=torch.float32, device=pool.device)
    _check(lib().kda_state_gather(_ptr(pool), _ptr(state_slots), pool.shape[0], _ptr(out), N, H,
                                  d_k, d_v, _stream_handle(stream, pool.device)),
           "kda_state_gather")
    return out


def state_scatter(src, pool, state_slots, *, stream=None):
    """pool[state_slots[n]] = src[n] (skipped for a slot outside the pool)."""
    _f32(src, "src"), _f32(pool, "pool")
    N = state_slots.numel()
    _slots(state_slots, pool, N)
    _, H, d_k, d_v = pool.shape
    _check(lib().kda_state_scatter(_ptr(src), _ptr(pool), _ptr(state_slots), pool.shape[0], N, H,
                                   d_k, d_v, _stream_handle(stream, pool.device)),
           "kda_state_scatter")
    return pool


def kda_decode_step(q, k, v, g, beta, state, *, o=None, stream=None):
    """One KDA decode step; ``state`` [N,H,d_k,d_v] fp32 is updated in place.
    q, k [N,H,d_k]; v [N,H,d_v]; g [N,H,d_k]; beta [N,H].  Returns o [N,H,d_v]."""
    return _decode("channel", q, k, v, g, beta, state, o, stream)


def gdn_decode_step(q, k, v, g, beta, state, *, o=None, stream=None):
    """One Gated DeltaNet decode step (scalar gate, q/k heads shared by groups of
    v heads); ``state`` is updated in place.  Returns o [N,H_v,d_v]."""
    return _decode("scalar", q, k, v, g, beta, state, o, stream)


def trace_enable(on: bool = True) -> None:
    """Record the device time of every library kernel launch (off by default)."""
    lib().kda_trace_enable(1 if on else 0)


def trace_read(capacity: int = 4096):
    """Wait for the traced launches; return [(kernel name, ms), ...] and clear."""
    L = lib()
    stride = 64
    names = ctypes.create_string_buffer(stride * capacity)
    ms = (ctypes.c_float * capacity)()
    n = L.kda_trace_read(names, stride, ms, capacity)
    return [(names.raw[i * stride:(i + 1) * stride].split(b"\0", 1)[0].decode(), float(ms[i]))
            for i in range(n)]


def selftest_wait_timeout(workspace, max_polls: int = 16, stream=None) -> None:
    """Run one bounded on-device wait that nothing completes; it expires and
    writes KDA_DEVICE_TIMEOUT into ``workspace``'s status word (read it with
    check_device_status).  Exercises the library's expired-wait path without
    faulting or hanging the GPU."""
    L = lib()
    _check(L.kda_selftest_wait_timeout(_ptr(workspace), int(max_polls),
                                       _stream_handle(stream, workspace.device)),
           "kda_selftest_wait_timeout")


def check_device_status(workspace, stream=None) -> Tuple[int, int]:
    """Synchronise ``stream`` and read the device status word of a prefill
    workspace.  Returns (status, device_code); raises on KDA_ERR_CUDA."""
    L = lib()
    code = ctypes.c_int32(0)
    st = L.kda_check_device_status(_ptr(workspace), _stream_handle(stream, workspace.device),
                                   ctypes.byref(code))
    if st == KDA_ERR_CUDA:
        _check(st, "kda_check_device_status")
    return st, code.value
