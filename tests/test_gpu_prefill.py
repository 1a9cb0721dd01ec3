"""Chunked prefill on the GPU against the fp64 oracle (same seeded inputs)."""
import os

import numpy as np
import pytest

from gated_delta_rule_87_b200 import workloads as W
from parity import (check_prefill_parity, oracle_prefill, prefill_device_inputs, rel_l2, to_host,
                    tol_for)

pytestmark = pytest.mark.gpu

# NaN guard bands around o and the final state: an out-of-range store by a
# kernel (a ragged tail row, a packed sequence's neighbour) overwrites them.
GUARD_TOKENS = 3
GUARD_FLOATS = 4096


def _label():
    return os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0].split("::")[-1]


def _run(x, **kw):
    import torch
    import gated_delta_rule_87_b200 as gdr
    d = prefill_device_inputs(x)
    fn = gdr.kda_chunk_fwd if x.w.gate == "channel" else gdr.gdn_chunk_fwd
    B, T = d["q"].shape[:2]
    row = x.w.H_v * x.w.d_v
    g_o = GUARD_TOKENS * row
    obuf = torch.full((B * T * row + 2 * g_o,), float("nan"), dtype=d["q"].dtype, device="cuda")
    o = obuf[g_o:g_o + B * T * row].view(B, T, x.w.H_v, x.w.d_v)
    n_state = x.num_seqs * x.w.H_v * x.w.d_k * x.w.d_v
    sbuf = torch.full((n_state + 2 * GUARD_FLOATS,), float("nan"), dtype=torch.float32,
                      device="cuda")
    sT = sbuf[GUARD_FLOATS:GUARD_FLOATS + n_state].view(x.num_seqs, x.w.H_v, x.w.d_k, x.w.d_v)
    o, sT, ws = fn(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"],
                   d["cu_seqlens"], o=o, final_state=sT, **kw)
    torch.cuda.synchronize()
    st, code = gdr.check_device_status(ws)
    assert st == gdr.KDA_OK, code
    for buf, gsz in ((obuf, g_o), (sbuf, GUARD_FLOATS)):
        assert torch.isnan(buf[:gsz]).all() and torch.isnan(buf[-gsz:]).all(), \
            "a kernel wrote outside o or final_state"
    o = to_host(o).reshape(x.total_tokens, x.w.H_v, x.w.d_v)
    return o, sT.cpu().numpy()


def _check(x, heads=None, tol=None, regress=None, **kw):
    o, sT = _run(x, **kw)
    ro, rs = oracle_prefill(x, heads, **kw)
    if heads is not None:
        o, sT = o[:, heads], sT[:, heads]
    tol = tol or tol_for(x.w.io_dtype)
    errs = check_prefill_parity(_label(), o, ro, sT, rs, x.cu_seqlens, tol, regress)
    return errs[0], errs[3]


def test_gdn_small_fp32_workload():
    """All-fp32 Gated DeltaNet, B=1 H=2 T=128 d=64, against the 1e-4 bound."""
    x = W.make_prefill(W.WORKLOADS["gdn_small_f32"], seed=0)
    _check(x)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 17, 63, 64, 65, 130, 257])
def test_kda_ragged_lengths(io, T):
    w = W.WORKLOADS["kda_prefill"].replace(T=T, H_qk=2, H_v=2, io_dtype=io)
    _check(W.make_prefill(w, seed=T))


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_kda_head_sizes(dk, dv):
    for io in ("f32", "bf16"):
        w = W.WORKLOADS["kda_prefill"].replace(T=200, H_qk=2, H_v=2, d_k=dk, d_v=dv, io_dtype=io)
        _check(W.make_prefill(w, seed=3))


def test_kda_dense_batch():
    w = W.WORKLOADS["kda_prefill"].replace(B=3, T=150, H_qk=2, H_v=2)
    _check(W.make_prefill(w, seed=4))


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_kda_packed_with_empty_sequences(io):
    w = W.WORKLOADS["kda_varlen"].replace(H_qk=2, H_v=2, io_dtype=io, init_state=True)
    x = W.make_prefill(w, seed=5, lengths=[70, 0, 1, 128, 0, 200])
    _check(x)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_gdn_shared_heads(io):
    w = W.WORKLOADS["gdn_long"].replace(T=300, H_qk=2, H_v=4, io_dtype=io, init_state=True)
    _check(W.make_prefill(w, seed=6))


@pytest.mark.parametrize("gate,scale", [("channel", 1.0), ("scalar", 1.0), ("scalar", 4.0)])
def test_strong_decay(gate, scale):
    """Strong gates: a per-token log-decay of about -0.7 x scale (up to ~ -5 x
    scale), so in-chunk cumulative decays reach e^{-40 scale} and the factors
    taken at a token and at the token before it differ by e^{g}, far beyond the
    tolerance.  The per-channel path's sub-chunk anchors and the scalar path's
    elementwise factors both have to keep every product finite and right."""
    base = "kda_prefill" if gate == "channel" else "gdn_long"
    w = W.WORKLOADS[base].replace(T=200, H_qk=2, H_v=2 if gate == "channel" else 4,
                                  gate_scale=scale, init_state=True)
    _check(W.make_prefill(w, seed=13))


@pytest.mark.parametrize("scale,order,mixed", [(1.5, "erase_then_decay", True),
                                               (2.0, "decay_then_erase", True),
                                               (4.0, "erase_then_decay", False),
                                               (8.0, "erase_then_decay", False)])
def test_kda_steep_decays(scale, order, mixed):
    """Steep per-channel decays on the bf16 tensor-core path.  The Gram scales
    its operands by up to the inverse decay product of 32 tokens; a chunk with
    a 16-token log-decay sum below -32 in some channel (so that a 32-token one
    could fall below -64 and push the operands past the fp32/bf16 range) has
    its Grams computed exactly instead.  At scales 1.5 and 2 both kinds of
    chunk occur in one call; at 4 and 8 (per-token log-decays down to -16 and
    -33) every chunk takes the exact Gram."""
    w = W.WORKLOADS["kda_prefill"].replace(T=200, H_qk=2, H_v=2, gate_scale=scale,
                                           init_state=True)
    x = W.make_prefill(w, seed=17)
    # sub-chunk sums of the log-decay per (16-token sub-chunk, head, channel)
    gp = np.zeros((256,) + x.g.shape[1:], np.float64)
    gp[:200] = x.g
    sums = gp.reshape(16, 16, *x.g.shape[1:]).sum(axis=1)
    steep = (sums < -32.0).any(axis=(-1,)).reshape(4, 4, -1).any(axis=1)  # per (chunk, head)
    assert steep.any() and (not steep.all()) == mixed
    if not mixed:
        assert x.g.min() <= -15.0
    _check(x, order=order)


def test_gdn_unshared_heads():
    """Scalar gate with as many q/k heads as v heads (no sharing), ragged length."""
    w = W.WORKLOADS["gdn_long"].replace(T=150, H_qk=3, H_v=3, init_state=True, gate_scale=0.3)
    _check(W.make_prefill(w, seed=16))


def test_gdn_packed_sequences():
    """Scalar gate, packed sequences (empty, one-token, chunk-aligned and
    ragged): a chunk's rows past its length hold the next sequence's tokens."""
    w = W.WORKLOADS["gdn_long"].replace(H_qk=2, H_v=4, init_state=True, gate_scale=0.5)
    _check(W.make_prefill(w, seed=14, lengths=[70, 0, 1, 128, 0, 200, 63, 65]))


def test_gdn_dense_batch_ragged_tail():
    """Scalar gate, B = 3 dense sequences of 100 tokens: each sequence's last
    chunk reads the next sequence's first 28 tokens as its rows 36..63."""
    w = W.WORKLOADS["gdn_long"].replace(B=3, T=100, H_qk=2, H_v=4, init_state=True,
                                        gate_scale=0.5)
    _check(W.make_prefill(w, seed=15))


def test_no_initial_state_no_final_state():
    import torch
    import gated_delta_rule_87_b200 as gdr
    w = W.WORKLOADS["kda_prefill"].replace(T=100, H_qk=2, H_v=2, init_state=False)
    x = W.make_prefill(w, seed=8)
    d = prefill_device_inputs(x)
    o, sT, _ = gdr.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None,
                                 output_final_state=False)
    torch.cuda.synchronize()
    assert sT is None
    ro, _ = oracle_prefill(x)
    assert rel_l2(to_host(o).reshape(ro.shape), ro) <= 2e-2


def test_split_prefill_carries_state():
    """prefill(T1) then prefill(T2) from its final state == prefill(T1 + T2)."""
    import torch
    import gated_delta_rule_87_b200 as gdr
    w = W.WORKLOADS["kda_prefill"].replace(T=320, H_qk=2, H_v=2)
    x = W.make_prefill(w, seed=9)
    d = prefill_device_inputs(x)
    o, s, _ = gdr.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"])
    cut = 137
    part = lambda t, a, b: t[:, a:b].contiguous()
    o1, s1, _ = gdr.kda_chunk_fwd(*(part(d[n], 0, cut) for n in ("q", "k", "v", "g", "beta")),
                                  d["initial_state"])
    o2, s2, _ = gdr.kda_chunk_fwd(*(part(d[n], cut, 320) for n in ("q", "k", "v", "g", "beta")),
                                  s1)
    torch.cuda.synchronize()
    full = to_host(o)
    split = np.concatenate([to_host(o1), to_host(o2)], axis=1)
    assert rel_l2(split, full) <= 1e-2
    assert rel_l2(s2.cpu().numpy(), s.cpu().numpy()) <= 1e-2


def test_decode_after_prefill_matches_longer_prefill():
    """A prefill of T tokens followed by n decode steps equals one prefill of
    T + n tokens (the state is the only carrier of the past)."""
    import torch
    import gated_delta_rule_87_b200 as gdr
    w = W.WORKLOADS["kda_prefill"].replace(T=96, H_qk=2, H_v=2)
    x = W.make_prefill(w, seed=10)
    d = prefill_device_inputs(x)
    T0 = 80
    part = lambda t, a, b: t[:, a:b].contiguous()
    _, s, _ = gdr.kda_chunk_fwd(*(part(d[n], 0, T0) for n in ("q", "k", "v", "g", "beta")),
                                d["initial_state"])
    outs = []
    for t in range(T0, 96):
        sl = lambda n: d[n][0, t].contiguous().unsqueeze(0)
        outs.append(to_host(gdr.kda_decode_step(sl("q"), sl("k"), sl("v"), sl("g"), sl("beta"), s)))
    torch.cuda.synchronize()
    ro, rs = oracle_prefill(x)
    assert rel_l2(np.concatenate(outs, axis=0), ro[T0:]) <= 2e-2
    assert rel_l2(s.cpu().numpy(), rs) <= 2e-2


def test_invalid_cu_seqlens_is_reported_on_device():
    import torch
    import gated_delta_rule_87_b200 as gdr
    w = W.WORKLOADS["kda_varlen"].replace(H_qk=2, H_v=2)
    x = W.make_prefill(w, seed=11, lengths=[64, 64])
    d = prefill_device_inputs(x)
    bad = torch.tensor([0, 80, 64], dtype=torch.int32, device="cuda")  # decreasing
    o = torch.full_like(d["v"], float("nan"))
    _, _, ws = gdr.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, bad, o=o)
    st, code = gdr.check_device_status(ws)
    assert st == gdr.KDA_ERR_DEVICE_CHECK and code == 1


# ----------------------------------------------------------------------------
# the full workloads (the bench's launch configuration), sampled where the
# oracle would take long
# ----------------------------------------------------------------------------
def test_kda_prefill_full_workload():
    x = W.make_prefill(W.WORKLOADS["kda_prefill"], seed=0)
    _check(x, regress=1e-2)


def test_kda_varlen_full_workload_sampled_heads():
    x = W.make_prefill(W.WORKLOADS["kda_varlen"], seed=0)
    assert list(np.diff(x.cu_seqlens)) == [14090, 10808, 8875, 5168, 5752, 1653, 2179, 1277]
    # eight heads: every quarter of the head range, both ends
    _check(x, heads=[0, 5, 9, 13, 18, 22, 27, 31], regress=1e-2)


def test_gdn_long_full_workload_sampled_heads():
    x = W.make_prefill(W.WORKLOADS["gdn_long"], seed=0)
    # eight v-heads: both v-heads of q/k heads 0 and 15, and four q/k heads between
    _check(x, heads=[0, 1, 9, 14, 17, 22, 30, 31], regress=1e-2)


@pytest.mark.parametrize("nseq", [8, 20])
def test_kda_column_slice_widths(nseq):
    """The scan splits each (sequence, v-head) state into 32-column slices (4
    CTAs) while the chains fit on the SMs in one wave, else 64-column slices
    (2 CTAs): both widths must agree with the oracle.  With 2 heads, 8
    sequences give 64 four-way chains (narrow); 20 give 160 > 148 SMs (wide)."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert (nseq * 2 * 4 <= sms) == (nseq == 8)
    w = W.WORKLOADS["kda_varlen"].replace(H_qk=2, H_v=2, init_state=True)
    rng = np.random.default_rng(12 + nseq)
    lengths = [int(x) for x in rng.integers(1, 200, nseq)]
    _check(W.make_prefill(w, seed=12, lengths=lengths))
