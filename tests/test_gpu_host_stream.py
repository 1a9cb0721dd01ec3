"""kda_chunk_fwd_host: the KDA prefill from pinned host memory with the
copies overlapped.  Its pieces are prefills chained through the fp32 state,
which is what one call computes between its chunks, so its results must equal
kda_chunk_fwd's bit for bit (same kernels, same inputs), and the oracle's
within the dtype's bound."""
import numpy as np
import pytest

from gated_delta_rule_87_b200 import workloads as W
from parity import check_prefill_parity, oracle_prefill, prefill_device_inputs, tol_for

pytestmark = pytest.mark.gpu


def _host(t):
    return t.cpu().pin_memory()


@pytest.mark.parametrize("io,B,T,pieces", [("bf16", 2, 1000, 3), ("bf16", 1, 4096, 8),
                                           ("bf16", 1, 130, 64), ("f32", 2, 300, 2),
                                           ("bf16", 3, 64, 1)])
def test_streamed_prefill_equals_device_call(io, B, T, pieces):
    import torch
    import gated_delta_rule_87_b200 as gdr
    w = W.WORKLOADS["kda_prefill"].replace(B=B, T=T, H_qk=4, H_v=4, io_dtype=io, init_state=True)
    x = W.make_prefill(w, seed=40 + T)
    d = prefill_device_inputs(x)
    o_ref, s_ref, _ = gdr.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                        d["initial_state"])
    h = {k_: _host(d[k_]) for k_ in ("q", "k", "v", "g", "beta", "initial_state")}
    o = torch.empty(o_ref.shape, dtype=o_ref.dtype).pin_memory()
    sT = torch.empty(s_ref.shape, dtype=torch.float32).pin_memory()
    buf = gdr.kda_chunk_fwd_host(h["q"], h["k"], h["v"], h["g"], h["beta"], h["initial_state"],
                                 o=o, final_state=sT, pieces=pieces)
    torch.cuda.synchronize()
    st, code = gdr.check_device_status(buf)
    assert st == gdr.KDA_OK, code
    assert torch.equal(o.view(torch.int16 if io == "bf16" else torch.int32),
                       o_ref.cpu().view(torch.int16 if io == "bf16" else torch.int32))
    assert torch.equal(sT.view(torch.int32), s_ref.cpu().view(torch.int32))
    ro, rs = oracle_prefill(x)
    oo = (o.float().numpy() if io == "bf16" else o.numpy()).reshape(ro.shape)
    check_prefill_parity(f"test_streamed_prefill ({io} B={B} T={T} pieces={pieces})", oo, ro,
                         sT.numpy(), rs, x.cu_seqlens, tol_for(io))


def test_streamed_prefill_without_states_and_reused_buffer():
    import torch
    import gated_delta_rule_87_b200 as gdr
    w = W.WORKLOADS["kda_prefill"].replace(B=1, T=777, H_qk=2, H_v=2)
    x = W.make_prefill(w, seed=5)
    d = prefill_device_inputs(x)
    o_ref, _, _ = gdr.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None)
    h = {k_: _host(d[k_]) for k_ in ("q", "k", "v", "g", "beta")}
    buf = None
    for _ in range(2):  # a second call on the same device buffer overwrites everything it reads
        o = torch.full(o_ref.shape, float("nan"), dtype=o_ref.dtype).pin_memory()
        buf = gdr.kda_chunk_fwd_host(h["q"], h["k"], h["v"], h["g"], h["beta"], None, o=o,
                                     device_buffer=buf, pieces=5)
        torch.cuda.synchronize()
        assert gdr.check_device_status(buf)[0] == gdr.KDA_OK
        assert torch.equal(o.view(torch.int16), o_ref.cpu().view(torch.int16))
