"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device
memory (a host that owns all device memory in its own pool and lets no
library allocate, or a path where a cudaMalloc, which may synchronise the
device, is not allowed).  It keeps its scratch in a fixed 64 MiB array
inside the library, so it takes no workspace argument.

Checked through the C ABI on two calls in a row with different inputs and
shapes, since the shared scratch keeps the previous call's contents: each
call must equal kda_chunk_fwd (the same kernels with a caller workspace) bit
for bit, and both must match the fp64 oracle.  This file is collected last
so a stop at the first failure has run every other test first; it also
passes alone in a fresh process (its first call does the address lookup)."""
import numpy as np
import pytest

from gated_delta_rule_87_b200 import workloads as W
from parity import TOL_BF16, check_prefill_parity, oracle_prefill, prefill_device_inputs, to_host

pytestmark = pytest.mark.gpu


def _call_noalloc(d, B, T, H, stream):
    import torch
    import gated_delta_rule_87_b200 as gdr
    L = gdr.lib()
    o = torch.full((B, T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    sT = torch.full((B, H, 128, 128), float("nan"), dtype=torch.float32, device="cuda")
    ptr = lambda t: None if t is None else t.data_ptr()
    st = L.kda_chunk_fwd_noalloc(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["g"]),
                                 ptr(d["beta"]), ptr(o), ptr(d["initial_state"]), ptr(sT),
                                 None, 0, B, T, H, 128, 128, 1, stream)
    return st, o, sT


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    import gated_delta_rule_87_b200 as gdr
    stream = torch.cuda.current_stream().cuda_stream
    for seed, T in ((21, 300), (22, 197)):   # two calls in a row, different shapes and data
        w = W.WORKLOADS["kda_prefill"].replace(T=T, H_qk=4, H_v=4)
        x = W.make_prefill(w, seed=seed)
        d = prefill_device_inputs(x)
        st, o, sT = _call_noalloc(d, 1, T, 4, stream)
        assert st == gdr.KDA_OK, gdr.lib().kda_last_error()
        ro, rs, _ = gdr.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                      d["initial_state"])
        torch.cuda.synchronize()
        # same kernels, same inputs: identical bits (stale scratch would show here)
        assert torch.equal(o.view(torch.int16), ro.view(torch.int16)), f"o differs (T={T})"
        assert torch.equal(sT.view(torch.int32), rs.view(torch.int32)), f"state differs (T={T})"
        oo, os_ = oracle_prefill(x)
        check_prefill_parity(f"test_noalloc (T={T})", to_host(o).reshape(oo.shape), oo,
                             sT.cpu().numpy(), os_, x.cu_seqlens, TOL_BF16)


def test_noalloc_rejects_problems_beyond_its_scratch():
    import gated_delta_rule_87_b200 as gdr
    L = gdr.lib()
    # 128 sequences x 32 heads: a 32 KB state image per chain alone is 128 MiB.
    # The size is checked here first: the call below passes unmapped pointers
    # and must never get past the library's host-side size check.
    B, T, H = 128, 64, 32
    assert L.kda_chunk_fwd_workspace_size(B, T, H, 128, 128, 0, 1) > (64 << 20)
    fake = 1 << 16
    st = L.kda_chunk_fwd_noalloc(fake, fake, fake, fake, fake, fake * 2, None, None, None, 0,
                                 B, T, H, 128, 128, 1, None)
    assert st == gdr.KDA_ERR_WORKSPACE
    assert b"64" in L.kda_last_error() or b"67108864" in L.kda_last_error()
