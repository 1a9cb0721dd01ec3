"""Failure detection on the GPU without a fault: an on-device wait that never
completes expires after its bound, the kernel writes KDA_DEVICE_TIMEOUT into the
workspace status word and returns, and the context stays usable."""
import numpy as np
import pytest

from gated_delta_rule_87_b200 import workloads as W
from parity import oracle_prefill, prefill_device_inputs, rel_l2, to_host

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_survives():
    import time
    import torch
    import gated_delta_rule_87_b200 as gdr
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    gdr.selftest_wait_timeout(ws, max_polls=16)
    st, code = gdr.check_device_status(ws)
    assert time.perf_counter() - t0 < 5.0
    assert st == gdr.KDA_ERR_DEVICE_CHECK and code == gdr.KDA_DEVICE_TIMEOUT
    # the same context runs a prefill correctly afterwards, with a clean status
    w = W.WORKLOADS["kda_prefill"].replace(T=100, H_qk=2, H_v=2)
    x = W.make_prefill(w, seed=21)
    d = prefill_device_inputs(x)
    o, sT, ws2 = gdr.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"])
    torch.cuda.synchronize()
    assert gdr.check_device_status(ws2) == (gdr.KDA_OK, gdr.KDA_DEVICE_OK)
    ro, rs = oracle_prefill(x)
    assert rel_l2(to_host(o).reshape(ro.shape), ro) <= 2e-2
    assert rel_l2(sT.cpu().numpy(), rs) <= 2e-2
    # and the status word of the self-test's buffer is reset by the next self-test
    gdr.selftest_wait_timeout(ws, max_polls=1)
    assert gdr.check_device_status(ws) == (gdr.KDA_ERR_DEVICE_CHECK, gdr.KDA_DEVICE_TIMEOUT)
