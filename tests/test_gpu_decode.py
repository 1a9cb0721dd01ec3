"""Decode step on the GPU against the fp64 oracle (same seeded inputs)."""
import numpy as np
import pytest

from gated_delta_rule_87_b200 import workloads as W
from parity import RECORDS, rel_l2, to_device, to_host, tol_for

pytestmark = pytest.mark.gpu


def _run_decode(x, gate, device="cuda"):
    import torch
    import gated_delta_rule_87_b200 as gdr
    io = x.w.io_dtype
    state = to_device(x.initial_state, "f32", device)
    outs = []
    for s in range(x.w.steps):
        q = to_device(x.q[s], io, device)
        k = to_device(x.k[s], io, device)
        v = to_device(x.v[s], io, device)
        g = to_device(x.g[s], "f32", device)
        b = to_device(x.beta[s], "f32", device)
        fn = gdr.kda_decode_step if gate == "channel" else gdr.gdn_decode_step
        outs.append(to_host(fn(q, k, v, g, b, state)))
    torch.cuda.synchronize()
    return np.stack(outs), state.cpu().numpy()


def _oracle(x, chains=None):
    import oracle
    if chains is None:
        return oracle.decode_steps(x.q32, x.k32, x.v32, x.g, x.beta, x.initial_state)
    n_idx = [c[0] for c in chains]
    h_idx = [c[1] for c in chains]
    group = x.w.H_v // x.w.H_qk
    hk = [h // group for h in h_idx]
    # each sampled chain becomes its own sequence with one head
    sel = lambda a, hh: a[:, n_idx, hh][:, :, None]
    o, s = oracle.decode_steps(sel(x.q32, hk), sel(x.k32, hk), sel(x.v32, h_idx),
                               sel(x.g, h_idx), sel(x.beta, h_idx),
                               x.initial_state[n_idx, h_idx][:, None])
    return o[:, :, 0], s[:, 0]


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_kda_decode_small(io, dk, dv):
    w = W.WORKLOADS["kda_decode"].replace(N=5, H_qk=3, H_v=3, d_k=dk, d_v=dv, steps=6,
                                          io_dtype=io)
    x = W.make_decode(w, seed=1)
    o, s = _run_decode(x, "channel")
    ro, rs = _oracle(x)
    assert rel_l2(o, ro) <= tol_for(io)
    assert rel_l2(s, rs) <= 1e-4          # state arithmetic is fp32 on both input dtypes
    # the fp32 path must be far inside its bound
    if io == "f32":
        assert rel_l2(o, ro) <= 1e-5


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_gdn_decode_shared_heads(io):
    w = W.Workload(name="gdn_dec", kind="decode", gate="scalar", io_dtype=io, N=4, H_qk=2,
                   H_v=6, d_k=128, d_v=128, gate_scale=0.05, init_state=True, steps=5)
    x = W.make_decode(w, seed=2)
    o, s = _run_decode(x, "scalar")
    ro, rs = _oracle(x)
    assert rel_l2(o, ro) <= tol_for(io)
    assert rel_l2(s, rs) <= 1e-4


def test_kda_decode_full_size_sampled():
    """The full decode workload (256 sequences x 32 heads, 64 steps, in place);
    64 sampled (sequence, head) chains checked against the oracle."""
    w = W.WORKLOADS["kda_decode"]
    x = W.make_decode(w, seed=0)
    o, s = _run_decode(x, "channel")
    rng = np.random.default_rng(7)
    chains = [(int(n), int(h)) for n, h in zip(rng.integers(0, w.N, 64), rng.integers(0, w.H_v, 64))]
    ro, rs = _oracle(x, chains)
    n_idx = [c[0] for c in chains]
    h_idx = [c[1] for c in chains]
    assert np.isfinite(o).all() and np.isfinite(s).all()
    os_, ss = o[:, n_idx, h_idx], s[n_idx, h_idx]
    eo, es = rel_l2(os_, ro), rel_l2(ss, rs)
    # per chain: each sampled (sequence, head) over its 64 steps, and its state
    ec = (np.linalg.norm(os_ - ro, axis=(0, 2)) / np.linalg.norm(ro, axis=(0, 2))).max()
    esc = (np.linalg.norm((ss - rs).reshape(64, -1), axis=1)
           / np.linalg.norm(rs.reshape(64, -1), axis=1)).max()
    RECORDS.append(("test_kda_decode_full_size_sampled", eo, ec, ec, es, esc, 2e-2))
    assert eo <= 2e-2 and ec <= 2e-2, (eo, ec)
    assert es <= 1e-4 and esc <= 1e-4, (es, esc)
    assert eo <= 1e-2  # regression bound near the measured error


def test_decode_zero_batch_is_noop():
    import torch
    import gated_delta_rule_87_b200 as gdr
    z = lambda *s, dt=torch.bfloat16: torch.zeros(s, dtype=dt, device="cuda")
    q = z(0, 2, 128); v = z(0, 2, 128)
    st = z(0, 2, 128, 128, dt=torch.float32)
    o = gdr.kda_decode_step(q, q.clone(), v, z(0, 2, 128, dt=torch.float32),
                            z(0, 2, dt=torch.float32), st)
    assert o.shape == (0, 2, 128)
