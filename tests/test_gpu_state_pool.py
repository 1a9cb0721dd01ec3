"""Serving state pool: prefill reading and writing pool slots in place, the
slot gather/scatter copies, and a later turn continuing from the pool."""
import numpy as np
import pytest

from gated_delta_rule_87_b200 import workloads as W
from parity import prefill_device_inputs, rel_l2, to_device, to_host, tol_for

pytestmark = pytest.mark.gpu


def _pool_with(x, slots, num_slots, seed=0):
    """A pool of random states with sequence n's initial state at slots[n]."""
    w = x.w
    rng = np.random.default_rng(seed)
    pool = (0.02 * rng.standard_normal((num_slots, w.H_v, w.d_k, w.d_v))).astype(np.float32)
    for n, sl in enumerate(slots):
        if 0 <= sl < num_slots:
            pool[sl] = x.initial_state[n]
    return pool


def _oracle(x, s0, order="erase_then_decay"):
    import oracle
    return oracle.gated_delta(x.q32, x.k32, x.v32, x.g, x.beta, s0,
                              x.cu_seqlens.astype(np.int64), order=order)


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("gate", ["channel", "scalar"])
def test_prefill_updates_pool_in_place(io, gate):
    import torch
    import gated_delta_rule_87_b200 as gdr
    base = W.WORKLOADS["kda_varlen" if gate == "channel" else "gdn_long"]
    w = base.replace(H_qk=2, H_v=2 if gate == "channel" else 4, io_dtype=io, init_state=True,
                     varlen=1)
    x = W.make_prefill(w, seed=31, lengths=[100, 0, 64, 230, 17])
    slots = np.array([6, 2, -1, 0, 9], dtype=np.int32)  # -1 and 9 (>= num_slots): no slot
    num_slots = 8
    pool0 = _pool_with(x, slots, num_slots)
    pool = to_device(pool0, "f32")
    d = prefill_device_inputs(x)
    fn = gdr.kda_chunk_fwd if gate == "channel" else gdr.gdn_chunk_fwd
    o, fin, ws = fn(d["q"], d["k"], d["v"], d["g"], d["beta"], None, d["cu_seqlens"],
                    state_pool=pool, state_slots=torch.from_numpy(slots).cuda())
    torch.cuda.synchronize()
    assert gdr.check_device_status(ws)[0] == gdr.KDA_OK
    assert fin is pool
    # sequences without a slot start from zeros
    s0 = x.initial_state.copy()
    live = (slots >= 0) & (slots < num_slots)
    s0[~live] = 0.0
    ro, rs = _oracle(x, s0)
    o = to_host(o).reshape(ro.shape)
    tol = tol_for(io)
    assert rel_l2(o, ro) <= tol
    p = pool.cpu().numpy()
    for n in np.nonzero(live)[0]:
        assert rel_l2(p[slots[n]], rs[n]) <= tol
    untouched = sorted(set(range(num_slots)) - set(slots[live].tolist()))
    assert np.array_equal(p[untouched], pool0[untouched])


def test_empty_prefill_leaves_pool_unchanged():
    import torch
    import gated_delta_rule_87_b200 as gdr
    pool = torch.randn((4, 2, 128, 128), dtype=torch.float32, device="cuda")
    before = pool.clone()
    z = lambda *s, dt=torch.bfloat16: torch.zeros(s, dtype=dt, device="cuda")
    gdr.kda_chunk_fwd(z(2, 0, 2, 128), z(2, 0, 2, 128), z(2, 0, 2, 128),
                      z(2, 0, 2, 128, dt=torch.float32), z(2, 0, 2, dt=torch.float32),
                      state_pool=pool, state_slots=torch.tensor([3, 1], dtype=torch.int32,
                                                                device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(pool, before)


def test_gather_scatter_are_exact_copies():
    import torch
    import gated_delta_rule_87_b200 as gdr
    pool = torch.randn((6, 3, 64, 128), dtype=torch.float32, device="cuda")
    slots = torch.tensor([4, -1, 0, 7], dtype=torch.int32, device="cuda")  # -1, 7: no slot
    out = gdr.state_gather(pool, slots)
    torch.cuda.synchronize()
    assert torch.equal(out[0], pool[4]) and torch.equal(out[2], pool[0])
    assert bool((out[1] == 0).all()) and bool((out[3] == 0).all())
    src = torch.randn((4, 3, 64, 128), dtype=torch.float32, device="cuda")
    before = pool.clone()
    gdr.state_scatter(src, pool, slots)
    torch.cuda.synchronize()
    assert torch.equal(pool[4], src[0]) and torch.equal(pool[0], src[2])
    for sl in (1, 2, 3, 5):
        assert torch.equal(pool[sl], before[sl])


@pytest.mark.parametrize("order", ["erase_then_decay", "decay_then_erase"])
def test_next_turn_continues_from_pool(order):
    """Turn 1: prefill writes each conversation's state into its slot.  Turn 2:
    a few tokens per conversation through the token-by-token path, read from
    the same slots.  Together they equal the oracle over both turns."""
    import torch
    import gated_delta_rule_87_b200 as gdr
    N, T1, T2, H = 3, 150, 4, 2
    w = W.WORKLOADS["kda_prefill"].replace(B=N, T=T1 + T2, H_qk=H, H_v=H, init_state=True)
    x = W.make_prefill(w, seed=41)
    ro, rs = _oracle(x, x.initial_state, order)
    slots = torch.tensor([2, 0, 3], dtype=torch.int32, device="cuda")
    pool = torch.zeros((4, H, 128, 128), dtype=torch.float32, device="cuda")
    gdr.state_scatter(to_device(x.initial_state, "f32"), pool, slots)
    d = prefill_device_inputs(x)  # [N, T1+T2, H, d]
    first = lambda a: a[:, :T1].contiguous()
    second = lambda a: a[:, T1:].contiguous()
    o1, _, _ = gdr.kda_chunk_fwd(first(d["q"]), first(d["k"]), first(d["v"]), first(d["g"]),
                                 first(d["beta"]), order=order, state_pool=pool,
                                 state_slots=slots)
    o2 = gdr.kda_recurrent_fwd(second(d["q"]), second(d["k"]), second(d["v"]), second(d["g"]),
                               second(d["beta"]), pool, state_slots=slots, order=order)
    torch.cuda.synchronize()
    o = torch.cat([o1, o2], dim=1)
    assert rel_l2(to_host(o).reshape(ro.shape), ro) <= 2e-2
    fin = gdr.state_gather(pool, slots)
    assert rel_l2(fin.cpu().numpy(), rs) <= 2e-2
