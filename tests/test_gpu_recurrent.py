"""Token-by-token path (a few tokens per sequence, state read and written once)
on the GPU against the fp64 oracle, in both decay orders and with a state pool."""
import numpy as np
import pytest

from gated_delta_rule_87_b200 import workloads as W
from parity import rel_l2, to_device, to_host, tol_for

pytestmark = pytest.mark.gpu

ORDERS = ("erase_then_decay", "decay_then_erase")


def _inputs(N, T, H_qk, H_v, dk, dv, io, gate="channel", seed=0):
    w = W.Workload(name="recurrent", kind="prefill", gate=gate, io_dtype=io, B=N, T=T,
                   H_qk=H_qk, H_v=H_v, d_k=dk, d_v=dv, gate_scale=0.1, init_state=True)
    return W.make_prefill(w, seed=seed)


def _dev(x, device="cuda"):
    """[N*T, H, d] host arrays -> [N, T, H, d] device tensors."""
    w = x.w
    shp = lambda a: a.reshape((w.B, w.T) + a.shape[1:])
    return dict(q=to_device(shp(x.q), w.io_dtype, device), k=to_device(shp(x.k), w.io_dtype, device),
                v=to_device(shp(x.v), w.io_dtype, device), g=to_device(shp(x.g), "f32", device),
                beta=to_device(shp(x.beta), "f32", device))


def _oracle(x, order="erase_then_decay"):
    import oracle
    return oracle.gated_delta(x.q32, x.k32, x.v32, x.g, x.beta, x.initial_state,
                              x.cu_seqlens.astype(np.int64), order=order)


def _recurrent(x, state, order="erase_then_decay", slots=None):
    import torch
    import gated_delta_rule_87_b200 as gdr
    d = _dev(x)
    if x.w.gate == "channel":
        o = gdr.kda_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], state,
                                  state_slots=slots, order=order)
    else:
        o = gdr.gdn_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], state,
                                  state_slots=slots)
    torch.cuda.synchronize()
    return to_host(o).reshape(x.total_tokens, x.w.H_v, x.w.d_v)


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("T", [1, 2, 7, 16, 64])
def test_kda_tokens_per_sequence(order, io, T):
    x = _inputs(N=3, T=T, H_qk=2, H_v=2, dk=128, dv=128, io=io, seed=T)
    state = to_device(x.initial_state, "f32")
    o = _recurrent(x, state, order)
    ro, rs = _oracle(x, order)
    assert rel_l2(o, ro) <= tol_for(io)
    assert rel_l2(state.cpu().numpy(), rs) <= 1e-4
    if io == "f32":
        assert rel_l2(o, ro) <= 1e-5


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_kda_tokens_head_sizes(order, dk, dv):
    x = _inputs(N=2, T=9, H_qk=3, H_v=3, dk=dk, dv=dv, io="f32", seed=dk + dv)
    state = to_device(x.initial_state, "f32")
    o = _recurrent(x, state, order)
    ro, rs = _oracle(x, order)
    assert rel_l2(o, ro) <= 1e-5
    assert rel_l2(state.cpu().numpy(), rs) <= 1e-5


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_gdn_tokens_shared_heads(io):
    x = _inputs(N=4, T=12, H_qk=2, H_v=6, dk=128, dv=128, io=io, gate="scalar", seed=5)
    state = to_device(x.initial_state, "f32")
    o = _recurrent(x, state)
    ro, rs = _oracle(x)
    assert rel_l2(o, ro) <= tol_for(io)
    assert rel_l2(state.cpu().numpy(), rs) <= 1e-4


def test_tokens_equal_repeated_single_steps():
    """T tokens in one call = T calls of one token each (the same arithmetic per
    token, so the two agree to rounding)."""
    import torch
    import gated_delta_rule_87_b200 as gdr
    x = _inputs(N=5, T=6, H_qk=2, H_v=2, dk=128, dv=128, io="bf16", seed=9)
    d = _dev(x)
    s_multi = to_device(x.initial_state, "f32")
    o_multi = gdr.kda_recurrent_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], s_multi)
    s_step = to_device(x.initial_state, "f32")
    outs = []
    for t in range(x.w.T):
        sl = lambda a: a[:, t:t + 1].contiguous()
        outs.append(gdr.kda_recurrent_fwd(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]),
                                          sl(d["beta"]), s_step))
    o_step = torch.cat(outs, dim=1)
    torch.cuda.synchronize()
    assert rel_l2(to_host(o_multi), to_host(o_step)) <= 1e-6
    assert rel_l2(s_multi.cpu().numpy(), s_step.cpu().numpy()) <= 1e-6


@pytest.mark.parametrize("order", ORDERS)
def test_state_pool_slots_and_padding(order):
    """Sequence n uses pool[slots[n]]; a slot outside the pool is a padding
    entry (zero output, no state touched); slots nobody names stay bit-exact."""
    import torch
    x = _inputs(N=4, T=5, H_qk=2, H_v=2, dk=128, dv=128, io="bf16", seed=11)
    num_slots = 7
    slots = np.array([5, 0, -1, 3], dtype=np.int32)
    rng = np.random.default_rng(3)
    pool0 = (0.02 * rng.standard_normal((num_slots, 2, 128, 128))).astype(np.float32)
    live = slots >= 0
    for n in np.nonzero(live)[0]:
        pool0[slots[n]] = x.initial_state[n]
    pool = to_device(pool0, "f32")
    o = _recurrent(x, pool, order, slots=torch.from_numpy(slots).cuda())
    ro, rs = _oracle(x, order)
    o = o.reshape(4, 5, 2, 128)
    ro = ro.reshape(4, 5, 2, 128)
    assert rel_l2(o[live], ro[live]) <= 2e-2
    assert np.all(o[~live] == 0)
    p = pool.cpu().numpy()
    for n in np.nonzero(live)[0]:
        assert rel_l2(p[slots[n]], rs[n]) <= 1e-4
    untouched = sorted(set(range(num_slots)) - set(slots[live].tolist()))
    assert np.array_equal(p[untouched], pool0[untouched])


def test_slot_past_pool_end_is_padding():
    import torch
    x = _inputs(N=2, T=3, H_qk=1, H_v=1, dk=64, dv=64, io="f32", seed=12)
    pool0 = np.ones((2, 1, 64, 64), dtype=np.float32)
    pool = to_device(pool0, "f32")
    slots = torch.tensor([1, 2], dtype=torch.int32, device="cuda")  # 2 is past the end
    o = _recurrent(x, pool, slots=slots).reshape(2, 3, 1, 64)
    assert np.all(o[1] == 0)
    assert np.isfinite(o[0]).all() and np.any(o[0] != 0)
    assert np.array_equal(pool.cpu().numpy()[0], pool0[0])


def test_zero_tokens_is_noop():
    import torch
    import gated_delta_rule_87_b200 as gdr
    z = lambda *s, dt=torch.bfloat16: torch.zeros(s, dtype=dt, device="cuda")
    st = torch.ones((3, 2, 128, 128), dtype=torch.float32, device="cuda")
    o = gdr.kda_recurrent_fwd(z(3, 0, 2, 128), z(3, 0, 2, 128), z(3, 0, 2, 128),
                              z(3, 0, 2, 128, dt=torch.float32), z(3, 0, 2, dt=torch.float32), st)
    torch.cuda.synchronize()
    assert o.shape == (3, 0, 2, 128)
    assert bool((st == 1).all())
