"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each ``pin_*`` function runs the oracle (optionally with a planted mistake,
``mut``) and returns ``(ok, detail)``.  ``test_oracle_pins.py`` requires every
pin to hold for the real operator and at least one pin to fail for every
planted mistake.

Sources of the pinned facts (all on the thethings.ai page "The argument, in
one page", table "Everything, in one table", unless noted):
  * rows "Linear attention", "Delta rule", "Gated DeltaNet", "KDA": the update
    rules, which nest (KDA with equal channels is Gated DeltaNet; alpha = 1 is
    the delta rule; no erase and beta = 1 is linear attention);
  * row "Delta rule", eviction column: the erase removes exactly what the key
    held -- with a unit key and beta = 1 the recall k^T S equals v^T;
  * paragraph "One operation, three axes": capacity of about d separable
    facts, because R^d has only d orthogonal directions;
  * row "Chunkwise / WY": the recurrence itself is unchanged by how it is
    computed, so state carried across calls must equal one long call
    (inferencex.semianalysis.com "Linear attention", "Why it matters": the
    state is the only carrier of the past).
"""
from __future__ import annotations

import numpy as np

import oracle
from oracle.brute import transition_products

from conftest import load_golden

RNG_SEED = 1234


def _rng(tag: int = 0):
    return np.random.default_rng(RNG_SEED + tag)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _problem(rng, T=6, H_qk=1, H_v=1, d_k=5, d_v=3, gate="channel", g_scale=0.3,
             unit_keys=False):
    q = rng.standard_normal((T, H_qk, d_k))
    k = rng.standard_normal((T, H_qk, d_k))
    if unit_keys:
        k = _unit(k)
    v = rng.standard_normal((T, H_v, d_v))
    if gate == "channel":
        g = -g_scale * rng.random((T, H_v, d_k))
    else:
        g = -g_scale * rng.random((T, H_v))
    beta = rng.random((T, H_v))
    s0 = rng.standard_normal((1, H_v, d_k, d_v))
    return q, k, v, g, beta, s0


def _run(q, k, v, g, beta, s0, mut, **kw):
    return oracle.gated_delta(q, k, v, g, beta, s0, mutation=mut, threads=1, **kw)


def _close(a, b, tol):
    err = float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) if np.size(a) else 0.0
    return err <= tol, err


# --------------------------------------------------------------------------- #
def pin_state_constant_without_write_or_decay(mut="none"):
    """beta = 0 and g = 0: nothing is erased, written or forgotten, so
    S_t = S_0 and o_t = S_0^T q_t for every t."""
    rng = _rng(1)
    q, k, v, g, beta, s0 = _problem(rng, T=7)
    g[:] = 0.0
    beta[:] = 0.0
    ok = True
    det = []
    for order in ("erase_then_decay", "decay_then_erase"):
        o, sT = _run(q, k, v, g, beta, s0, mut, order=order)
        exp_o = np.einsum("tc,cj->tj", q[:, 0], s0[0, 0])
        a, e1 = _close(o[:, 0], exp_o, 1e-13)
        b, e2 = _close(sT, s0, 0.0)
        ok &= a and b
        det.append(f"{order}: o err {e1:.2e}, state err {e2:.2e}")
    return ok, "; ".join(det)


def pin_pure_decay_closed_form(mut="none"):
    """beta = 0: S_t = Diag(exp(sum_{s<=t} g_s)) S_0 (row i decays by its own
    channel), for the per-channel and the scalar gate."""
    rng = _rng(2)
    ok = True
    det = []
    for gate in ("channel", "scalar"):
        q, k, v, g, beta, s0 = _problem(rng, T=6, gate=gate, g_scale=0.7)
        beta[:] = 0.0
        o, sT = _run(q, k, v, g, beta, s0, mut)
        G = np.cumsum(g[:, 0], axis=0)                  # [T, d_k] or [T]
        if gate == "scalar":
            G = np.repeat(G[:, None], q.shape[2], axis=1)
        St = np.exp(G)[:, :, None] * s0[0, 0][None]     # [T, d_k, d_v]
        exp_o = np.einsum("tc,tcj->tj", q[:, 0], St)
        a, e1 = _close(o[:, 0], exp_o, 1e-13)
        b, e2 = _close(sT[0, 0], St[-1], 1e-13)
        ok &= a and b
        det.append(f"{gate}: o err {e1:.2e}, state err {e2:.2e}")
    return ok, "; ".join(det)


def pin_one_hot_gate_indexing(mut="none"):
    """g = 0 except g[t0, c] = -1, beta = 0: row c of the state is multiplied by
    exp(-1) from token t0 on (the gate acts at its own token) and no other
    element ever changes."""
    rng = _rng(3)
    q, k, v, g, beta, s0 = _problem(rng, T=6, d_k=5, d_v=3)
    g[:] = 0.0
    beta[:] = 0.0
    t0, c = 3, 1
    g[t0, 0, c] = -1.0
    o, sT = _run(q, k, v, g, beta, s0, mut)
    e = np.exp(-1.0)
    St = np.repeat(s0[0, 0][None], 6, axis=0)
    St[t0:, c, :] *= e
    exp_o = np.einsum("tc,tcj->tj", q[:, 0], St)
    a, e1 = _close(o[:, 0], exp_o, 1e-14)
    rows = [i for i in range(5) if i != c]
    b = np.array_equal(sT[0, 0][rows], s0[0, 0][rows])
    cc, e3 = _close(sT[0, 0][c], e * s0[0, 0][c], 1e-15)
    return a and b and cc, f"o err {e1:.2e}, other rows exact {b}, row c err {e3:.2e}"


def pin_recall_identity(mut="none"):
    """g = 0, beta = 1, unit keys: after token t, k_t^T S_t = v_t^T (the erase
    removes what k_t held, the write puts v_t there).  With q_t = k_t the
    readout (after the update) therefore returns v_t."""
    rng = _rng(4)
    q, k, v, g, beta, s0 = _problem(rng, T=6, unit_keys=True)
    g[:] = 0.0
    beta[:] = 1.0
    worst = 0.0
    for t in range(1, 7):
        _, St = _run(q[:t], k[:t], v[:t], g[:t], beta[:t], s0, mut)
        rec = k[t - 1, 0] @ St[0, 0]
        worst = max(worst, float(np.max(np.abs(rec - v[t - 1, 0]))))
    o, _ = _run(k.copy(), k, v, g, beta, s0, mut)      # q_t = k_t
    e2 = float(np.max(np.abs(o[:, 0] - v[:, 0])))
    return worst < 1e-12 and e2 < 1e-12, f"recall err {worst:.2e}, readout err {e2:.2e}"


def pin_orthonormal_capacity(mut="none"):
    """g = 0, beta = 1, m <= d_k orthonormal keys: after all m writes every key
    still recalls its own value (d orthogonal directions hold d facts).  With
    d_k + 1 unit keys the earlier recalls are no longer exact."""
    rng = _rng(5)
    d_k, d_v = 6, 4
    Qm, _ = np.linalg.qr(rng.standard_normal((d_k, d_k)))
    keys = Qm.T[:, None, :]                             # [m, 1, d_k], orthonormal rows
    m = d_k
    v = rng.standard_normal((m, 1, d_v))
    g = np.zeros((m, 1, d_k))
    beta = np.ones((m, 1))
    s0 = rng.standard_normal((1, 1, d_k, d_v))
    _, S = _run(keys, keys, v, g, beta, s0, mut)
    rec = keys[:, 0] @ S[0, 0]
    e1 = float(np.max(np.abs(rec - v[:, 0])))
    # one key too many: interference
    k2 = _unit(rng.standard_normal((d_k + 1, 1, d_k)))
    v2 = rng.standard_normal((d_k + 1, 1, d_v))
    _, S2 = _run(k2, k2, v2, np.zeros((d_k + 1, 1, d_k)), np.ones((d_k + 1, 1)),
                 np.zeros((1, 1, d_k, d_v)), mut)
    rec2 = k2[:-1, 0] @ S2[0, 0]
    e2 = float(np.max(np.abs(rec2 - v2[:-1, 0])))
    return e1 < 1e-12 and e2 > 1e-3, f"orthonormal recall err {e1:.2e}, overfull err {e2:.2e}"


def pin_linear_attention(mut="none"):
    """Erase term removed, g = 0, beta = 1: S_t = S_0 + sum_{i<=t} k_i v_i^T
    (row "Linear attention": S += k^T v)."""
    rng = _rng(6)
    q, k, v, g, beta, s0 = _problem(rng, T=5)
    g[:] = 0.0
    beta[:] = 1.0
    o, sT = _run(q, k, v, g, beta, s0, mut, rule="linear")
    St = s0[0, 0][None] + np.cumsum(np.einsum("tc,tj->tcj", k[:, 0], v[:, 0]), axis=0)
    exp_o = np.einsum("tc,tcj->tj", q[:, 0], St)
    a, e1 = _close(o[:, 0], exp_o, 1e-12)
    b, e2 = _close(sT[0, 0], St[-1], 1e-12)
    return a and b, f"o err {e1:.2e}, state err {e2:.2e}"


def pin_uniform_channels_equal_scalar_gate(mut="none"):
    """A per-channel gate whose channels are all equal is the scalar gate
    (KDA reduces to Gated DeltaNet), for both operator orders."""
    rng = _rng(7)
    q, k, v, g, beta, s0 = _problem(rng, T=8, gate="scalar")
    gc = np.repeat(g[:, :, None], q.shape[2], axis=2)
    ok = True
    det = []
    for order in ("erase_then_decay", "decay_then_erase"):
        o1, s1 = _run(q, k, v, g, beta, s0, mut, order=order)
        o2, s2 = _run(q, k, v, gc, beta, s0, mut, order=order)
        a, e1 = _close(o1, o2, 1e-13)
        b, e2 = _close(s1, s2, 1e-13)
        ok &= a and b
        det.append(f"{order}: {e1:.1e}/{e2:.1e}")
    # both orders coincide for a scalar gate
    o3, s3 = _run(q, k, v, g, beta, s0, mut, order="decay_then_erase")
    o4, s4 = _run(q, k, v, g, beta, s0, mut, order="erase_then_decay")
    c, e3 = _close(o3, o4, 1e-13)
    return ok and c, "; ".join(det) + f"; scalar orders agree {e3:.1e}"


def pin_brute_force(mut="none"):
    """Token loop == explicit product of transition matrices (T <= 8), for both
    orders, both rules, per-channel and scalar gates."""
    rng = _rng(8)
    worst = 0.0
    for gate in ("channel", "scalar"):
        for order in ("erase_then_decay", "decay_then_erase"):
            for rule in ("delta", "linear"):
                q, k, v, g, beta, s0 = _problem(rng, T=8, gate=gate, g_scale=0.5)
                o, sT = _run(q, k, v, g, beta, s0, mut, order=order, rule=rule)
                ob, sb = transition_products(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0],
                                             s0[0, 0], order=order, rule=rule)
                worst = max(worst, float(np.max(np.abs(o[:, 0] - ob))),
                            float(np.max(np.abs(sT[0, 0] - sb))))
    # a square state (d_k = d_v) so that a transposed readout cannot hide
    q, k, v, g, beta, s0 = _problem(rng, T=5, d_k=4, d_v=4)
    o, sT = _run(q, k, v, g, beta, s0, mut)
    ob, sb = transition_products(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], s0[0, 0])
    worst = max(worst, float(np.max(np.abs(o[:, 0] - ob))), float(np.max(np.abs(sT[0, 0] - sb))))
    return worst < 1e-12, f"max |oracle - brute| = {worst:.2e}"


def pin_worked_example(mut="none"):
    """The hand-worked d_k = 2, d_v = 1 step in tests/golden/kda_worked_step.txt."""
    gd = load_golden("kda_worked_step.txt")
    q = np.array(gd["q"]).reshape(1, 1, 2)
    k = np.array(gd["k"]).reshape(1, 1, 2)
    v = np.array(gd["v"]).reshape(1, 1, 1)
    g = np.log(np.array(gd["a"])).reshape(1, 1, 2)
    beta = np.array(gd["beta"]).reshape(1, 1)
    s0 = np.array(gd["S0"]).reshape(1, 1, 2, 1)
    ok = True
    det = []
    for order in ("erase_then_decay", "decay_then_erase"):
        o, s1 = _run(q, k, v, g, beta, s0, mut, order=order)
        a, e1 = _close(s1.reshape(2), gd["S1_" + order], 1e-14)
        b, e2 = _close(o.reshape(1), gd["o_" + order], 1e-14)
        c, e3 = _close([float(k.reshape(2) @ s1.reshape(2))], gd["recall_" + order], 1e-14)
        ok &= a and b and c
        det.append(f"{order}: {e1:.1e}/{e2:.1e}/{e3:.1e}")
    return ok, "; ".join(det)


def pin_linearity(mut="none"):
    """The recurrence is linear in (S_0, v) jointly: scaling both by lambda
    scales every output and the final state by lambda."""
    rng = _rng(9)
    q, k, v, g, beta, s0 = _problem(rng, T=8)
    lam = 3.7
    o1, s1 = _run(q, k, v, g, beta, s0, mut)
    o2, s2 = _run(q, k, lam * v, g, beta, lam * s0, mut)
    a, e1 = _close(o2, lam * o1, 1e-12)
    b, e2 = _close(s2, lam * s1, 1e-12)
    return a and b, f"{e1:.1e}/{e2:.1e}"


def pin_head_grouping(mut="none"):
    """H_qk = 2 q/k heads shared by H_v = 4 v heads: v-heads 0,1 read q/k head 0
    and v-heads 2,3 read q/k head 1 (contiguous groups)."""
    rng = _rng(10)
    q, k, v, g, beta, s0 = _problem(rng, T=6, H_qk=2, H_v=4)
    o, sT = _run(q, k, v, g, beta, s0, mut)
    worst = 0.0
    for h in range(4):
        hk = h // 2
        o1, s1 = _run(q[:, hk:hk + 1], k[:, hk:hk + 1], v[:, h:h + 1], g[:, h:h + 1],
                      beta[:, h:h + 1], s0[:, h:h + 1], mut)
        worst = max(worst, float(np.max(np.abs(o[:, h] - o1[:, 0]))),
                    float(np.max(np.abs(sT[:, h] - s1[:, 0]))))
    return worst == 0.0, f"max diff {worst:.1e}"


def pin_split_call_state_carry(mut="none"):
    """Carrying the final state of a T1-token call into a T2-token call equals
    one (T1+T2)-token call."""
    rng = _rng(11)
    q, k, v, g, beta, s0 = _problem(rng, T=9)
    o, sT = _run(q, k, v, g, beta, s0, mut)
    oa, sa = _run(q[:4], k[:4], v[:4], g[:4], beta[:4], s0, mut)
    ob, sb = _run(q[4:], k[4:], v[4:], g[4:], beta[4:], sa, mut)
    a, e1 = _close(np.concatenate([oa, ob]), o, 0.0)
    b, e2 = _close(sb, sT, 0.0)
    return a and b, f"{e1:.1e}/{e2:.1e}"


def pin_packed_sequences(mut="none"):
    """Packed sequences (with a zero-length one) equal separate calls; an empty
    sequence returns its initial state."""
    rng = _rng(12)
    lens = [5, 0, 7, 1]
    T = sum(lens)
    q, k, v, g, beta, _ = _problem(rng, T=T)
    s0 = rng.standard_normal((len(lens), 1, 5, 3))
    offs = np.concatenate([[0], np.cumsum(lens)])
    o, sT = oracle.gated_delta(q, k, v, g, beta, s0, offs, mutation=mut, threads=3)
    worst = 0.0
    for n, (a, b) in enumerate(zip(offs[:-1], offs[1:])):
        if b == a:
            worst = max(worst, float(np.max(np.abs(sT[n] - s0[n]))))
            continue
        o1, s1 = _run(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], s0[n:n + 1], mut)
        worst = max(worst, float(np.max(np.abs(o[a:b] - o1))), float(np.max(np.abs(sT[n] - s1[0]))))
    return worst == 0.0, f"max diff {worst:.1e}"


ALL_PINS = [
    pin_state_constant_without_write_or_decay,
    pin_pure_decay_closed_form,
    pin_one_hot_gate_indexing,
    pin_recall_identity,
    pin_orthonormal_capacity,
    pin_linear_attention,
    pin_uniform_channels_equal_scalar_gate,
    pin_brute_force,
    pin_worked_example,
    pin_linearity,
    pin_head_grouping,
    pin_split_call_state_carry,
    pin_packed_sequences,
]
