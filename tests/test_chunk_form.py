"""The chunk form the prefill kernels compute, re-derived in fp64 NumPy and
checked against the token-by-token oracle (no GPU).

For one chunk of C tokens entering with state S0, with G_t the in-chunk
cumulative log-decay through token t and Gp_t the one through t - 1 (row
"KDA" of the table "Everything, in one table", thethings.ai "The argument,
in one page"; chunking per row "Chunkwise / WY"; literal order: erase from the
old state, then decay):

  recall     (I + tril_-1(A_e) diag(beta)) R = (K e^{Gp}) S0 + tril_-1(A_w) diag(beta) V
  state      S_t = e^{G_t} [S0 + sum_{i<=t} beta_i (e^{-G_i} k_i v_i^T - e^{-Gp_i} k_i r_i^T)]
  output     o_t = S0^T (e^{G_t} q_t) + sum_{i<=t} beta_i [B_w[t,i] v_i - B_e[t,i] r_i]

with A_w[i,j] = k_i^T e^{Gp_i - G_j} k_j, A_e[i,j] = k_i^T e^{Gp_i - Gp_j} k_j,
B_w[t,j] = q_t^T e^{G_t - G_j} k_j, B_e[t,j] = q_t^T e^{G_t - Gp_j} k_j; and
the affine map the scan applies, S_L = P S0 + Qc, o = Q' S0 + O_intra, with
W = T^{-1}(K e^{Gp}), U = T^{-1} tril_-1(A_w) diag(beta) V,
P = Diag(e^{G_L}) - K_b^T diag(beta) W, Qc = K_a^T diag(beta) V - K_b^T diag(beta) U,
Q' = Q e^{G} - tril(B_e) diag(beta) W, O_intra = tril(B_w) diag(beta) V - tril(B_e) diag(beta) U,
K_a = K e^{G_L - G}, K_b = K e^{G_L - Gp}.  The decode readout computes
o = S'^T q in one pass over the old state: o = p - beta (k.(a q)) r + beta (k.q) v
with r = S^T k, p = S^T (a q).
"""
import numpy as np
import pytest

import oracle


def _chunk(q, k, v, g, beta, S0):
    """One chunk by the formulas above; returns (o [C, d_v], S_L, (P, Qc, Qp, Oi))."""
    C = q.shape[0]
    G = np.cumsum(g, axis=0)
    Gp = G - g
    lower = np.tril(np.ones((C, C)), -1)
    incl = np.tril(np.ones((C, C)))
    # pair factors formed directly from exponent differences (fp64, small C)
    Aw = np.einsum("ic,ijc,jc->ij", k, np.exp(Gp[:, None, :] - G[None, :, :]), k) * lower
    Ae = np.einsum("ic,ijc,jc->ij", k, np.exp(Gp[:, None, :] - Gp[None, :, :]), k) * lower
    Bw = np.einsum("tc,tjc,jc->tj", q, np.exp(G[:, None, :] - G[None, :, :]), k) * incl
    Be = np.einsum("tc,tjc,jc->tj", q, np.exp(G[:, None, :] - Gp[None, :, :]), k) * incl
    Tm = np.eye(C) + Ae * beta[None, :]
    R = np.linalg.solve(Tm, (k * np.exp(Gp)) @ S0 + (Aw * beta[None, :]) @ v)
    # states and outputs token by token from the closed forms
    o = np.empty((C, v.shape[1]))
    for t in range(C):
        o[t] = S0.T @ (np.exp(G[t]) * q[t]) + sum(
            beta[i] * (Bw[t, i] * v[i] - Be[t, i] * R[i]) for i in range(t + 1))
    L = C - 1
    S_L = np.exp(G[L])[:, None] * (S0 + sum(
        beta[i] * (np.outer(np.exp(-G[i]) * k[i], v[i]) - np.outer(np.exp(-Gp[i]) * k[i], R[i]))
        for i in range(C)))
    # the affine map of the scan
    W = np.linalg.solve(Tm, k * np.exp(Gp))
    U = np.linalg.solve(Tm, (Aw * beta[None, :]) @ v)
    Ka = k * np.exp(G[L] - G)
    Kb = k * np.exp(G[L] - Gp)
    P = np.diag(np.exp(G[L])) - Kb.T @ (beta[:, None] * W)
    Qc = Ka.T @ (beta[:, None] * v) - Kb.T @ (beta[:, None] * U)
    Qp = q * np.exp(G) - (Be * beta[None, :]) @ W
    Oi = (Bw * beta[None, :]) @ v - (Be * beta[None, :]) @ U
    assert np.allclose(R, W @ S0 + U, rtol=1e-12, atol=1e-12)  # R = W S0 + U
    return o, S_L, (P, Qc, Qp, Oi)


def _problem(rng, T, d_k, d_v, gate, scale):
    q = rng.standard_normal((T, 1, d_k))
    k = rng.standard_normal((T, 1, d_k))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, 1, d_v))
    g = -scale * rng.random((T, 1, d_k) if gate == "channel" else (T, 1))
    beta = rng.random((T, 1))
    s0 = rng.standard_normal((1, 1, d_k, d_v))
    return q, k, v, g, beta, s0


@pytest.mark.parametrize("gate", ["channel", "scalar"])
@pytest.mark.parametrize("C,chunks,scale", [(8, 3, 0.3), (16, 2, 1.5), (5, 4, 0.05)])
def test_chunk_form_and_affine_map_equal_the_token_loop(gate, C, chunks, scale):
    rng = np.random.default_rng(7 + C + chunks)
    d_k, d_v = 6, 4
    T = C * chunks
    q, k, v, g, beta, s0 = _problem(rng, T, d_k, d_v, gate, scale)
    ro, rs = oracle.gated_delta(q, k, v, g, beta, s0, threads=1)
    S = s0[0, 0].copy()
    S_map = s0[0, 0].copy()
    for u in range(chunks):
        sl = slice(u * C, (u + 1) * C)
        gc = g[sl, 0] if gate == "channel" else np.repeat(g[sl, 0][:, None], d_k, axis=1)
        o, S_L, (P, Qc, Qp, Oi) = _chunk(q[sl, 0], k[sl, 0], v[sl, 0], gc, beta[sl, 0], S)
        np.testing.assert_allclose(o, ro[sl, 0], rtol=1e-10, atol=1e-12)
        # the same chunk through the affine map, from the map's own carried state
        np.testing.assert_allclose(Qp @ S_map + Oi, ro[sl, 0], rtol=1e-10, atol=1e-12)
        S, S_map = S_L, P @ S_map + Qc
    np.testing.assert_allclose(S, rs[0, 0], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S_map, rs[0, 0], rtol=1e-10, atol=1e-12)


def test_one_pass_decode_readout_equals_the_updated_state_read():
    rng = np.random.default_rng(11)
    d_k, d_v = 7, 5
    for _ in range(5):
        S = rng.standard_normal((d_k, d_v))
        q, k, v = rng.standard_normal(d_k), rng.standard_normal(d_k), rng.standard_normal(d_v)
        k /= np.linalg.norm(k)
        a = np.exp(-rng.random(d_k))
        b = rng.random()
        r, p = S.T @ k, S.T @ (a * q)
        o = p - b * (k @ (a * q)) * r + b * (k @ q) * v
        S_new = a[:, None] * (S - b * np.outer(k, r)) + b * np.outer(k, v)
        np.testing.assert_allclose(o, S_new.T @ q, rtol=1e-12, atol=1e-12)
        ro, rs = oracle.gated_delta(q[None, None], k[None, None], v[None, None],
                                    np.log(a)[None, None], np.array([[b]]), S[None, None],
                                    threads=1)
        np.testing.assert_allclose(o, ro[0, 0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S_new, rs[0, 0], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("scale", [0.05, 1.0, 4.0])
def test_scalar_gate_gram_factorisation(scale):
    """With one gate value per token the Grams are the raw dot products times
    factors that are all <= 1: left of the diagonal 16-token block, a row factor
    e^{row - E_J} times a column factor e^{E_J - G_j} (E_J: G at the end of key
    block J); inside it, the product of the decays a_s of the tokens strictly
    between the pair; the erase Grams are the write Grams times a_j."""
    rng = np.random.default_rng(17)
    C, d_k = 64, 8
    q = rng.standard_normal((C, d_k))
    k = rng.standard_normal((C, d_k))
    g = -scale * np.log1p(np.exp(rng.standard_normal(C)))  # -scale * softplus(N)
    G = np.cumsum(g)
    Gp = G - g
    a = np.exp(g)
    E = G[15::16]
    KK, QK = k @ k.T, q @ k.T
    Aw = np.zeros((C, C)); Bw = np.zeros((C, C))
    for r in range(C):
        for j in range(C):
            I, J = r // 16, j // 16
            if J < I:
                Aw[r, j] = KK[r, j] * np.exp(Gp[r] - E[J]) * np.exp(E[J] - G[j])
                Bw[r, j] = QK[r, j] * np.exp(G[r] - E[J]) * np.exp(E[J] - G[j])
            elif J == I:
                d = np.prod(a[j + 1:r]) if j < r else 0.0  # e^{Gp_r - G_j}
                Aw[r, j] = KK[r, j] * d
                Bw[r, j] = QK[r, j] * (d * a[r] if j < r else (1.0 if j == r else 0.0))
    Ae, Be = Aw * a[None, :], Bw * a[None, :]
    lower, incl = np.tril(np.ones((C, C)), -1), np.tril(np.ones((C, C)))
    np.testing.assert_allclose(Aw, KK * np.exp(Gp[:, None] - G[None, :]) * lower, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(Ae, KK * np.exp(Gp[:, None] - Gp[None, :]) * lower, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(Bw, QK * np.exp(G[:, None] - G[None, :]) * incl, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(Be, QK * np.exp(G[:, None] - Gp[None, :]) * incl, rtol=1e-12, atol=1e-300)
