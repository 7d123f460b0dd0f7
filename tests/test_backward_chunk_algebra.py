"""The chunk regroupings the tensor-core backward kernels compute, restated in
float64 numpy and checked against the token-by-token gradient oracle
(oracle.ttt_backward_f64) on small ragged sequences.  CPU only: this pins the
algebra of chunked_tc.cuh's reverse mode and of backward_mom_tc.cuh, not the
kernels (the GPU tests compare those with the oracle).

- Without momentum: u_t = G_t k_t, with G_t = dL/dW_T + sum_{t' >= t} do_t' q_t'^T,
  is the chunked forward over the chunks last to first with the anti-causal
  mask j >= i inside a chunk, on (q, k, v) := (k, q, do), eta = 1, from dL/dW_T.
- With momentum, the reverse chunkwise recurrence carrying (G, X = beta H)
  with the suffix weights e_i and w_ij = e_i - beta^(j+1-i) e_{j+1}.
- deta with momentum, forward order, carrying (M, P = -G) from dL/dW_0, with
  the rectangle sums through a strictly-lower ones matrix.
"""
import numpy as np
import pytest

import oracle


def _case(T, d, seed, asc):
    rng = np.random.default_rng(seed)
    q, k, v, dO = (rng.standard_normal((T, d)) for _ in range(4))
    eta = rng.uniform(0.01, 0.2, T)
    S0, M0 = 0.3 * rng.standard_normal((d, d)), 0.3 * rng.standard_normal((d, d))
    dWT, dMT = rng.standard_normal((d, d)), rng.standard_normal((d, d))
    return q, k, v, dO, eta, S0, M0, dWT, dMT, (-1.0 if asc else 1.0)


def _reverse_plain(Kq, Kk, Kv, G, C):
    """Chunked forward with eta = 1 over the chunks last to first, anti-causal
    inside a chunk: O_c = triu(Q K^T) V + Q G^T, then G += V^T K."""
    T = Kq.shape[0]
    out = np.zeros((T, Kv.shape[1]))
    for c in range((T + C - 1) // C - 1, -1, -1):
        a, b = c * C, min(T, c * C + C)
        Q, K, V = Kq[a:b], Kk[a:b], Kv[a:b]
        out[a:b] = np.triu(Q @ K.T) @ V + Q @ G.T
        G = G + V.T @ K
    return out, G


@pytest.mark.parametrize("T,d,C,asc", [(37, 8, 8, False), (64, 6, 16, True), (5, 4, 8, False)])
def test_plain_reverse_passes_give_the_gradient(T, d, C, asc):
    q, k, v, dO, eta, S0, _, dWT, _, sigma = _case(T, d, 10 + T, asc)
    ref = oracle.ttt_backward_f64(q, k, v, eta, dO, dWT, None, beta=0.0, ascent=asc, S0=S0)
    u, dW0 = _reverse_plain(k, q, dO, dWT, C)          # (q, k, v) := (k, q, do)
    r, _ = _reverse_plain(v, dO, q, dWT.T, C)          # (q, k, v) := (v, do, q)
    scale = (sigma * eta)[:, None]
    for got, want in ((scale * u, ref["dv"]), (scale * r, ref["dk"]), (sigma * np.einsum("tn,tn->t", v, u), ref["deta"]),
                      (dW0, ref["dW0"])):
        np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-10 * np.abs(want).max())


def _mom_reverse(Kr, Qr, Dr, eta, G, X, beta, sigma, C):
    """Rows -sigma H_t Kr_t for the chunks last to first, carrying G and X = beta H."""
    T = Kr.shape[0]
    out = np.zeros((T, Dr.shape[1]))
    for c in range((T + C - 1) // C - 1, -1, -1):
        a = c * C
        n = min(C, T - a)
        K, Q, D = Kr[a:a + n], Qr[a:a + n], Dr[a:a + n]
        e = np.zeros(n + 1)
        for i in range(n - 1, -1, -1):
            e[i] = eta[a + i] + beta * e[i + 1]
        w = np.array([[e[i] - beta ** (j + 1 - i) * e[j + 1] if j >= i else 0.0 for j in range(n)] for i in range(n)])
        bp = beta ** (n - 1 - np.arange(n))
        out[a:a + n] = (-sigma * bp)[:, None] * (K @ X.T) + (sigma * e[:n])[:, None] * (K @ G.T) + (sigma * w * (K @ Q.T)) @ D
        X = beta ** n * X - beta * e[0] * G - (D * (beta * w[0])[:, None]).T @ Q
        G = G + D.T @ Q
    return out, G, X


def _mom_deta(q, k, v, dO, M, P, beta, sigma, C):
    """deta_t = -<G_t, M_t> for the chunks first to last, carrying M and P = -G."""
    T = q.shape[0]
    deta = np.zeros(T)
    for c in range((T + C - 1) // C):
        a = c * C
        n = min(C, T - a)
        Q, K, V, D = q[a:a + n], k[a:a + n], v[a:a + n], dO[a:a + n]
        G = -P
        g0 = np.sum(G * M)
        y = np.einsum("jn,jn->j", D, Q @ M.T)
        z = np.einsum("sn,sn->s", V, K @ G.T)
        F = np.tril(np.ones((n, n)), -1) @ ((Q @ K.T) * (D @ V.T))
        for i in range(n):
            pw = beta ** (i - np.arange(i + 1))
            val = beta ** (i + 1) * (g0 - y[:i].sum()) - sigma * pw @ z[:i + 1] + sigma * pw @ F[i, :i + 1]
            deta[a + i] = -val
        M = beta ** n * M + V.T @ ((-sigma * beta ** (n - 1 - np.arange(n)))[:, None] * K)
        P = P + D.T @ Q
    return deta


@pytest.mark.parametrize("T,d,C,asc", [(37, 8, 8, False), (64, 6, 16, True), (5, 4, 8, False), (50, 8, 16, True)])
def test_momentum_chunkwise_recurrences_give_the_gradient(T, d, C, asc):
    q, k, v, dO, eta, S0, M0, dWT, dMT, sigma = _case(T, d, 40 + T, asc)
    beta = 0.9
    ref = oracle.ttt_backward_f64(q, k, v, eta, dO, dWT, dMT, beta=beta, ascent=asc, S0=S0, M0=M0)
    dv, dW0, dM0 = _mom_reverse(k, q, dO, eta, dWT, dMT, beta, sigma, C)
    dk, _, _ = _mom_reverse(v, dO, q, eta, dWT.T, dMT.T, beta, sigma, C)
    deta = _mom_deta(q, k, v, dO, M0, -dW0, beta, sigma, C)
    for got, name in ((dv, "dv"), (dk, "dk"), (dW0, "dW0"), (dM0, "dM0"), (deta, "deta")):
        want = ref[name]
        np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-9 * np.abs(want).max(), err_msg=name)


def test_suffix_weights_need_no_division():
    """w_ij = e_i - beta^(j+1-i) e_{j+1} equals sum_{r=i}^{j} beta^(r-i) eta_r;
    the factorisation beta^-i (P_j - P_{i-1}) loses digits as beta^-C grows."""
    rng = np.random.default_rng(3)
    C, beta = 128, 0.9
    eta = rng.uniform(0.01, 0.2, C).astype(np.float32)
    e = np.zeros(C + 1, dtype=np.float32)
    for i in range(C - 1, -1, -1):
        e[i] = np.float32(eta[i] + np.float32(beta) * e[i + 1])
    i, j = 100, 120
    exact = sum(float(eta[r]) * beta ** (r - i) for r in range(i, j + 1))
    stable = float(e[i] - np.float32(beta ** (j + 1 - i)) * e[j + 1])
    Pf = np.cumsum(eta * (np.float32(beta) ** np.arange(C, dtype=np.float32))).astype(np.float32)
    factored = float(np.float32(beta) ** -i * (Pf[j] - Pf[i - 1]))
    assert abs(stable - exact) / exact < 1e-5
    assert abs(factored - exact) / exact > 10 * abs(stable - exact) / exact
