"""Pins for the float64 gradient oracle, against things other than itself.

* central finite differences of L = sum_t <o_t, dO_t> + <W_T, dW_T> +
  <M_T, dM_T>, computed through the forward oracle, for every input (q, k,
  v, per-token eta, W_0, M_0), with and without momentum, descent and ascent;
* one token by hand: o = (W_0 + sigma eta v k^T) q gives
  dq = W_0^T dO + sigma eta (v . dO) k, dv = sigma eta (k . q) dO,
  dk = sigma eta (v . dO) q, deta = sigma (v . dO)(k . q), dW_0 = dO q^T;
* eta = 0: no gradient reaches k or v, and dq_t = W_0^T dO_t;
* linearity in the upstream gradient.
"""
import numpy as np
import pytest

from oracle import ttt_backward_f64, ttt_recurrence_f64


def _rand(seed, B=1, H=2, T=6, dk=3, dv=4):
    r = np.random.default_rng(seed)
    return dict(
        q=r.standard_normal((B, H, T, dk)), k=r.standard_normal((B, H, T, dk)), v=r.standard_normal((B, H, T, dv)),
        eta=r.uniform(0.1, 0.5, (B, H, T)), S0=r.standard_normal((B, H, dv, dk)), M0=r.standard_normal((B, H, dv, dk)),
        dO=r.standard_normal((B, H, T, dv)), dW=r.standard_normal((B, H, dv, dk)), dM=r.standard_normal((B, H, dv, dk)))


def _loss(x, beta, ascent):
    o, W, M = ttt_recurrence_f64(x["q"], x["k"], x["v"], x["eta"], beta=beta, ascent=ascent, S0=x["S0"],
                                 M0=x["M0"] if beta else None)
    L = np.sum(o * x["dO"]) + np.sum(W * x["dW"])
    if beta:
        L += np.sum(M * x["dM"])
    return L


@pytest.mark.parametrize("beta,ascent", [(0.0, False), (0.0, True), (0.8, False), (0.5, True)])
def test_gradient_matches_finite_differences(beta, ascent):
    x = _rand(3)
    g = ttt_backward_f64(x["q"], x["k"], x["v"], x["eta"], x["dO"], x["dW"], x["dM"] if beta else None, beta=beta,
                         ascent=ascent, S0=x["S0"], M0=x["M0"] if beta else None)
    names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("eta", "deta"), ("S0", "dW0")] + ([("M0", "dM0")] if beta else [])
    h = 1e-6
    for inp, out in names:
        fd = np.zeros_like(x[inp])
        for idx in np.ndindex(*x[inp].shape):
            xp = {n: a.copy() for n, a in x.items()}
            xm = {n: a.copy() for n, a in x.items()}
            xp[inp][idx] += h
            xm[inp][idx] -= h
            fd[idx] = (_loss(xp, beta, ascent) - _loss(xm, beta, ascent)) / (2 * h)
        np.testing.assert_allclose(g[out], fd, rtol=1e-6, atol=1e-6 * max(1.0, np.max(np.abs(fd))), err_msg=inp)


@pytest.mark.parametrize("ascent", [False, True])
def test_one_token_by_hand(ascent):
    x = _rand(4, B=1, H=1, T=1, dk=3, dv=2)
    s = -1.0 if ascent else 1.0
    q, k, v, e = x["q"][0, 0, 0], x["k"][0, 0, 0], x["v"][0, 0, 0], x["eta"][0, 0, 0]
    W0, dO = x["S0"][0, 0], x["dO"][0, 0, 0]
    g = ttt_backward_f64(x["q"], x["k"], x["v"], x["eta"], x["dO"], ascent=ascent, S0=x["S0"])
    np.testing.assert_allclose(g["dq"][0, 0, 0], W0.T @ dO + s * e * (v @ dO) * k, rtol=1e-13)
    np.testing.assert_allclose(g["dv"][0, 0, 0], s * e * (k @ q) * dO, rtol=1e-13)
    np.testing.assert_allclose(g["dk"][0, 0, 0], s * e * (v @ dO) * q, rtol=1e-13)
    np.testing.assert_allclose(g["deta"][0, 0, 0], s * (v @ dO) * (k @ q), rtol=1e-13)
    np.testing.assert_allclose(g["dW0"][0, 0], np.outer(dO, q), rtol=1e-13)


def test_zero_learning_rate_and_linearity():
    x = _rand(5)
    g = ttt_backward_f64(x["q"], x["k"], x["v"], 0.0 * x["eta"], x["dO"], S0=x["S0"])
    assert not np.any(g["dk"]) and not np.any(g["dv"])
    np.testing.assert_allclose(g["dq"], np.einsum("bhnk,bhtn->bhtk", x["S0"], x["dO"]), rtol=1e-13)
    for beta in (0.0, 0.7):
        a = ttt_backward_f64(x["q"], x["k"], x["v"], x["eta"], x["dO"], x["dW"], beta=beta, S0=x["S0"])
        b = ttt_backward_f64(x["q"], x["k"], x["v"], x["eta"], -2.5 * x["dO"], -2.5 * x["dW"], beta=beta,
                             S0=x["S0"])
        for n in ("dq", "dk", "dv", "deta", "dW0", "dM0"):
            np.testing.assert_allclose(b[n], -2.5 * a[n], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("ascent", [False, True])
def test_plain_gradient_is_three_forward_passes(ascent):
    """Without momentum the backward is three runs of the forward layer:
      dq_t = W_t^T do_t            forward on (q=dO, k=v, v=k), W_0 -> W_0^T
      u_t  = G_t k_t               forward on the reversed sequence of (q=k, k=q, v=dO),
                                   eta = 1, descent, starting from dL/dW_T
      r_t  = G_t^T v_t             the same with (q=v, k=dO, v=q), starting from dL/dW_T^T
    then dv = sigma eta u, dk = sigma eta r, deta = sigma v . u, and dW_0 is the
    second run's final state.  An independent route to the same numbers."""
    x = _rand(6, T=9, dk=4, dv=4)
    s = -1.0 if ascent else 1.0
    g = ttt_backward_f64(x["q"], x["k"], x["v"], x["eta"], x["dO"], x["dW"], ascent=ascent, S0=x["S0"])
    tr = lambda m: np.swapaxes(m, -1, -2)  # noqa: E731
    rev = lambda a: a[..., ::-1, :]  # noqa: E731
    dq, _, _ = ttt_recurrence_f64(x["dO"], x["v"], x["k"], x["eta"], ascent=ascent, S0=tr(x["S0"]))
    u_rev, G1, _ = ttt_recurrence_f64(rev(x["k"]), rev(x["q"]), rev(x["dO"]), 1.0, S0=x["dW"])
    r_rev, _, _ = ttt_recurrence_f64(rev(x["v"]), rev(x["dO"]), rev(x["q"]), 1.0, S0=tr(x["dW"]))
    u, r = rev(u_rev), rev(r_rev)
    e = x["eta"][..., None]
    np.testing.assert_allclose(g["dq"], dq, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dv"], s * e * u, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dk"], s * e * r, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["deta"], s * np.sum(x["v"] * u, axis=-1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dW0"], G1, rtol=1e-12, atol=1e-12)
