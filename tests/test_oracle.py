"""Pins for the float64 oracle, checked against things other than itself.

* a worked example derived by hand (tests/golden), compared exactly;
* an exact-rational re-derivation with fractions.Fraction on the same example;
* the gradient of the binding loss by central finite differences;
* textbook causal linear attention, eta * tril(Q K^T) V, via numpy matmul
  (standard linear attention, Table 2 caption of the thelatestinai.com listing);
* the closed-form linear-attention sum (kualia.ai explainer, section "The
  Linear Attention Equivalence") against the literal recurrence;
* invariants: eta = 0, ascent negation (Table 1), beta = 0 through the momentum
  path, linearity in V and in eta, T = 1, chunk-size independence including a
  ragged last chunk, sequence splitting through the carried state, Q := K.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import (binding_loss_f64, ttt_chunked_f64, ttt_closed_form_f64,
                    ttt_recurrence_f64)

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_example_dk3_dv2_T3.json")


def _rand(seed, B=2, H=2, T=11, dk=5, dv=3, token_eta=True):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, H, T, dk))
    k = r.standard_normal((B, H, T, dk))
    v = r.standard_normal((B, H, T, dv))
    eta = r.uniform(0.05, 0.6, (B, H, T)) if token_eta else 0.3
    S0 = r.standard_normal((B, H, dv, dk))
    M0 = r.standard_normal((B, H, dv, dk))
    return q, k, v, eta, S0, M0


def _close(a, b, tol=1e-12):
    a, b = np.asarray(a), np.asarray(b)
    scale = max(1.0, float(np.max(np.abs(b))))
    assert np.max(np.abs(a - b)) <= tol * scale, np.max(np.abs(a - b))


# ---------------------------------------------------------------- golden ----
def _golden():
    with open(GOLD) as f:
        return json.load(f)


@pytest.mark.parametrize("case_idx", range(4))
def test_hand_example_recurrence(case_idx):
    g = _golden()
    c = g["cases"][case_idx]
    x = g["inputs"]
    q, k, v, eta = (np.array(x[n], float) for n in ("q", "k", "v", "eta"))
    o, W, M = ttt_recurrence_f64(q, k, v, eta, beta=c["beta"], ascent=c["ascent"],
                                 S0=c["S0"], M0=c["M0"])
    assert np.array_equal(o, np.array(c["o"], float))
    assert np.array_equal(W, np.array(c["W"], float))
    if "M" in c:
        assert np.array_equal(M, np.array(c["M"], float))


@pytest.mark.parametrize("case_idx", range(4))
def test_hand_example_closed_form_and_chunked(case_idx):
    g = _golden()
    c = g["cases"][case_idx]
    x = g["inputs"]
    q, k, v, eta = (np.array(x[n], float) for n in ("q", "k", "v", "eta"))
    kw = dict(beta=c["beta"], ascent=c["ascent"], S0=c["S0"], M0=c["M0"])
    for fn in (lambda: ttt_closed_form_f64(q, k, v, eta, **kw),
               lambda: ttt_chunked_f64(q, k, v, eta, 2, **kw)):
        o, W, M = fn()
        _close(o, c["o"], 1e-15)
        _close(W, c["W"], 1e-15)
        if "M" in c:
            _close(M, c["M"], 1e-15)


def test_hand_example_exact_rationals():
    """Re-derive the golden numbers with exact rationals, element by element,
    from the update rule alone (no numpy), so the fixture itself is checked."""
    g = _golden()
    x = g["inputs"]
    F = Fraction
    q = [[F(a) for a in r] for r in x["q"]]
    k = [[F(a) for a in r] for r in x["k"]]
    v = [[F(a) for a in r] for r in x["v"]]
    eta = [F(a).limit_denominator() for a in x["eta"]]
    for c in g["cases"]:
        sig = -1 if c["ascent"] else 1
        beta = F(c["beta"]).limit_denominator()
        W = [[F(a).limit_denominator() for a in r] for r in (c["S0"] or [[0] * 3] * 2)]
        M = [[F(a).limit_denominator() for a in r] for r in (c["M0"] or [[0] * 3] * 2)]
        outs = []
        for t in range(3):
            for n in range(2):
                for j in range(3):
                    grad = -sig * v[t][n] * k[t][j]
                    if beta != 0:
                        M[n][j] = beta * M[n][j] + grad
                        W[n][j] -= eta[t] * M[n][j]
                    else:
                        W[n][j] -= eta[t] * grad
            outs.append([sum(W[n][j] * q[t][j] for j in range(3)) for n in range(2)])
        assert outs == [[F(a).limit_denominator() for a in r] for r in c["o"]]
        assert W == [[F(a).limit_denominator() for a in r] for r in c["W"]]
        if "M" in c:
            assert M == [[F(a).limit_denominator() for a in r] for r in c["M"]]


# ------------------------------------------------------- loss gradient ----
@pytest.mark.parametrize("ascent", [False, True])
def test_update_is_a_gradient_step_on_binding_loss(ascent):
    """One recurrence step from W0 equals W0 - eta * dL/dW with dL/dW taken by
    central finite differences of the binding loss (exact for a linear loss)."""
    r = np.random.default_rng(5)
    dk, dv = 4, 3
    W0 = r.standard_normal((dv, dk))
    q, k, v = r.standard_normal(dk), r.standard_normal(dk), r.standard_normal(dv)
    eta, h = 0.37, 1e-3
    num = np.zeros_like(W0)
    for i in range(dv):
        for j in range(dk):
            E = np.zeros_like(W0)
            E[i, j] = h
            num[i, j] = (binding_loss_f64(W0 + E, q, k, v, ascent)
                         - binding_loss_f64(W0 - E, q, k, v, ascent)) / (2 * h)
    _, W1, _ = ttt_recurrence_f64(q[None], k[None], v[None], [eta], ascent=ascent, S0=W0)
    _close(W1, W0 - eta * num, 1e-10)
    # momentum path, first step from M0 = 0: M1 = grad, W1 = W0 - eta * grad
    _, W1m, M1 = ttt_recurrence_f64(q[None], k[None], v[None], [eta], beta=0.9,
                                    ascent=ascent, S0=W0)
    _close(M1, num, 1e-10)
    _close(W1m, W0 - eta * num, 1e-10)


# --------------------------------------------------------- textbook -------
def test_textbook_causal_linear_attention():
    """Constant eta, no momentum, zero initial state: the layer is eta times
    unnormalised causal linear attention with identity feature map."""
    q, k, v, _, _, _ = _rand(1, T=17)
    eta = 0.25
    o, W, _ = ttt_recurrence_f64(q, k, v, eta)
    ref = eta * np.matmul(np.tril(np.matmul(q, np.swapaxes(k, -1, -2))), v)
    _close(o, ref)
    _close(W, eta * np.matmul(np.swapaxes(v, -1, -2), k))


# ---------------------------------------------------- closed form ---------
@pytest.mark.parametrize("beta", [0.0, 0.9, 0.5])
@pytest.mark.parametrize("ascent", [False, True])
def test_closed_form_equals_recurrence(beta, ascent):
    q, k, v, eta, S0, M0 = _rand(2, B=1, H=2, T=9, dk=4, dv=3)
    a = ttt_recurrence_f64(q, k, v, eta, beta, ascent, S0, M0)
    b = ttt_closed_form_f64(q, k, v, eta, beta, ascent, S0, M0)
    for x, y in zip(a, b):
        _close(x, y, 1e-12)


# ------------------------------------------------------- invariants -------
@pytest.mark.parametrize("beta", [0.0, 0.9])
def test_eta_zero_leaves_fast_weight(beta):
    q, k, v, _, S0, M0 = _rand(3)
    o, W, M = ttt_recurrence_f64(q, k, v, 0.0, beta, False, S0, M0)
    _close(W, S0, 0)
    _close(o, np.einsum("bhnk,bhtk->bhtn", S0, q))
    if beta:
        T = q.shape[2]
        Mref = beta ** T * M0 - np.einsum("t,bhtn,bhtk->bhnk",
                                          beta ** np.arange(T - 1, -1, -1.0), v, k)
        _close(M, Mref)
    else:
        _close(M, M0, 0)


@pytest.mark.parametrize("beta", [0.0, 0.9])
def test_ascent_negates_update(beta):
    q, k, v, eta, _, _ = _rand(4)
    od, Wd, Md = ttt_recurrence_f64(q, k, v, eta, beta, False)
    oa, Wa, Ma = ttt_recurrence_f64(q, k, v, eta, beta, True)
    _close(oa, -od)
    _close(Wa, -Wd)
    _close(Ma, -Md)


def test_beta_zero_momentum_path_equals_plain():
    q, k, v, eta, S0, _ = _rand(6)
    a = ttt_recurrence_f64(q, k, v, eta, 0.0, False, S0, None, momentum=False)
    b = ttt_recurrence_f64(q, k, v, eta, 0.0, False, S0, None, momentum=True)
    _close(a[0], b[0])
    _close(a[1], b[1])


@pytest.mark.parametrize("beta", [0.0, 0.9])
def test_linear_in_v_and_in_eta(beta):
    q, k, v, eta, _, _ = _rand(7)
    v2 = np.random.default_rng(8).standard_normal(v.shape)
    o1 = ttt_recurrence_f64(q, k, v, eta, beta)[0]
    o2 = ttt_recurrence_f64(q, k, v2, eta, beta)[0]
    o12 = ttt_recurrence_f64(q, k, v + v2, eta, beta)[0]
    _close(o12, o1 + o2)
    o3 = ttt_recurrence_f64(q, k, v, 3.0 * eta, beta)[0]
    _close(o3, 3.0 * o1)


@pytest.mark.parametrize("beta", [0.0, 0.9])
def test_single_token(beta):
    q, k, v, eta, S0, M0 = _rand(9, T=1)
    o, _, _ = ttt_recurrence_f64(q, k, v, eta, beta, False, S0, M0)
    qk = np.einsum("bhtk,bhtk->bht", q, k)
    ref = np.einsum("bhnk,bhtk->bhtn", S0, q) + (eta * qk)[..., None] * v
    if beta:
        ref -= (eta * beta)[..., None] * np.einsum("bhnk,bhtk->bhtn", M0, q)
    _close(o, ref)


@pytest.mark.parametrize("beta", [0.0, 0.9])
@pytest.mark.parametrize("chunk", [1, 3, 4, 8, 64])
def test_chunked_regrouping_independent_of_chunk(beta, chunk):
    q, k, v, eta, S0, M0 = _rand(10, T=21)
    a = ttt_recurrence_f64(q, k, v, eta, beta, True, S0, M0)
    b = ttt_chunked_f64(q, k, v, eta, chunk, beta, True, S0, M0)
    for x, y in zip(a, b):
        _close(x, y, 1e-12)


@pytest.mark.parametrize("beta", [0.0, 0.9])
def test_split_sequence_through_carried_state(beta):
    q, k, v, eta, S0, M0 = _rand(11, T=19)
    o, W, M = ttt_recurrence_f64(q, k, v, eta, beta, False, S0, M0)
    t1 = 7
    oa, Wa, Ma = ttt_recurrence_f64(q[..., :t1, :], k[..., :t1, :], v[..., :t1, :],
                                    eta[..., :t1], beta, False, S0, M0)
    ob, Wb, Mb = ttt_recurrence_f64(q[..., t1:, :], k[..., t1:, :], v[..., t1:, :],
                                    eta[..., t1:], beta, False, Wa, Ma)
    _close(np.concatenate([oa, ob], axis=-2), o)
    _close(Wb, W)
    _close(Mb, M)


def test_query_replaced_by_key():
    """Table 1 ablation 'Replace Q with K': reading with the key is allowed."""
    q, k, v, eta, _, _ = _rand(12)
    o, _, _ = ttt_recurrence_f64(k, k, v, eta)
    ref = ttt_closed_form_f64(k, k, v, eta)[0]
    _close(o, ref)


# -------------------------------------------- planted mistakes are caught --
def test_pins_catch_planted_mistakes():
    """Variants of the recurrence with one plausible slip each must fail the
    golden example: exclusive diagonal, eta applied before the momentum
    buffer, wrong gradient sign, dropped M0 term.  (A transposed fast weight
    cannot even be applied: the example has d_k = 3 != d_v = 2.)"""
    g = _golden()
    x = g["inputs"]
    q, k, v, eta = (np.array(x[n], float) for n in ("q", "k", "v", "eta"))
    c = g["cases"][3]
    S0, M0, beta = np.array(c["S0"], float), np.array(c["M0"], float), c["beta"]

    def run(exclusive=False, eta_first=False, flip_sign=False, drop_m0=False):
        W, M = S0.copy(), (np.zeros_like(M0) if drop_m0 else M0.copy())
        out = []
        for t in range(3):
            o_prev = W @ q[t]
            G = np.outer(v[t], k[t]) * (-1.0 if flip_sign else 1.0)
            if eta_first:
                M = beta * M - eta[t] * G
                W = W - M
            else:
                M = beta * M - G
                W = W - eta[t] * M
            out.append(o_prev if exclusive else W @ q[t])
        return np.array(out)

    good = np.array(c["o"], float)
    assert np.array_equal(run(), good)
    for bad in (dict(exclusive=True), dict(eta_first=True), dict(flip_sign=True),
                dict(drop_m0=True)):
        assert not np.allclose(run(**bad), good), bad
