"""Pins for the float64 feature-map oracle, checked against things other than
its own formula.

* hand values at pre-activations +-ln 3, where sigmoid is exactly 3/4 or 1/4;
* the odd part phi(x; W1, W3) - phi(x; -W1, W3) = (W1 x)(W3 x), against
  explicit loops (fixes which weight is gated and which head uses which
  weights; a sigmoid in place of silu, or W1 and W3 swapped, fails it);
* the even part, (W1 x)(W3 x) tanh((W1 x)/2), against numpy's tanh;
* the ReLU limit for large pre-activations; W1 = 0 or W3 = 0 gives zero;
* the layer on phi against the kernelised causal linear-attention sum written
  out with loops (kualia.ai explainer, section "The Linear Attention
  Equivalence"), and with momentum against the closed-form oracle.
"""
import math

import numpy as np
import pytest

from oracle import (feature_map_f64, silu_f64, ttt_closed_form_f64,
                    ttt_feature_layer_f64)


def _rand(seed, B=2, H=3, T=5, d_in=4, d_out=6):
    r = np.random.default_rng(seed)
    x = r.standard_normal((B, H, T, d_in))
    W1 = r.standard_normal((H, d_out, d_in))
    W3 = r.standard_normal((H, d_out, d_in))
    return x, W1, W3


def _loops_preact(x, W):
    B, H, T, d_in = x.shape
    d_out = W.shape[1]
    out = np.zeros((B, H, T, d_out))
    for b in range(B):
        for h in range(H):
            for t in range(T):
                for o in range(d_out):
                    out[b, h, t, o] = sum(W[h, o, i] * x[b, h, t, i] for i in range(d_in))
    return out


def test_hand_values_at_plus_minus_ln3():
    # x = e_0; head 0 row 0: W1 x = ln 3, W3 x = 4 -> silu(ln 3) * 4 = (3/4) ln 3 * 4 = 3 ln 3
    #          head 0 row 1: W1 x = -ln 3, W3 x = 2 -> silu(-ln 3) * 2 = -(1/4) ln 3 * 2 = -ln 3 / 2
    #          head 0 row 2: W1 x = 0 -> 0 whatever W3 x is
    L = math.log(3.0)
    x = np.array([[[[1.0, 0.0]]]])
    W1 = np.array([[[L, 7.0], [-L, -1.0], [0.0, 2.0]]])
    W3 = np.array([[[4.0, 9.0], [2.0, 0.5], [5.0, 5.0]]])
    phi = feature_map_f64(x, W1, W3)
    assert phi.shape == (1, 1, 1, 3)
    np.testing.assert_allclose(phi[0, 0, 0], [3.0 * L, -L / 2.0, 0.0], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(silu_f64([L, -L, 0.0]), [0.75 * L, -0.25 * L, 0.0], rtol=1e-15, atol=0)


@pytest.mark.parametrize("seed", [0, 1])
def test_odd_part_is_the_bilinear_product(seed):
    x, W1, W3 = _rand(seed)
    odd = feature_map_f64(x, W1, W3) - feature_map_f64(x, -W1, W3)
    expect = _loops_preact(x, W1) * _loops_preact(x, W3)
    np.testing.assert_allclose(odd, expect, rtol=1e-12, atol=1e-12)


def test_even_part_is_the_tanh_form():
    x, W1, W3 = _rand(2)
    even = feature_map_f64(x, W1, W3) + feature_map_f64(x, -W1, W3)
    a, b = _loops_preact(x, W1), _loops_preact(x, W3)
    np.testing.assert_allclose(even, a * b * np.tanh(a / 2.0), rtol=1e-12, atol=1e-12)


def test_relu_limit_and_zero_weights():
    x, W1, W3 = _rand(3)
    a = _loops_preact(x, W1)
    c = 1e6
    lim = feature_map_f64(x, c * W1, W3) / c
    far = np.abs(a) > 1e-4  # exp(-c |a|) below 1e-43 there
    assert far.mean() > 0.9
    np.testing.assert_allclose(lim[far], (np.maximum(a, 0.0) * _loops_preact(x, W3))[far], rtol=1e-9, atol=1e-9)
    assert not np.any(feature_map_f64(x, np.zeros_like(W1), W3))
    assert not np.any(feature_map_f64(x, W1, np.zeros_like(W3)))
    # very negative pre-activations: a vanishing gate, with no overflow on the way
    with np.errstate(over="raise"):
        assert np.all(np.abs(silu_f64([-800.0, -1e6])) < 1e-290)


def test_heads_use_their_own_weights():
    x, W1, W3 = _rand(4)
    perm = [2, 0, 1]
    a = feature_map_f64(x[:, perm], W1[perm], W3[perm])
    b = feature_map_f64(x, W1, W3)[:, perm]
    np.testing.assert_array_equal(a, b)
    with pytest.raises(ValueError):
        feature_map_f64(x, W1[:2], W3[:2])


def _phi_loops(x, W1, W3):
    a, b = _loops_preact(x, W1), _loops_preact(x, W3)
    out = np.zeros_like(a)
    for idx in np.ndindex(*a.shape):
        out[idx] = a[idx] / (1.0 + math.exp(-a[idx])) * b[idx]
    return out


@pytest.mark.parametrize("ascent", [False, True])
def test_layer_is_kernelised_linear_attention(ascent):
    r = np.random.default_rng(5)
    B, H, T, d_in, d_out, d_v = 1, 2, 6, 3, 4, 2
    q = r.standard_normal((B, H, T, d_in))
    k = r.standard_normal((B, H, T, d_in))
    v = r.standard_normal((B, H, T, d_v))
    eta = r.uniform(0.1, 0.5, (B, H, T))
    W1 = r.standard_normal((H, d_out, d_in))
    W3 = r.standard_normal((H, d_out, d_in))
    S0 = r.standard_normal((B, H, d_v, d_out))
    o, W_T, _ = ttt_feature_layer_f64(q, k, v, eta, W1, W3, ascent=ascent, S0=S0)
    fq, fk = _phi_loops(q, W1, W3), _phi_loops(k, W1, W3)
    sigma = -1.0 if ascent else 1.0
    for b in range(B):
        for h in range(H):
            W = S0[b, h].copy()
            for t in range(T):
                expect = S0[b, h] @ fq[b, h, t]
                for s in range(t + 1):
                    expect = expect + sigma * eta[b, h, s] * float(fq[b, h, t] @ fk[b, h, s]) * v[b, h, s]
                np.testing.assert_allclose(o[b, h, t], expect, rtol=1e-11, atol=1e-11)
                W = W + sigma * eta[b, h, t] * np.outer(v[b, h, t], fk[b, h, t])
            np.testing.assert_allclose(W_T[b, h], W, rtol=1e-11, atol=1e-11)


def test_layer_with_momentum_matches_the_closed_form():
    r = np.random.default_rng(6)
    B, H, T, d_in, d_out = 1, 2, 7, 3, 5
    q, k = r.standard_normal((2, B, H, T, d_in))
    v = r.standard_normal((B, H, T, d_out))
    eta = r.uniform(0.1, 0.5, (B, H, T))
    W1, W3 = r.standard_normal((2, H, d_out, d_in))
    S0, M0 = r.standard_normal((2, B, H, d_out, d_out))
    o, W_T, M_T = ttt_feature_layer_f64(q, k, v, eta, W1, W3, beta=0.8, S0=S0, M0=M0)
    fq, fk = _phi_loops(q, W1, W3), _phi_loops(k, W1, W3)
    o2, W2, M2 = ttt_closed_form_f64(fq, fk, v, eta, beta=0.8, S0=S0, M0=M0)
    np.testing.assert_allclose(o, o2, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(W_T, W2, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(M_T, M2, rtol=1e-10, atol=1e-10)
