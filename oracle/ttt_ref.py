"""Float64 CPU oracle for the causal TTT layer with one linear fast weight.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may call it.  It shares no code with the CUDA library.

What it computes
----------------
The pages ("Test-Time Training with KV Binding Is Secretly Linear Attention",
Liu et al.; the explainer "Test Time Training" on wpnews.pro and the abstract
on thelatestinai.com) describe a sequence layer whose fast weight, a matrix
that does not grow with sequence length and is reset for every sequence, takes
one gradient step per token on a key-value binding loss.  Table 2 of the
thelatestinai.com listing reduces the general layer step by step; Variants 3-5
keep a single linear fast weight W with a per-token learning rate eta_t
(Variant 3), optional SGD momentum (Variants 3-4) and, without momentum,
become standard linear attention (Variant 5).

The pages print no equation.  The readings taken here (each one listed with
its reason in the design notes) are:

* binding loss  L_t(W) = -sigma * v_t^T W k_t  (inner-product loss), so
  grad_t = dL_t/dW = -sigma * v_t k_t^T.  sigma = +1 is gradient descent;
  sigma = -1 is the gradient-ascent ablation of Table 1 (same page).
* update, then read (inclusive diagonal):  o_t = W_t q_t.
* momentum is plain SGD momentum on the gradient, learning rate applied after
  the buffer:  M_t = beta M_{t-1} + grad_t ;  W_t = W_{t-1} - eta_t M_t.
  Without momentum:  W_t = W_{t-1} - eta_t grad_t = W_{t-1} + sigma eta_t v_t k_t^T.
* no normaliser in the output ("denominator" of the kualia.ai explainer,
  section "The Linear Attention Equivalence", is not given; o = W q is used).

Layouts: q, k are [..., T, d_k], v is [..., T, d_v], eta is [..., T] or a
scalar, W and M are [..., d_v, d_k].  The leading axes (batch, heads) are
independent sequences; the loops below run over tokens and vectorise over them.

Functions whose result is pinned by ``tests/test_oracle.py`` against something
other than this file: ``ttt_recurrence_f64`` (hand-derived exact example,
finite-difference gradient of the loss, textbook causal linear attention,
invariants) and ``ttt_closed_form_f64`` (agreement with the recurrence on random
inputs, hand example).  ``ttt_chunked_f64`` is pinned against both.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "ttt_recurrence_f64",
    "ttt_closed_form_f64",
    "ttt_chunked_f64",
    "binding_loss_f64",
]


def _f64(x):
    return np.array(x, dtype=np.float64, copy=True)


def _prep(q, k, v, eta, S0, M0):
    q, k, v = _f64(q), _f64(k), _f64(v)
    lead = q.shape[:-2]
    T, dk = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    if k.shape != q.shape:
        raise ValueError("q and k must have the same shape")
    if v.shape[:-1] != q.shape[:-1]:
        raise ValueError("v must share the leading and token axes of q")
    eta = np.broadcast_to(_f64(eta), lead + (T,)).copy()
    W = np.zeros(lead + (dv, dk)) if S0 is None else _f64(S0).reshape(lead + (dv, dk))
    M = np.zeros(lead + (dv, dk)) if M0 is None else _f64(M0).reshape(lead + (dv, dk))
    return q, k, v, eta, W, M


def binding_loss_f64(W, q_unused, k, v, ascent=False):
    """Per-token key-value binding loss L(W) = -sigma * v^T W k (reading: the
    inner-product loss; the pages name the loss only as "KV binding").
    Used by the tests to pin the gradient sign by finite differences."""
    sigma = -1.0 if ascent else 1.0
    return -sigma * np.einsum("...n,...nk,...k->...", _f64(v), _f64(W), _f64(k))


def ttt_recurrence_f64(q, k, v, eta, beta=0.0, ascent=False, S0=None, M0=None,
                       momentum=None):
    """The literal token-by-token inner loop: one gradient step on the binding
    loss per token, then the read-out o_t = W_t q_t.

    momentum: None -> use the momentum buffer iff beta != 0; True/False forces
    the code path (True with beta=0 must equal the plain path).
    Returns (o [...,T,d_v], W_T [...,d_v,d_k], M_T [...,d_v,d_k]).  Without
    momentum, M_T is M0 unchanged (zeros if M0 is None).
    """
    q, k, v, eta, W, M = _prep(q, k, v, eta, S0, M0)
    use_mom = (beta != 0.0) if momentum is None else bool(momentum)
    sigma = -1.0 if ascent else 1.0
    T = q.shape[-2]
    o = np.zeros(v.shape)
    for t in range(T):
        # gradient of L_t(W) = -sigma v_t^T W k_t with respect to W
        grad = -sigma * v[..., t, :, None] * k[..., t, None, :]
        if use_mom:
            M = beta * M + grad
            W = W - eta[..., t, None, None] * M
        else:
            W = W - eta[..., t, None, None] * grad
        o[..., t, :] = np.einsum("...nk,...k->...n", W, q[..., t, :])
    return o, W, M


def _coeff(eta_row, beta, t, s, use_mom):
    """c_{t,s}: total weight with which token s's outer product v_s k_s^T has
    entered W by the end of token t (s <= t).  Plain SGD: eta_s.  Momentum:
    sum_{r=s}^{t} eta_r beta^(r-s) (token s's gradient is carried in the
    buffer and applied once per later step)."""
    if not use_mom:
        return eta_row[s]
    return sum(eta_row[r] * beta ** (r - s) for r in range(s, t + 1))


def ttt_closed_form_f64(q, k, v, eta, beta=0.0, ascent=False, S0=None, M0=None,
                        momentum=None):
    """The same layer written as causal linear attention with per-pair weights
    (the equivalence of the kualia.ai explainer, section "The Linear Attention
    Equivalence"; abstract of the paper): brute-force O(T^2) double sum,

      o_t = S0 q_t - (sum_{r<=t} eta_r beta^(r+1)) M0 q_t
            + sigma * sum_{s<=t} c_{t,s} (q_t . k_s) v_s       (0-based t, r, s)

    with the M0 term present only on the momentum path.  Slow; for tiny inputs.
    Returns (o, W_T, M_T) with the final states from the same sums.
    """
    q, k, v, eta, S0f, M0f = _prep(q, k, v, eta, S0, M0)
    use_mom = (beta != 0.0) if momentum is None else bool(momentum)
    sigma = -1.0 if ascent else 1.0
    lead = q.shape[:-2]
    T, dk, dv = q.shape[-2], q.shape[-1], v.shape[-1]
    o = np.zeros(v.shape)
    W_T = np.zeros(lead + (dv, dk))
    M_T = np.zeros(lead + (dv, dk))
    for idx in np.ndindex(*lead):
        e = eta[idx]
        S0i, M0i = S0f[idx], M0f[idx]
        for t in range(T):
            acc = S0i @ q[idx][t]
            if use_mom:
                g = sum(e[r] * beta ** (r + 1) for r in range(t + 1))
                acc = acc - g * (M0i @ q[idx][t])
            for s in range(t + 1):
                c = _coeff(e, beta, t, s, use_mom)
                acc = acc + sigma * c * float(q[idx][t] @ k[idx][s]) * v[idx][s]
            o[idx][t] = acc
        Wf = S0i.copy()
        if use_mom:
            Wf -= sum(e[r] * beta ** (r + 1) for r in range(T)) * M0i
        for s in range(T):
            Wf += sigma * _coeff(e, beta, T - 1, s, use_mom) * np.outer(v[idx][s], k[idx][s])
        W_T[idx] = Wf
        if use_mom:
            Mf = beta ** T * M0i
            for s in range(T):
                Mf = Mf - sigma * beta ** (T - 1 - s) * np.outer(v[idx][s], k[idx][s])
            M_T[idx] = Mf
        else:
            M_T[idx] = M0i
    return o, W_T, M_T


def ttt_chunked_f64(q, k, v, eta, chunk, beta=0.0, ascent=False, S0=None, M0=None,
                    momentum=None):
    """Chunk-parallel regrouping of the same sums ("fully parallel formulations",
    abstract; "cumulant matrices", kualia.ai explainer): within a chunk of
    tokens (t0, t0+C] the intra-chunk part is a masked (Q K^T * coefficients) V
    product and everything before the chunk enters through the carried state.

    Per chunk, with local indices i, j in [0, C) and coefficients computed by
    the stable backward recursion c_{i,i} = eta_i, c_{i,j} = eta_j + beta c_{i,j+1}:
      o_i   = W q_i - g_i M q_i + sigma sum_{j<=i} c_{i,j} (q_i . k_j) v_j,
      g_i   = beta * c_{i,0}                          (momentum only)
      W'    = W - g_{C-1} M + sigma sum_j c_{C-1,j} v_j k_j^T
      M'    = beta^C M - sigma sum_j beta^(C-1-j) v_j k_j^T
    Without momentum c_{i,j} = eta_j, g = 0 and M is untouched.  A ragged last
    chunk simply has fewer tokens.  Reference for debugging the GPU blocking;
    it is not used as the parity oracle (the recurrence is).
    """
    q, k, v, eta, W, M = _prep(q, k, v, eta, S0, M0)
    use_mom = (beta != 0.0) if momentum is None else bool(momentum)
    sigma = -1.0 if ascent else 1.0
    T = q.shape[-2]
    o = np.zeros(v.shape)
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        n = t1 - t0
        Q, K, V, E = q[..., t0:t1, :], k[..., t0:t1, :], v[..., t0:t1, :], eta[..., t0:t1]
        if use_mom:
            c = np.zeros(E.shape[:-1] + (n, n))
            for i in range(n):
                c[..., i, i] = E[..., i]
                for j in range(i - 1, -1, -1):
                    c[..., i, j] = E[..., j] + beta * c[..., i, j + 1]
            g = beta * c[..., :, 0]
        else:
            c = np.tril(np.broadcast_to(E[..., None, :], E.shape[:-1] + (n, n)))
            g = np.zeros(E.shape)
        A = np.einsum("...ik,...jk->...ij", Q, K) * c
        o_intra = sigma * np.einsum("...ij,...jn->...in", A, V)
        o_state = np.einsum("...nk,...ik->...in", W, Q)
        o_mom = g[..., :, None] * np.einsum("...nk,...ik->...in", M, Q)
        o[..., t0:t1, :] = o_state - o_mom + o_intra
        cl = c[..., n - 1, :]
        dW = sigma * np.einsum("...j,...jn,...jk->...nk", cl, V, K)
        if use_mom:
            bp = beta ** np.arange(n - 1, -1, -1, dtype=np.float64)
            dM = -sigma * np.einsum("j,...jn,...jk->...nk", bp, V, K)
            W = W - g[..., n - 1, None, None] * M + dW
            M = beta ** n * M + dM
        else:
            W = W + dW
    return o, W, M
