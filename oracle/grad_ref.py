"""Float64 CPU oracle for the gradient of the causal TTT layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may
call it.  It shares no code with the CUDA library.

What it computes
----------------
Figure 4 of the thelatestinai.com listing of "Test-Time Training with KV
Binding Is Secretly Linear Attention" trains models whose TTT layer runs in
the parallel form, so the layer needs its backward pass.  For an upstream
gradient dO = dL/do_t (and optionally dL/dW_T, dL/dM_T on the final states)
of the layer of ``ttt_ref`` (update, then read; sigma = +1 descent, -1
ascent):

  forward   M_t = beta M_{t-1} - sigma v_t k_t^T ;  W_t = W_{t-1} - eta_t M_t
            (without momentum W_t = W_{t-1} + sigma eta_t v_t k_t^T)
            o_t = W_t q_t

the chain rule taken backwards over the tokens gives, with
G_t = dL/dW_t (everything W_t reaches: o_t and W_{t+1}) and
H_t = dL/dM_t (everything M_t reaches: W_t and M_{t+1}):

  G_t   = G_{t+1} + do_t q_t^T,          G_{T+1} = dL/dW_T
  H_t   = beta H_{t+1} - eta_t G_t  (t < T),   H_T = dL/dM_T - eta_T G_T
  dq_t  = W_t^T do_t
  dv_t  = -sigma H_t k_t,   dk_t = -sigma H_t^T v_t,   deta_t = -<G_t, M_t>
  dW_0  = G_1,   dM_0 = beta H_1

and without momentum (M absent):

  dv_t = sigma eta_t G_t k_t,  dk_t = sigma eta_t G_t^T v_t,
  deta_t = sigma v_t^T G_t k_t,  dW_0 = G_1.

These are written out below as a loop over the tokens in reverse, on the
stored forward states.  The function is pinned (``tests/test_oracle_grad.py``)
by central finite differences of the scalar
  L = sum_t <o_t, dO_t> + <W_T, dW_T> + <M_T, dM_T>
with respect to every input, and by hand-derived formulas for one token.
"""
from __future__ import annotations

import numpy as np

from .ttt_ref import _prep

__all__ = ["ttt_backward_f64"]


def ttt_backward_f64(q, k, v, eta, dO, dW_T=None, dM_T=None, beta=0.0, ascent=False, S0=None, M0=None):
    """Gradients of the layer with respect to q, k, v, eta (per token), W_0
    and M_0.  Shapes as in ``ttt_recurrence_f64``; dO is [..., T, d_v],
    dW_T and dM_T are [..., d_v, d_k] or None (zero).  Momentum is used iff
    beta != 0.  Returns a dict with dq, dk, dv, deta, dW0 and dM0 (dM0 is
    zeros without momentum)."""
    q, k, v, eta, W, M = _prep(q, k, v, eta, S0, M0)
    dO = np.array(dO, dtype=np.float64)
    use_mom = beta != 0.0
    sigma = -1.0 if ascent else 1.0
    T = q.shape[-2]
    lead = q.shape[:-2]
    dv_, dk_ = v.shape[-1], q.shape[-1]

    # forward, keeping W_t and M_t for every token
    Ws, Ms = [], []
    for t in range(T):
        if use_mom:
            M = beta * M - sigma * v[..., t, :, None] * k[..., t, None, :]
            W = W - eta[..., t, None, None] * M
        else:
            W = W + sigma * eta[..., t, None, None] * v[..., t, :, None] * k[..., t, None, :]
        Ws.append(W)
        Ms.append(M)

    G = np.zeros(lead + (dv_, dk_)) if dW_T is None else np.array(dW_T, dtype=np.float64).reshape(lead + (dv_, dk_))
    Hn = np.zeros(lead + (dv_, dk_)) if dM_T is None else np.array(dM_T, dtype=np.float64).reshape(lead + (dv_, dk_))
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    deta = np.zeros(eta.shape)
    H = None
    for t in range(T - 1, -1, -1):
        G = G + dO[..., t, :, None] * q[..., t, None, :]
        dq[..., t, :] = np.einsum("...nk,...n->...k", Ws[t], dO[..., t, :])
        if use_mom:
            # H_t = beta H_{t+1} - eta_t G_t, where the dM_T term enters at t = T
            H = (Hn if t == T - 1 else beta * H) - eta[..., t, None, None] * G
            dv[..., t, :] = -sigma * np.einsum("...nk,...k->...n", H, k[..., t, :])
            dk[..., t, :] = -sigma * np.einsum("...nk,...n->...k", H, v[..., t, :])
            deta[..., t] = -np.einsum("...nk,...nk->...", G, Ms[t])
        else:
            Gk = np.einsum("...nk,...k->...n", G, k[..., t, :])
            dv[..., t, :] = sigma * eta[..., t, None] * Gk
            dk[..., t, :] = sigma * eta[..., t, None] * np.einsum("...nk,...n->...k", G, v[..., t, :])
            deta[..., t] = sigma * np.einsum("...n,...n->...", v[..., t, :], Gk)
    dM0 = beta * H if use_mom else np.zeros(lead + (dv_, dk_))
    return dict(dq=dq, dk=dk, dv=dv, deta=deta, dW0=G, dM0=dM0)
