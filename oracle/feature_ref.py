"""Float64 CPU oracle for the frozen-MLP feature map and the layer built on it.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may call it.  It shares no code with the CUDA library.

What it computes
----------------
Table 2 of the thelatestinai.com listing of "Test-Time Training with KV
Binding Is Secretly Linear Attention" walks the general TTT layer down to
linear attention.  Its Variant 1 keeps a multi-layer MLP as the fast weight
but lets the inner loop update only the MLP's last layer; Variant 2 also drops
weight normalisation; Variant 3 then swaps the MLP for one linear layer (the
layer of ``ttt_ref``).  In Variants 1-2 every layer before the last is held
fixed during the sequence, so it acts as a feature map phi on the keys (which
the inner loop trains on) and on the queries (which read the fast weight), and
the updated last layer is the linear fast weight W of ``ttt_ref`` acting on
phi(k) and phi(q).  This is the learned kernel feature map phi of the
(phi(Q) phi(K)^T) V form in the kualia.ai explainer, section "The Linear
Attention Equivalence".

Readings (the pages print no formula for the MLP):

* the frozen part is one gated hidden layer of the "GLU Variants Improve
  Transformer" form (SwiGLU, listed among the works the paper builds on in the
  mlsanity.com summary):  phi(x) = silu(W1 x) * (W3 x), elementwise product,
  silu(a) = a / (1 + exp(-a));
* W1, W3 are per-head matrices of shape [d_out, d_in], shared by q and k;
* the weights are seeded random stand-ins for trained ones (no checkpoint is
  published).

Layouts: x is [B, H, T, d_in]; W1, W3 are [H, d_out, d_in]; phi(x) is
[B, H, T, d_out].

Pins (``tests/test_oracle_feature.py``): hand-computed values; the
odd-part identity phi(x; W1, W3) - phi(x; -W1, W3) = (W1 x) * (W3 x) against
an explicit double loop; the ReLU limit for large pre-activations; W1 = 0 and
W3 = 0 give phi = 0; the layer on phi against the textbook kernelised causal
linear attention sum written out with loops.
"""
from __future__ import annotations

import numpy as np

from .ttt_ref import ttt_recurrence_f64

__all__ = ["silu_f64", "feature_map_f64", "ttt_feature_layer_f64"]


def silu_f64(a):
    """silu(a) = a * sigmoid(a) = a / (1 + exp(-a)), in float64.  The
    exponent is clipped at 700 so that exp stays finite; beyond it the
    quotient is below 1e-290 in magnitude (zero for any purpose here)."""
    a = np.asarray(a, dtype=np.float64)
    return a / (1.0 + np.exp(np.minimum(-a, 700.0)))


def feature_map_f64(x, W1, W3):
    """phi(x) = silu(W1 x) * (W3 x) per token, with head h of x using W1[h],
    W3[h].  x: [B, H, T, d_in]; W1, W3: [H, d_out, d_in].  Returns float64
    [B, H, T, d_out]."""
    x = np.asarray(x, dtype=np.float64)
    W1 = np.asarray(W1, dtype=np.float64)
    W3 = np.asarray(W3, dtype=np.float64)
    if x.ndim != 4 or W1.ndim != 3 or W1.shape != W3.shape:
        raise ValueError("x must be [B,H,T,d_in], W1 and W3 [H,d_out,d_in]")
    if W1.shape[0] != x.shape[1] or W1.shape[2] != x.shape[3]:
        raise ValueError("W1/W3 head count or input width does not match x")
    a = np.einsum("bhti,hoi->bhto", x, W1)  # W1 x for every token
    b = np.einsum("bhti,hoi->bhto", x, W3)  # W3 x for every token
    return silu_f64(a) * b


def ttt_feature_layer_f64(q, k, v, eta, W1, W3, beta=0.0, ascent=False, S0=None, M0=None):
    """The TTT layer whose fast weight is the last layer of the frozen-MLP
    network: the linear layer's token-by-token recurrence (``ttt_recurrence_f64``)
    run on phi(q), phi(k) and v.  S0, M0: [B, H, d_v, d_out].
    Returns (o [B,H,T,d_v], W_T, M_T)."""
    return ttt_recurrence_f64(feature_map_f64(q, W1, W3), feature_map_f64(k, W1, W3), v, eta,
                              beta=beta, ascent=ascent, S0=S0, M0=M0)
