"""Seeded synthetic inputs for the causal TTT / linear-attention layer.

Shared by the tests, the benchmark and the smoke check.  This module holds
the input recipe only (random draws, per-token L2 normalisation of q and k,
the learning-rate schedule eta_t = sigmoid(z_t)/sqrt(d_k)); none of the
layer's own arithmetic lives here, and it imports neither the oracle nor the
CUDA library.

Recipe (the pages publish no workload beyond "the TTT layer on the LLM task",
Table 2 of the thelatestinai.com listing, so every tensor is synthetic):
  q, k ~ N(0, 1) per element, then divided by their L2 norm per token;
  v ~ N(0, 1);  z ~ N(0, 1) per (b, h, t) and eta_t = sigmoid(z_t)/sqrt(d_k)
  for a per-token learning rate, or the constant 1/sqrt(d_k);
  all drawn in fp32 from one torch.Generator in the order q, k, v, z, then
  rounded to the working dtype (bf16 or fp32).
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["LayerCase", "CONFIGS", "make_case", "make_qkv", "get_config", "make_feature_weights"]


@dataclasses.dataclass(frozen=True)
class LayerCase:
    """One workload: shapes, dtype, learning-rate mode, momentum, chunk."""
    name: str
    B: int
    H: int
    T: int
    d_k: int
    d_v: int
    dtype: str            # "f32" or "bf16"
    eta_mode: str         # "const" or "token"
    beta: float
    chunk: int
    seed: int
    ascent: bool = False

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def eta_const(self) -> float:
        return 1.0 / math.sqrt(self.d_k)

    def replace(self, **kw) -> "LayerCase":
        return dataclasses.replace(self, **kw)


# The five workloads the layer is measured and checked on.
CONFIGS = {
    # tiny fp32 layer: constant eta, no momentum (Variant 5)
    "tiny_f32": LayerCase("tiny_f32", 1, 2, 256, 32, 32, "f32", "const", 0.0, 64, 0),
    # LLM-shaped layer: per-token eta, no momentum
    "llm_d64": LayerCase("llm_d64", 4, 16, 4096, 64, 64, "bf16", "token", 0.0, 64, 1),
    # momentum layer: per-token eta, SGD momentum 0.9 (Variant 3, linear W)
    "momentum_d128": LayerCase("momentum_d128", 2, 16, 8192, 128, 128, "bf16", "token", 0.9, 128, 2),
    # long-context throughput: constant eta, no momentum
    "long_d128": LayerCase("long_d128", 1, 8, 65536, 128, 128, "bf16", "const", 0.0, 128, 3),
}

# Batched decode: 256 sequences x 16 heads, d = 128, 2048-token prefill then
# 512 single-token steps, constant eta, no momentum.
DECODE = dict(N=256, H=16, d=128, prefill=2048, steps=512, seed=4, dtype="bf16")


def get_config(name: str) -> LayerCase:
    return CONFIGS[name]


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True).clamp_min(1e-12)


def make_qkv(shape_lead, T, d_k, d_v, seed, device="cpu", with_z=True):
    """fp32 draws in the fixed order q, k, v, z from one generator."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = torch.randn(*shape_lead, T, d_k, generator=g, device=device)
    k = torch.randn(*shape_lead, T, d_k, generator=g, device=device)
    v = torch.randn(*shape_lead, T, d_v, generator=g, device=device)
    z = torch.randn(*shape_lead, T, generator=g, device=device) if with_z else None
    return _unit(q), _unit(k), v, z


def make_case(case: LayerCase, device="cpu", B=None, H=None, T=None):
    """Inputs for ``case`` (optionally with B, H or T overridden for a reduced
    sample).  Returns a dict with q, k, v in the case dtype, eta as a
    [B, H, T] fp32 tensor (per-token mode) or None, eta_const, beta, chunk."""
    B = case.B if B is None else B
    H = case.H if H is None else H
    T = case.T if T is None else T
    q, k, v, z = make_qkv((B, H), T, case.d_k, case.d_v, case.seed, device)
    dt = case.torch_dtype
    eta = None
    if case.eta_mode == "token":
        eta = (torch.sigmoid(z) / math.sqrt(case.d_k)).float().contiguous()
    return dict(
        q=q.to(dt).contiguous(), k=k.to(dt).contiguous(), v=v.to(dt).contiguous(),
        eta=eta, eta_const=case.eta_const, beta=case.beta, chunk=case.chunk,
        ascent=case.ascent,
    )


def make_decode_inputs(device="cuda", N=None, H=None, prefill=None, steps=None, d=None, seed=None):
    """Inputs of the batched decode workload: a bf16 prefill [N,H,T,d] (q, k
    unit-norm per token, v normal) and per-step bf16 q, k, v [steps,N,H,d],
    drawn on `device` from one generator in the order prefill q, k, v, then
    step q, k, v.  Constant learning rate 1/sqrt(d), no momentum."""
    N = DECODE["N"] if N is None else N
    H = DECODE["H"] if H is None else H
    T = DECODE["prefill"] if prefill is None else prefill
    S = DECODE["steps"] if steps is None else steps
    d = DECODE["d"] if d is None else d
    g = torch.Generator(device=device)
    g.manual_seed(DECODE["seed"] if seed is None else seed)

    def draw(*shape, unit):
        x = torch.randn(*shape, generator=g, device=device)
        if unit:
            x = _unit(x)
        return x.to(torch.bfloat16)

    pq, pk, pv = draw(N, H, T, d, unit=True), draw(N, H, T, d, unit=True), draw(N, H, T, d, unit=False)
    sq, sk, sv = draw(S, N, H, d, unit=True), draw(S, N, H, d, unit=True), draw(S, N, H, d, unit=False)
    return dict(prefill=(pq, pk, pv), steps=(sq, sk, sv), eta_const=1.0 / math.sqrt(d))


def make_feature_weights(H, d_in, d_out, seed, dtype=torch.bfloat16, device="cpu"):
    """Seeded stand-ins for the frozen gated layer of the feature map,
    phi(x) = silu(W1 x) * (W3 x): W1 and W3 [H, d_out, d_in] with N(0, 1)
    entries, drawn in fp32 in the order W1, W3 from one generator and rounded
    to `dtype`.  With unit-norm q and k every pre-activation is then N(0, 1),
    the range where the gate is neither linear nor saturated."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    W1 = torch.randn(H, d_out, d_in, generator=g, device=device)
    W3 = torch.randn(H, d_out, d_in, generator=g, device=device)
    return W1.to(dtype).contiguous(), W3.to(dtype).contiguous()
