"""Helpers shared by the GPU parity tests: oracle calls on the exact inputs
given to the GPU, and the error measures with the stated tolerances.

Tolerances (against the float64 oracle):
  fp32 inputs: max |x - ref| / max |ref| <= 1e-4, per output tensor;
  bf16 inputs (fp32 accumulation): ||x - ref||_F / ||ref||_F <= 2e-2 for every
  (b, h) slice, plus the same ratio over the whole tensor.
"""
import numpy as np
import torch

import oracle

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def f64(t):
    return None if t is None else t.detach().float().cpu().double().numpy()


def oracle_forward(q, k, v, eta, eta_const, beta=0.0, ascent=False, S0=None, M0=None):
    e = f64(eta) if eta is not None else eta_const
    return oracle.ttt_recurrence_f64(f64(q), f64(k), f64(v), e, beta=beta, ascent=ascent,
                                     S0=f64(S0), M0=f64(M0))


def max_rel(x, ref):
    x = f64(x) if torch.is_tensor(x) else x
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-30))


def fro_rel_per_slice(x, ref, lead=2):
    """Worst per-(b,h) relative Frobenius error and the global one."""
    x = f64(x) if torch.is_tensor(x) else x
    xs = x.reshape(int(np.prod(x.shape[:lead])), -1)
    rs = ref.reshape(xs.shape)
    num = np.linalg.norm(xs - rs, axis=1)
    den = np.maximum(np.linalg.norm(rs, axis=1), 1e-30)
    glob = float(np.linalg.norm(xs - rs) / max(np.linalg.norm(rs), 1e-30))
    return float(np.max(num / den)), glob


def assert_f32(x, ref, what=""):
    e = max_rel(x, ref)
    assert e <= TOL_F32, f"{what}: max-rel error {e:.3e} > {TOL_F32}"
    return e


def assert_bf16(x, ref, what="", lead=2):
    worst, glob = fro_rel_per_slice(x, ref, lead)
    assert worst <= TOL_BF16 and glob <= TOL_BF16, f"{what}: rel-Frobenius worst {worst:.3e}, global {glob:.3e}"
    return worst
