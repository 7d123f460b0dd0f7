"""The seeded input recipe: deterministic, unit-norm q/k, eta range."""
import math

import torch

from synth import CONFIGS, make_case


def test_deterministic_and_recipe():
    c = CONFIGS["llm_d64"]
    a = make_case(c, B=1, H=2, T=64)
    b = make_case(c, B=1, H=2, T=64)
    for n in ("q", "k", "v", "eta"):
        assert torch.equal(a[n], b[n])
    assert a["q"].dtype == torch.bfloat16
    nq = torch.linalg.vector_norm(a["q"].float(), dim=-1)
    assert torch.allclose(nq, torch.ones_like(nq), atol=1e-2)
    e = a["eta"]
    assert e.shape == (1, 2, 64) and e.dtype == torch.float32
    assert float(e.min()) > 0 and float(e.max()) < 1 / math.sqrt(64)


def test_const_eta_case():
    c = CONFIGS["tiny_f32"]
    a = make_case(c)
    assert a["eta"] is None and a["q"].dtype == torch.float32
    assert abs(a["eta_const"] - 1 / math.sqrt(32)) < 1e-12
    assert a["q"].shape == (1, 2, 256, 32)
