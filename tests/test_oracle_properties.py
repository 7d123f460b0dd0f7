"""Property tests of the float64 oracle over random shapes (hypothesis):
the chunk regrouping the GPU kernels implement equals the literal
recurrence for any chunk size, ragged tail, momentum and sign; the
backward is linear in the upstream gradient and its dot product with a
random direction matches the derivative of the forward."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import ttt_backward_f64, ttt_chunked_f64, ttt_recurrence_f64

shapes = st.tuples(st.integers(1, 2), st.integers(1, 2), st.integers(1, 23), st.integers(1, 5), st.integers(1, 5))


def _draw(seed, B, H, T, dk, dv):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B, H, T, dk)), r.standard_normal((B, H, T, dk)), r.standard_normal((B, H, T, dv)),
            r.uniform(0.05, 0.6, (B, H, T)), r.standard_normal((B, H, dv, dk)), r.standard_normal((B, H, dv, dk)))


@settings(max_examples=40, deadline=None)
@given(shapes, st.integers(1, 9), st.sampled_from([0.0, 0.3, 0.9]), st.booleans(), st.integers(0, 2**31 - 1))
def test_chunked_regrouping_equals_recurrence(shape, chunk, beta, ascent, seed):
    q, k, v, eta, S0, M0 = _draw(seed, *shape)
    a = ttt_recurrence_f64(q, k, v, eta, beta=beta, ascent=ascent, S0=S0, M0=M0)
    b = ttt_chunked_f64(q, k, v, eta, chunk, beta=beta, ascent=ascent, S0=S0, M0=M0)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-10, atol=1e-10)


@settings(max_examples=25, deadline=None)
@given(shapes, st.sampled_from([0.0, 0.7]), st.booleans(), st.integers(0, 2**31 - 1))
def test_backward_directional_derivative(shape, beta, ascent, seed):
    q, k, v, eta, S0, M0 = _draw(seed, *shape)
    r = np.random.default_rng(seed + 1)
    dO = r.standard_normal(v.shape)
    dirs = [r.standard_normal(x.shape) for x in (q, k, v, eta)]
    g = ttt_backward_f64(q, k, v, eta, dO, beta=beta, ascent=ascent, S0=S0, M0=M0 if beta else None)

    def L(h):
        o, _, _ = ttt_recurrence_f64(q + h * dirs[0], k + h * dirs[1], v + h * dirs[2], eta + h * dirs[3],
                                     beta=beta, ascent=ascent, S0=S0, M0=M0 if beta else None)
        return float(np.sum(o * dO))

    h = 1e-6
    fd = (L(h) - L(-h)) / (2 * h)
    an = sum(float(np.sum(g[n] * d)) for n, d in zip(("dq", "dk", "dv", "deta"), dirs))
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (fd, an)
