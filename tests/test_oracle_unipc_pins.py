"""Pins of the oracle's UniPC multistep sampler (the sampler the "Wan2.2 I2V
inference trace" names for the latent update; steps from the UniPC paper's
data-prediction form with B(h) = e^h - 1). Independent checks: the first-order
predictor alone is the flow-matching Euler step, and on an ODE with a known
solution each variant converges at its order (1, 2 with the corrector, 3 for
order 2 with the corrector when the last step keeps full order)."""
import math

import numpy as np

from oracle import wan_oracle as O

# A data prediction that depends only on lambda: m(lambda) = cubic, velocity
# v = (x - m) / sigma. The exact flow solution from lambda_a to lambda_b is
# x_b = (sigma_b / sigma_a) x_a + sigma_b int e^lambda m(lambda) dlambda.
C = np.array([[0.3, -0.2], [0.5, 0.1], [-0.2, 0.25], [0.05, -0.04]])
LA, LB = -1.5, 1.5


def _m(lam):
    return C[0] + C[1] * lam + C[2] * lam ** 2 + C[3] * lam ** 3


def _sigma(lam):
    return 1.0 / (1.0 + math.exp(lam))           # alpha / sigma = e^lambda with alpha = 1 - sigma


def _vel(x, s, i):
    return (x - _m(O.flow_lambda(s))) / s


def _primitive(lam):
    c0, c1, c2, c3 = C
    p = c0 + c1 * lam + c2 * lam ** 2 + c3 * lam ** 3
    p1 = c1 + 2 * c2 * lam + 3 * c3 * lam ** 2
    p2 = 2 * c2 + 6 * c3 * lam
    return math.exp(lam) * (p - p1 + p2 - 6 * c3)


def _error(n, **kw):
    sig = [_sigma(l) for l in np.linspace(LA, LB, n + 1)]
    x0 = np.array([0.4, -0.7])
    xf, _ = O.unipc_sample(x0, _vel, sig, **kw)
    exact = (sig[-1] / sig[0]) * x0 + sig[-1] * (_primitive(LB) - _primitive(LA))
    return np.abs(xf - exact).max()


def _ratio(**kw):
    return _error(64, **kw) / _error(128, **kw)


def test_flow_lambda():
    assert O.flow_lambda(0.5) == 0.0
    assert math.isclose(O.flow_lambda(0.2), math.log(4.0))
    assert O.flow_lambda(0.0) == math.inf


def test_first_order_predictor_is_euler():
    rng = np.random.default_rng(0)
    sig = O.flow_sigmas(12)
    vs = [rng.standard_normal(6) for _ in range(12)]
    x0 = rng.standard_normal(6)
    got, _ = O.unipc_sample(x0, lambda x, s, i: vs[i], sig, order=1, corrector=False)
    ref = x0.copy()
    for i in range(12):
        ref = ref + (sig[i + 1] - sig[i]) * vs[i]
    assert np.abs(got - ref).max() <= 1e-12


def test_convergence_orders():
    assert 1.8 <= _ratio(order=1, corrector=False) <= 2.2        # Euler: first order
    assert 3.6 <= _ratio(order=1) <= 4.4                         # UniC-1 raises it to 2
    assert 3.6 <= _ratio(order=2, corrector=False) <= 4.4        # UniP-2: second order
    assert 7.2 <= _ratio(order=2, lower_order_final=False) <= 8.8    # UniPC-2: third order
    # the default (first-order last step) is second order and more accurate than Euler
    assert 3.6 <= _ratio(order=2) <= 4.4
    assert _error(32, order=2) < 0.2 * _error(32, order=1, corrector=False)


def test_schedule_and_final_step():
    sig = O.flow_sigmas(8, shift=5.0)
    assert sig[-1] == 0.0 and sig[0] < 1.0 and np.all(np.diff(sig) < 0)
    # the last step lands on the data prediction of the last evaluation
    rng = np.random.default_rng(1)
    vs = [rng.standard_normal(3) for _ in range(8)]
    got, seen = O.unipc_sample(rng.standard_normal(3), lambda x, s, i: vs[i], sig)
    assert np.allclose(got, seen[-1] - sig[-2] * vs[-1], rtol=0, atol=1e-12)
