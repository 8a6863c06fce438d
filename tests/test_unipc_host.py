"""The library's host-side UniPC coefficients (wan_unipc_coefficients, no GPU
needed) against the oracle's corrector and predictor, whose outputs are
linear in the previous sample, the new sample and the data predictions: the
coefficients are read off the oracle by feeding it unit vectors."""
import ctypes

import numpy as np
import pytest

from oracle import wan_oracle as O
from video_diffusion_transformer_fwd_b200 import wan


def _lib_coef(sigmas, step, order, lof):
    sig = (ctypes.c_double * len(sigmas))(*sigmas)
    coef = (ctypes.c_double * 8)()
    wan.check(wan.wan_unipc_coefficients(sig, len(sigmas), step, order, 1 if lof else 0, coef))
    return np.array(list(coef))


def _oracle_coef(sigmas, i, order, lof):
    n = len(sigmas) - 1

    def this_order(j):
        return min(order, n - j if lof else order, j + 1)
    e = np.eye(5)          # basis: x, last, m_{i-1}, m_{i-2}, m_i
    x, last, m1, m2, mi = e
    if i > 0:
        oc = this_order(i - 1)
        hist = [m2, m1] if oc == 2 else [m1]
        xc = O.unipc_correct(last, hist, mi, sigmas, i, oc)
    else:
        xc = x
    op = this_order(i)
    xn = O.unipc_predict(xc, [m1, mi] if op == 2 else [mi], sigmas, i, op)
    # x_next in terms of (x_c, m_i, m_{i-1}): x_c enters with weight xn / xc on
    # the basis vector that carries x_c (last if corrected, x otherwise)
    carrier = 1 if i > 0 else 0
    p_xc = xn[carrier] / xc[carrier]
    p_mi = xn[4] - p_xc * xc[4]
    p_m1 = xn[2] - p_xc * xc[2]
    return np.array([xc[0], xc[1], xc[2], xc[3], xc[4], p_xc, p_mi, p_m1])


@pytest.mark.parametrize("n,shift", [(4, 5.0), (10, 3.0), (25, 1.0)])
@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("lof", [True, False])
def test_coefficients_match_oracle(n, shift, order, lof):
    sig = list(O.flow_sigmas(n, shift))
    if not lof:
        sig[-1] = sig[-2] * 0.5          # a last sigma above 0 keeps the full order
    for i in range(n):
        got = _lib_coef(sig, i, order, lof)
        ref = _oracle_coef(sig, i, order, lof)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), (i, got, ref)


def test_coefficients_reject_bad_schedules():
    coef = (ctypes.c_double * 8)()
    bad = (ctypes.c_double * 3)(0.5, 0.7, 0.0)           # increasing
    assert wan.wan_unipc_coefficients(bad, 3, 0, 2, 1, coef) == wan.WAN_EINVAL
    ok = (ctypes.c_double * 3)(0.9, 0.5, 0.0)
    assert wan.wan_unipc_coefficients(ok, 3, 2, 2, 1, coef) == wan.WAN_EINVAL      # step out of range
    assert wan.wan_unipc_coefficients(ok, 3, 0, 3, 1, coef) == wan.WAN_EUNSUPPORTED
    one = (ctypes.c_double * 3)(1.0, 0.5, 0.0)
    assert wan.wan_unipc_coefficients(one, 3, 0, 2, 1, coef) == wan.WAN_EINVAL     # sigma 1 (alpha 0)
