"""Pins of the oracle's dt surroundings (dt + bias, softplus, clamp).

softplus is pinned by closed forms: softplus(0) = ln 2, softplus(v) - softplus(-v) = v,
softplus(v) -> v for large v and -> e^v for very negative v; the bias is added per head
and the clamp only acts when dt_max > 0.
"""
import math

import numpy as np

import oracle


def test_identity_without_options():
    dt = np.array([[0.1, 0.02], [0.3, 1e-3]], dtype=np.float32)
    np.testing.assert_array_equal(oracle.dt_effective(dt), dt.astype(np.float64))


def test_softplus_closed_forms():
    assert abs(oracle.dt_effective(np.zeros(1), softplus=True)[0] - math.log(2.0)) < 1e-15
    v = np.linspace(-30.0, 30.0, 121)
    sp = oracle.dt_effective(v, softplus=True)
    spn = oracle.dt_effective(-v, softplus=True)
    np.testing.assert_allclose(sp - spn, v, rtol=0, atol=1e-12)
    big = np.array([40.0, 80.0])
    np.testing.assert_allclose(oracle.dt_effective(big, softplus=True), big, rtol=1e-15)
    small = np.array([-40.0, -60.0])
    np.testing.assert_allclose(oracle.dt_effective(small, softplus=True), np.exp(small), rtol=1e-12)


def test_bias_is_per_head_and_clamp_only_when_asked():
    dt = np.zeros((2, 3, 4))
    bias = np.array([0.0, 1.0, -2.0, 3.0])
    got = oracle.dt_effective(dt, dt_bias=bias)
    np.testing.assert_array_equal(got, np.broadcast_to(bias, dt.shape))
    clamped = oracle.dt_effective(dt, dt_bias=bias, dt_min=0.5, dt_max=2.0)
    np.testing.assert_array_equal(clamped[0, 0], [0.5, 1.0, 0.5, 2.0])
    assert (oracle.dt_effective(dt, dt_bias=bias, dt_min=0.5, dt_max=0.0) == got).all()
