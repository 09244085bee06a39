"""Pins of the oracle's short convolution and pre-gate normalisation (oracle/module.py) against what
the definitions fix independently: special kernels (identity, delay), a library convolution,
linearity, closed forms on constant inputs, and the normalisation invariants.  CPU only."""
import numpy as np
import pytest

from oracle import module as M

CU = [0, 5, 6, 13, 13, 20]   # ragged, with a length-1 and an empty sequence


def _x(T=20, H=2, d=8, seed=0):
    return np.random.default_rng(seed).standard_normal((T, H, d))


@pytest.mark.parametrize("W", [1, 2, 3, 4])
def test_last_tap_delta_is_identity(W):
    x = _x()
    w = np.zeros((2, 8, W))
    w[:, :, W - 1] = 1.0
    assert np.array_equal(M.short_conv(x, w, CU), x)


@pytest.mark.parametrize("W", [2, 3, 4])
def test_previous_tap_delta_is_a_delay_inside_each_sequence(W):
    x = _x()
    w = np.zeros((2, 8, W))
    w[:, :, W - 2] = 1.0
    y = M.short_conv(x, w, CU)
    for n in range(len(CU) - 1):
        s, e = CU[n], CU[n + 1]
        if e > s:
            assert np.all(y[s] == 0.0)              # nothing leaks in from the previous sequence
            assert np.array_equal(y[s + 1:e], x[s:e - 1])


@pytest.mark.parametrize("W", [1, 2, 4])
def test_matches_numpy_convolve_per_channel(W):
    x = _x(seed=1)
    w = np.random.default_rng(2).standard_normal((2, 8, W))
    y = M.short_conv(x, w, CU)
    for n in range(len(CU) - 1):
        s, e = CU[n], CU[n + 1]
        if e == s:
            continue
        for h in range(2):
            for c in range(8):
                ref = np.convolve(x[s:e, h, c], w[h, c, ::-1])[: e - s]   # causal, taps oldest first
                assert np.allclose(y[s:e, h, c], ref, atol=1e-12)


def test_linear_in_the_input():
    x1, x2 = _x(seed=3), _x(seed=4)
    w = np.random.default_rng(5).standard_normal((2, 8, 3))
    lhs = M.short_conv(2.5 * x1 - 0.5 * x2, w, CU)
    rhs = 2.5 * M.short_conv(x1, w, CU) - 0.5 * M.short_conv(x2, w, CU)
    assert np.allclose(lhs, rhs, atol=1e-12)


def test_constant_input_closed_form():
    T, W = 10, 4
    x = np.ones((T, 1, 8)) * 0.75
    w = np.random.default_rng(6).standard_normal((1, 8, W))
    y = M.short_conv(x, w, [0, T])
    for t in range(T):
        taps = w[0, :, W - 1 - min(t, W - 1):].sum(axis=-1)   # the taps that see the sequence
        assert np.allclose(y[t, 0], 0.75 * taps, atol=1e-12)


def test_l2norm_rows_are_unit_and_scale_free():
    x = _x(seed=7)
    w = np.random.default_rng(8).standard_normal((2, 8, 3))
    y = M.short_conv(x, w, CU, l2norm=True)
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-9)
    assert np.allclose(M.short_conv(3.0 * x, w, CU, l2norm=True), y, atol=1e-9)


def test_norm_gate_closed_forms():
    o = np.random.default_rng(9).standard_normal((6, 3, 16))
    ones = np.ones(16)
    y = M.output_norm_gate(o, None, ones, eps=0.0)
    assert np.allclose(np.mean(y * y, axis=-1), 1.0)                       # RMS of the result is 1
    assert np.allclose(M.output_norm_gate(4.0 * o, None, ones, eps=0.0), y)  # scale invariant
    zero_gate = np.zeros_like(o)
    assert np.allclose(M.output_norm_gate(o, zero_gate, ones, eps=0.0), 0.5 * y)   # sigmoid(0) = 1/2
    gain = np.linspace(0.5, 2.0, 16)
    assert np.allclose(M.output_norm_gate(o, None, gain, eps=0.0), y * gain)
    eps = 0.3
    ye = M.output_norm_gate(o, None, ones, eps=eps)
    ms = np.mean(o * o, axis=-1)
    assert np.allclose(np.mean(ye * ye, axis=-1), ms / (ms + eps))
