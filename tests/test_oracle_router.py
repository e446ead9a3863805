"""Pins of the router oracle (oracle.router) against what the definition fixes by itself:
element loops, a hand-worked example, unit-vector inputs, central finite differences of the
oracle's own forward (the backward must be its derivative), and the bf16 rounding of the
logits' gradient on constructed ties."""
import numpy as np
import pytest

import synth
from oracle import router as orr
from oracle.layer import bf16_bits_to_f64


def _bits(vals):
    """bf16 bit patterns of values that bf16 holds exactly (small integers, halves ...)."""
    return synth.f32_to_bf16_bits(np.asarray(vals, np.float32))


def test_hand_worked_example():
    # x = [[1, 2], [3, -1]], W_r = [[2, 0.5], [-1, 1], [0, 4]]:
    # logits[0] = [1*2 + 2*0.5, -1 + 2, 8] = [3, 1, 8]; logits[1] = [6 - 0.5, -3 - 1, -4]
    x = _bits([[1, 2], [3, -1]])
    w = _bits([[2, 0.5], [-1, 1], [0, 4]])
    assert np.array_equal(orr.router_logits(x, w), [[3.0, 1.0, 8.0], [5.5, -4.0, -4.0]])
    # with G = [[1, 0, 0], [0, 0, 2]]: dx_r = G W_r, dW_r = G^T x
    g = np.array([[1.0, 0.0, 0.0], [0.0, 0.0, 2.0]])
    dx, dw = orr.router_backward(g, x, w)
    assert np.array_equal(dx, [[2.0, 0.5], [0.0, 8.0]])
    assert np.array_equal(dw, [[1.0, 2.0], [0.0, 0.0], [6.0, -2.0]])


def test_unit_vectors_pick_weight_columns():
    rng = np.random.default_rng(3)
    d, E = 16, 5
    w = synth.f32_to_bf16_bits(rng.standard_normal((E, d)).astype(np.float32))
    x = _bits(np.eye(d))
    assert np.array_equal(orr.router_logits(x, w), bf16_bits_to_f64(w).T)


@pytest.mark.parametrize("T,d,E", [(1, 3, 1), (5, 7, 4), (9, 12, 8)])
def test_vectorised_matches_loops(T, d, E):
    rng = np.random.default_rng(T * 100 + d * 10 + E)
    x = synth.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    w = synth.f32_to_bf16_bits(rng.standard_normal((E, d)).astype(np.float32))
    g = rng.standard_normal((T, E)).astype(np.float32)
    np.testing.assert_allclose(orr.router_logits(x, w), orr.router_logits_bruteforce(x, w),
                               rtol=1e-13, atol=1e-13)
    dx, dw = orr.router_backward(g, x, w)
    bx, bw = orr.router_backward_bruteforce(g, x, w)
    np.testing.assert_allclose(dx, bx, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(dw, bw, rtol=1e-13, atol=1e-13)


def test_backward_is_the_derivative_of_the_forward():
    # L = sum(G * logits(x, W_r)) with G exactly representable in bf16 (the rounding of G is
    # then the identity): dL/dx = dx_r and dL/dW_r = dW_r, by central differences of the
    # oracle's own forward (L is linear in each operand: the difference quotient is exact
    # up to fp64 rounding).
    rng = np.random.default_rng(11)
    T, d, E = 4, 6, 3
    x = rng.standard_normal((T, d))
    w = rng.standard_normal((E, d))
    g = bf16_bits_to_f64(_bits(np.round(rng.standard_normal((T, E)) * 8) / 8))
    dx, dw = orr.router_backward(g, _bits(x), _bits(w))
    xb, wb = bf16_bits_to_f64(_bits(x)), bf16_bits_to_f64(_bits(w))

    def loss(xv, wv):
        return float(np.sum(g * orr.router_logits_values(xv, wv)))
    h = 0.5
    for t in range(T):
        for i in range(d):
            e = np.zeros_like(xb)
            e[t, i] = h
            fd = (loss(xb + e, wb) - loss(xb - e, wb)) / (2 * h)
            assert abs(fd - dx[t, i]) <= 1e-12 * (1 + abs(fd)), (t, i)
    for r in range(E):
        for i in range(d):
            e = np.zeros_like(wb)
            e[r, i] = h
            fd = (loss(xb, wb + e) - loss(xb, wb - e)) / (2 * h)
            assert abs(fd - dw[r, i]) <= 1e-12 * (1 + abs(fd)), (r, i)


def test_gradient_is_rounded_to_bf16_ties_to_even():
    # bf16 keeps 8 significant bits: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 and
    # rounds to the even 1; 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6 and
    # rounds to the even 1 + 2^-6.  With x = W_r = [[1]] the gradients equal rounded G.
    one = _bits([[1.0]])
    for g, want in [(1 + 2.0 ** -8, 1.0), (1 + 3 * 2.0 ** -8, 1 + 2.0 ** -6),
                    (-(1 + 2.0 ** -8), -1.0), (1 + 2.0 ** -7, 1 + 2.0 ** -7)]:
        dx, dw = orr.router_backward(np.array([[g]]), one, one)
        assert dx[0, 0] == want and dw[0, 0] == want, g


def test_planted_mistakes_fail_the_pins(monkeypatch):
    # a backward that skips the bf16 rounding of G, and one that uses W_r's transpose
    # pattern wrongly (rows of W_r indexed by the feature), must each fail a pin above
    real = orr.router_backward

    def no_rounding(dlogits, x_bits, wr_bits):
        g = np.asarray(dlogits, np.float64)
        return g @ bf16_bits_to_f64(wr_bits), g.T @ bf16_bits_to_f64(x_bits)

    def reversed_features(dlogits, x_bits, wr_bits):
        dx, dw = real(dlogits, x_bits, wr_bits)
        return dx[:, ::-1], dw

    monkeypatch.setattr(orr, "router_backward", no_rounding)
    with pytest.raises(AssertionError):
        test_gradient_is_rounded_to_bf16_ties_to_even()
    monkeypatch.setattr(orr, "router_backward", reversed_features)
    with pytest.raises(AssertionError):
        test_backward_is_the_derivative_of_the_forward()
