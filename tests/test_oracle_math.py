"""The oracle's elementwise and row-wise steps against closed forms and library routines."""
import numpy as np
import pytest
import scipy.special

from oracle import silu, softmax_rows, swiglu_ffn

from conftest import read_golden


def test_silu_matches_library_sigmoid():
    z = np.linspace(-30, 30, 2001)
    np.testing.assert_allclose(silu(z), z * scipy.special.expit(z), rtol=1e-13, atol=1e-300)


def test_silu_closed_forms():
    assert silu(0.0) == 0.0
    # sigma(-z) = 1 - sigma(z)  =>  SiLU(-z) = SiLU(z) - z  (catches a sign slip)
    z = np.linspace(-8, 8, 161)
    np.testing.assert_allclose(silu(-z), silu(z) - z, rtol=0, atol=1e-13)
    # saturation: SiLU(z) -> z for large z, -> 0 for very negative z
    assert abs(silu(60.0) - 60.0) < 1e-20 * 60 + 1e-12
    assert abs(silu(-60.0)) < 1e-24
    assert np.isfinite(silu(-1000.0))


def test_softmax_matches_library_and_invariants():
    rng = np.random.default_rng(1)
    s = rng.normal(size=(7, 13)) * 5
    p = softmax_rows(s)
    np.testing.assert_allclose(p, scipy.special.softmax(s, axis=1), rtol=1e-13)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    # shift invariance and uniform output on equal scores
    np.testing.assert_allclose(softmax_rows(s + 123.0), p, rtol=1e-12)
    np.testing.assert_allclose(softmax_rows(np.zeros((2, 9))), np.full((2, 9), 1 / 9), rtol=1e-15)
    # huge scores do not overflow (max-subtracted form)
    big = softmax_rows(np.array([[1000.0, 1000.0, -1000.0]]))
    np.testing.assert_allclose(big, [[0.5, 0.5, 0.0]], atol=1e-300)


def test_swiglu_hand_worked_example():
    (want,) = read_golden("swiglu_worked.txt")
    u = np.array([[1.0, 1.5]])
    W1 = np.array([[1.0, 0.0]])
    W3 = np.array([[0.0, 2.0]])
    W2 = np.array([[1.0], [-1.0]])
    out = swiglu_ffn(u, W1, W3, W2)
    np.testing.assert_allclose(out[0], [float(want[0]), float(want[1])], rtol=1e-15)


def test_swiglu_against_scalar_loops():
    # element-by-element definition on a rectangular case (d != f catches a transposed W)
    rng = np.random.default_rng(2)
    d, f, n = 5, 3, 4
    u = rng.normal(size=(n, d))
    W1, W3 = rng.normal(size=(f, d)), rng.normal(size=(f, d))
    W2 = rng.normal(size=(d, f))
    want = np.zeros((n, d))
    for r in range(n):
        for c in range(d):
            acc = 0.0
            for i in range(f):
                a = sum(W1[i, q] * u[r, q] for q in range(d))
                b = sum(W3[i, q] * u[r, q] for q in range(d))
                acc += W2[c, i] * (a * scipy.special.expit(a)) * b
            want[r, c] = acc
    np.testing.assert_allclose(swiglu_ffn(u, W1, W3, W2), want, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("bad", ["W1", "W3", "W2"])
def test_swiglu_rejects_wrong_layout(bad):
    rng = np.random.default_rng(3)
    d, f = 6, 4
    mats = {"W1": rng.normal(size=(f, d)), "W3": rng.normal(size=(f, d)),
            "W2": rng.normal(size=(d, f))}
    mats[bad] = mats[bad].T
    with pytest.raises(ValueError):
        swiglu_ffn(rng.normal(size=(2, d)), mats["W1"], mats["W3"], mats["W2"])
