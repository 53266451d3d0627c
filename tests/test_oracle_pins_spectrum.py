"""Pins for the oracle's explicit-spectrum cast and its 2-D transform.

Checked against hand values (tests/golden), numpy's FFT (an independent library
routine; the oracle computes by DFT matrices), closed forms, the reduction to the
1-D transform, Parseval and round trips; the last test plants plausible mistakes in
copies of the oracle and checks that some pin catches each.
"""
import numpy as np
import pytest

import oracle
from synthetic import normal

SHAPES = [(2, 2), (2, 4), (4, 2), (4, 4), (8, 16), (16, 8), (2, 64), (64, 2), (32, 32)]


# ------------------------------------------------------------ 1-D complex cast
@pytest.mark.parametrize("p", [2, 4, 8, 64, 512])
def test_packed_to_rfft_is_library_rfft(p):
    x = normal(40 + p, (3, p))
    np.testing.assert_allclose(oracle.packed_to_rfft(oracle.dft_packed(x)), np.fft.rfft(x, axis=-1),
                               atol=1e-9 * p)


def test_rfft_to_packed_hand_values(golden):
    for (p,), xs, ys in golden("packed_hand_values.txt"):
        x = np.array([float(v) for v in xs])
        y = np.array([float(v) for v in ys])
        np.testing.assert_allclose(oracle.rfft_to_packed(np.fft.rfft(x)), y, atol=1e-12)


@pytest.mark.parametrize("p", [2, 4, 32, 4096])
def test_cast_round_trip_is_exact(p):
    y = normal(41, (5, p))
    z = oracle.packed_to_rfft(y)
    assert z.shape == (5, p // 2 + 1)
    assert np.all(z[:, 0].imag == 0) and np.all(z[:, -1].imag == 0)
    assert np.array_equal(oracle.rfft_to_packed(z), y)          # moves values only


# ------------------------------------------------------------------------ 2-D
def test_2d_hand_values(golden):
    rows = golden("packed2d_hand_values.txt")
    assert len(rows) >= 5
    for (R, C), xs, ys in rows:
        R, C = int(R), int(C)
        x = np.array([float(v) for v in xs]).reshape(R, C)
        y = np.array([float(v) for v in ys]).reshape(R, C)
        np.testing.assert_allclose(oracle.dft2_packed(x), y, atol=1e-12)
        np.testing.assert_allclose(oracle.idft2_packed(y), x, atol=1e-12)


@pytest.mark.parametrize("R,C", SHAPES)
def test_2d_full_spectrum_is_library_fft2(R, C):
    x = normal(42, (2, R, C))
    want = np.fft.fft2(x)
    np.testing.assert_allclose(oracle.dft2_full(x), want, atol=1e-10 * R * C)
    np.testing.assert_allclose(oracle.unpack2_spectrum(oracle.dft2_packed(x)), want, atol=1e-10 * R * C)


@pytest.mark.parametrize("R,C", SHAPES)
def test_2d_round_trips(R, C):
    x = normal(43, (3, R, C))
    np.testing.assert_allclose(oracle.idft2_packed(oracle.dft2_packed(x)), x, atol=1e-12)
    y = normal(44, (3, R, C))       # every real array is the packed spectrum of a real image
    np.testing.assert_allclose(oracle.dft2_packed(oracle.idft2_packed(y)), y, atol=1e-12)


@pytest.mark.parametrize("R,C", [(4, 8), (16, 4), (8, 8)])
def test_2d_separable_image(R, C):
    u, v = normal(45, (R,)), normal(46, (C,))
    Y = oracle.unpack2_spectrum(oracle.dft2_packed(np.outer(u, v)))
    np.testing.assert_allclose(Y, np.outer(np.fft.fft(u), np.fft.fft(v)), atol=1e-10)


@pytest.mark.parametrize("R,C", [(4, 8), (8, 4), (16, 16)])
def test_2d_reduces_to_1d_on_a_single_row(R, C):
    """Only row 0 nonzero: Y[k1, k2] = X[k2] for every k1 (X the 1-D spectrum)."""
    x = np.zeros((R, C))
    x[0] = normal(47, (C,))
    y1 = oracle.dft_packed(x[0])
    y2 = oracle.dft2_packed(x)
    h = C // 2
    for k2 in range(1, h):
        np.testing.assert_allclose(y2[:, k2], y1[k2], atol=1e-12)
        np.testing.assert_allclose(y2[:, C - k2], y1[C - k2], atol=1e-12)
    for k2 in (0, h):                 # a constant real column: its packed column
        col = np.zeros(R)
        col[: R // 2 + 1] = y1[k2]
        np.testing.assert_allclose(y2[:, k2], col, atol=1e-12)


@pytest.mark.parametrize("R,C", [(4, 8), (32, 16)])
def test_2d_reduces_to_1d_on_a_single_column(R, C):
    """Only column 0 nonzero: Y[k1, k2] = X[k1] for every k2."""
    x = np.zeros((R, C))
    x[:, 0] = normal(48, (R,))
    X = np.fft.fft(x[:, 0])
    y2 = oracle.dft2_packed(x)
    for k2 in range(1, C // 2):
        np.testing.assert_allclose(y2[:, k2], X.real, atol=1e-12)
        np.testing.assert_allclose(y2[:, C - k2], X.imag, atol=1e-12)
    for k2 in (0, C // 2):
        np.testing.assert_allclose(y2[:, k2], oracle.dft_packed(x[:, 0]), atol=1e-12)


@pytest.mark.parametrize("R,C", [(8, 8), (4, 32)])
def test_2d_plane_wave(R, C):
    """cos(2 pi (a r / R + b c / C)) has Y = RC/2 at (a, b) and at (-a, -b)."""
    r, c = np.meshgrid(np.arange(R), np.arange(C), indexing="ij")
    a, b = 1, 3
    y = oracle.dft2_packed(np.cos(2 * np.pi * (a * r / R + b * c / C)))
    want = np.zeros((R, C))
    want[a, b] = R * C / 2          # Re Y[a, b]; Y[R - a, b] = 0, Im parts 0
    np.testing.assert_allclose(y, want, atol=1e-9)


@pytest.mark.parametrize("R,C", [(8, 16), (64, 4)])
def test_2d_parseval(R, C):
    x = normal(49, (R, C))
    Y = oracle.unpack2_spectrum(oracle.dft2_packed(x))
    np.testing.assert_allclose(np.sum(np.abs(Y) ** 2) / (R * C), np.sum(x ** 2), rtol=1e-12)


# ------------------------------------------------------------ planted mistakes
def _mutants():
    def transposed(x):                  # axes swapped (needs a square image)
        return np.swapaxes(oracle.dft2_packed(np.swapaxes(x, -1, -2)), -1, -2)

    def im_columns_reversed(x):         # Im Y[., k2] stored at column k2 + C/2
        y = oracle.dft2_packed(x)
        C = y.shape[-1]
        y[..., C // 2 + 1:] = y[..., C // 2 + 1:][..., ::-1]
        return y

    def column0_as_pair(x):             # column 0 stored as plain Re (no packing down it)
        y = oracle.dft2_packed(x)
        y[..., :, 0] = oracle.dft2_full(x)[..., :, 0].real
        return y

    def conj_sign(x):                   # e^{+i} along the rows
        y = oracle.dft2_packed(x)
        y[..., :, y.shape[-1] // 2 + 1:] *= -1
        return y

    return [transposed, im_columns_reversed, column0_as_pair, conj_sign]


def test_2d_pins_catch_planted_mistakes(golden):
    rows = golden("packed2d_hand_values.txt")
    for mutant in _mutants():
        caught = False
        for (R, C), xs, ys in rows:
            R, C = int(R), int(C)
            x = np.array([float(v) for v in xs]).reshape(R, C)
            y = np.array([float(v) for v in ys]).reshape(R, C)
            if R == C or mutant.__name__ != "transposed":
                if not np.allclose(mutant(x), y, atol=1e-12):
                    caught = True
        x = normal(50, (8, 8))
        if not np.allclose(oracle.unpack2_spectrum(mutant(x)), np.fft.fft2(x), atol=1e-9):
            caught = True
        assert caught, mutant.__name__


def test_2d_single_slots_hand_values(golden):
    for (R, C), xs, ys in golden("packed2d_hand_values.txt"):
        R, C = int(R), int(C)
        x = np.array([float(v) for v in xs]).reshape(R, C)
        y = np.array([float(v) for v in ys]).reshape(R, C)
        slots = [(r, c) for r in range(R) for c in range(C)]
        np.testing.assert_allclose(oracle.dft2_packed_at(x, slots), y.ravel(), atol=1e-12)


@pytest.mark.parametrize("R,C", [(8, 16), (16, 4), (2, 8)])
def test_2d_single_slots_read_fft2(R, C):
    """Each slot is Re or Im of the fft2 entry that the layout assigns it."""
    x = normal(51, (R, C))
    F = np.fft.fft2(x)
    slots = [(r, c) for r in range(R) for c in range(C)]
    got = oracle.dft2_packed_at(x, slots)
    for (r, c), v in zip(slots, got):
        if 0 < c < C // 2:
            want = F[r, c].real
        elif c > C // 2:
            want = F[r, C - c].imag
        elif r <= R // 2:
            want = F[r, c].real
        else:
            want = F[R - r, c].imag
        assert abs(v - want) <= 1e-10, (r, c)
