"""Pins for the float64 oracle: facts fixed by the pages and by the mathematics.

None of these retypes the oracle's formulas. They check it against hand values,
closed forms, invariants (Parseval, round trip, adjoint, linearity), a library FFT
on the cases that reduce to one, and finite differences. The last test plants
plausible mistakes in copies of the oracle and checks that some pin catches each.
"""
import numpy as np
import pytest

import oracle
from synthetic import normal

POW2 = [2, 4, 8, 16, 32, 64, 128]


def _packed_from_rfft(x):
    """Packed layout read off numpy's rfft (an independent library FFT)."""
    R = np.fft.rfft(x, axis=-1)
    p = x.shape[-1]
    h = p // 2
    out = np.empty_like(x)
    out[..., : h + 1] = R.real
    for k in range(1, h):
        out[..., p - k] = R[..., k].imag
    return out


# ---------------------------------------------------------------- hand values
def test_hand_values(golden):
    rows = golden("packed_hand_values.txt")
    assert len(rows) >= 6
    for (p,), xs, ys in rows:
        x = np.array([float(v) for v in xs])
        y = np.array([float(v) for v in ys])
        assert x.size == int(p) == y.size
        np.testing.assert_allclose(oracle.dft_packed(x), y, atol=1e-12)
        np.testing.assert_allclose(oracle.idft_packed(y), x, atol=1e-12)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("p", POW2)
def test_delta_is_flat_spectrum(p):
    x = np.zeros(p)
    x[0] = 1.0
    want = np.zeros(p)
    want[: p // 2 + 1] = 1.0          # real parts 1, imaginary slots 0
    np.testing.assert_allclose(oracle.dft_packed(x), want, atol=1e-12)


@pytest.mark.parametrize("p", POW2)
def test_constant(p):
    x = np.full(p, 0.75)
    want = np.zeros(p)
    want[0] = 0.75 * p
    np.testing.assert_allclose(oracle.dft_packed(x), want, atol=1e-11)


@pytest.mark.parametrize("p", [4, 8, 16, 64])
def test_cosine_and_sine(p):
    n = np.arange(p)
    for m in range(1, p // 2):
        want = np.zeros(p)
        want[m] = p / 2
        got = oracle.dft_packed(np.cos(2 * np.pi * m * n / p))
        np.testing.assert_allclose(got, want, atol=1e-10)
        # sin(2 pi m n / p) = (e^{i..} - e^{-i..}) / 2i -> Y_m = -i p/2: slot p-m holds -p/2
        want = np.zeros(p)
        want[p - m] = -p / 2
        got = oracle.dft_packed(np.sin(2 * np.pi * m * n / p))
        np.testing.assert_allclose(got, want, atol=1e-10)
    # Nyquist cosine (-1)^n -> p at index p/2
    want = np.zeros(p)
    want[p // 2] = p
    np.testing.assert_allclose(oracle.dft_packed((-1.0) ** n), want, atol=1e-10)


@pytest.mark.parametrize("p", [8, 32])
def test_shifted_delta(p):
    for s in (1, 3, p - 1):
        x = np.zeros(p)
        x[s] = 1.0
        k = np.arange(p // 2 + 1)
        want = np.zeros(p)
        want[: p // 2 + 1] = np.cos(2 * np.pi * k * s / p)
        for kk in range(1, p // 2):
            want[p - kk] = -np.sin(2 * np.pi * kk * s / p)
        np.testing.assert_allclose(oracle.dft_packed(x), want, atol=1e-12)


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("p", POW2 + [512])
def test_packed_parseval(p):
    x = normal(11, (5, p))
    y = oracle.dft_packed(x)
    h = p // 2
    w = np.full(p, 2.0)
    w[0] = 1.0
    w[h] = 1.0
    np.testing.assert_allclose((x * x).sum(-1), (w * y * y).sum(-1) / p, rtol=1e-12)


@pytest.mark.parametrize("p", POW2 + [1024])
def test_round_trips(p):
    x = normal(12, (4, p))
    np.testing.assert_allclose(oracle.idft_packed(oracle.dft_packed(x)), x, atol=1e-11)
    # every real vector is a valid packed spectrum
    y = normal(13, (4, p))
    np.testing.assert_allclose(oracle.dft_packed(oracle.idft_packed(y)), y, atol=1e-10)


def test_linearity():
    x1, x2 = normal(14, (3, 64)), normal(15, (3, 64))
    a, b = 0.3, -1.7
    np.testing.assert_allclose(oracle.dft_packed(a * x1 + b * x2),
                               a * oracle.dft_packed(x1) + b * oracle.dft_packed(x2),
                               atol=1e-11)


# ---------------------------------------------------------------- library FFT
@pytest.mark.parametrize("p", POW2 + [256, 512, 1024, 4096])
def test_matches_library_rfft(p):
    rows = 3 if p >= 1024 else 6
    x = normal(16 + p, (rows, p))
    ref = _packed_from_rfft(x)
    scale = np.abs(ref).max()
    assert np.abs(oracle.dft_packed(x) - ref).max() <= 1e-12 * scale * np.log2(p) + 1e-14
    y = normal(17 + p, (rows, p))
    Y = oracle.unpack_spectrum(y)
    lib = np.fft.irfft(Y[..., : p // 2 + 1], n=p, axis=-1)
    np.testing.assert_allclose(oracle.idft_packed(y), lib, atol=1e-12 * np.abs(lib).max() * p)


def test_unpack_is_hermitian():
    y = normal(18, (2, 16))
    Y = oracle.unpack_spectrum(y)
    for k in range(1, 16):
        np.testing.assert_allclose(Y[:, 16 - k], np.conj(Y[:, k]))
    assert np.all(Y[:, 0].imag == 0) and np.all(Y[:, 8].imag == 0)


# ---------------------------------------------------------------- circulant layer
def _block_conv_fft(x, c):
    """y_i = sum_j circular_conv(c_ij, x_j) by numpy's FFT (convolution theorem)."""
    q, _, p = c.shape
    B = x.shape[0]
    X = np.fft.rfft(x.reshape(B, q, p), axis=-1)
    Cf = np.fft.rfft(c, axis=-1)
    Y = np.einsum("ijk,bjk->bik", Cf, X)
    return np.fft.irfft(Y, n=p, axis=-1).reshape(B, q * p)


def test_identity_and_shift():
    q, p = 3, 8
    x = normal(20, (2, q * p))
    c = np.zeros((q, q, p))
    for i in range(q):
        c[i, i, 0] = 1.0
    np.testing.assert_allclose(oracle.circ_forward(x, c), x, atol=1e-14)
    c = np.zeros((q, q, p))
    for i in range(q):
        c[i, i, 3] = 1.0          # first column delta at 3: y[n] = x[n - 3]
    want = np.roll(x.reshape(2, q, p), 3, axis=-1).reshape(2, q * p)
    np.testing.assert_allclose(oracle.circ_forward(x, c), want, atol=1e-14)


def test_block_orientation():
    """c[i, j] maps input block j to output block i (not the transpose)."""
    q, p = 3, 4
    x = normal(21, (1, q * p))
    c = np.zeros((q, q, p))
    c[0, 2, 0] = 1.0              # output block 0 <- input block 2
    y = oracle.circ_forward(x, c).reshape(q, p)
    np.testing.assert_allclose(y[0], x.reshape(q, p)[2], atol=1e-14)
    np.testing.assert_allclose(y[1:], 0.0, atol=1e-14)


@pytest.mark.parametrize("q,p", [(1, 16), (2, 8), (4, 4), (3, 32)])
def test_forward_matches_convolution_theorem(q, p):
    x = normal(22, (5, q * p))
    c = normal(23, (q, q, p))
    np.testing.assert_allclose(oracle.circ_forward(x, c), _block_conv_fft(x, c), atol=1e-11)


@pytest.mark.parametrize("q,p", [(1, 8), (2, 4), (3, 16)])
def test_grad_x_adjoint(q, p):
    x = normal(24, (4, q * p))
    g = normal(25, (4, q * p))
    c = normal(26, (q, q, p))
    y = oracle.circ_forward(x, c)
    gx, _ = oracle.circ_backward(g, x, c)
    assert np.isclose((y * g).sum(), (x * gx).sum(), rtol=1e-12)
    # adjoint of a circulant is the circulant of the reversed column: also via FFT
    c_adj = np.roll(c[:, :, ::-1], 1, axis=-1).transpose(1, 0, 2)
    np.testing.assert_allclose(gx, _block_conv_fft(g, c_adj), atol=1e-11)


@pytest.mark.parametrize("q,p", [(1, 4), (2, 8), (3, 4)])
def test_grad_c_finite_differences(q, p):
    B = 3
    x = normal(27, (B, q * p))
    g = normal(28, (B, q * p))
    c = normal(29, (q, q, p))
    _, gc = oracle.circ_backward(g, x, c)

    def loss(cc):
        return (oracle.circ_forward(x, cc) * g).sum()

    eps = 1e-3
    for i in range(q):
        for j in range(q):
            for k in range(p):
                e = np.zeros_like(c)
                e[i, j, k] = eps
                fd = (loss(c + e) - loss(c - e)) / (2 * eps)
                assert abs(fd - gc[i, j, k]) <= 1e-9 * (1 + abs(fd)), (i, j, k)


def test_grad_c_as_cross_correlation():
    """grad_c_ij[k] = sum_b sum_n g_i[n] x_j[n - k]: checked with numpy FFT correlation."""
    q, p, B = 2, 16, 5
    x = normal(30, (B, q * p)).reshape(B, q, p)
    g = normal(31, (B, q * p)).reshape(B, q, p)
    c = normal(32, (q, q, p))
    _, gc = oracle.circ_backward(g.reshape(B, -1), x.reshape(B, -1), c)
    G = np.fft.rfft(g, axis=-1)
    X = np.fft.rfft(x, axis=-1)
    S = np.einsum("bik,bjk->ijk", G, np.conj(X))
    np.testing.assert_allclose(gc, np.fft.irfft(S, n=p, axis=-1), atol=1e-11)


# ---------------------------------------------------------------- planted mistakes
def _mutants():
    """Copies of the oracle's transforms with one plausible mistake each."""
    def wrong_sign(x):            # e^{+i} convention
        y = oracle.dft_packed(x)
        p = y.shape[-1]
        y[..., p // 2 + 1:] *= -1
        return y

    def im_slot_swapped(x):       # Im Y_k stored at k instead of p-k
        y = oracle.dft_packed(x)
        p = y.shape[-1]
        y[..., p // 2 + 1:] = y[..., p // 2 + 1:][..., ::-1]
        return y

    def dropped_nyquist(x):       # y_{p/2} forgotten
        y = oracle.dft_packed(x)
        y[..., y.shape[-1] // 2] = 0
        return y

    def scaled_forward(x):        # 1/p put on the forward
        return oracle.dft_packed(x) / x.shape[-1]

    return [wrong_sign, im_slot_swapped, dropped_nyquist, scaled_forward]


def test_pins_catch_planted_mistakes(golden):
    rows = golden("packed_hand_values.txt")
    for mutant in _mutants():
        caught = False
        for (p,), xs, ys in rows:
            x = np.array([float(v) for v in xs])
            y = np.array([float(v) for v in ys])
            if not np.allclose(mutant(x), y, atol=1e-12):
                caught = True
        x = normal(33, (2, 16))
        if not np.allclose(mutant(x), _packed_from_rfft(x), atol=1e-9):
            caught = True
        assert caught, mutant.__name__
    # a transposed layer (c[j, i] used for c[i, j]) fails the orientation pin
    q, p = 3, 4
    c = np.zeros((q, q, p))
    c[0, 2, 0] = 1.0
    x = normal(34, (1, q * p))
    y_t = oracle.circ_forward(x, c.transpose(1, 0, 2)).reshape(q, p)
    assert not np.allclose(y_t[0], x.reshape(q, p)[2])
