"""Plain float64 reference computations (test infrastructure only; see oracle/__init__.py).

Conventions (the pages leave these open; the readings taken are listed with the
reason in the design notes of the repository):
  * DFT sign: Y_k = sum_n x_n exp(-2 pi i k n / p), forward unnormalised, inverse
    carries 1/p.
  * Slot p-k of the packed row holds +Im Y_k.
  * p is a power of two, p >= 2. For p = 2 the packed row is [Y_0, Y_1].
  * Circulant block c_ij is the first column of its p x p block:
    C_ij[n][m] = c_ij[(n - m) mod p]; i indexes output blocks, j input blocks.
"""
from __future__ import annotations

import numpy as np


def _check_p(p: int) -> None:
    if p < 2 or (p & (p - 1)) != 0:
        raise ValueError(f"p must be a power of two >= 2, got {p}")


def _dft_cos_sin(p: int):
    """cos and sin of 2 pi (k n mod p) / p for k, n in [0, p).

    The angle is reduced with exact integer arithmetic before the float64 cos/sin
    library calls, so every entry is as accurate as the library routine.
    """
    k = np.arange(p, dtype=np.int64)
    kn = np.outer(k, k) % p
    ang = (2.0 * np.pi / p) * kn.astype(np.float64)
    return np.cos(ang), np.sin(ang)


def dft_packed(x: np.ndarray) -> np.ndarray:
    """Packed real DFT of each row of x (shape (..., p)), float64.

    Definition: Y_k = sum_{n<p} x_n e^{-2 pi i k n/p}, i.e.
    Re Y_k = sum_n x_n cos(2 pi k n/p), Im Y_k = -sum_n x_n sin(2 pi k n/p).
    Packed layout ("Memory-Efficient Training with In-Place FFT Implementation",
    paper-notes page, method section "Squeeze N+2 -> N"; summary page "Approach"):
    out[0] = Y_0, out[p/2] = Y_{p/2}, out[k] = Re Y_k and out[p-k] = Im Y_k for
    0 < k < p/2. Y_0 and Y_{p/2} are real for real input.
    """
    x = np.asarray(x, dtype=np.float64)
    p = x.shape[-1]
    _check_p(p)
    cos, sin = _dft_cos_sin(p)
    h = p // 2
    re = x @ cos[: h + 1].T            # Re Y_k, k = 0..p/2
    im = -(x @ sin[1:h].T)             # Im Y_k, k = 1..p/2-1
    out = np.empty_like(x)
    out[..., : h + 1] = re
    if h > 1:
        out[..., h + 1:] = im[..., ::-1]   # slot p-k holds Im Y_k
    return out


def unpack_spectrum(y: np.ndarray) -> np.ndarray:
    """Full complex spectrum Y_0..Y_{p-1} (complex128) of packed rows y.

    Reads the packed layout of dft_packed and fills the other half by conjugate
    symmetry Y_{p-k} = conj(Y_k) of a real signal's spectrum (paper-notes page,
    "Squeeze N+2 -> N").
    """
    y = np.asarray(y, dtype=np.float64)
    p = y.shape[-1]
    _check_p(p)
    h = p // 2
    Y = np.zeros(y.shape, dtype=np.complex128)
    Y[..., 0] = y[..., 0]
    Y[..., h] = y[..., h]
    for k in range(1, h):
        Y[..., k] = y[..., k] + 1j * y[..., p - k]
        Y[..., p - k] = y[..., k] - 1j * y[..., p - k]
    return Y


def idft_packed(y: np.ndarray) -> np.ndarray:
    """Inverse of dft_packed: x_n = (1/p) sum_{k<p} Y_k e^{+2 pi i k n/p}, float64.

    Y is the conjugate-symmetric spectrum read from the packed rows, so the sum is
    real; the real part is returned. The 1/p factor is the product of the halving
    in every inverse butterfly level described on the paper-notes page ("In-place
    IFFT design": x_a = (y_a + y_b)/2, x_b = (y_a - y_b)/(2 W)).
    """
    y = np.asarray(y, dtype=np.float64)
    p = y.shape[-1]
    Y = unpack_spectrum(y)
    cos, sin = _dft_cos_sin(p)
    # e^{+i theta} = cos + i sin; keep the real part of Y * e^{+i theta}.
    re = Y.real @ cos - Y.imag @ sin
    return re / p


def circulant_matrix(c: np.ndarray) -> np.ndarray:
    """Dense D x D weight of a block-circulant layer, float64.

    c has shape (q, q, p): c[i, j] is the first column of the circulant block in
    block-row i (output block) and block-column j (input block), so
    W[i*p + n, j*p + m] = c[i, j, (n - m) mod p]. ("Memory-Efficient Training with
    In-Place FFT Implementation", paper-notes page, "Circulant matrix training
    adaptation": y = IFFT(FFT(c) (.) FFT(x)) is the product with this circulant.)
    """
    c = np.asarray(c, dtype=np.float64)
    q, q2, p = c.shape
    if q != q2:
        raise ValueError("c must have shape (q, q, p)")
    _check_p(p)
    n = np.arange(p)
    idx = (n[:, None] - n[None, :]) % p          # (n, m) -> (n - m) mod p
    blocks = c[:, :, idx]                         # (i, j, n, m)
    return blocks.transpose(0, 2, 1, 3).reshape(q * p, q * p)


def circ_forward(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """y = W x for every token row of x (shape (B, D)), W = circulant_matrix(c)."""
    W = circulant_matrix(c)
    x = np.asarray(x, dtype=np.float64)
    return x @ W.T


def circ_backward(g: np.ndarray, x: np.ndarray, c: np.ndarray):
    """Gradients of L = sum_b <g_b, W x_b> with respect to x and c.

    grad_x = W^T g (per token). grad_c by the chain rule through the entries of W:
    dL/dW = sum_b g_b x_b^T, and c[i, j, k] appears in W exactly at the entries
    (i*p + n, j*p + m) with (n - m) mod p = k, so
    grad_c[i, j, k] = sum_n dL/dW[i*p + n, j*p + (n - k) mod p].
    ("Gradient computation likewise keeps the symmetry", paper-notes page,
    "Circulant matrix training adaptation".)
    """
    c = np.asarray(c, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    q, _, p = c.shape
    W = circulant_matrix(c)
    grad_x = g @ W
    dW = (g.T @ x).reshape(q, p, q, p)            # [i, n, j, m]
    n = np.arange(p)
    grad_c = np.empty((q, q, p), dtype=np.float64)
    for k in range(p):
        m = (n - k) % p
        grad_c[:, :, k] = dW[:, n, :, m].sum(axis=0)   # advanced dims first: (p, q, q)
    return grad_x, grad_c


# ------------------------------------------------------ explicit complex spectrum
def packed_to_rfft(y: np.ndarray) -> np.ndarray:
    """Bins Y_0..Y_{p/2} (complex128, shape (..., p/2 + 1)) of packed rows y.

    The explicit complex spectrum that the packed layout encodes implicitly
    ("Memory-Efficient Training with In-Place FFT Implementation", summary page,
    "Limitations": reaching it needs a cast out of the in-place buffer, since p
    reals become p/2 + 1 complex values). Bins 0 and p/2 have zero imaginary part.
    """
    Y = unpack_spectrum(y)
    return Y[..., : y.shape[-1] // 2 + 1].copy()


def rfft_to_packed(z: np.ndarray) -> np.ndarray:
    """Packed rows (float64, shape (..., p)) of bins z = Y_0..Y_{p/2}, p = 2 (n - 1).

    Inverse of packed_to_rfft on spectra of real rows: slot k takes Re Y_k and slot
    p - k takes Im Y_k for 0 < k < p/2; the imaginary parts of Y_0 and Y_{p/2}
    (zero for a real row) are not stored.
    """
    z = np.asarray(z, dtype=np.complex128)
    p = 2 * (z.shape[-1] - 1)
    _check_p(p)
    h = p // 2
    out = np.empty(z.shape[:-1] + (p,), dtype=np.float64)
    out[..., : h + 1] = z.real
    for k in range(1, h):
        out[..., p - k] = z[..., k].imag
    return out


# ------------------------------------------------------------------- 2-D rdFFT
def _dft_matrix(n: int) -> np.ndarray:
    """F[k, m] = exp(-2 pi i (k m mod n) / n), complex128."""
    cos, sin = _dft_cos_sin(n)
    return cos - 1j * sin


def dft2_full(x: np.ndarray) -> np.ndarray:
    """2-D DFT Y[k1, k2] = sum_{r, c} x[r, c] e^{-2 pi i (k1 r / R + k2 c / C)} of the
    last two axes of real x (shape (..., R, C)), complex128, by the definition."""
    x = np.asarray(x, dtype=np.float64)
    R, C = x.shape[-2:]
    return _dft_matrix(R) @ x @ _dft_matrix(C).T


def dft2_packed(x: np.ndarray) -> np.ndarray:
    """Packed 2-D real DFT of the last two axes of x (shape (..., R, C)), float64.

    The pages leave the 2-D transform open (paper-notes page, "Limitations and
    outlook": only 1-D is done). The reading taken is the packed layout applied per
    axis, so that every slot holds one real number of the spectrum, as in 1-D:
      * columns 0 < k2 < C/2: slot [k1, k2] = Re Y[k1, k2] and slot [k1, C - k2] =
        Im Y[k1, k2] for every row k1 < R;
      * columns k2 in {0, C/2}: Y[., k2] is the spectrum of a real sequence
        (conjugate symmetric in k1), stored in the 1-D packed layout down the
        column: [0] = Y[0, k2], [R/2] = Y[R/2, k2], [k1] = Re Y[k1, k2],
        [R - k1] = Im Y[k1, k2] for 0 < k1 < R/2.
    Every value of the non-redundant half-spectrum appears exactly once.
    """
    x = np.asarray(x, dtype=np.float64)
    R, C = x.shape[-2:]
    _check_p(R)
    _check_p(C)
    Y = dft2_full(x)
    out = np.empty_like(x)
    h = C // 2
    for k2 in range(1, h):
        out[..., :, k2] = Y[..., :, k2].real
        out[..., :, C - k2] = Y[..., :, k2].imag
    for k2 in (0, h):
        col = Y[..., :, k2]
        out[..., 0, k2] = col[..., 0].real
        out[..., R // 2, k2] = col[..., R // 2].real
        for k1 in range(1, R // 2):
            out[..., k1, k2] = col[..., k1].real
            out[..., R - k1, k2] = col[..., k1].imag
    return out


def unpack2_spectrum(y: np.ndarray) -> np.ndarray:
    """Full 2-D spectrum Y[k1, k2] (complex128, shape (..., R, C)) of packed y.

    Reads dft2_packed's layout and fills the rest by the symmetry of a real
    image's spectrum, Y[(R - k1) mod R, (C - k2) mod C] = conj(Y[k1, k2]).
    """
    y = np.asarray(y, dtype=np.float64)
    R, C = y.shape[-2:]
    _check_p(R)
    _check_p(C)
    h = C // 2
    Y = np.zeros(y.shape, dtype=np.complex128)
    for k2 in range(1, h):
        Y[..., :, k2] = y[..., :, k2] + 1j * y[..., :, C - k2]
    for k2 in (0, h):
        Y[..., 0, k2] = y[..., 0, k2]
        Y[..., R // 2, k2] = y[..., R // 2, k2]
        for k1 in range(1, R // 2):
            Y[..., k1, k2] = y[..., k1, k2] + 1j * y[..., R - k1, k2]
            Y[..., R - k1, k2] = y[..., k1, k2] - 1j * y[..., R - k1, k2]
    k1 = np.arange(R)
    for k2 in range(h + 1, C):
        Y[..., :, k2] = np.conj(Y[..., (R - k1) % R, C - k2])
    return Y


def idft2_packed(y: np.ndarray) -> np.ndarray:
    """Inverse of dft2_packed: x[r, c] = (1/(R C)) sum_{k1, k2} Y[k1, k2]
    e^{+2 pi i (k1 r / R + k2 c / C)}, float64 (the real part of the sum)."""
    Y = unpack2_spectrum(y)
    R, C = Y.shape[-2:]
    x = np.conj(_dft_matrix(R)) @ Y @ np.conj(_dft_matrix(C)).T
    return x.real / (R * C)


def dft2_packed_at(x: np.ndarray, slots) -> np.ndarray:
    """Values of the packed 2-D spectrum of one image x (R x C) at the given slots
    [(row, col), ...], each by the definition alone (O(R C) per slot), for images too
    large for dft2_packed. Slot (row, col) holds, by the layout of dft2_packed:
      0 < col < C/2 : Re Y[row, col];  C/2 < col : Im Y[row, C - col];
      col in {0, C/2}: row in {0, R/2} -> Y[row, col]; 0 < row < R/2 -> Re Y[row, col];
                       R/2 < row -> Im Y[R - row, col].
    """
    x = np.asarray(x, dtype=np.float64)
    R, C = x.shape
    _check_p(R)
    _check_p(C)
    out = []
    for row, col in slots:
        if 0 < col < C // 2:
            k1, k2, part = row, col, "re"
        elif col > C // 2:
            k1, k2, part = row, C - col, "im"
        elif row == 0 or row == R // 2 or row < R // 2:
            k1, k2, part = row, col, "re"
        else:
            k1, k2, part = R - row, col, "im"
        ar = 2.0 * np.pi * ((k1 * np.arange(R)) % R) / R
        ac = 2.0 * np.pi * ((k2 * np.arange(C)) % C) / C
        Y = np.exp(-1j * ar) @ x @ np.exp(-1j * ac)
        out.append(Y.real if part == "re" else Y.imag)
    return np.array(out)
