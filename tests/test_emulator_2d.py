"""The 2-D rdFFT's per-thread column code (rdfft2d_steps.cuh) and the row code, run
on the host by the emulator CTA by CTA, against the oracle's 2-D packed DFT."""
import ctypes
import os

import numpy as np
import pytest

import oracle
from conftest import ROOT
from synthetic import bf16_bits_to_f64, sample

# Every column length, each with a width that leaves a ragged last strip pair
# (C/2 + 1 left columns are never a multiple of the strip width), several images.
SHAPES = [(2, 2), (2, 64), (4, 8), (8, 2), (16, 32), (32, 4), (64, 2), (64, 64), (128, 8), (256, 128),
          (512, 4), (1024, 16), (2048, 2), (4096, 4), (8, 4096), (64, 1024)]


@pytest.fixture(scope="module")
def emu():
    from block_circulant_layers_b200 import build
    build.build_emulator()
    L = ctypes.CDLL(os.path.join(ROOT, "block_circulant_layers_b200", "librdfft_hostemu.so"))
    L.rdfft2_emulate.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_int]
    return L


def _images(R, C):
    return 3 if R * C <= 1 << 14 else 1


@pytest.mark.parametrize("R,C", SHAPES)
def test_2d_forward_fp32_matches_oracle(emu, R, C):
    n = _images(R, C)
    s = sample(7000 + R + C, (n, R, C), "f32")
    a = s.stored.copy()
    assert emu.rdfft2_emulate(a.ctypes.data, n, R, C, 0, 0) == 0
    ref = oracle.dft2_packed(s.exact)
    assert np.abs(a - ref).max() <= 1e-5 * np.abs(ref).max()


@pytest.mark.parametrize("R,C", SHAPES)
def test_2d_inverse_fp32_matches_oracle(emu, R, C):
    n = _images(R, C)
    s = sample(8000 + R + C, (n, R, C), "f32")
    a = s.stored.copy()
    assert emu.rdfft2_emulate(a.ctypes.data, n, R, C, 0, 1) == 0
    ref = oracle.idft2_packed(s.exact)
    assert np.abs(a - ref).max() <= 1e-5 * np.abs(ref).max()


@pytest.mark.parametrize("R,C", [(4, 16), (256, 64), (4096, 2)])
def test_2d_bf16(emu, R, C):
    s = sample(9000 + R, (2, R, C), "bf16")
    a = s.stored.copy()
    assert emu.rdfft2_emulate(a.ctypes.data, 2, R, C, 1, 0) == 0
    ref = oracle.dft2_packed(s.exact)
    assert np.all(np.abs(bf16_bits_to_f64(a) - ref) <= 2e-2 * np.sqrt(np.mean(ref ** 2)))


def test_2d_unsupported_and_empty(emu):
    a = np.zeros((4, 6), dtype=np.float32)
    assert emu.rdfft2_emulate(a.ctypes.data, 1, 4, 6, 0, 0) == 1
    assert emu.rdfft2_emulate(None, 0, 64, 64, 0, 0) == 0


@pytest.mark.parametrize("C", [32, 64])
@pytest.mark.parametrize("inverse", [0, 1])
def test_2d_bf16_r4096_interior_strips(emu, C, inverse):
    """R = 4096, 16-bit, with interior strip pairs (away from columns 0 and C/2) as well as
    the edge ones, forward and inverse against the oracle: a strip's left columns and their
    mirrors land in the right tile rows and come back to the right image columns."""
    s = sample(9100 + C + inverse, (1, 4096, C), "bf16")
    a = s.stored.copy()
    assert emu.rdfft2_emulate(a.ctypes.data, 1, 4096, C, 1, inverse) == 0
    ref = (oracle.idft2_packed if inverse else oracle.dft2_packed)(s.exact)
    got = bf16_bits_to_f64(a)
    assert np.all(np.abs(got - ref) <= 2e-2 * np.sqrt(np.mean(ref ** 2)))
    # every column pair is right, not just most of the image: the worst column's error
    # stays at bf16 rounding size relative to that column's own scale
    col_err = np.abs(got - ref).max(axis=(0, 1))
    col_rms = np.sqrt(np.mean(ref ** 2, axis=(0, 1)))
    assert np.all(col_err <= 2e-2 * np.maximum(col_rms, 1e-30) + 1e-6 * np.sqrt(np.mean(ref ** 2)))
