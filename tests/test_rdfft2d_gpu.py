"""GPU parity of the 2-D rdFFT (rdfft2_fwd / rdfft2_inv) against the float64 oracle,
through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, to_device, to_host_f64
from synthetic import sample

pytestmark = pytest.mark.gpu

# every column length; widths that leave a ragged last strip pair; several images
SHAPES = [(2, 2), (2, 4096), (4, 8), (8, 2), (16, 32), (32, 4), (32, 1024), (64, 2), (64, 64), (128, 8),
          (256, 128), (512, 4), (1024, 16), (2048, 2), (4096, 4), (8, 4096), (64, 1024)]


@pytest.fixture(scope="module")
def rd():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for the gpu tests")
    import block_circulant_layers_b200 as rd
    return rd


def _n(R, C):
    return 5 if R * C <= 1 << 14 else 2


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("R,C", SHAPES)
def test_2d_forward(rd, R, C, dtype):
    s = sample(40_000 + R * 7 + C, (_n(R, C), R, C), dtype)
    t = to_device(s, dtype)
    rd.rdfft2_fwd(t)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(t), oracle.dft2_packed(s.exact), dtype, f"2d fwd {R}x{C}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("R,C", SHAPES)
def test_2d_inverse(rd, R, C, dtype):
    s = sample(50_000 + R * 7 + C, (_n(R, C), R, C), dtype)
    t = to_device(s, dtype)
    rd.rdfft2_inv(t)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(t), oracle.idft2_packed(s.exact), dtype, f"2d inv {R}x{C}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("R,C", [(4096, 4096), (1024, 2048), (2048, 512)])
def test_2d_large_sampled_and_round_trip(rd, R, C, dtype):
    """Large images: sampled slots against the definition (edges, the self-mirrored
    columns 0 and C/2, rows 0 and R/2, and random slots), then the round trip."""
    n = 2
    s = sample(60_000 + R + C, (n, R, C), dtype)
    t = to_device(s, dtype)
    rd.rdfft2_fwd(t)
    torch.cuda.synchronize()
    got = to_host_f64(t)
    rng = np.random.default_rng(R + C)
    slots = [(0, 0), (0, C // 2), (R // 2, 0), (R // 2, C // 2), (R - 1, 0), (1, C // 2), (R - 1, C - 1),
             (1, 1), (R // 2, 3), (R // 2 + 1, C - 3)]
    slots += [(int(a), int(b)) for a, b in zip(rng.integers(0, R, 6), rng.integers(0, C, 6))]
    img = n - 1
    ref = oracle.dft2_packed_at(s.exact[img], slots)
    vals = np.array([got[img, a, b] for a, b in slots])
    # By Parseval the packed slots (Re and Im parts of half the spectrum) have
    # rms = sqrt(R C / 2) * rms(x). bf16: the bar itself, 2e-2 * rms. f32: the bar is
    # 1e-5 * max|ref|, and max|ref| over R C Gaussian slots exceeds 5 * rms, so
    # 5e-5 * rms is at least as strict.
    rms = np.sqrt(R * C / 2) * np.sqrt(np.mean(s.exact[img] ** 2))
    tol = (5e-5 if dtype == "f32" else 2e-2) * rms
    assert np.all(np.abs(vals - ref) <= tol), np.abs(vals - ref).max() / rms
    rd.rdfft2_inv(t)
    torch.cuda.synchronize()
    back = to_host_f64(t)
    if dtype == "f32":
        assert_parity(back, s.exact, dtype, f"2d round trip {R}x{C}")
    else:
        # two bf16 transforms, each held to the one-transform bar: twice the bar
        err = np.abs(back - s.exact).max() / np.sqrt(np.mean(s.exact ** 2))
        assert err <= 2 * 2e-2, err


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("C", [64, 128])
def test_2d_r4096_every_slot(rd, C, dtype):
    """R = 4096, where a column CTA holds W = 8 tile rows (4 left columns and their
    mirrors): C = 64 gives 9 strips and C = 128 gives 17, the last one holding only the
    column C/2. Every slot of the forward and of the inverse against the definition."""
    R = 4096
    s = sample(61_000 + C, (1, R, C), dtype)
    t = to_device(s, dtype)
    rd.rdfft2_fwd(t)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(t), oracle.dft2_packed(s.exact), dtype, f"2d fwd {R}x{C}")
    s2 = sample(62_000 + C, (1, R, C), dtype)
    t2 = to_device(s2, dtype)
    rd.rdfft2_inv(t2)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(t2), oracle.idft2_packed(s2.exact), dtype, f"2d inv {R}x{C}")


def test_2d_empty_and_neighbours_untouched(rd):
    R, C = 256, 64
    buf = torch.full((3 * R * C + 256,), 7.0, device="cuda")
    body = buf[64:64 + 3 * R * C].view(3, R, C)
    s = sample(70_000, (3, R, C), "f32")
    body.copy_(torch.from_numpy(s.stored.astype(np.float32)).cuda())
    rd.rdfft2_fwd(body)
    rd.rdfft2_fwd(buf[:0].view(0, R, C))
    torch.cuda.synchronize()
    assert torch.all(buf[:64] == 7.0) and torch.all(buf[64 + 3 * R * C:] == 7.0)
    assert_parity(to_host_f64(body), oracle.dft2_packed(s.exact), "f32", "2d in a slice")


def test_2d_rejects_bad_shapes(rd):
    t = torch.zeros(2, 48, 64, device="cuda")
    with pytest.raises(rd.RdfftError):
        rd.rdfft2_fwd(t)
    t = torch.zeros(2, 64, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(TypeError):
        rd.rdfft2_fwd(t)
