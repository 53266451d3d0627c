"""GPU parity of the packed <-> complex-bin cast (rdfft_to_complex / rdfft_from_complex):
the kernels only move values, so the results must equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import to_device, to_host_f64
from synthetic import sample

pytestmark = pytest.mark.gpu

PS = [2, 4, 8, 64, 512, 4096]


@pytest.fixture(scope="module")
def rd():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for the gpu tests")
    import block_circulant_layers_b200 as rd
    return rd


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("p", PS)
def test_to_complex_exact(rd, p, dtype):
    rows = 37 if p >= 512 else 301
    s = sample(80_000 + p, (rows, p), dtype)
    t = to_device(s, dtype)
    z = rd.rdfft_to_complex(t, p)
    torch.cuda.synchronize()
    assert z.shape == (rows, p // 2 + 1, 2)
    ref = oracle.packed_to_rfft(s.exact)
    got = to_host_f64(z)
    assert np.array_equal(got[..., 0], ref.real) and np.array_equal(got[..., 1], ref.imag)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("p", PS)
def test_from_complex_exact(rd, p, dtype):
    rows = 37 if p >= 512 else 301
    s = sample(90_000 + p, (rows, p // 2 + 1, 2), dtype)
    z = to_device(s, dtype)
    t = rd.rdfft_from_complex(z)
    torch.cuda.synchronize()
    ref = oracle.rfft_to_packed(s.exact[..., 0] + 1j * s.exact[..., 1])
    assert np.array_equal(to_host_f64(t), ref)


def test_cast_of_a_transform_is_the_library_rfft(rd):
    """rdfft_fwd then the cast gives the complex rfft of the rows (within the f32 bar)."""
    p, rows = 1024, 64
    s = sample(91_000, (rows, p), "f32")
    t = to_device(s, "f32")
    rd.rdfft_fwd(t, p)
    z = torch.view_as_complex(rd.rdfft_to_complex(t, p))
    torch.cuda.synchronize()
    ref = np.fft.rfft(s.exact, axis=-1)
    err = np.abs(z.cpu().numpy().astype(np.complex128) - ref).max()
    assert err <= 1e-5 * np.abs(ref).max()


def test_cast_large_and_empty(rd):
    p, rows = 512, 1 << 16
    s = sample(92_000, (rows, p), "bf16")
    t = to_device(s, "bf16")
    z = rd.rdfft_to_complex(t, p)
    back = rd.rdfft_from_complex(z)
    torch.cuda.synchronize()
    assert torch.equal(back.view(torch.int16), t.view(torch.int16))
    e = torch.empty(0, p, device="cuda")
    assert rd.rdfft_to_complex(e, p).shape == (0, p // 2 + 1, 2)
