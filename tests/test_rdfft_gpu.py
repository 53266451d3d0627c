"""GPU parity of rdfft_fwd / rdfft_inv against the float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, to_device, to_host_f64
from synthetic import sample

pytestmark = pytest.mark.gpu

PS = [2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096]


@pytest.fixture(scope="module")
def rd():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for the gpu tests")
    import block_circulant_layers_b200 as rd
    return rd


def _rows(p):
    per_cta = 128 if p <= 32 else max(1, 128 // (p // 32))
    return 3 * per_cta + 5          # several CTAs plus a ragged tail


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("p", PS)
def test_forward_all_p(rd, p, dtype):
    rows = _rows(p)
    s = sample(10_000 + p, (rows, p), dtype)
    t = to_device(s, dtype)
    rd.rdfft_fwd(t, p)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(t), oracle.dft_packed(s.exact), dtype, f"fwd p={p}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("p", PS)
def test_inverse_all_p(rd, p, dtype):
    rows = _rows(p)
    s = sample(20_000 + p, (rows, p), dtype)
    t = to_device(s, dtype)
    rd.rdfft_inv(t, p)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(t), oracle.idft_packed(s.exact), dtype, f"inv p={p}")


@pytest.mark.parametrize("rows", [1, 3, 147, 149, 1000])
def test_odd_row_counts(rd, rows):
    p = 512
    s = sample(30_000 + rows, (rows, p), "f32")
    t = to_device(s, "f32")
    rd.rdfft_fwd(t, p)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(t), oracle.dft_packed(s.exact), "f32", f"rows={rows}")


def test_in_bounds_of_a_slice(rd):
    """Transforming rows 2..5 of a buffer leaves rows 0, 1 and 6.. bit-identical."""
    p = 4096
    s = sample(31_000, (9, p), "f32")
    t = to_device(s, "f32")
    before = t.clone()
    rd.rdfft_fwd(t[2:6], p)
    torch.cuda.synchronize()
    assert torch.equal(t[:2], before[:2]) and torch.equal(t[6:], before[6:])
    assert_parity(to_host_f64(t[2:6]), oracle.dft_packed(s.exact[2:6]), "f32", "slice")


def test_config_small_round_trip(rd):
    """64 rows of p = 16, fp32, N(0,1): packed spectrum vs the oracle, then back to x."""
    s = sample(1, (64, 16), "f32")
    t = to_device(s, "f32")
    rd.rdfft_fwd(t, 16)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(t), oracle.dft_packed(s.exact), "f32", "config p=16 fwd")
    rd.rdfft_inv(t, 16)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(t), s.exact, "f32", "config p=16 round trip")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("p", [512, 4096])
def test_config_standalone_full_size(rd, p, dtype):
    """256 x 4096 reals viewed as rows of p, N(0,1): forward and inverse, every element."""
    seed = {"f32": 2, "bf16": 3}[dtype]
    s = sample(seed, (256 * 4096 // p, p), dtype)
    t = to_device(s, dtype)
    rd.rdfft_fwd(t, p)
    torch.cuda.synchronize()
    spec = to_host_f64(t)
    assert_parity(spec, oracle.dft_packed(s.exact), dtype, f"full fwd p={p}")
    rd.rdfft_inv(t, p)
    torch.cuda.synchronize()
    # the inverse is checked against the oracle on the same stored spectrum
    assert_parity(to_host_f64(t), oracle.idft_packed(spec), dtype, f"full inv p={p}")


def test_closed_forms_on_gpu(rd):
    p = 4096
    n = np.arange(p)
    rows = np.stack([np.eye(1, p, 0)[0], np.full(p, 0.5), np.cos(2 * np.pi * 5 * n / p),
                     np.sin(2 * np.pi * 7 * n / p)])
    t = to_device(rows.astype(np.float32), "f32")
    rd.rdfft_fwd(t, p)
    torch.cuda.synchronize()
    got = to_host_f64(t)
    want = np.zeros((4, p))
    want[0, : p // 2 + 1] = 1
    want[1, 0] = 0.5 * p
    want[2, 5] = p / 2
    want[3, p - 7] = -p / 2
    assert np.abs(got - want).max() <= 1e-5 * p


def test_streams_and_empty(rd):
    p = 256
    s = sample(32_000, (64, p), "f32")
    t = to_device(s, "f32")
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        rd.rdfft_fwd(t, p)
    st.synchronize()
    assert_parity(to_host_f64(t), oracle.dft_packed(s.exact), "f32", "side stream")
    e = torch.empty(0, device="cuda")
    rd.rdfft_fwd(e, p)


def test_errors_raise(rd):
    t = torch.zeros(3 * 512, device="cuda")
    with pytest.raises(rd.RdfftError):
        rd.rdfft_fwd(t, 3)
    with pytest.raises(TypeError):
        rd.rdfft_fwd(torch.zeros(512, device="cuda", dtype=torch.float16), 512)


def test_bounded_wait_error_path(rd):
    """No wait times out in normal use; the self-test's wait runs out and is reported,
    once, without any fault."""
    p = 4096
    t = torch.randn(300, p, device="cuda").to(torch.bfloat16)
    rd.rdfft_fwd(t, p)
    rd.rdfft_inv(t, p)
    torch.cuda.synchronize()
    assert rd.take_device_error() == 0
    rd.selftest_wait_timeout()
    torch.cuda.synchronize()
    assert rd.take_device_error() == rd.RDFFT_ETIMEOUT
    assert rd.take_device_error() == 0
    # the transforms still work afterwards
    s = sample(33_000, (5, p), "f32")
    x = to_device(s, "f32")
    rd.rdfft_fwd(x, p)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(x), oracle.dft_packed(s.exact), "f32", "after self-test")
