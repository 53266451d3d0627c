"""GPU tests of circ_bwd_deterministic: grad_c summed over the token slices in a fixed
order through a workspace. Parity with the float64 oracle, the same bits on every run
(also after the workspace was filled with NaN), grad_x bit for bit as circ_bwd's, and
the workspace rules, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, to_device, to_host_f64
from synthetic import sample

pytestmark = pytest.mark.gpu

ESPACE = 8


@pytest.fixture(scope="module")
def rd():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for the gpu tests")
    import block_circulant_layers_b200 as rd
    return rd


def make(B, D, p, dtype, seeds):
    q = D // p
    c = sample(seeds[0], (q, q, p), "f32", sigma=1.0 / np.sqrt(D))
    x = sample(seeds[1], (B, D), dtype)
    g = sample(seeds[2], (B, D), dtype)
    return c, x, g


# (B, D, p, with grad_x): the one-kernel backward over input-block groups in tensor memory
# (p = 128, 512, 1024 at D = 4096), the register form for one and two blocks, and the
# grad_c kernel of the two-kernel path (p = 64 and 256, and any call without grad_x)
CASES = [
    (256, 4096, 128, True),
    (1027, 4096, 512, True),
    (300, 4096, 1024, True),
    (700, 1024, 512, True),
    (301, 4096, 4096, True),
    (256, 4096, 128, False),
    (3001, 1024, 64, True),
    (517, 4096, 256, True),
    (999, 2048, 1024, False),
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,D,p,with_gx", CASES)
def test_deterministic_grad_c(rd, B, D, p, with_gx, dtype):
    c, x, g = make(B, D, p, dtype, (300 + p, 301 + B, 302 + D))
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    xd, gd = to_device(x, dtype), to_device(g, dtype)
    tdt = xd.dtype
    need = rd.circ_bwd_workspace_size(B, D, p, tdt, with_grad_x=with_gx)
    q = D // p
    assert need > 0 and need % (q * q * p * 4) == 0         # several token slices here
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    runs = []
    for fill in (0.0, float("nan")):
        ws.view(torch.float32).fill_(fill)                   # stale workspace contents never leak in
        gc = torch.full(c_hat.shape, float("nan"), device="cuda")
        gx = torch.empty_like(gd) if with_gx else None
        rd.circ_bwd(gd, xd, c_hat, p, grad_x=gx, grad_c=gc, need_grad_x=with_gx, deterministic=True,
                    workspace=ws)
        torch.cuda.synchronize()
        runs.append((gx, gc.clone()))
    assert torch.equal(runs[0][1], runs[1][1]), "grad_c differs between two runs"
    gx_ref, gc_ref = oracle.circ_backward(g.exact, x.exact, c.exact)
    assert_parity(to_host_f64(runs[0][1]), gc_ref, dtype, f"deterministic grad_c B={B} D={D} p={p}")
    # against circ_bwd: grad_x the same bits, grad_c within the same tolerance
    gx2, gc2 = rd.circ_bwd(gd, xd, c_hat, p, need_grad_x=with_gx)
    torch.cuda.synchronize()
    if with_gx:
        assert torch.equal(runs[0][0], gx2), "grad_x differs from circ_bwd's"
        assert_parity(to_host_f64(runs[0][0]), gx_ref, dtype, f"deterministic grad_x B={B} D={D} p={p}")
    assert_parity(to_host_f64(gc2), gc_ref, dtype, f"circ_bwd grad_c B={B} D={D} p={p}")


@pytest.mark.parametrize("B,D,p", [(1, 4096, 128), (2, 4096, 512), (1, 4096, 1024), (2, 1024, 1024), (2, 512, 64)])
def test_one_slice_needs_no_workspace(rd, B, D, p):
    """A handful of tokens: one slice per block group stores grad_c, no workspace, and the
    result equals circ_bwd's bit for bit."""
    assert rd.circ_bwd_workspace_size(B, D, p, torch.bfloat16) == 0
    c, x, g = make(B, D, p, "bf16", (310, 311 + B, 312 + p))
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    xd, gd = to_device(x, "bf16"), to_device(g, "bf16")
    rc = rd.lib.circ_bwd_deterministic(gd.data_ptr(), xd.data_ptr(), c_hat.data_ptr(), None, None, B, D, p, 1,
                                       None, 0, torch.cuda.current_stream().cuda_stream)
    assert rc == 0                                           # nothing asked: nothing to do
    gx, gc = rd.circ_bwd(gd, xd, c_hat, p, deterministic=True)
    gx2, gc2 = rd.circ_bwd(gd, xd, c_hat, p)
    torch.cuda.synchronize()
    assert torch.equal(gx, gx2) and torch.equal(gc, gc2)
    _, gc_ref = oracle.circ_backward(g.exact, x.exact, c.exact)
    assert_parity(to_host_f64(gc), gc_ref, "bf16", "one-slice grad_c")


def test_workspace_too_small_is_refused(rd):
    B, D, p = 256, 4096, 128
    c, x, g = make(B, D, p, "bf16", (320, 321, 322))
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    xd, gd = to_device(x, "bf16"), to_device(g, "bf16")
    need = rd.circ_bwd_workspace_size(B, D, p, torch.bfloat16)
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(rd.RdfftError) as e:
        rd.circ_bwd(gd, xd, c_hat, p, deterministic=True, workspace=small)
    assert e.value.code == ESPACE


def test_module_backward_is_reproducible(rd):
    """BlockCirculantLinear(deterministic=True), and any layer under
    torch.use_deterministic_algorithms(True), give the same c.grad on every run."""
    D, p, B = 4096, 512, 2048
    gen = torch.Generator(device="cuda").manual_seed(7)
    x = torch.randn(B, D, device="cuda", generator=gen).to(torch.bfloat16)
    gy = torch.randn(B, D, device="cuda", generator=gen).to(torch.bfloat16)

    def grad_of(layer):
        layer.c.grad = None
        layer(x).backward(gy)
        torch.cuda.synchronize()
        return layer.c.grad.clone()

    layer = rd.BlockCirculantLinear(D, p, device="cuda", generator=gen, deterministic=True)
    a, b = grad_of(layer), grad_of(layer)
    assert torch.equal(a, b)
    plain = rd.BlockCirculantLinear(D, p, device="cuda")
    plain.c.data.copy_(layer.c.data)
    was = torch.are_deterministic_algorithms_enabled()
    torch.use_deterministic_algorithms(True)
    try:
        c1, c2 = grad_of(plain), grad_of(plain)
    finally:
        torch.use_deterministic_algorithms(was)
    assert torch.equal(c1, c2) and torch.equal(c1, a)
    # and the default (atomic) backward agrees within fp32 rounding of the sum
    d = grad_of(plain)
    assert torch.allclose(d, a, rtol=0, atol=1e-5 * float(a.abs().max()))
