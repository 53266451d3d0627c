"""GPU parity of circ_fwd / circ_bwd (block-circulant layer) against the dense
float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, to_device, to_host_f64
from synthetic import sample

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rd():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA GPU is required for the gpu tests")
    import block_circulant_layers_b200 as rd
    return rd


def make_layer(B, D, p, dtype, seeds):
    q = D // p
    cs, xs, gs = seeds
    c = sample(cs, (q, q, p), "f32", sigma=1.0 / np.sqrt(D))
    x = sample(xs, (B, D), dtype)
    g = sample(gs, (B, D), dtype)
    return c, x, g


def run_layer(rd, B, D, p, dtype, seeds, grads=True):
    c, x, g = make_layer(B, D, p, dtype, seeds)
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    xd, gd = to_device(x, dtype), to_device(g, dtype)
    y = rd.circ_fwd(xd, c_hat, p)
    gx = gc = None
    if grads:
        gx, gc = rd.circ_bwd(gd, xd, c_hat, p)
    torch.cuda.synchronize()
    return c, x, g, y, gx, gc


def check_all(rd, B, D, p, dtype, seeds, tokens=None):
    c, x, g, y, gx, gc = run_layer(rd, B, D, p, dtype, seeds)
    sel = slice(None) if tokens is None else tokens
    y_ref = oracle.circ_forward(x.exact[sel], c.exact)
    assert_parity(to_host_f64(y)[sel], y_ref, dtype, f"y B={B} D={D} p={p}")
    gx_ref, _ = oracle.circ_backward(g.exact[sel], x.exact[sel], c.exact)
    assert_parity(to_host_f64(gx)[sel], gx_ref, dtype, f"grad_x B={B} D={D} p={p}")
    _, gc_ref = oracle.circ_backward(g.exact, x.exact, c.exact)
    assert_parity(to_host_f64(gc), gc_ref, dtype, f"grad_c B={B} D={D} p={p}")


# small layers over every supported block size: several CTAs, ragged token counts
SMALL = [(5, 256, 64), (7, 512, 128), (3, 1024, 256), (9, 1024, 512), (4, 2048, 1024),
         (6, 4096, 2048), (5, 4096, 4096), (33, 512, 64), (70, 256, 128), (300, 128, 64)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,D,p", SMALL)
def test_small_layers(rd, B, D, p, dtype):
    check_all(rd, B, D, p, dtype, (100 + p, 200 + B, 300 + D))


@pytest.mark.parametrize("D,p", [(768, 256), (3072, 1024), (1536, 512)])
def test_non_power_of_two_block_counts(rd, D, p):
    check_all(rd, 11, D, p, "f32", (400, 401, 402))


def test_identity_layer_is_exact(rd):
    """c_ii = delta, c_ij = 0: y = x and grad_x = g."""
    B, D, p = 16, 1024, 256
    q = D // p
    c = np.zeros((q, q, p), dtype=np.float32)
    for i in range(q):
        c[i, i, 0] = 1.0
    x = sample(410, (B, D), "f32")
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    xd = to_device(x, "f32")
    y = rd.circ_fwd(xd, c_hat, p)
    gx, _ = rd.circ_bwd(xd, xd, c_hat, p)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(y), x.exact, "f32", "identity y")
    assert_parity(to_host_f64(gx), x.exact, "f32", "identity grad_x")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B", [1, 256])
def test_config_d4096_p128(rd, B, dtype):
    """D = 4096, p = 128 (q = 32), c ~ N(0, 1/D), x, g ~ N(0, 1), B in {1, 256}."""
    check_all(rd, B, 4096, 128, dtype, (4, 5, 6))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B", [1, 3, 5, 9, 37, 149, 297, 301])
@pytest.mark.parametrize("p", [512, 1024])
def test_fused_backward_shapes(rd, p, B, dtype):
    """D = 4096 at p = 512 (q = 8) and p = 1024 (q = 4): circ_bwd computes grad_x and grad_c
    in one kernel (the cross-spectrum accumulated in tensor memory). Ragged token counts:
    one CTA storing grad_c, and several adding into it; the smaller token tiles (2 tokens at
    p = 512 up to 296 tokens, 1 at p = 1024 up to 148) and the larger ones beyond."""
    check_all(rd, B, 4096, p, dtype, (110 + p, 120 + B, 130 + B))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B", [1, 3, 8, 16, 33, 64, 77, 256, 259, 301])
def test_fused_backward_p128_block_groups(rd, B, dtype):
    """D = 4096 at p = 128 (q = 32) at any batch size: the fused backward splits the input
    blocks into 4 groups (grid y), each CTA transforming g in full and x for its group, with
    a ragged last token tile and several token slices adding into grad_c; tiles of 2 tokens
    up to 74 tokens (one tile per CTA in one wave), of 4 above."""
    check_all(rd, B, 4096, 128, dtype, (150, 151 + B, 152 + B))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B", [1, 3, 130])
@pytest.mark.parametrize("p", [512, 1024, 2048, 4096])
def test_fused_backward_one_block(rd, p, B, dtype):
    """q = 1 (D = p): the one-kernel backward keeps each thread's bins of the cross-spectrum
    in registers; ragged token tiles, one CTA storing grad_c (few tokens) or several adding."""
    check_all(rd, B, p, p, dtype, (170 + p // 512, 171 + B, 172 + B))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B", [1, 3, 130])
@pytest.mark.parametrize("p", [512, 1024, 2048, 4096])
def test_fused_backward_two_blocks(rd, p, B, dtype):
    """q = 2 (D = 2 p): the same register-form backward with the 2 x 2 blocks' cross-spectra
    per bin and each grad_x block summed over both output blocks."""
    check_all(rd, B, 2 * p, p, dtype, (190 + p // 512, 191 + B, 192 + B))


@pytest.mark.parametrize("p,B", [(512, 3), (4096, 2)])
def test_fused_backward_one_block_stores_every_grad_c_element(rd, p, B):
    """q = 1 with one CTA (one token tile: 4 tokens at p = 512, 2 at p = 4096): grad_c is
    stored, not added; a NaN-filled grad_c must come out finite and right."""
    c, x, g = make_layer(B, p, p, "bf16", (180, 181, 182))
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    gc = torch.full(c_hat.shape, float("nan"), device="cuda")
    gx = torch.empty(B, p, device="cuda", dtype=torch.bfloat16)
    rd.circ_bwd(to_device(g, "bf16"), to_device(x, "bf16"), c_hat, p, grad_x=gx, grad_c=gc)
    torch.cuda.synchronize()
    gx_ref, gc_ref = oracle.circ_backward(g.exact, x.exact, c.exact)
    assert_parity(to_host_f64(gc), gc_ref, "bf16", "one-block grad_c from NaN")
    assert_parity(to_host_f64(gx), gx_ref, "bf16", "one-block grad_x")


@pytest.mark.parametrize("p,B", [(512, 1), (512, 2), (1024, 1)])
def test_fused_backward_stores_every_grad_c_element(rd, p, B):
    """With a single CTA (one token tile) the fused kernel stores grad_c instead of adding
    into a zeroed buffer: a grad_c full of NaN must come out finite and right."""
    D = 4096
    c, x, g = make_layer(B, D, p, "bf16", (140, 141, 142))
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    gc = torch.full(c_hat.shape, float("nan"), device="cuda")
    gx = torch.empty(B, D, device="cuda", dtype=torch.bfloat16)
    rd.circ_bwd(to_device(g, "bf16"), to_device(x, "bf16"), c_hat, p, grad_x=gx, grad_c=gc)
    torch.cuda.synchronize()
    gx_ref, gc_ref = oracle.circ_backward(g.exact, x.exact, c.exact)
    assert_parity(to_host_f64(gc), gc_ref, "bf16", "fused grad_c from NaN")
    assert_parity(to_host_f64(gx), gx_ref, "bf16", "fused grad_x")


@pytest.mark.parametrize("D,p", [(4096, 128), (1024, 1024), (4096, 4096), (256, 64)])
def test_circ_prepare_out_of_place_and_in_place(rd, D, p):
    """circ_prepare equals rdfft_fwd of a copy of c bit for bit, leaves c untouched, and
    works in place (out = c); c_hat against the oracle's packed DFT."""
    q = D // p
    c = sample(90 + p, (q, q, p), "f32", sigma=1.0 / np.sqrt(D))
    cd = to_device(c, "f32")
    c0 = cd.clone()
    ch = rd.circ_prepare(cd)
    ref = rd.rdfft_fwd(cd.clone(), p)
    torch.cuda.synchronize()
    assert torch.equal(cd, c0)
    assert torch.equal(ch, ref)
    assert_parity(to_host_f64(ch), oracle.dft_packed(c.exact), "f32", f"c_hat p={p}")
    same = rd.circ_prepare(cd, out=cd)
    torch.cuda.synchronize()
    assert same.data_ptr() == cd.data_ptr() and torch.equal(cd, ref)
    with pytest.raises(TypeError):
        rd.circ_prepare(c0.to(torch.bfloat16))


@pytest.mark.parametrize("B", [1, 2, 3, 5, 130, 256, 1027])
def test_tensor_core_d4096_p128_bf16(rd, B):
    """circ_fwd_tc / circ_bwd_x_tc (contraction on the tensor cores) at D = 4096, p = 128,
    bf16, four tokens per CTA: the workload's B in {1, 256} and token counts that leave a
    partial last CTA, every element against the oracle."""
    D, p = 4096, 128
    c, x, g = make_layer(B, D, p, "bf16", (4, 50 + B, 60 + B))
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    y = rd.circ_fwd_tc(to_device(x, "bf16"), c_hat, p)
    gx = rd.circ_bwd_x_tc(to_device(g, "bf16"), c_hat, p)
    torch.cuda.synchronize()
    assert_parity(to_host_f64(y), oracle.circ_forward(x.exact, c.exact), "bf16", f"tc y B={B}")
    gx_ref, _ = oracle.circ_backward(g.exact, x.exact, c.exact)
    assert_parity(to_host_f64(gx), gx_ref, "bf16", f"tc grad_x B={B}")
    assert rd.take_device_error() == 0


def test_tensor_core_shape_rules(rd):
    """The tensor-core entry points cover bf16 at p = 128, D = 4096 only; empty is a no-op."""
    c_hat = torch.zeros(32, 32, 128, device="cuda")
    x = torch.zeros(2, 4096, device="cuda")
    with pytest.raises(rd.RdfftError):
        rd.circ_fwd_tc(x, c_hat, 128)                     # fp32
    xb = torch.zeros(2, 2048, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(rd.RdfftError):
        rd.circ_fwd_tc(xb, torch.zeros(16, 16, 128, device="cuda"), 128)   # D = 2048
    e = torch.empty(0, 4096, device="cuda", dtype=torch.bfloat16)
    assert rd.circ_fwd_tc(e, c_hat, 128).shape == (0, 4096)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,D", [(256, 2048), (257, 8192), (256, 1024)])
def test_p128_many_token_shapes(rd, B, D, dtype):
    """p = 128 from 256 tokens with q = 16, 64 and 8: the 512-thread forward / grad_x CTAs
    cover 16 output blocks (q = 16), two groups of 32 (q = 64, one token left over), or keep
    the 256-thread shape (q < 16); the backward runs the two kernels (D != 4096)."""
    check_all(rd, B, D, 128, dtype, (160, 161 + D // 128, 162 + B))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("D,p,seed", [(4096, 1024, 7), (4096, 4096, 8), (1024, 1024, 9)])
def test_config_block_size_extremes(rd, D, p, seed, dtype):
    check_all(rd, 256, D, p, dtype, (seed, seed + 10, seed + 20))


def test_config_adapter_stack_shape_sampled(rd):
    """One adapter of the LLaMA2-7B-shaped stack at full size: D = 4096, p = 512,
    4096 tokens, bf16. y and grad_x on the first and last 32 tokens, grad_c in full."""
    B, D, p = 4096, 4096, 512
    toks = np.r_[0:32, B - 32:B]
    check_all(rd, B, D, p, "bf16", (300, 100, 200), tokens=toks)


def test_grad_c_only_and_grad_x_only(rd):
    B, D, p = 20, 1024, 128
    c, x, g = make_layer(B, D, p, "f32", (500, 501, 502))
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    xd, gd = to_device(x, "f32"), to_device(g, "f32")
    gx, gc = rd.circ_bwd(gd, xd, c_hat, p, need_grad_c=False)
    assert gc is None
    gx2, gc2 = rd.circ_bwd(gd, xd, c_hat, p, need_grad_x=False)
    assert gx2 is None
    torch.cuda.synchronize()
    gx_ref, gc_ref = oracle.circ_backward(g.exact, x.exact, c.exact)
    assert_parity(to_host_f64(gx), gx_ref, "f32", "grad_x only")
    assert_parity(to_host_f64(gc2), gc_ref, "f32", "grad_c only")


def test_grad_c_overwrites_and_empty_batch(rd):
    B, D, p = 8, 512, 64
    c, x, g = make_layer(B, D, p, "f32", (510, 511, 512))
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    xd, gd = to_device(x, "f32"), to_device(g, "f32")
    gc = torch.full(c_hat.shape, 123.0, device="cuda")
    rd.circ_bwd(gd, xd, c_hat, p, grad_c=gc, need_grad_x=False)
    torch.cuda.synchronize()
    _, gc_ref = oracle.circ_backward(g.exact, x.exact, c.exact)
    assert_parity(to_host_f64(gc), gc_ref, "f32", "grad_c overwrite")
    e = torch.empty((0, D), device="cuda")
    gc.fill_(5.0)
    rd.circ_bwd(e, e, c_hat, p, grad_c=gc, need_grad_x=False)
    torch.cuda.synchronize()
    assert torch.all(gc == 0)


@pytest.mark.parametrize("B,D,p", [(1, 4096, 128), (2, 4096, 128), (1, 1024, 1024), (1, 4096, 4096),
                                   (2, 512, 64), (3, 1536, 512)])
def test_grad_c_single_token_slice_writes_every_element(rd, B, D, p):
    """With so few tokens that one CTA per input-block group covers them all, grad_c is
    stored instead of accumulated into a zeroed buffer: every element must be written
    (grad_c starts as NaN here), and the values match the oracle."""
    c, x, g = make_layer(B, D, p, "bf16", (520 + B, 521, 522))
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    xd, gd = to_device(x, "bf16"), to_device(g, "bf16")
    gc = torch.full(c_hat.shape, float("nan"), device="cuda")
    gx = torch.empty_like(xd)
    rd.circ_bwd(gd, xd, c_hat, p, grad_x=gx, grad_c=gc)
    y = rd.circ_fwd(xd, c_hat, p)
    torch.cuda.synchronize()
    assert not torch.isnan(gc).any()
    gx_ref, gc_ref = oracle.circ_backward(g.exact, x.exact, c.exact)
    assert_parity(to_host_f64(gc), gc_ref, "bf16", f"grad_c B={B} D={D} p={p}")
    assert_parity(to_host_f64(gx), gx_ref, "bf16", f"grad_x B={B} D={D} p={p}")
    assert_parity(to_host_f64(y), oracle.circ_forward(x.exact, c.exact), "bf16", f"y B={B} D={D} p={p}")


@pytest.mark.parametrize("D,p,B", [(4096, 512, 31), (4096, 512, 64), (4096, 512, 255), (4096, 512, 256),
                                   (4096, 512, 512), (2048, 512, 128), (1024, 256, 256), (4096, 256, 64),
                                   (1024, 64, 64)])
def test_forward_token_tile_choices(rd, D, p, B):
    """The forward's token tile (4, 2 or 1 tokens per CTA, the largest whose grid keeps a
    token's output blocks in one CTA) on both sides of each choice, and the backward beside it."""
    check_all(rd, B, D, p, "bf16", (500 + p, 501 + B, 502 + D))


@pytest.mark.parametrize("D,p,B", [(4096, 128, 16), (4096, 128, 64), (4096, 128, 129), (4096, 512, 16),
                                   (4096, 512, 148), (4096, 512, 300), (4096, 1024, 64), (4096, 1024, 149),
                                   (1024, 64, 100), (4096, 256, 77)])
def test_grad_c_token_tile_choices(rd, D, p, B):
    """grad_c alone (the grad_c kernel) with half-size token tiles at few tokens and full ones
    above, against the oracle; a NaN-filled grad_c must come out finite and right."""
    c, x, g = make_layer(B, D, p, "bf16", (510 + p, 511 + B, 512 + D))
    c_hat = rd.circ_prepare(to_device(c, "f32"))
    gc = torch.full(c_hat.shape, float("nan"), device="cuda")
    rd.circ_bwd(to_device(g, "bf16"), to_device(x, "bf16"), c_hat, p, grad_c=gc, need_grad_x=False)
    torch.cuda.synchronize()
    _, gc_ref = oracle.circ_backward(g.exact, x.exact, c.exact)
    assert_parity(to_host_f64(gc), gc_ref, "bf16", f"grad_c alone B={B} D={D} p={p}")
