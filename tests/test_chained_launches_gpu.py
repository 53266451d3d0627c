"""Launches chained on one stream with no host synchronisation between them.

The rows kernel is launched with programmatic stream serialization: the next launch
in the stream may be scheduled while the previous one drains, and every CTA waits
(griddepcontrol.wait) before it touches global memory. These tests check that each
launch of a chain sees the complete output of the launch before it, in a plain
stream and replayed from a CUDA graph. The kernels are deterministic, so a chain run
without synchronisation must be bit-identical to the same chain run one launch at a
time with the device synchronised after each launch; the first step of that
reference chain is also held to the oracle.
"""
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


def _rows(p):
    per_cta = 128 if p <= 32 else max(1, 128 // (p // 32))
    return 40 * per_cta + 3           # many CTAs, so launches overlap, plus a ragged tail


def _chain_rows(rd, t, p):
    """Four forward/inverse pairs on the same rows, then the rows viewed at another
    length (a different kernel on the same bytes)."""
    ops = []
    for _ in range(4):
        ops.append(lambda: rd.rdfft_fwd(t, p))
        ops.append(lambda: rd.rdfft_inv(t, p))
    q = 4096 if p != 4096 else 512
    if t.numel() % q == 0:
        flat = t.view(-1)
        ops.append(lambda: rd.rdfft_fwd(flat, q))
        ops.append(lambda: rd.rdfft_inv(flat, q))
    ops.append(lambda: rd.rdfft_fwd(t, p))
    return ops


def _run_synced(ops):
    for op in ops:
        op()
        torch.cuda.synchronize()


def _run_chained(ops, mode, scratch_ops):
    if mode == "stream":
        st = torch.cuda.Stream()
        st.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(st):
            for op in ops:
                op()
        st.synchronize()
        return
    # graph: warm up on scratch buffers of the same shapes (sets the kernels'
    # attributes), capture the chain on the real buffer, then replay it once
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for op in scratch_ops:
            op()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for op in ops:
            op()
    g.replay()
    torch.cuda.synchronize()
    del g


@pytest.mark.parametrize("mode", ["stream", "graph"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("p", [16, 512, 4096])
def test_rows_chain_without_sync(rd, p, dtype, mode):
    rows = _rows(p)
    rows -= rows % max(1, 4096 // p)           # whole 4096-rows, so the chain can re-view the bytes
    s = sample(80_000 + p, (rows, p), dtype)
    ref = to_device(s, dtype)
    ref_ops = _chain_rows(rd, ref, p)
    rd.rdfft_fwd(ref, p)                       # first step alone, against the oracle
    torch.cuda.synchronize()
    assert_parity(to_host_f64(ref), oracle.dft_packed(s.exact), dtype, f"chain first step p={p}")
    ref.copy_(to_device(s, dtype))
    _run_synced(ref_ops)

    got = to_device(s, dtype)
    scratch = torch.empty_like(got)
    _run_chained(_chain_rows(rd, got, p), mode, _chain_rows(rd, scratch, p))
    assert torch.equal(got.view(torch.int16 if dtype == "bf16" else torch.int32),
                       ref.view(torch.int16 if dtype == "bf16" else torch.int32)), \
        f"chained launches differ from synchronised ones (p={p}, {dtype}, {mode})"


def _chain_2d(rd, t):
    ops = []
    for _ in range(2):
        ops.append(lambda: rd.rdfft2_fwd(t))          # rows kernel, then columns kernel
        ops.append(lambda: rd.rdfft2_inv(t))          # columns kernel, then rows kernel
    ops.append(lambda: rd.rdfft2_fwd(t))
    return ops


@pytest.mark.parametrize("mode", ["stream", "graph"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("R,C", [(512, 512), (4096, 64)])
def test_2d_chain_without_sync(rd, R, C, dtype, mode):
    s = sample(81_000 + R + C, (3, R, C), dtype)
    ref = to_device(s, dtype)
    _run_synced(_chain_2d(rd, ref))
    got = to_device(s, dtype)
    scratch = torch.empty_like(got)
    _run_chained(_chain_2d(rd, got), mode, _chain_2d(rd, scratch))
    iv = torch.int16 if dtype == "bf16" else torch.int32
    assert torch.equal(got.view(iv), ref.view(iv)), f"2-D chain differs ({R}x{C}, {dtype}, {mode})"


def test_layer_chain_without_sync(rd):
    """prepare -> forward -> backward, chained, equals the synchronised sequence."""
    B, D, p = 64, 1024, 128
    q = D // p
    c = torch.from_numpy(sample(82_000, (q, q, p), "f32", sigma=D ** -0.5).stored).cuda()
    x = to_device(sample(82_001, (B, D), "bf16"), "bf16")
    g = to_device(sample(82_002, (B, D), "bf16"), "bf16")

    def run(sync):
        ch = torch.empty_like(c)
        y = torch.empty_like(x)
        gx = torch.empty_like(x)
        gc = torch.empty_like(c)
        ops = [lambda: rd.circ_prepare(c, out=ch), lambda: rd.circ_fwd(x, ch, p, y=y),
               lambda: rd.circ_bwd(g, x, ch, p, grad_x=gx, grad_c=gc), lambda: rd.rdfft_fwd(gx, p)]
        for op in ops:
            op()
            if sync:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return y, gx, gc

    y0, gx0, gc0 = run(True)
    y1, gx1, gc1 = run(False)
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    assert torch.equal(gx0.view(torch.int16), gx1.view(torch.int16))
    # grad_c is a sum over token slices added with atomics: order may differ
    assert np.allclose(gc0.cpu().numpy(), gc1.cpu().numpy(), rtol=1e-5, atol=1e-6 * gc0.abs().max().item())


def _chain_layer_det(rd, bufs, p):
    """prepare -> forward -> deterministic backward -> rdFFT of grad_c's rows, twice: the
    second backward overwrites grad_c and the workspace while the grid before it may still be
    draining (programmatic dependent launch)."""
    c, x, g, ch, y, gx, gc, ws, spec = bufs
    ops = []
    for _ in range(2):
        ops.append(lambda: rd.circ_prepare(c, out=ch))
        ops.append(lambda: rd.circ_fwd(x, ch, p, y=y))
        ops.append(lambda: rd.circ_bwd(g, x, ch, p, grad_x=gx, grad_c=gc, deterministic=True, workspace=ws))
        ops.append(lambda: spec.copy_(gc))
        ops.append(lambda: rd.rdfft_fwd(spec, p))
    return ops


@pytest.mark.parametrize("mode", ["stream", "graph"])
@pytest.mark.parametrize("D,p,B", [(4096, 128, 256), (4096, 512, 64), (1024, 1024, 256), (1024, 64, 300)])
def test_deterministic_layer_chain_without_sync(rd, D, p, B, mode):
    """The deterministic backward chained with the layer's other calls, in a stream and in a
    captured CUDA graph, gives the same bits as the synchronised sequence: the zeroing,
    per-slice, ordered-sum and rdIFFT launches keep their order without a host sync."""
    q = D // p

    def make():
        c = torch.from_numpy(sample(83_000 + p, (q, q, p), "f32", sigma=D ** -0.5).stored).cuda()
        x = to_device(sample(83_001 + B, (B, D), "bf16"), "bf16")
        g = to_device(sample(83_002 + B, (B, D), "bf16"), "bf16")
        need = max(16, rd.circ_bwd_workspace_size(B, D, p, torch.bfloat16))
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        return [c, x, g, torch.empty_like(c), torch.empty_like(x), torch.empty_like(x), torch.empty_like(c), ws,
                torch.empty_like(c)]

    ref = make()
    _run_synced(_chain_layer_det(rd, ref, p))
    got = make()
    _run_chained(_chain_layer_det(rd, got, p), mode, _chain_layer_det(rd, make(), p))
    for name, i in (("y", 4), ("grad_x", 5)):
        assert torch.equal(got[i].view(torch.int16), ref[i].view(torch.int16)), f"{name} ({D}, {p}, {B}, {mode})"
    for name, i in (("grad_c", 6), ("rdFFT of grad_c", 8)):
        assert torch.equal(got[i], ref[i]), f"{name} ({D}, {p}, {B}, {mode})"
