"""PyTorch autograd module of the block-circulant linear layer over the C ABI.

"Memory-Efficient Training with In-Place FFT Implementation" (paper-notes page,
"Training strategy": the circulant structure replaces linear-layer weights, forward
and backward run in place in the real domain, and the operator integrates with an
autograd framework). The weight is D x D, made of q x q circulant blocks of size p
given by c[i][j] (first columns, fp32). Every step of the computation runs in the
library's kernels (rdfft_fwd / circ_fwd / circ_bwd / rdfft_inv); this file only
marshals tensors.

inplace_spectrum (default False) chooses where c_hat lives during a call:
  * False: torch allocates a temporary fp32 c_hat (q x q x p) for each forward and
    backward call, and c itself is never written. Exact: training sees c as the
    optimizer left it.
  * True: no second copy of c. The spectrum is computed in c's own buffer
    (rdfft_fwd), used, and turned back into c (rdfft_inv) within the same call, so
    the layer's extra memory is the activations alone (the in-place memory saving
    the method is about). The fp32 round trip is not exact, and because it applies
    the same rounding map to nearly the same c on every call its errors accumulate
    linearly, not as a random walk: about 1.2e-7 relative (rms over c) per call,
    2.5e-4 after 1000 forward + backward calls at p = 128 to 4096, measured on the
    kernels' own arithmetic (tests/test_emulator.py) and on the GPU
    (tests/test_layer_module_gpu.py). Use it where that drift is small against the
    optimizer's updates. While a call runs, c holds its spectrum: work on another
    stream must not read c until the call's stream has reached its end.

The gradient of c is a sum over tokens. By default the token slices add into it with
fp32 atomics, so its last bits can change from run to run; with deterministic=True, or
whenever torch.use_deterministic_algorithms(True) is in force, the backward calls
circ_bwd_deterministic instead (the slices summed in a fixed order through a workspace
from torch's caching allocator).
"""
from __future__ import annotations

import math

import torch

from . import _binding as _b


class _CirculantFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, c, p, inplace, deterministic):
        ctx.p = p
        ctx.inplace = inplace
        ctx.deterministic = deterministic or torch.are_deterministic_algorithms_enabled()
        shape = x.shape
        x2 = x.reshape(-1, shape[-1]).contiguous()
        with torch.no_grad():
            if inplace:
                c_hat = _b.rdfft_fwd(c.data, p)
            else:
                c_hat = _b.circ_prepare(c.detach())
            y = _b.circ_fwd(x2, c_hat, p)
            if inplace:
                _b.rdfft_inv(c.data, p)
        ctx.save_for_backward(x2, c)
        return y.reshape(shape)

    @staticmethod
    def backward(ctx, gy):
        x2, c = ctx.saved_tensors
        p = ctx.p
        g2 = gy.reshape(-1, gy.shape[-1]).contiguous().to(x2.dtype)
        need_x, need_c = ctx.needs_input_grad[0], ctx.needs_input_grad[1]
        with torch.no_grad():
            if ctx.inplace:
                c_hat = _b.rdfft_fwd(c.data, p)
            else:
                c_hat = _b.circ_prepare(c.detach())
            gx, gc = _b.circ_bwd(g2, x2, c_hat, p, need_grad_x=need_x, need_grad_c=need_c,
                                 deterministic=ctx.deterministic)
            if ctx.inplace:
                _b.rdfft_inv(c.data, p)
        if gx is not None:
            gx = gx.reshape(gy.shape)
        return gx, gc, None, None, None


def block_circulant(x: torch.Tensor, c: torch.Tensor, p: int, inplace_spectrum: bool = False,
                    deterministic: bool = False) -> torch.Tensor:
    """y = W(c) x over the last dimension of x (bf16 or fp32); c: (q, q, p) fp32."""
    return _CirculantFn.apply(x, c, p, inplace_spectrum, deterministic)


class BlockCirculantLinear(torch.nn.Module):
    """Linear layer D -> D whose weight is block circulant with block size p.

    Parameters: c of shape (D/p, D/p, p), fp32, initialised i.i.d. N(0, 1/D) (the
    synthetic initialisation used throughout this repository). Inputs may be bf16
    or fp32; the arithmetic is fp32 and the output has the input's dtype.
    """

    def __init__(self, features: int, block: int, inplace_spectrum: bool = False, device=None,
                 generator: torch.Generator | None = None, deterministic: bool = False):
        super().__init__()
        if block < 64 or block & (block - 1) or features % block:
            raise ValueError("block must be a power of two >= 64 dividing features")
        q = features // block
        c = torch.randn(q, q, block, device=device, dtype=torch.float32, generator=generator)
        self.c = torch.nn.Parameter(c / math.sqrt(features))
        self.features = features
        self.block = block
        self.inplace_spectrum = inplace_spectrum
        self.deterministic = deterministic

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        return block_circulant(x, self.c, self.block, self.inplace_spectrum, self.deterministic)

    def extra_repr(self) -> str:
        return (f"features={self.features}, block={self.block}, inplace_spectrum={self.inplace_spectrum}, "
                f"deterministic={self.deterministic}")
