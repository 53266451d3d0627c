"""B200-native rdFFT: in-place real-domain FFT and the block-circulant layer.

Thin Python binding over the C ABI of include/rdfft.h (librdfft.so, built in-tree by
``python -m block_circulant_layers_b200.build``). Every function marshals its
arguments and calls the library; all of the computation runs in the library's CUDA
kernels. There is no fallback: without the compiled library, importing the binding
raises, and the functions accept CUDA tensors only.

Tensor functions (torch is used for device memory and the current stream):
    rdfft_fwd(t, p)                       in place, packed spectrum of each row
    rdfft_inv(t, p)                       in place, inverse
    rdfft_to_complex(t, p)                (..., p/2+1, 2) complex bins, out of place
    rdfft_from_complex(z)                 packed rows from complex bins, out of place
    rdfft2_fwd(t) / rdfft2_inv(t)         in place, 2-D packed spectrum of (..., R, C)
    circ_fwd(x, c_hat, p, y=None)         y = W x
    circ_bwd(g, x, c_hat, p, grad_x=..., grad_c=..., deterministic=False)
    circ_bwd_workspace_size(B, D, p, dtype)  device bytes the deterministic backward needs
    circ_prepare(c)                       c_hat = packed rdfft_fwd of fp32 c
    circ_fwd_tc / circ_bwd_x_tc           forward / grad_x with the contraction on the tensor
                                          cores (bf16, p = 128, D = 4096; slower, kept measured)
    BlockCirculantLinear(D, p)            torch.nn.Module with autograd over the above
Raw entry points on integer device pointers: ``lib`` (the ctypes handle).
"""
from __future__ import annotations

_EXPORTS = ("RDFFT_BF16", "RDFFT_F32", "RDFFT_ETIMEOUT", "RdfftError", "circ_bwd", "circ_fwd", "circ_prepare",
            "circ_fwd_tc", "circ_bwd_x_tc", "circ_bwd_workspace_size",
            "lib", "lib_path", "rdfft_fwd", "rdfft_inv", "rdfft_to_complex", "rdfft_from_complex", "rdfft2_fwd",
            "rdfft2_inv", "take_device_error", "selftest_wait_timeout")
_LAYER = ("BlockCirculantLinear", "block_circulant")

__all__ = list(_EXPORTS + _LAYER)


def __getattr__(name):
    # Loaded on first use so that `python -m block_circulant_layers_b200.build` can run
    # before the library exists; any use of the API without it raises ImportError.
    if name in _EXPORTS:
        from . import _binding
        return getattr(_binding, name)
    if name in _LAYER:
        from . import layer
        return getattr(layer, name)
    raise AttributeError(name)
