"""ctypes binding of librdfft.so (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "librdfft.so")

RDFFT_F32 = 0
RDFFT_BF16 = 1

if not os.path.exists(lib_path):
    raise ImportError(
        f"{lib_path} is missing: build it with `python -m block_circulant_layers_b200.build` "
        "(the package has no non-CUDA fallback)")

lib = ctypes.CDLL(lib_path)

_i64, _int, _vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
lib.rdfft_fwd.argtypes = [_vp, _i64, _int, _int, _vp]
lib.rdfft_inv.argtypes = [_vp, _i64, _int, _int, _vp]
lib.rdfft_to_complex.argtypes = [_vp, _vp, _i64, _int, _int, _vp]
lib.rdfft_from_complex.argtypes = [_vp, _vp, _i64, _int, _int, _vp]
lib.rdfft2_fwd.argtypes = [_vp, _i64, _int, _int, _int, _vp]
lib.rdfft2_inv.argtypes = [_vp, _i64, _int, _int, _int, _vp]
lib.circ_prepare.argtypes = [_vp, _vp, _int, _int, _vp]
lib.circ_fwd.argtypes = [_vp, _vp, _vp, _i64, _int, _int, _int, _vp]
lib.circ_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _int, _int, _int, _vp]
lib.circ_fwd_tc.argtypes = [_vp, _vp, _vp, _i64, _int, _int, _int, _vp]
lib.circ_bwd_x_tc.argtypes = [_vp, _vp, _vp, _i64, _int, _int, _int, _vp]
lib.circ_bwd_workspace_size.argtypes = [_i64, _int, _int, _int, _int, ctypes.POINTER(ctypes.c_size_t)]
lib.circ_bwd_deterministic.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _int, _int, _int, _vp, ctypes.c_size_t, _vp]
lib.circ_bwd_deterministic_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _int, _int, _int, _vp]
for _f in (lib.rdfft_fwd, lib.rdfft_inv, lib.rdfft_to_complex, lib.rdfft_from_complex, lib.rdfft2_fwd,
           lib.rdfft2_inv, lib.circ_prepare, lib.circ_fwd, lib.circ_bwd, lib.circ_fwd_tc, lib.circ_bwd_x_tc,
           lib.circ_bwd_workspace_size, lib.circ_bwd_deterministic, lib.circ_bwd_deterministic_noalloc):
    _f.restype = _int
lib.rdfft_strerror.argtypes = [_int]
lib.rdfft_strerror.restype = ctypes.c_char_p
lib.rdfft_version.argtypes = []
lib.rdfft_version.restype = _int
lib.rdfft_take_device_error.argtypes = []
lib.rdfft_take_device_error.restype = _int
lib.rdfft_selftest_wait_timeout.argtypes = [_vp]
lib.rdfft_selftest_wait_timeout.restype = _int

RDFFT_ETIMEOUT = 7


class RdfftError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {lib.rdfft_strerror(code).decode()} (code {code})")


def _check(code: int, where: str) -> None:
    if code != 0:
        raise RdfftError(code, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RDFFT_F32
    if t.dtype == torch.bfloat16:
        return RDFFT_BF16
    raise TypeError(f"rdfft supports float32 and bfloat16 tensors, got {t.dtype}")


def _cuda_dense(t: torch.Tensor, name: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def rdfft_fwd(t: torch.Tensor, p: int) -> torch.Tensor:
    """In-place packed rdFFT of every length-p row of `t` (numel a multiple of p)."""
    _cuda_dense(t, "t")
    if p <= 0 or t.numel() % p:
        raise ValueError("numel must be a multiple of p")
    with torch.cuda.device(t.device):
        _check(lib.rdfft_fwd(t.data_ptr(), t.numel() // p, p, _dtype_code(t), _stream(t)), "rdfft_fwd")
    return t


def rdfft_inv(t: torch.Tensor, p: int) -> torch.Tensor:
    """In-place inverse rdFFT (with 1/p) of every packed length-p row of `t`."""
    _cuda_dense(t, "t")
    if p <= 0 or t.numel() % p:
        raise ValueError("numel must be a multiple of p")
    with torch.cuda.device(t.device):
        _check(lib.rdfft_inv(t.data_ptr(), t.numel() // p, p, _dtype_code(t), _stream(t)), "rdfft_inv")
    return t


def rdfft_to_complex(t: torch.Tensor, p: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """Complex bins Y_0..Y_{p/2} of packed rows `t` (..., p), out of place, as a tensor of
    shape (..., p/2 + 1, 2) of t's dtype holding (re, im); for float32 use
    torch.view_as_complex on it."""
    _cuda_dense(t, "t")
    if p <= 0 or t.shape[-1] != p:
        raise ValueError("the last dimension of t must be p")
    shape = t.shape[:-1] + (p // 2 + 1, 2)
    if out is None:
        out = torch.empty(shape, dtype=t.dtype, device=t.device)
    _cuda_dense(out, "out")
    if out.shape != shape or out.dtype != t.dtype:
        raise ValueError(f"out must have shape {tuple(shape)} and dtype {t.dtype}")
    with torch.cuda.device(t.device):
        _check(lib.rdfft_to_complex(t.data_ptr(), out.data_ptr(), t.numel() // p, p, _dtype_code(t), _stream(t)),
               "rdfft_to_complex")
    return out


def rdfft_from_complex(z: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """Packed rows (..., p) from complex bins z (..., p/2 + 1, 2), out of place."""
    _cuda_dense(z, "z")
    if z.dim() < 2 or z.shape[-1] != 2:
        raise ValueError("z must have shape (..., p/2 + 1, 2)")
    p = 2 * (z.shape[-2] - 1)
    shape = z.shape[:-2] + (p,)
    if out is None:
        out = torch.empty(shape, dtype=z.dtype, device=z.device)
    _cuda_dense(out, "out")
    if out.shape != shape or out.dtype != z.dtype:
        raise ValueError(f"out must have shape {tuple(shape)} and dtype {z.dtype}")
    rows = out.numel() // p if p > 0 else 0
    with torch.cuda.device(z.device):
        _check(lib.rdfft_from_complex(z.data_ptr(), out.data_ptr(), rows, p, _dtype_code(z), _stream(z)),
               "rdfft_from_complex")
    return out


def _images(t: torch.Tensor):
    if t.dim() < 2:
        raise ValueError("t must have shape (..., R, C)")
    R, C = t.shape[-2], t.shape[-1]
    return t.numel() // (R * C) if R * C else 0, R, C


def rdfft2_fwd(t: torch.Tensor) -> torch.Tensor:
    """In-place 2-D rdFFT of every R x C image in the last two dimensions of `t`."""
    _cuda_dense(t, "t")
    n, R, C = _images(t)
    with torch.cuda.device(t.device):
        _check(lib.rdfft2_fwd(t.data_ptr(), n, R, C, _dtype_code(t), _stream(t)), "rdfft2_fwd")
    return t


def rdfft2_inv(t: torch.Tensor) -> torch.Tensor:
    """In-place inverse 2-D rdFFT (with 1/(R C)) of every packed R x C spectrum in `t`."""
    _cuda_dense(t, "t")
    n, R, C = _images(t)
    with torch.cuda.device(t.device):
        _check(lib.rdfft2_inv(t.data_ptr(), n, R, C, _dtype_code(t), _stream(t)), "rdfft2_inv")
    return t


def circ_prepare(c: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """c_hat for circ_fwd / circ_bwd: the packed rdFFT of fp32 c (q x q x p), computed out
    of place into `out` (a new tensor by default; `out` may be c itself)."""
    _cuda_dense(c, "c")
    if c.dim() != 3 or c.shape[0] != c.shape[1]:
        raise ValueError("c must have shape (q, q, p)")
    if c.dtype != torch.float32:
        raise TypeError("c must be float32")
    q, p = c.shape[0], c.shape[2]
    if out is None:
        out = torch.empty_like(c)
    _cuda_dense(out, "out")
    if out.shape != c.shape or out.dtype != torch.float32:
        raise ValueError("out must match c in shape and be float32")
    with torch.cuda.device(c.device):
        _check(lib.circ_prepare(c.data_ptr(), out.data_ptr(), q * p, p, _stream(c)), "circ_prepare")
    return out


def _layer_dims(x: torch.Tensor, p: int):
    D = x.shape[-1]
    B = x.numel() // D if D else 0
    return B, D


def circ_fwd(x: torch.Tensor, c_hat: torch.Tensor, p: int, y: torch.Tensor | None = None) -> torch.Tensor:
    """y = W x of the block-circulant layer, for x of shape (..., D)."""
    _cuda_dense(x, "x")
    _cuda_dense(c_hat, "c_hat")
    if c_hat.dtype != torch.float32:
        raise TypeError("c_hat must be float32")
    if y is None:
        y = torch.empty_like(x)
    _cuda_dense(y, "y")
    if y.dtype != x.dtype or y.shape != x.shape:
        raise ValueError("y must match x in shape and dtype")
    B, D = _layer_dims(x, p)
    with torch.cuda.device(x.device):
        _check(lib.circ_fwd(x.data_ptr(), c_hat.data_ptr(), y.data_ptr(), B, D, p, _dtype_code(x),
                            _stream(x)), "circ_fwd")
    return y


def circ_bwd_workspace_size(B: int, D: int, p: int, dtype: torch.dtype, with_grad_x: bool = True) -> int:
    """Bytes of workspace circ_bwd(..., deterministic=True) needs on the current device (0: none)."""
    n = ctypes.c_size_t()
    code = RDFFT_BF16 if dtype == torch.bfloat16 else RDFFT_F32
    _check(lib.circ_bwd_workspace_size(B, D, p, code, int(with_grad_x), ctypes.byref(n)), "circ_bwd_workspace_size")
    return n.value


def circ_bwd(g: torch.Tensor, x: torch.Tensor, c_hat: torch.Tensor, p: int,
             grad_x: torch.Tensor | None = None, grad_c: torch.Tensor | None = None,
             need_grad_x: bool = True, need_grad_c: bool = True, deterministic: bool = False,
             workspace: torch.Tensor | None = None):
    """(grad_x, grad_c) of the block-circulant layer for upstream gradient g.

    deterministic=True calls circ_bwd_deterministic: grad_c is then the same bit for bit
    from run to run. Its workspace (device bytes, circ_bwd_workspace_size) is taken from
    `workspace` if given, else allocated here through torch's caching allocator."""
    _cuda_dense(g, "g")
    _cuda_dense(x, "x")
    _cuda_dense(c_hat, "c_hat")
    if c_hat.dtype != torch.float32:
        raise TypeError("c_hat must be float32")
    if x.dtype != g.dtype or x.shape != g.shape:
        raise ValueError("g must match x in shape and dtype")
    B, D = _layer_dims(x, p)
    if need_grad_x and grad_x is None:
        grad_x = torch.empty_like(g)
    if need_grad_c and grad_c is None:
        grad_c = torch.empty(c_hat.shape, dtype=torch.float32, device=c_hat.device)
    gx_ptr = grad_x.data_ptr() if (need_grad_x and grad_x is not None) else None
    gc_ptr = grad_c.data_ptr() if (need_grad_c and grad_c is not None) else None
    with torch.cuda.device(x.device):
        if not deterministic:
            _check(lib.circ_bwd(g.data_ptr(), x.data_ptr(), c_hat.data_ptr(), gx_ptr, gc_ptr, B, D, p,
                                _dtype_code(x), _stream(x)), "circ_bwd")
        else:
            need = circ_bwd_workspace_size(B, D, p, x.dtype, gx_ptr is not None) if gc_ptr is not None else 0
            if workspace is None:
                workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
            _cuda_dense(workspace, "workspace")
            _check(lib.circ_bwd_deterministic(g.data_ptr(), x.data_ptr(), c_hat.data_ptr(), gx_ptr, gc_ptr, B, D,
                                              p, _dtype_code(x), workspace.data_ptr(),
                                              workspace.numel() * workspace.element_size(), _stream(x)),
                   "circ_bwd_deterministic")
    return (grad_x if need_grad_x else None), (grad_c if need_grad_c else None)


def circ_fwd_tc(x: torch.Tensor, c_hat: torch.Tensor, p: int, y: torch.Tensor | None = None) -> torch.Tensor:
    """circ_fwd with the per-bin contraction on the tensor cores (bf16, p = 128, D = 4096)."""
    _cuda_dense(x, "x")
    _cuda_dense(c_hat, "c_hat")
    if y is None:
        y = torch.empty_like(x)
    _cuda_dense(y, "y")
    if y.dtype != x.dtype or y.shape != x.shape:
        raise ValueError("y must match x in shape and dtype")
    B, D = _layer_dims(x, p)
    with torch.cuda.device(x.device):
        _check(lib.circ_fwd_tc(x.data_ptr(), c_hat.data_ptr(), y.data_ptr(), B, D, p, _dtype_code(x), _stream(x)),
               "circ_fwd_tc")
    return y


def circ_bwd_x_tc(g: torch.Tensor, c_hat: torch.Tensor, p: int, grad_x: torch.Tensor | None = None) -> torch.Tensor:
    """grad_x of circ_bwd with the per-bin contraction on the tensor cores (bf16, p = 128, D = 4096)."""
    _cuda_dense(g, "g")
    _cuda_dense(c_hat, "c_hat")
    if grad_x is None:
        grad_x = torch.empty_like(g)
    _cuda_dense(grad_x, "grad_x")
    if grad_x.dtype != g.dtype or grad_x.shape != g.shape:
        raise ValueError("grad_x must match g in shape and dtype")
    B, D = _layer_dims(g, p)
    with torch.cuda.device(g.device):
        _check(lib.circ_bwd_x_tc(g.data_ptr(), c_hat.data_ptr(), grad_x.data_ptr(), B, D, p, _dtype_code(g),
                                 _stream(g)), "circ_bwd_x_tc")
    return grad_x


def take_device_error() -> int:
    """Device error state of the transform kernels since the last call (then cleared):
    0, or RDFFT_ETIMEOUT when a bounded wait gave up. Synchronises with the device."""
    code = lib.rdfft_take_device_error()
    if code not in (0, RDFFT_ETIMEOUT):
        raise RdfftError(code, "rdfft_take_device_error")
    return code


def selftest_wait_timeout() -> None:
    """Enqueue the self-test kernel whose bounded wait runs out (about 1 ms)."""
    _check(lib.rdfft_selftest_wait_timeout(torch.cuda.current_stream().cuda_stream), "rdfft_selftest_wait_timeout")
