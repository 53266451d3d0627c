"""C ABI checks that need no GPU: the library loads, exports every declared symbol,
rejects bad arguments before touching CUDA, and its objects call no allocator."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

from conftest import ROOT

PKG = os.path.join(ROOT, "block_circulant_layers_b200")
HEADER = os.path.join(ROOT, "include", "rdfft.h")

OK, EINVAL, ENULL, EALIGN, EDTYPE, ECUDA, EOVERLAP, ETIMEOUT, ESPACE = range(9)
F32, BF16 = 0, 1


@pytest.fixture(scope="module")
def lib():
    from block_circulant_layers_b200 import build
    build.build_lib()
    L = ctypes.CDLL(os.path.join(PKG, "librdfft.so"))
    i64, i, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    L.rdfft_fwd.argtypes = [vp, i64, i, i, vp]
    L.rdfft_inv.argtypes = [vp, i64, i, i, vp]
    L.rdfft_to_complex.argtypes = [vp, vp, i64, i, i, vp]
    L.rdfft_from_complex.argtypes = [vp, vp, i64, i, i, vp]
    L.rdfft2_fwd.argtypes = [vp, i64, i, i, i, vp]
    L.rdfft2_inv.argtypes = [vp, i64, i, i, i, vp]
    L.circ_prepare.argtypes = [vp, vp, i, i, vp]
    L.circ_fwd.argtypes = [vp, vp, vp, i64, i, i, i, vp]
    L.circ_bwd.argtypes = [vp, vp, vp, vp, vp, i64, i, i, i, vp]
    L.circ_fwd_tc.argtypes = [vp, vp, vp, i64, i, i, i, vp]
    L.circ_bwd_x_tc.argtypes = [vp, vp, vp, i64, i, i, i, vp]
    L.circ_bwd_workspace_size.argtypes = [i64, i, i, i, i, ctypes.POINTER(ctypes.c_size_t)]
    L.circ_bwd_deterministic.argtypes = [vp, vp, vp, vp, vp, i64, i, i, i, vp, ctypes.c_size_t, vp]
    L.circ_bwd_deterministic_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i, i, i, vp]
    L.rdfft_strerror.argtypes = [i]
    L.rdfft_strerror.restype = ctypes.c_char_p
    return L


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"^\s*(?:int|const char\*)\s+(\w+)\s*\(", src, flags=re.M)


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("rdfft_fwd", "rdfft_inv", "rdfft_to_complex", "rdfft_from_complex", "rdfft2_fwd", "rdfft2_inv",
              "circ_prepare", "circ_fwd", "circ_bwd", "circ_fwd_tc", "circ_bwd_x_tc", "circ_bwd_workspace_size",
              "circ_bwd_deterministic", "circ_bwd_deterministic_noalloc", "rdfft_strerror",
              "rdfft_version",
              "rdfft_take_device_error",
              "rdfft_selftest_wait_timeout"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", os.path.join(PKG, "librdfft.so")],
                         capture_output=True, text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    for name in declared_functions():
        assert name in exported, name


def test_version_and_messages(lib):
    assert lib.rdfft_version() >= 100
    for code in range(9):
        assert lib.rdfft_strerror(code)
    assert b"workspace" in lib.rdfft_strerror(ESPACE)
    assert b"unknown" in lib.rdfft_strerror(99)


A = 0x10000          # aligned fake device addresses: validation fails before any use
Bp = 0x20000000


def test_rdfft_argument_errors(lib):
    for fn in (lib.rdfft_fwd, lib.rdfft_inv):
        assert fn(None, 0, 512, F32, None) == OK          # empty work: nothing enqueued
        assert fn(None, 4, 512, F32, None) == ENULL
        assert fn(A, 4, 3, F32, None) == EINVAL
        assert fn(A, 4, 1, F32, None) == EINVAL
        assert fn(A, 4, 8192, F32, None) == EINVAL
        assert fn(A, -1, 512, F32, None) == EINVAL
        assert fn(A, 4, 512, 2, None) == EDTYPE
        assert fn(A + 4, 4, 512, BF16, None) == EALIGN


def test_complex_cast_argument_errors(lib):
    for fn in (lib.rdfft_to_complex, lib.rdfft_from_complex):
        assert fn(None, None, 0, 512, F32, None) == OK
        assert fn(None, Bp, 4, 512, F32, None) == ENULL
        assert fn(A, None, 4, 512, F32, None) == ENULL
        assert fn(A, Bp, 4, 6, F32, None) == EINVAL
        assert fn(A, Bp, -2, 512, F32, None) == EINVAL
        assert fn(A, Bp, 4, 512, 3, None) == EDTYPE
        assert fn(A + 8, Bp, 4, 512, F32, None) == EALIGN
        assert fn(A, Bp + 2, 4, 512, BF16, None) == EALIGN
        assert fn(A, A, 4, 512, F32, None) == EOVERLAP
    # packed rows 4 x 512 f32 = 8192 B; complex rows 4 x 514 f32 = 8224 B (only
    # overlapping pairs here: a disjoint pair would pass validation and launch)
    assert lib.rdfft_to_complex(A, A + 8176, 4, 512, F32, None) == EOVERLAP
    assert lib.rdfft_from_complex(A, A + 8208, 4, 512, F32, None) == EOVERLAP


def test_2d_argument_errors(lib):
    for fn in (lib.rdfft2_fwd, lib.rdfft2_inv):
        assert fn(None, 0, 64, 64, F32, None) == OK
        assert fn(None, 2, 64, 64, F32, None) == ENULL
        assert fn(A, 2, 48, 64, F32, None) == EINVAL
        assert fn(A, 2, 64, 8192, F32, None) == EINVAL
        assert fn(A, 2, 1, 64, F32, None) == EINVAL
        assert fn(A, -1, 64, 64, F32, None) == EINVAL
        assert fn(A, 1 << 40, 4096, 4096, F32, None) == EINVAL      # images * R * C overflows int64
        assert fn(A, 2, 64, 64, 7, None) == EDTYPE
        assert fn(A + 2, 2, 64, 64, BF16, None) == EALIGN


def test_circ_argument_errors(lib):
    D, p = 4096, 128
    assert lib.circ_fwd(A, Bp, A + (1 << 26), 0, D, p, BF16, None) == OK
    assert lib.circ_fwd(A, Bp, A + (1 << 26), 4, 4000, p, BF16, None) == EINVAL   # D % p
    assert lib.circ_fwd(A, Bp, A + (1 << 26), 4, 16384, p, BF16, None) == EINVAL  # D too large
    assert lib.circ_fwd(A, Bp, A + (1 << 26), 4, 1024, 32, BF16, None) == EINVAL  # p < 64
    assert lib.circ_fwd(A, Bp, A + (1 << 26), 4, D, p, 5, None) == EDTYPE
    assert lib.circ_fwd(None, Bp, A, 4, D, p, BF16, None) == ENULL
    assert lib.circ_fwd(A, None, A + (1 << 26), 4, D, p, BF16, None) == ENULL
    assert lib.circ_fwd(A, Bp + 8, A + (1 << 26), 4, D, p, BF16, None) == EALIGN
    assert lib.circ_fwd(A, Bp, A, 4, D, p, BF16, None) == EOVERLAP                 # y == x
    assert lib.circ_fwd(A, Bp, A + 4096, 4, D, p, BF16, None) == EOVERLAP          # partial overlap
    # backward
    assert lib.circ_bwd(A, A, Bp, None, None, 4, D, p, BF16, None) == OK           # nothing asked
    assert lib.circ_bwd(None, A, Bp, A + (1 << 26), None, 4, D, p, BF16, None) == ENULL
    assert lib.circ_bwd(A, None, Bp, None, Bp + (1 << 24), 4, D, p, BF16, None) == ENULL
    assert lib.circ_bwd(A, A, Bp, A, None, 4, D, p, BF16, None) == EOVERLAP        # grad_x == g
    assert lib.circ_bwd(A, A + (1 << 25), Bp, None, A, 4, D, p, BF16, None) == EOVERLAP
    assert lib.circ_bwd(A, A + (1 << 25), Bp, A + (1 << 26), None, 4, 4000, p, BF16, None) == EINVAL


def workspace_size(lib, B, D, p, dtype=BF16, with_gx=1):
    n = ctypes.c_size_t(12345)
    rc = lib.circ_bwd_workspace_size(B, D, p, dtype, with_gx, ctypes.byref(n))
    return rc, n.value


def test_deterministic_backward_workspace_size(lib):
    """The workspace query runs the launchers' own shape choice without a GPU (148 SMs
    assumed): slices x q^2 p x 4 bytes, 0 for one slice, and the usual shape errors."""
    assert lib.circ_bwd_workspace_size(4, 4096, 128, BF16, 1, None) == ENULL
    assert workspace_size(lib, 4, 4000, 128) == (EINVAL, 0)
    assert workspace_size(lib, 4, 4096, 32) == (EINVAL, 0)
    assert workspace_size(lib, 4, 4096, 128, dtype=3) == (EDTYPE, 0)
    assert workspace_size(lib, 0, 4096, 128) == (OK, 0)              # empty batch
    assert workspace_size(lib, 1, 4096, 128) == (OK, 0)              # one slice stores grad_c
    assert workspace_size(lib, 2, 4096, 512) == (OK, 0)              # one tile of 2 tokens
    # D = 4096, p = 128, B = 256: 4 input-block groups x 32 slices of two 4-token tiles, both
    # with grad_x (one kernel) and without (the grad_c kernel); 32 x 512 KiB
    assert workspace_size(lib, 256, 4096, 128) == (OK, 32 * 32 * 32 * 128 * 4)
    assert workspace_size(lib, 256, 4096, 128, with_gx=0) == (OK, 32 * 32 * 32 * 128 * 4)
    # the adapter shape, D = 4096, p = 512, B = 4096: 147 slices of 7 tiles
    assert workspace_size(lib, 4096, 4096, 512) == (OK, 147 * 8 * 8 * 512 * 4)
    # one block, p = 4096, B = 4096, 2-token tiles: 147 slices
    assert workspace_size(lib, 4096, 4096, 4096) == (OK, 147 * 4096 * 4)
    for B in (1, 2, 5, 64, 255, 256, 1000, 4097):
        for D, p in ((4096, 128), (4096, 512), (1024, 64), (2048, 1024), (8192, 4096)):
            rc, n = workspace_size(lib, B, D, p)
            q = D // p
            assert rc == OK and n % (q * q * p * 4) == 0 and n // (q * q * p * 4) <= 148


def test_deterministic_backward_argument_errors(lib):
    """Checked before anything is enqueued: the circ_bwd checks, then the workspace's."""
    B, D, p = 256, 4096, 128
    need = 32 * 32 * 32 * 128 * 4                     # 16 MiB (see the test above)
    g, x, gx = A, A + (1 << 22), A + (1 << 23)        # 2 MiB bf16 activations each
    ch, gc, ws = Bp, Bp + (1 << 20), Bp + (1 << 24)   # c_hat, grad_c: 512 KiB each
    f = lib.circ_bwd_deterministic
    assert f(g, x, ch, None, None, B, D, p, BF16, None, 0, None) == OK         # nothing asked
    assert f(g, x, ch, gx, gc, B, 4000, p, BF16, ws, need, None) == EINVAL
    assert f(g, x, ch, gx, gc, B, D, p, 7, ws, need, None) == EDTYPE
    assert f(None, x, ch, gx, gc, B, D, p, BF16, ws, need, None) == ENULL
    assert f(g, x, ch, g, gc, B, D, p, BF16, ws, need, None) == EOVERLAP       # grad_x == g
    assert f(g, x, ch, gx, gc, B, D, p, BF16, None, need, None) == ENULL       # workspace needed
    assert f(g, x, ch, gx, gc, B, D, p, BF16, ws + 4, need, None) == EALIGN
    assert f(g, x, ch, gx, gc, B, D, p, BF16, ws, need - 16, None) == ESPACE
    assert f(g, x, ch, gx, gc, B, D, p, BF16, g, need, None) == EOVERLAP       # workspace over g
    assert f(g, x, ch, gx, gc, B, D, p, BF16, gc - 4096, need, None) == EOVERLAP


def test_noalloc_backward_argument_errors(lib):
    """The built-in-scratch variant checks like circ_bwd and refuses, before enqueuing
    anything, a call whose workspace would exceed its 16 MiB."""
    f = lib.circ_bwd_deterministic_noalloc
    B, D, p = 256, 4096, 128
    g, x, gx = A, A + (1 << 22), A + (1 << 23)
    ch, gc = Bp, Bp + (1 << 20)
    assert f(g, x, ch, None, None, B, D, p, BF16, None) == OK                 # nothing asked
    assert f(g, x, ch, gx, gc, B, 4000, p, BF16, None) == EINVAL
    assert f(g, x, ch, gx, gc, B, D, p, 9, None) == EDTYPE
    assert f(g, None, ch, gx, gc, B, D, p, BF16, None) == ENULL
    assert f(g, x, ch, gx + 2, gc, B, D, p, BF16, None) == EALIGN
    assert f(g, x, ch, gc, gc, B, D, p, BF16, None) == EOVERLAP
    # D = 8192, p = 64 (q = 128: 4 MiB of grad_c per token slice), B = 4096: 5 slices, 20 MiB;
    # the adapter shape D = 4096, p = 512, B = 4096: 147 slices, 18.4 MiB
    for B, D, p in ((4096, 8192, 64), (4096, 4096, 512)):
        rc, need = workspace_size(lib, B, D, p)
        assert rc == OK and need > (16 << 20)
        q = D // p
        g, x, gx = A, A + (1 << 27), A + (1 << 28)      # up to 64 MiB bf16 activations each
        ch, gc = Bp, Bp + (1 << 23)                     # up to 4 MiB c_hat / grad_c
        assert f(g, x, ch, gx, gc, B, D, p, BF16, None) == ESPACE
    # the same tokens without grad_x take the grad_c kernel: one input-block group of 147
    # slices, 18.4 MiB
    rc, need = workspace_size(lib, 4096, 4096, 512, with_gx=0)
    assert rc == OK and need > (16 << 20)
    assert f(A, A + (1 << 27), Bp, None, Bp + (1 << 23), 4096, 4096, 512, BF16, None) == ESPACE


def test_circ_prepare_argument_errors(lib):
    D, p = 4096, 128                                   # c: 32 x 32 x 128 fp32 = 512 KiB
    assert lib.circ_prepare(Bp, Bp + (1 << 20), D, 100, None) == EINVAL        # p not a power of two
    assert lib.circ_prepare(Bp, Bp + (1 << 20), D, 32, None) == EINVAL         # p < 64
    assert lib.circ_prepare(Bp, Bp + (1 << 20), 4000, p, None) == EINVAL       # D % p
    assert lib.circ_prepare(None, Bp, D, p, None) == ENULL
    assert lib.circ_prepare(Bp, None, D, p, None) == ENULL
    assert lib.circ_prepare(Bp + 4, Bp + (1 << 20), D, p, None) == EALIGN
    assert lib.circ_prepare(Bp, Bp + 4096, D, p, None) == EOVERLAP             # partial overlap


def test_tensor_core_layer_argument_errors(lib):
    """The tensor-core entry points check like circ_fwd and cover bf16, p = 128, D = 4096."""
    D, p = 4096, 128
    for f in (lib.circ_fwd_tc, lib.circ_bwd_x_tc):
        assert f(A, Bp, A + (1 << 26), 0, D, p, BF16, None) == OK                 # empty
        assert f(A, Bp, A + (1 << 26), 4, D, p, F32, None) == EINVAL              # fp32
        assert f(A, Bp, A + (1 << 26), 4, 2048, p, BF16, None) == EINVAL          # D != 4096
        assert f(A, Bp, A + (1 << 26), 4, D, 256, BF16, None) == EINVAL           # p != 128
        assert f(A, Bp, A + (1 << 26), 4, D, p, 5, None) == EDTYPE
        assert f(None, Bp, A, 4, D, p, BF16, None) == ENULL
        assert f(A, Bp + 8, A + (1 << 26), 4, D, p, BF16, None) == EALIGN
        assert f(A, Bp, A, 4, D, p, BF16, None) == EOVERLAP                       # output == input


def test_objects_call_no_allocator():
    """The library allocates nothing: none of its own objects references an allocator."""
    from block_circulant_layers_b200 import build
    build.build_lib()
    objs = glob.glob(os.path.join(PKG, "_build", "*.o"))
    assert objs
    for o in objs:
        und = subprocess.run(["nm", "-u", o], capture_output=True, text=True, check=True).stdout
        for sym in ("cudaMalloc", "cudaMallocAsync", "cudaMallocManaged", "cudaMallocHost", "cuMemAlloc",
                    "cudaHostAlloc", "cudaMallocPitch", "cudaMalloc3D"):
            assert not re.search(rf"\b{sym}\w*\b", und), (o, sym)
