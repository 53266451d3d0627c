"""The block-circulant layer launchers' shape rules (csrc/layer_policy.h), run on the
CPU through the host test library: output blocks per forward / grad_x CTA, input
blocks per grad_c group and grad_c token slices. The rules only reshape grids that
would leave most SMs idle; the shapes measured at B >= 256 stay as they are."""
import ctypes
import os

import pytest

from conftest import ROOT

N_SM = 148


@pytest.fixture(scope="module")
def emu():
    from block_circulant_layers_b200 import build
    build.build_emulator()
    L = ctypes.CDLL(os.path.join(ROOT, "block_circulant_layers_b200", "librdfft_hostemu.so"))
    L.rdfft_layer_qi.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int]
    L.rdfft_layer_qj.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int]
    L.rdfft_layer_gc_slices.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_int64)]
    return L


def largest_divisor_leq(q, cap):
    return max(d for d in range(1, cap + 1) if q % d == 0)


# (what, q, output blocks a CTA's slots cover, token groups of the grid, expected QI)
QI_CASES = [
    ("D=4096 p=128 B=256: 4 tokens, 16 blocks per CTA", 32, 16, 64, 16),
    ("D=4096 p=512 B=4096 (adapter): 4 tokens, 8 blocks", 8, 8, 1024, 8),
    ("D=4096 p=1024 B=256: 1 token, 4 blocks", 4, 4, 256, 4),
    ("D=4096 p=4096 B=256: q = 1", 1, 1, 256, 1),
    ("D=4096 p=128 B=1: one output block per CTA, 32 CTAs", 32, 8, 1, 1),
    ("D=4096 p=128 B=8: 2 blocks per CTA, 128 CTAs", 32, 8, 8, 2),
]


@pytest.mark.parametrize("what,q,qi_max,gx,want", QI_CASES)
def test_output_blocks_per_cta(emu, what, q, qi_max, gx, want):
    assert emu.rdfft_layer_qi(q, qi_max, gx, N_SM) == want, what


def test_output_blocks_rule_properties(emu):
    for q in range(1, 65):
        for qi_max in (1, 2, 4, 8, 16, 32):
            for gx in (1, 2, 3, 5, 8, 17, 40, 64, 128, 1024):
                qi = emu.rdfft_layer_qi(q, qi_max, gx, N_SM)
                first = largest_divisor_leq(q, qi_max)
                assert q % qi == 0 and 1 <= qi <= first
                if gx * (q // first) >= N_SM // 2:
                    assert qi == first                     # a full grid keeps its shape
                if qi > 1:
                    assert gx * (q // qi) >= N_SM // 2    # a shrunk grid covers half the SMs
                # and the rule shrank no further than needed: every larger divisor of q it
                # passed over (from the slots' cover down) left the grid under half the SMs
                d = first
                while d > qi:
                    assert gx * (q // d) < N_SM // 2
                    d = largest_divisor_leq(q, d - 1)
                assert d == qi


# (what, q, bins p/2, token tiles, expected QJ); at most 32 x 512 accumulators per CTA
QJ_CASES = [
    ("D=4096 p=128 B=256, 4-token tiles", 32, 64, 64, 8),
    ("D=4096 p=512 B=4096 (adapter)", 8, 256, 1024, 8),
    ("D=4096 p=1024 B=256, 2-token tiles", 4, 512, 128, 4),
    ("D=4096 p=4096 B=256", 1, 2048, 256, 1),
    ("D=4096 p=128 B=1: one input block per group, 32 CTAs", 32, 64, 1, 1),
    ("D=8192 p=64: accumulator limit", 128, 32, 1024, 4),
]


@pytest.mark.parametrize("what,q,hb,ntiles,want", QJ_CASES)
def test_input_blocks_per_grad_c_group(emu, what, q, hb, ntiles, want):
    assert emu.rdfft_layer_qj(q, hb, 32 * 512, ntiles, N_SM) == want, what


def test_input_block_rule_properties(emu):
    for q in range(1, 129):
        for hb in (32, 64, 128, 256, 512, 1024, 2048):
            for ntiles in (1, 2, 4, 16, 64, 1024):
                qj = emu.rdfft_layer_qj(q, hb, 32 * 512, ntiles, N_SM)
                assert q % qj == 0 and 1 <= qj <= 8
                assert qj == 1 or hb * q * qj <= 32 * 512
                if qj > 1:
                    assert ntiles * (q // qj) >= N_SM // 2


def test_grad_c_token_slices(emu):
    tp = ctypes.c_int64()
    # D=4096 p=128 B=256 with 4-token tiles: 4 groups x 32 slices of 2 tiles
    assert emu.rdfft_layer_gc_slices(4, 64, N_SM, ctypes.byref(tp)) == 32 and tp.value == 2
    # one tile (a handful of tokens): a single slice, so grad_c is stored, not accumulated
    assert emu.rdfft_layer_gc_slices(32, 1, N_SM, ctypes.byref(tp)) == 1 and tp.value == 1
    for njgroups in (1, 2, 4, 8, 16, 32, 64, 128, 200):
        for ntiles in (1, 2, 3, 7, 37, 64, 148, 1000, 4096):
            s = emu.rdfft_layer_gc_slices(njgroups, ntiles, N_SM, ctypes.byref(tp))
            assert s >= 1 and tp.value >= 1
            assert s * tp.value >= ntiles                 # every tile is covered
            assert (s - 1) * tp.value < ntiles            # and no slice is empty
            assert s <= max(1, -(-N_SM // njgroups))      # about one CTA per SM
            # a single slice (grad_c stored, no zeroing) exactly when one tile or one CTA
            # per group is all there is
            assert (s == 1) == (ntiles == 1 or -(-N_SM // njgroups) == 1)


def test_forward_token_tiles(emu):
    """The largest token tile whose grid keeps a token's output blocks in one CTA."""
    f = emu.rdfft_layer_x_tokens
    f.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    # D = 4096, p = 512 (q = 8, 8 output blocks per CTA): 64 groups of 4 tokens would need the
    # output blocks split in two; 2-token tiles give 128 CTAs of all 8
    assert f(256, 8, 8, N_SM, 4) == 2
    assert f(512, 8, 8, N_SM, 4) == 4
    assert f(4096, 8, 8, N_SM, 4) == 4
    assert f(64, 8, 8, N_SM, 2) == 1
    # D = 4096, p = 256 (q = 16): two output-block groups of 8 at B = 256 either way
    assert f(256, 16, 8, N_SM, 4) == 4
    for q in (1, 2, 4, 8, 16, 32, 64, 128):
        full = emu.rdfft_layer_qi(q, 8, 1 << 30, N_SM)
        for B in (1, 5, 32, 64, 200, 256, 300, 512, 1024, 4096):
            for tt_max in (1, 2, 4):
                tt = f(B, q, 8, N_SM, tt_max)
                assert tt in (1, 2, 4) and tt <= tt_max
                if tt > 1:                   # the chosen tile keeps the output blocks whole
                    assert emu.rdfft_layer_qi(q, 8, -(-B // tt), N_SM) == full
                if tt < tt_max:              # and every larger one would split them
                    for t2 in (2 * tt, 4 * tt):
                        if t2 <= tt_max:
                            assert emu.rdfft_layer_qi(q, 8, -(-B // t2), N_SM) != full


def test_fused_backward_token_tiles(emu):
    """The one-kernel backward takes its smaller token tile while every CTA then holds one
    tile and all fit in one wave of one CTA per SM."""
    f = emu.rdfft_layer_fused_small_tiles
    f.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    assert f(256, 2, 1, N_SM) == 1 and f(296, 2, 1, N_SM) == 1 and f(297, 2, 1, N_SM) == 0   # p = 512
    assert f(148, 1, 1, N_SM) == 1 and f(149, 1, 1, N_SM) == 0                             # p = 1024
    assert f(74, 2, 4, N_SM) == 1 and f(75, 2, 4, N_SM) == 0 and f(256, 2, 4, N_SM) == 0   # p = 128


def test_grad_c_token_tiles(emu):
    """The grad_c kernel halves its token tile while that leaves at most half the SMs' worth of
    tiles and its grid fits one wave."""
    f = emu.rdfft_layer_gc_half_tiles
    f.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int]
    S = 32 * 512
    # D = 4096: p = 512 (q = 8, 256 bins), p = 128 (q = 32, 64 bins), p = 1024 (q = 4, 512 bins)
    assert f(16, 4, 8, 256, S, N_SM) == 1 and f(128, 4, 8, 256, S, N_SM) == 1
    assert f(256, 4, 8, 256, S, N_SM) == 0
    assert f(16, 4, 32, 64, S, N_SM) == 1 and f(64, 4, 32, 64, S, N_SM) == 1
    assert f(128, 4, 32, 64, S, N_SM) == 0
    assert f(64, 2, 4, 512, S, N_SM) == 1 and f(128, 2, 4, 512, S, N_SM) == 0
    assert f(5, 1, 4, 512, S, N_SM) == 0                  # no tile smaller than one token
    for q, hb in ((1, 2048), (4, 512), (8, 256), (16, 128), (32, 64), (64, 32), (128, 32)):
        for B in (1, 2, 7, 16, 64, 100, 128, 256, 1000):
            for tt in (2, 4):
                if f(B, tt, q, hb, S, N_SM):
                    nt = -(-B // (tt // 2))
                    qj = emu.rdfft_layer_qj(q, hb, S, nt, N_SM)
                    assert nt <= N_SM // 2 and nt * (q // qj) <= N_SM
