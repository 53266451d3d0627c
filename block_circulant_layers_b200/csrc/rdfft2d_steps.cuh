// Per-thread steps of the column half of the 2-D rdFFT over an image of R x C.
//
// The 2-D transform is the packed layout applied per axis ("Memory-Efficient
// Training with In-Place FFT Implementation": the packed layout of the summary page,
// "Approach"; the paper-notes page, "Limitations and outlook", leaves 2-D open). After
// the in-place rdFFT of every image row (the standalone row kernel), column k of the
// image holds a[r] = Re Z_r(k) and column C - k holds b[r] = Im Z_r(k), Z_r being the
// spectrum of row r. The 2-D spectrum is Y[k1, k] = DFT(a)[k1] + i DFT(b)[k1]. With
// A = rdFFT(a) and B = rdFFT(b) (packed down the columns), for 0 < k1 < R/2:
//     Re Y[k1, k]     = Ar - Bi      Im Y[k1, k]     = Ai + Br
//     Re Y[R - k1, k] = Ar + Bi      Im Y[R - k1, k] = Br - Ai
// (Ar = A[k1], Ai = A[R - k1], likewise B), and rows 0, R/2 keep A and B as they are.
// So the column pass transforms every column in place and combines each pair (k, C-k)
// into Re / Im of Y; columns 0 and C/2 hold real row bins, their column spectrum is
// conjugate symmetric and stays in the 1-D packed layout down the column.
//
// The inverse undoes the combine (halving the sums and differences), then runs the
// inverse column transform in its Hartley form, rdIFFT = (1/R) M rdFFT M with M the
// mirror (slot k <- y_k - y_{R-k}, slot R-k <- y_k + y_{R-k}): un-combine and the
// first M in one sweep over the tile, forward passes, the second M and 1/R on the
// store. The row inverse (standalone row kernel) follows.
//
// GPU shape (ours): a CTA owns the strip pair of H = W/2 "left" columns k0..k0+H-1
// (those <= C/2; tile rows 0..H-1) and their mirrors C - k (tile rows H..W-1), read
// from HBM once (consecutive threads read consecutive columns of one image row) into
// an fp32 shared tile with one tile row per column, and written back once.
#pragma once

#include "packed_fft.cuh"

namespace rdfft {

// Columns per CTA and CTA size for column length R >= 64: the tile (W columns of R
// fp32 plus pad) stays near 64 KiB for R <= 1024 and 132 KiB above; one thread per
// TPR-th of every column (up to 1024 threads), at least 128.
template <int R>
struct ColTiling {
  static constexpr int W = R >= 4096 ? 8 : (R >= 1024 ? 16 : 32);
  static constexpr int TPR = Geo<R, kEPT>::TPR;
  static constexpr int NT = W * TPR > 1024 ? 1024 : (W * TPR < 128 ? 128 : W * TPR);
};

// The row geometry of a column tile. For R >= 1024 (a warp per tile row in the
// passes) the row stride gets an extra pad so that it is 32/W modulo the 32 banks:
// the W tile rows that one load or store round touches at the same image row then
// fall in distinct banks. Shorter columns keep the row-kernel layout, whose row
// offsets already spread them.
template <int R, int W>
struct ColGeo : Geo<R, kEPT> {
  using Base = Geo<R, kEPT>;
  static constexpr bool WIDE = Base::TPR >= 32;
  static constexpr int XPAD = WIDE ? ((32 / W) - Base::RS % 32 + 32) % 32 : 0;
  static constexpr int RS = Base::RS + XPAD;
  RD_HD static constexpr int row_base(int r) { return WIDE ? r * RS : Base::row_base(r); }
  RD_HD static constexpr int words(int rows) { return row_base(rows) + 1; }
};

// Image column of tile row j of the strip pair starting at left column k0, or -1.
RD_HD int strip_col(int j, int H, int k0, int C) {
  if (j < H) {
    const int k = k0 + j;
    return k <= C / 2 ? k : -1;
  }
  const int k = k0 + j - H;
  return (k > 0 && k < C / 2) ? C - k : -1;
}

// Number of strip pairs (CTAs) per image: left columns 0..C/2.
RD_HD constexpr int col_groups(int C, int H) { return (C / 2 + H) / H; }

// HBM -> tile (forward). Thread tid owns tile row j = tid % W, a fixed image column,
// and image rows r0 + i STEP (r0 = tid / W, STEP = NT / W), so its tile addresses
// are one base plus compile-time offsets (STEP and 2^S divide one another) and its
// global addresses one base plus multiples of STEP rows. Loads are issued in batches
// of LB before their shared-memory stores, to keep LB loads in flight per thread.
template <class G, int W, int NT, typename T>
RD_HD void cols_load(float* tile, const T* img, int C, int k0, int tid) {
  constexpr int R = G::P, H = W / 2, STEP = NT / W, ITER = R / STEP;
  constexpr int LB = ITER < 16 ? ITER : 16;
  static_assert(NT % W == 0 && R % STEP == 0 && ITER % LB == 0, "whole rounds");
  static_assert(STEP % (1 << G::S) == 0 || (1 << G::S) % STEP == 0, "compile-time tile offsets");
  const int j = tid % W, r0 = tid / W;
  const int col = strip_col(j, H, k0, C);
  float* trow = tile + G::row_base(j) + G::at(r0);
  const T* src = img + (int64_t)r0 * C + (col >= 0 ? col : 0);
  const int64_t gstep = (int64_t)STEP * C;
#pragma unroll
  for (int i0 = 0; i0 < ITER; i0 += LB) {
    float v[LB];
#pragma unroll
    for (int b = 0; b < LB; ++b) v[b] = col >= 0 ? ld(src + (i0 + b) * gstep) : 0.0f;
#pragma unroll
    for (int b = 0; b < LB; ++b) {
      const int c = (i0 + b) * STEP;
      trow[c + (c >> G::S)] = v[b];
    }
  }
}

// HBM -> tile (inverse), fused with the first sweep of the inverse: un-combine each
// pair (k, C-k) back to the packed column spectra A, B and apply the mirror M to every
// column (slots 0 and R/2 unchanged). With u, u2 = Re Y at k1, R-k1 and w, w2 = Im Y:
//   Ar = (u + u2)/2, Bi = (u2 - u)/2, Br = (w + w2)/2, Ai = (w - w2)/2, and
//   M A: [k1] = Ar - Ai, [R-k1] = Ar + Ai;  M B: [k1] = Br - Bi, [R-k1] = Br + Bi.
// Thread tid owns left column k = k0 + tid % H (and its mirror) and the row pairs
// (k1, R - k1) for k1 = q0 + i STEP (q0 = tid / H, STEP = NT / H); k1 = 0 stands for
// the rows (0, R/2), which are copied.
template <class G, int W, int NT, typename T>
RD_HD void cols_load_unpair(float* tile, const T* img, int C, int k0, int tid) {
  constexpr int R = G::P, H = W / 2, Q = R / 2, STEP = NT / H, ITER = Q / STEP;
  constexpr int LB = ITER < 8 ? ITER : 8;
  static_assert(NT % H == 0 && Q % STEP == 0 && ITER % LB == 0, "whole rounds");
  const int jl = tid % H, q0 = tid / H;
  const int k = k0 + jl;
  const bool valid = k <= C / 2, paired = k > 0 && k < C / 2;
  float* A = tile + G::row_base(jl);
  float* B = tile + G::row_base(jl + H);
  const T* ca = img + (valid ? k : 0);
  const T* cb = img + (paired ? C - k : 0);
#pragma unroll
  for (int i0 = 0; i0 < ITER; i0 += LB) {
    float u[LB], u2[LB], w[LB], w2[LB];
#pragma unroll
    for (int b = 0; b < LB; ++b) {
      const int k1 = q0 + (i0 + b) * STEP;
      const int lo = k1, hi = k1 == 0 ? Q : R - k1;
      u[b] = valid ? ld(ca + (int64_t)lo * C) : 0.0f;
      u2[b] = valid ? ld(ca + (int64_t)hi * C) : 0.0f;
      w[b] = paired ? ld(cb + (int64_t)lo * C) : 0.0f;
      w2[b] = paired ? ld(cb + (int64_t)hi * C) : 0.0f;
    }
#pragma unroll
    for (int b = 0; b < LB; ++b) {
      const int k1 = q0 + (i0 + b) * STEP;
      const int lo = G::at(k1), hi = G::at(k1 == 0 ? Q : R - k1);
      if (k1 == 0) {
        A[lo] = u[b];
        A[hi] = u2[b];
        B[lo] = w[b];
        B[hi] = w2[b];
      } else if (paired) {
        const float su = u[b] + u2[b], du = u[b] - u2[b], sw = w[b] + w2[b], dw = w[b] - w2[b];
        A[lo] = 0.5f * (su - dw);
        A[hi] = 0.5f * (su + dw);
        B[lo] = 0.5f * (sw + du);
        B[hi] = 0.5f * (sw - du);
      } else {
        A[lo] = u[b] - u2[b];
        A[hi] = u[b] + u2[b];
        B[lo] = 0.0f;
        B[hi] = 0.0f;
      }
    }
  }
}

// Orbit pass K >= 1 (tile -> tile) of the forward column transform over tile rows
// [0, NR): generic orbits row by row, then the NR * NB merged orbits one per thread
// (disjoint positions, so both halves run without a barrier between them).
template <class G, int K>
RD_HD void cols_orbit_pass(float* tile, int NR, int tid, int NT) {
  constexpr int TPR = G::TPR;
  constexpr int NB = PassShape<G, K>::NB;
  const int v = tid % TPR;
  for (int r = tid / TPR; r < NR; r += NT / TPR)
    generic_pass<G, K, false, 0, 0>(tile, r, v, (float*)nullptr, false);
  for (int mu = tid; mu < NR * NB; mu += NT)
    merged_orbit<G, K, false, 0, 0>(tile, mu / NB, mu % NB, (float*)nullptr, false);
}

// Forward, tile -> HBM: combine each pair into Re / Im of Y (see the top of the file).
// Thread tid owns left column k = k0 + tid % H (and its mirror) and the row pairs
// (k1, R - k1), k1 = q0 + i STEP, as cols_load_unpair; k1 = 0 stands for (0, R/2).
template <class G, int W, int NT, typename T>
RD_HD void cols_store_fwd(const float* tile, T* img, int C, int k0, int tid) {
  constexpr int R = G::P, H = W / 2, Q = R / 2, STEP = NT / H, ITER = Q / STEP;
  const int jl = tid % H, q0 = tid / H;
  const int k = k0 + jl;
  if (k > C / 2) return;
  const bool paired = k > 0 && k < C / 2;
  const float* A = tile + G::row_base(jl);
  const float* B = tile + G::row_base(jl + H);
  T* ca = img + k;
  T* cb = img + (paired ? C - k : 0);
#pragma unroll 4
  for (int i = 0; i < ITER; ++i) {
    const int k1 = q0 + i * STEP;
    const int rlo = k1, rhi = k1 == 0 ? Q : R - k1;
    const float ar = A[G::at(rlo)], ai = A[G::at(rhi)];
    if (!paired) {
      ca[(int64_t)rlo * C] = from_f32<T>(ar);
      ca[(int64_t)rhi * C] = from_f32<T>(ai);
      continue;
    }
    const float br = B[G::at(rlo)], bi = B[G::at(rhi)];
    if (k1 == 0) {
      ca[0] = from_f32<T>(ar);
      ca[(int64_t)Q * C] = from_f32<T>(ai);
      cb[0] = from_f32<T>(br);
      cb[(int64_t)Q * C] = from_f32<T>(bi);
    } else {
      ca[(int64_t)rlo * C] = from_f32<T>(ar - bi);
      ca[(int64_t)rhi * C] = from_f32<T>(ar + bi);
      cb[(int64_t)rlo * C] = from_f32<T>(ai + br);
      cb[(int64_t)rhi * C] = from_f32<T>(br - ai);
    }
  }
}

// Inverse, tile -> HBM: the second mirror and the 1/R of the Hartley-form inverse.
// Thread tid owns tile row j = tid % W and the row pairs (k1, R - k1), k1 = q0 + i
// STEP (q0 = tid / W, STEP = NT / W); k1 = 0 stands for (0, R/2).
template <class G, int W, int NT, typename T>
RD_HD void cols_store_inv(const float* tile, T* img, int C, int k0, int tid) {
  constexpr int R = G::P, H = W / 2, Q = R / 2, STEP = NT / W, ITER = Q / STEP;
  constexpr float scale = 1.0f / R;
  const int j = tid % W, q0 = tid / W;
  const int col = strip_col(j, H, k0, C);
  if (col < 0) return;
  const float* X = tile + G::row_base(j);
  T* dst = img + col;
#pragma unroll 4
  for (int i = 0; i < ITER; ++i) {
    const int k1 = q0 + i * STEP;
    const int rlo = k1, rhi = k1 == 0 ? Q : R - k1;
    const float a = X[G::at(rlo)], b = X[G::at(rhi)];
    float lo, hi;
    if (k1 == 0) {
      lo = a * scale;
      hi = b * scale;
    } else {
      lo = (a - b) * scale;
      hi = (a + b) * scale;
    }
    dst[(int64_t)rlo * C] = from_f32<T>(lo);
    dst[(int64_t)rhi * C] = from_f32<T>(hi);
  }
}

// Columns of R <= 32: one thread owns left column k and its mirror C - k in
// registers (forward DIT stages on bit-reversed input, as the row kernel's small
// rows), with the same combine / un-combine and Hartley-form inverse as above.
template <int R, bool INV, typename T>
RD_HD void col_small(T* img, int C, int k) {
  constexpr int e = ilog2(R);
  const bool paired = k > 0 && k < C / 2;
  float a[R], b[R];
  if constexpr (!INV) {
#pragma unroll
    for (int j = 0; j < R; ++j) {
      a[bitrev(j, e)] = ld(img + (int64_t)j * C + k);
      b[bitrev(j, e)] = paired ? ld(img + (int64_t)j * C + (C - k)) : 0.0f;
    }
    stages_contig<2, R, R, 0, false>(a);
    stages_contig<2, R, R, 0, false>(b);
    if (!paired) {
#pragma unroll
      for (int j = 0; j < R; ++j) img[(int64_t)j * C + k] = from_f32<T>(a[j]);
      return;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float re, im;
      if (r == 0 || r == R / 2) {
        re = a[r];
        im = b[r];
      } else {
        const int k1 = r < R / 2 ? r : R - r;
        const float ar = a[k1], ai = a[R - k1], br = b[k1], bi = b[R - k1];
        re = r < R / 2 ? ar - bi : ar + bi;
        im = r < R / 2 ? ai + br : br - ai;
      }
      img[(int64_t)r * C + k] = from_f32<T>(re);
      img[(int64_t)r * C + (C - k)] = from_f32<T>(im);
    }
  } else {
    float u[R], w[R];
#pragma unroll
    for (int j = 0; j < R; ++j) {
      u[j] = ld(img + (int64_t)j * C + k);
      w[j] = paired ? ld(img + (int64_t)j * C + (C - k)) : 0.0f;
    }
    // un-combine + mirror into bit-reversed registers
    a[0] = u[0];
    b[0] = w[0];
    a[bitrev(R / 2, e)] = u[R / 2];
    b[bitrev(R / 2, e)] = w[R / 2];
#pragma unroll
    for (int k1 = 1; k1 < R / 2; ++k1) {
      if (paired) {
        const float su = u[k1] + u[R - k1], du = u[k1] - u[R - k1];
        const float sw = w[k1] + w[R - k1], dw = w[k1] - w[R - k1];
        a[bitrev(k1, e)] = 0.5f * (su - dw);
        a[bitrev(R - k1, e)] = 0.5f * (su + dw);
        b[bitrev(k1, e)] = 0.5f * (sw + du);
        b[bitrev(R - k1, e)] = 0.5f * (sw - du);
      } else {
        a[bitrev(k1, e)] = u[k1] - u[R - k1];
        a[bitrev(R - k1, e)] = u[k1] + u[R - k1];
        b[bitrev(k1, e)] = 0.0f;
        b[bitrev(R - k1, e)] = 0.0f;
      }
    }
    stages_contig<2, R, R, 0, false>(a);
    stages_contig<2, R, R, 0, false>(b);
    constexpr float scale = 1.0f / R;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float xa, xb;
      if (r == 0 || r == R / 2) {
        xa = a[r] * scale;
        xb = b[r] * scale;
      } else if (r < R / 2) {
        xa = (a[r] - a[R - r]) * scale;
        xb = (b[r] - b[R - r]) * scale;
      } else {
        xa = (a[R - r] + a[r]) * scale;
        xb = (b[R - r] + b[r]) * scale;
      }
      img[(int64_t)r * C + k] = from_f32<T>(xa);
      if (paired) img[(int64_t)r * C + (C - k)] = from_f32<T>(xb);
    }
  }
}

}  // namespace rdfft
