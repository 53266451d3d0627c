// Per-thread steps of the standalone batched rdFFT / rdIFFT over rows of length P.
//
// A CTA owns ROWS consecutive rows and Plan<P>::TPR threads per row. Step k of the
// forward transform runs pass k; step k of the inverse runs pass NPASS-1-k with the
// inverse butterflies ("In-place IFFT design" on the paper-notes page of "Memory-
// Efficient Training with In-Place FFT Implementation": the inverse reverses the
// forward graph). Consecutive steps are separated by a CTA barrier on the GPU and by
// a full sweep over the threads in the host emulator. The first step reads the row
// from global memory and the last one writes it back in place, so the only other
// storage is the CTA's fp32 shared-memory tile.
#pragma once

#include "packed_fft.cuh"

namespace rdfft {

template <int P, bool INV, int K, typename T>
RD_HD void row_step(float* tile, int lrow, int v, T* g, bool active) {
  constexpr int NP = Plan<P>::NPASS;
  static_assert(NP >= 2, "multi-pass rows only");
  if constexpr (!INV) {
    if constexpr (K == 0) fwd_pass0<P, T>(tile, lrow, v, g, active);
    else if constexpr (K == NP - 1) orbit_pass<P, K, false, 0, 1>(tile, lrow, v, g, active);
    else orbit_pass<P, K, false, 0, 0>(tile, lrow, v, g, active);
  } else {
    constexpr int PASS = NP - 1 - K;
    if constexpr (PASS == 0) inv_pass0<P, T>(tile, lrow, v, g, active);
    else if constexpr (K == 0) orbit_pass<P, PASS, true, 1, 0>(tile, lrow, v, g, active);
    else orbit_pass<P, PASS, true, 0, 0>(tile, lrow, v, g, active);
  }
}

// Rows of P <= 32: one thread per row, everything in registers.
template <int P, bool INV, typename T>
RD_HD void row_small(T* g) {
  constexpr int e = ilog2(P);
  float a[P];
  if constexpr (!INV) {
#pragma unroll
    for (int j = 0; j < P; ++j) a[bitrev(j, e)] = ld(g + j);
    stages_contig<2, P, P, 0, false>(a);
#pragma unroll
    for (int j = 0; j < P; ++j) g[j] = from_f32<T>(a[j]);
  } else {
#pragma unroll
    for (int j = 0; j < P; ++j) a[j] = ld(g + j);
    stages_contig<2, P, P, 0, true>(a);
    constexpr float scale = 1.0f / P;
#pragma unroll
    for (int j = 0; j < P; ++j) g[bitrev(j, e)] = from_f32<T>(a[j] * scale);
  }
}

// Rows per CTA: 128 threads for the multi-pass rows, 128 rows for the small ones.
template <int P>
struct RowTiling {
  static constexpr int THREADS = 128;
  static constexpr int ROWS = (P <= 32) ? THREADS : THREADS / Plan<P>::TPR;
};

}  // namespace rdfft
