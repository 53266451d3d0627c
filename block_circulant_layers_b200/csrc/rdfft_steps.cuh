// Per-thread steps of the standalone batched rdFFT / rdIFFT over rows of length P.
//
// A CTA owns ROWS consecutive rows and RowGeo<P>::TPR threads per row. Step k of the
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

// Step K for CTA thread tid = lrow * TPR + v. `rowptr(r)` gives the global row of
// tile row r and `rowok(r)` whether it exists. Orbit passes run the thread's generic
// orbits, then threads 0..NM-1 each run one merged orbit of the CTA's NM.
template <class G, bool INV, int K, int ROWS, typename T, typename RowPtr, typename RowOk>
RD_HD void row_step(float* tile, int lrow, int v, RowPtr rowptr, RowOk rowok) {
  constexpr int NP = G::NPASS;
  static_assert(NP >= 2, "multi-pass rows only");
  constexpr int PASS = INV ? NP - 1 - K : K;
  T* g = rowptr(lrow);
  const bool active = rowok(lrow);
  if constexpr (PASS == 0) {
    if constexpr (!INV) fwd_pass0<G, T>(tile, lrow, v, g, active);
    else inv_pass0<G, T>(tile, lrow, v, g, active);
  } else {
    constexpr int SRC = (INV && K == 0) ? 1 : 0;
    constexpr int DST = (!INV && K == NP - 1) ? 1 : 0;
    generic_pass<G, PASS, INV, SRC, DST>(tile, lrow, v, g, active);
    constexpr int NB = PassShape<G, PASS>::NB;
    const int tid = lrow * G::TPR + v;
    if (tid < ROWS * NB) {
      const int mrow = tid / NB, beta = tid % NB;
      merged_orbit<G, PASS, INV, SRC, DST>(tile, mrow, beta, rowptr(mrow), rowok(mrow));
    }
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

// Rows per CTA: 32 threads (two rows) at p = 512, 128 threads otherwise (measured best
// on B200 among 32..256 threads); 128 rows of one thread each for p <= 32.
template <int P>
struct RowTiling {
  static constexpr int THREADS = P == 512 ? 32 : 128;
  static constexpr int ROWS = (P <= 32) ? THREADS : THREADS / RowGeo<P>::TPR;
};

}  // namespace rdfft
