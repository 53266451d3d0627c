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

// Rows of P <= 32: one thread per row, everything in registers. The row is read from
// src and written to dst (the same row when in place: every element is read first).
template <int P, bool INV, typename T>
RD_HD void row_small(const T* src, T* dst) {
  constexpr int e = ilog2(P);
  float a[P];
  if constexpr (!INV) {
#pragma unroll
    for (int j = 0; j < P; ++j) a[bitrev(j, e)] = ld(src + j);
    stages_contig<2, P, P, 0, false>(a);
#pragma unroll
    for (int j = 0; j < P; ++j) dst[j] = from_f32<T>(a[j]);
  } else {
#pragma unroll
    for (int j = 0; j < P; ++j) a[j] = ld(src + j);
    stages_contig<2, P, P, 0, true>(a);
    constexpr float scale = 1.0f / P;
#pragma unroll
    for (int j = 0; j < P; ++j) dst[bitrev(j, e)] = from_f32<T>(a[j] * scale);
  }
}

// Rows per CTA: 128 threads (8 rows at p = 512, one at p = 4096), measured best on
// B200 among 32..512 threads with the bulk-copy staging (wider CTAs put more rows'
// merged orbits in one warp, narrower ones wait less at barriers); 128 rows of one
// thread each for p <= 32.
template <int P>
struct RowTiling {
  static constexpr int THREADS = 128;
  static constexpr int ROWS = (P <= 32) ? THREADS : THREADS / RowGeo<P>::TPR;
};

// Shared-memory plan of a rows CTA (p >= 64), dynamic: the staging buffer of the
// rows as they are in HBM, the fp32 tile, the mbarrier. A step of pass 0 has the
// TPR lanes of a row read TPR consecutive elements (SEG bytes, at least 16), and the
// RW rows of a warp read at once; staged row r starts at r (RAW_ROW + SEG) +
// 16 (r / RW) bytes. So staged rows are 16-byte aligned for the bulk copies and never
// overlap, the RW rows of a warp read disjoint banks, and consecutive warp groups are
// shifted by one more 16-byte bank group (for the merged orbits, which one warp
// stores for many rows at the same in-row position). 16-bit rows of p = 256 and 512
// take twice that SEG: with TPR*2 bytes, rows r and r + 3 (p = 512) of the merged
// orbits' accesses fall in one bank.
template <int P, typename T>
struct RowSmem {
  static constexpr int ROWS = RowTiling<P>::ROWS;
  static constexpr int TPR = RowGeo<P>::TPR;
  static constexpr int RW = TPR < 32 ? 32 / TPR : 1;
  static constexpr int RAW_ROW = P * (int)sizeof(T);
  static constexpr int SEG1 = TPR * (int)sizeof(T) < 16 ? 16 : TPR * (int)sizeof(T);
  static constexpr int SEG = (sizeof(T) == 2 && (P == 256 || P == 512)) ? 2 * SEG1 : SEG1;
  RD_HD static constexpr int raw_off(int r) { return r * (RAW_ROW + SEG) + 16 * (r / RW); }
  static constexpr int TILE_OFF = raw_off(ROWS - 1) + RAW_ROW;
  static constexpr int MBAR_OFF = TILE_OFF + ((RowGeo<P>::words(ROWS) * 4 + 15) / 16) * 16;
  static constexpr int BYTES = MBAR_OFF + 16;
  static_assert(RAW_ROW % 16 == 0 && SEG % 16 == 0 && TILE_OFF % 16 == 0, "16-byte alignment");
};

}  // namespace rdfft
