// Host emulation of the standalone rdFFT kernels, for the CPU tests.
//
// Runs the very per-thread pass functions of packed_fft.cuh / rdfft_steps.cuh that
// the GPU kernels run, CTA by CTA, with every CTA barrier replaced by a sweep over
// all of the CTA's threads. Compiled by g++ (no CUDA), with floating-point
// contraction off, so its results are what the kernels compute, operation for
// operation. Not part of the product path.
#include <stdint.h>

#include <vector>

#include "rdfft_steps.cuh"

namespace rdfft {
namespace {

template <int P, bool INV, int K, typename T>
void emu_steps(float* tile, int rows_in_cta, int64_t row0, int64_t rows, T* data) {
  if constexpr (K < Plan<P>::NPASS) {
    constexpr int TPR = Plan<P>::TPR;
    for (int tid = 0; tid < rows_in_cta * TPR; ++tid) {
      const int lrow = tid / TPR, v = tid % TPR;
      const int64_t row = row0 + lrow;
      const bool active = row < rows;
      T* g = data + (active ? row : 0) * P;
      row_step<P, INV, K, T>(tile, lrow, v, g, active);
    }
    emu_steps<P, INV, K + 1, T>(tile, rows_in_cta, row0, rows, data);
  }
}

template <int P, bool INV, typename T>
void emu_rows(T* data, int64_t rows) {
  constexpr int ROWS = RowTiling<P>::ROWS;
  if constexpr (P <= 32) {
    for (int64_t r = 0; r < rows; ++r) row_small<P, INV, T>(data + r * P);
  } else {
    std::vector<float> tile(ROWS * P, 0.0f);
    for (int64_t row0 = 0; row0 < rows; row0 += ROWS)
      emu_steps<P, INV, 0, T>(tile.data(), ROWS, row0, rows, data);
  }
}

template <typename T>
int emu_t(void* data, int64_t rows, int p, bool inv) {
  T* d = static_cast<T*>(data);
#define RD_CASE(PP)                                   \
  case PP:                                            \
    if (inv) emu_rows<PP, true, T>(d, rows);          \
    else emu_rows<PP, false, T>(d, rows);             \
    return 0;
  switch (p) {
    RD_CASE(2) RD_CASE(4) RD_CASE(8) RD_CASE(16) RD_CASE(32) RD_CASE(64) RD_CASE(128)
    RD_CASE(256) RD_CASE(512) RD_CASE(1024) RD_CASE(2048) RD_CASE(4096)
    default: return 1;
  }
#undef RD_CASE
}

}  // namespace
}  // namespace rdfft

extern "C" {

// In-place emulated rdfft_fwd (inverse = 0) or rdfft_inv (inverse = 1) on host
// memory; dtype 0 = fp32, 1 = bf16 bits. Returns 0, or 1 for an unsupported p.
int rdfft_emulate(void* data, int64_t rows, int p, int dtype, int inverse) {
  if (dtype == 0) return rdfft::emu_t<float>(data, rows, p, inverse != 0);
  return rdfft::emu_t<rdfft::bf16_t>(data, rows, p, inverse != 0);
}

// Positions of the first n elements of the generic orbit with residue r of a pass
// that starts at block size H (the kernels' orbit_pos), for the index-model test.
void rdfft_orbit_positions(int H, int r, int n, int* out) {
  for (int i = 0; i < n; ++i) out[i] = rdfft::orbit_pos(H, i, r);
}

// Pass plan of the kernels for row length p: fills s0[i], s1[i] (stages s0+1..s1 of
// pass i) and returns the number of passes.
int rdfft_plan(int p, int* s0, int* s1) {
  int L = 0;
  while ((1 << L) < p) ++L;
  const int E = p < rdfft::kEPT ? p : rdfft::kEPT;
  int e = 0;
  while ((1 << e) < E) ++e;
  int n = 0;
  s0[n] = 0;
  s1[n] = e;
  ++n;
  int cur = e;
  while (cur < L) {
    const int nxt = cur + e - 1 < L ? cur + e - 1 : L;
    s0[n] = cur;
    s1[n] = nxt;
    ++n;
    cur = nxt;
  }
  return n;
}

}  // extern "C"
