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

template <class G, bool INV, int K, int ROWS, typename T>
void emu_steps(float* tile, int64_t row0, int64_t rows, T* data) {
  if constexpr (K < G::NPASS) {
    constexpr int TPR = G::TPR;
    auto rowok = [&](int r) { return row0 + r < rows; };
    auto rowptr = [&](int r) { return data + (row0 + r < rows ? row0 + r : (int64_t)0) * G::P; };
    for (int tid = 0; tid < ROWS * TPR; ++tid)
      row_step<G, INV, K, ROWS, T>(tile, tid / TPR, tid % TPR, rowptr, rowok);
    emu_steps<G, INV, K + 1, ROWS, T>(tile, row0, rows, data);
  }
}

// Emulates the row transform of geometry G with ROWS rows per CTA.
template <class G, int ROWS, bool INV, typename T>
void emu_geo(T* data, int64_t rows) {
  std::vector<float> tile(G::words(ROWS), 0.0f);
  for (int64_t row0 = 0; row0 < rows; row0 += ROWS)
    emu_steps<G, INV, 0, ROWS, T>(tile.data(), row0, rows, data);
}

template <int P, bool INV, typename T>
void emu_rows(T* data, int64_t rows, int ept) {
  if constexpr (P <= 32) {
    for (int64_t r = 0; r < rows; ++r) row_small<P, INV, T>(data + r * P);
  } else {
    if (ept == 0) {
      emu_geo<RowGeo<P>, RowTiling<P>::ROWS, INV, T>(data, rows);
    } else {
      // the layer kernels' geometry: 32 elements per thread, rows of a 128-thread CTA
      using G = Geo<P, kEPT>;
      emu_geo<G, (128 / G::TPR > 0 ? 128 / G::TPR : 1), INV, T>(data, rows);
    }
  }
}

template <typename T>
int emu_t(void* data, int64_t rows, int p, bool inv, int ept) {
  T* d = static_cast<T*>(data);
#define RD_CASE(PP)                                   \
  case PP:                                            \
    if (inv) emu_rows<PP, true, T>(d, rows, ept);     \
    else emu_rows<PP, false, T>(d, rows, ept);        \
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
  if (dtype == 0) return rdfft::emu_t<float>(data, rows, p, inverse != 0, 0);
  return rdfft::emu_t<rdfft::bf16_t>(data, rows, p, inverse != 0, 0);
}

// The same with the layer kernels' row geometry (32 elements per thread).
int rdfft_emulate_layer_rows(void* data, int64_t rows, int p, int dtype, int inverse) {
  if (dtype == 0) return rdfft::emu_t<float>(data, rows, p, inverse != 0, 32);
  return rdfft::emu_t<rdfft::bf16_t>(data, rows, p, inverse != 0, 32);
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
  const int E = p < rdfft::ept_for(p) ? p : rdfft::ept_for(p);
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
