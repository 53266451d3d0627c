// Host emulation of the standalone rdFFT kernels, for the CPU tests.
//
// Runs the very per-thread pass functions of packed_fft.cuh / rdfft_steps.cuh that
// the GPU kernels run, CTA by CTA, with every CTA barrier replaced by a sweep over
// all of the CTA's threads. Compiled by g++ (no CUDA), with floating-point
// contraction off, so its results are what the kernels compute, operation for
// operation. Not part of the product path.
#include <stdint.h>

#include <vector>

#include "layer_policy.h"
#include "rdfft2d_steps.cuh"
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

// Forward orbit passes K.. of the Hartley-form inverse; the last one writes rows to
// global memory with the mirror epilogue.
template <class G, int K, typename T>
void emu_hartley_rest(float* tile, int nr, T* rows) {
  constexpr int TPR = G::TPR;
  constexpr bool LAST = (K == G::NPASS - 1);
  for (int tid = 0; tid < nr * TPR; ++tid) {
    const int r = tid / TPR;
    if constexpr (LAST) generic_pass<G, K, false, 0, 1, T, 1>(tile, r, tid % TPR, rows + (int64_t)r * G::P, true);
    else generic_pass<G, K, false, 0, 0, T>(tile, r, tid % TPR, (T*)nullptr, false);
  }
  constexpr int NB = PassShape<G, K>::NB;
  for (int mu = 0; mu < nr * NB; ++mu) {
    const int r = mu / NB;
    if constexpr (LAST) merged_orbit<G, K, false, 0, 1, T, 1>(tile, r, mu % NB, rows + (int64_t)r * G::P, true);
    else merged_orbit<G, K, false, 0, 0, T>(tile, r, mu % NB, (T*)nullptr, false);
  }
  if constexpr (!LAST) emu_hartley_rest<G, K + 1, T>(tile, nr, rows);
}

template <class G, int W, int NT, int K>
void emu_col_passes(float* tile) {
  if constexpr (K < G::NPASS) {
    for (int tid = 0; tid < NT; ++tid) cols_orbit_pass<G, K>(tile, W, tid, NT);
    emu_col_passes<G, W, NT, K + 1>(tile);
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
    for (int64_t r = 0; r < rows; ++r) row_small<P, INV, T>(data + r * P, data + r * P);
  } else {
    if (ept == 0) {
      emu_geo<RowGeo<P>, RowTiling<P>::ROWS, INV, T>(data, rows);
    } else {
      // the layer kernels' geometry: 32 elements per thread, rows of a 128-thread CTA
      using G = LayerGeo<P>;
      emu_geo<G, (128 / G::TPR > 0 ? 128 / G::TPR : 1), INV, T>(data, rows);
    }
  }
}

// The layer kernels' Hartley-form inverse of packed rows: mirror the spectrum (as
// their contraction epilogue does), pass 0 from the tile, forward orbit passes, last
// pass to global with the mirror epilogue. ROWS rows per emulated CTA.
template <int P, typename T>
void emu_hartley_inverse(T* data, int64_t rows) {
  using G = LayerGeo<P>;
  constexpr int TPR = G::TPR;
  constexpr int ROWS = 128 / TPR > 0 ? 128 / TPR : 1;
  std::vector<float> tile(G::words(ROWS), 0.0f);
  std::vector<float> regs((size_t)ROWS * TPR * G::E);
  for (int64_t row0 = 0; row0 < rows; row0 += ROWS) {
    const int nr = (int)((rows - row0) < ROWS ? (rows - row0) : ROWS);
    for (int r = 0; r < nr; ++r) {
      const T* y = data + (row0 + r) * P;
      float* trow = tile.data() + G::row_base(r);
      trow[G::at(0)] = to_f32(y[0]);
      trow[G::at(P / 2)] = to_f32(y[P / 2]);
      for (int k = 1; k < P / 2; ++k) {
        const float re = to_f32(y[k]), im = to_f32(y[P - k]);
        trow[G::at(k)] = re - im;
        trow[G::at(P - k)] = re + im;
      }
    }
    // pass 0: every thread gathers, then every thread scatters
    for (int tid = 0; tid < nr * TPR; ++tid) {
      float(&a)[G::E] = *reinterpret_cast<float(*)[G::E]>(&regs[(size_t)tid * G::E]);
      fwd_pass0_load_tile<G>(a, tid % TPR, tile.data() + G::row_base(tid / TPR));
    }
    for (int tid = 0; tid < nr * TPR; ++tid) {
      float(&a)[G::E] = *reinterpret_cast<float(*)[G::E]>(&regs[(size_t)tid * G::E]);
      fwd_pass0_finish<G>(a, tid % TPR, tile.data() + G::row_base(tid / TPR));
    }
    emu_hartley_rest<G, 1, T>(tile.data(), nr, data + row0 * P);
  }
}

// Column half of the 2-D transform, CTA by CTA as k_cols / k_cols_small run it.
template <int R, bool INV, typename T>
void emu_cols(T* data, int64_t images, int C) {
  if constexpr (R <= 32) {
    for (int64_t img = 0; img < images; ++img)
      for (int k = 0; k <= C / 2; ++k) col_small<R, INV, T>(data + img * (int64_t)R * C, C, k);
  } else {
    using CT = ColTiling<R>;
    constexpr int W = CT::W, NT = CT::NT;
    using G = ColGeo<R, W>;
    constexpr int TPR = G::TPR;
    std::vector<float> tile(G::words(W), 0.0f);
    std::vector<float> regs((size_t)W * TPR * G::E);
    const int ngroups = col_groups(C, W / 2);
    for (int64_t img = 0; img < images; ++img) {
      T* base = data + img * (int64_t)R * C;
      for (int grp = 0; grp < ngroups; ++grp) {
        const int k0 = grp * (W / 2);
        float* t = tile.data();
        for (int tid = 0; tid < NT; ++tid) {
          if (INV) cols_load_unpair<G, W, NT, T>(t, base, C, k0, tid);
          else cols_load<G, W, NT, T>(t, base, C, k0, tid);
        }
        for (int i = 0; i < W * TPR; ++i) {
          float(&a)[G::E] = *reinterpret_cast<float(*)[G::E]>(&regs[(size_t)i * G::E]);
          fwd_pass0_load_tile<G>(a, i % TPR, t + G::row_base(i / TPR));
        }
        for (int i = 0; i < W * TPR; ++i) {
          float(&a)[G::E] = *reinterpret_cast<float(*)[G::E]>(&regs[(size_t)i * G::E]);
          fwd_pass0_finish<G>(a, i % TPR, t + G::row_base(i / TPR));
        }
        emu_col_passes<G, W, NT, 1>(t);
        for (int tid = 0; tid < NT; ++tid) {
          if (INV) cols_store_inv<G, W, NT, T>(t, base, C, k0, tid);
          else cols_store_fwd<G, W, NT, T>(t, base, C, k0, tid);
        }
      }
    }
  }
}

template <bool INV, typename T>
int emu_cols_t(T* data, int64_t images, int R, int C) {
#define RD_CCASE(RR) \
  case RR: emu_cols<RR, INV, T>(data, images, C); return 0;
  switch (R) {
    RD_CCASE(2) RD_CCASE(4) RD_CCASE(8) RD_CCASE(16) RD_CCASE(32) RD_CCASE(64) RD_CCASE(128)
    RD_CCASE(256) RD_CCASE(512) RD_CCASE(1024) RD_CCASE(2048) RD_CCASE(4096)
    default: return 1;
  }
#undef RD_CCASE
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

template <class SM, int P>
static void plan_of(int64_t* out) {
  out[0] = SM::ROWS;
  out[1] = SM::RAW_ROW;
  out[2] = SM::TILE_OFF;
  out[3] = SM::MBAR_OFF;
  out[4] = SM::BYTES;
  out[5] = rdfft::RowGeo<P>::words(SM::ROWS);
  out[6] = SM::TPR;
  for (int r = 0; r < SM::ROWS; ++r) out[7 + r] = SM::raw_off(r);
}

extern "C" {

// In-place emulated rdfft_fwd (inverse = 0) or rdfft_inv (inverse = 1) on host
// memory; dtype 0 = fp32, 1 = bf16 bits. Returns 0, or 1 for an unsupported p.
int rdfft_emulate(void* data, int64_t rows, int p, int dtype, int inverse) {
  if (dtype == 0) return rdfft::emu_t<float>(data, rows, p, inverse != 0, 0);
  return rdfft::emu_t<rdfft::bf16_t>(data, rows, p, inverse != 0, 0);
}

// The layer kernels' Hartley-form inverse (mirrored spectrum, forward transform,
// mirror epilogue), in place on host rows; returns 1 for an unsupported p.
int rdfft_emulate_hartley_inverse(void* data, int64_t rows, int p, int dtype) {
#define RD_HCASE(PP)                                                                        \
  case PP:                                                                                  \
    if (dtype == 0) rdfft::emu_hartley_inverse<PP, float>(static_cast<float*>(data), rows); \
    else rdfft::emu_hartley_inverse<PP, rdfft::bf16_t>(static_cast<rdfft::bf16_t*>(data), rows); \
    return 0;
  switch (p) {
    RD_HCASE(64) RD_HCASE(128) RD_HCASE(256) RD_HCASE(512) RD_HCASE(1024) RD_HCASE(2048) RD_HCASE(4096)
    default: return 1;
  }
#undef RD_HCASE
}

// The same with the layer kernels' row geometry (32 elements per thread).
int rdfft_emulate_layer_rows(void* data, int64_t rows, int p, int dtype, int inverse) {
  if (dtype == 0) return rdfft::emu_t<float>(data, rows, p, inverse != 0, 32);
  return rdfft::emu_t<rdfft::bf16_t>(data, rows, p, inverse != 0, 32);
}

// Emulated rdfft2_fwd / rdfft2_inv on host images (row kernel, then column kernel,
// or the reverse); returns 1 for an unsupported R or C.
int rdfft2_emulate(void* data, int64_t images, int R, int C, int dtype, int inverse) {
  const int64_t rows = images * R;
  if (dtype == 0) {
    float* d = static_cast<float*>(data);
    if (!inverse) {
      if (rdfft::emu_t<float>(d, rows, C, false, 0)) return 1;
      return rdfft::emu_cols_t<false>(d, images, R, C);
    }
    if (rdfft::emu_cols_t<true>(d, images, R, C)) return 1;
    return rdfft::emu_t<float>(d, rows, C, true, 0);
  }
  rdfft::bf16_t* d = static_cast<rdfft::bf16_t*>(data);
  if (!inverse) {
    if (rdfft::emu_t<rdfft::bf16_t>(d, rows, C, false, 0)) return 1;
    return rdfft::emu_cols_t<false>(d, images, R, C);
  }
  if (rdfft::emu_cols_t<true>(d, images, R, C)) return 1;
  return rdfft::emu_t<rdfft::bf16_t>(d, rows, C, true, 0);
}

// Shared-memory plan of the rows kernel for row length p >= 64 and dtype: out[0..6] =
// rows per CTA, bytes per staged row, tile offset, mbarrier offset, total bytes, tile
// words, threads per row; out[7 + r] = byte offset of staged row r (out must hold
// 7 + rows per CTA values). Returns 1 for an unsupported p.
int rdfft_row_smem_plan(int p, int dtype, int64_t* out) {
#define RD_PCASE(PP)                                                                   \
  case PP:                                                                             \
    if (dtype == 0) plan_of<rdfft::RowSmem<PP, float>, PP>(out);                       \
    else plan_of<rdfft::RowSmem<PP, rdfft::bf16_t>, PP>(out);                          \
    return 0;
  switch (p) {
    RD_PCASE(64) RD_PCASE(128) RD_PCASE(256) RD_PCASE(512) RD_PCASE(1024) RD_PCASE(2048) RD_PCASE(4096)
    default: return 1;
  }
#undef RD_PCASE
}

// Tile geometry of the rows kernel for row length p: out[0] = S (one pad word per 2^S
// elements), out[1] = rows per CTA, out[2 + r] = word offset of tile row r.
int rdfft_row_tile_plan(int p, int64_t* out) {
#define RD_TCASE(PP)                                                                   \
  case PP: {                                                                           \
    using G = rdfft::RowGeo<PP>;                                                       \
    constexpr int R = rdfft::RowTiling<PP>::ROWS;                                      \
    out[0] = G::S;                                                                     \
    out[1] = R;                                                                        \
    for (int r = 0; r < R; ++r) out[2 + r] = G::row_base(r);                           \
    return 0;                                                                          \
  }
  switch (p) {
    RD_TCASE(64) RD_TCASE(128) RD_TCASE(256) RD_TCASE(512) RD_TCASE(1024) RD_TCASE(2048) RD_TCASE(4096)
    default: return 1;
  }
#undef RD_TCASE
}

// Tile geometry of the layer kernels for row length p: out[0] = S, out[1 + r] = word
// offset of tile row r for r < rows.
int rdfft_layer_tile_plan(int p, int rows, int64_t* out) {
#define RD_LCASE(PP)                                                                   \
  case PP: {                                                                           \
    using G = rdfft::LayerGeo<PP>;                                                     \
    out[0] = G::S;                                                                     \
    for (int r = 0; r < rows; ++r) out[1 + r] = G::row_base(r);                        \
    return 0;                                                                          \
  }
  switch (p) {
    RD_LCASE(64) RD_LCASE(128) RD_LCASE(256) RD_LCASE(512) RD_LCASE(1024) RD_LCASE(2048) RD_LCASE(4096)
    default: return 1;
  }
#undef RD_LCASE
}

// The layer launchers' shape rules (layer_policy.h), for the CPU tests.
int rdfft_layer_qi(int q, int qi_max, int64_t gx, int n_sm) { return rdfft::layer_qi(q, qi_max, gx, n_sm); }
int rdfft_layer_qj(int q, int hb, int64_t max_slots, int64_t ntiles, int n_sm) {
  return rdfft::layer_qj(q, hb, max_slots, ntiles, n_sm);
}
int rdfft_layer_x_tokens(int64_t B, int q, int qi_max, int n_sm, int tt_max) {
  return rdfft::layer_x_tokens(B, q, qi_max, n_sm, tt_max);
}
int rdfft_layer_fused_small_tiles(int64_t B, int tt_small, int njgroups, int n_sm) {
  return rdfft::layer_fused_small_tiles(B, tt_small, njgroups, n_sm) ? 1 : 0;
}
int rdfft_layer_gc_half_tiles(int64_t B, int tt, int q, int hb, int64_t max_slots, int n_sm) {
  return rdfft::layer_gc_half_tiles(B, tt, q, hb, max_slots, n_sm) ? 1 : 0;
}
int rdfft_layer_gc_slices(int njgroups, int64_t ntiles, int n_sm, int64_t* tiles_per) {
  return rdfft::layer_gc_slices(njgroups, ntiles, n_sm, tiles_per);
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
