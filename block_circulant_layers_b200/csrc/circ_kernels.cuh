// Block-circulant linear layer kernels (sm_100a): forward, grad_x and grad_c.
//
// "Memory-Efficient Training with In-Place FFT Implementation", paper-notes page,
// "Circulant matrix training adaptation": y = IFFT(FFT(c) (.) FFT(x)) per circulant
// block; the product of conjugate-symmetric spectra stays conjugate symmetric, so
// every spectrum lives in the packed layout and every transform is the in-place
// rdFFT of packed_fft.cuh. With D = q p:
//     forward : y_i      = IFFT( sum_j  C_ij (.) X_j )
//     grad_x  : grad_x_j = IFFT( sum_i conj(C_ij) (.) G_i )
//     grad_c  : grad_c_ij = IFFT( sum_b G_i^b (.) conj(X_j^b) )
// where C = c_hat (packed, fp32), X = rdFFT(x), G = rdFFT(g) per block.
//
// Kernel shapes (ours):
//  * k_circ_x (forward and grad_x): a CTA owns TT tokens and a group of QI output
//    blocks. It rdFFTs the TT*q input rows straight from HBM into an fp32 shared
//    tile, contracts them against c_hat (read through L2) with CUDA-core FMA into
//    registers, writes the output spectra over the tile and rdIFFTs them straight
//    back to HBM. HBM traffic: the input, c_hat, the output.
//  * k_circ_gc (grad_c): a persistent CTA owns a group of QJ input blocks j and a
//    slice of the tokens; it keeps its part of the packed cross-spectrum
//    S_ij = sum_b G_i conj(X_j) in registers across all its token tiles and adds it
//    into grad_c once (fp32 red.add into a grad_c zeroed by k_zero_f4; a plain store
//    when a single token slice covers all tokens, and grad_c then needs no zeroing).
//    grad_c is rdIFFT'd in place after, so the output buffer is the only global
//    storage used. In the deterministic mode (circ_bwd_deterministic) each slice
//    instead stores its sums into its own q x q x p part of a caller workspace, and
//    the slices are summed in a fixed order (k_sum_slices, circ_launch.cu).
//  * For some shapes circ_bwd with both gradients runs one kernel instead of k_circ_x
//    (grad_x) and k_circ_gc (circ_bwd_fused.cu).
#pragma once

#include <cuda_runtime.h>

#include "internal.h"
#include "layer_policy.h"
#include "packed_fft.cuh"
#include "pdl.cuh"

namespace rdfft {

// The layer kernels' tiles use LayerGeo (packed_fft.cuh): 32 elements per thread,
// three passes at p >= 1024, since their registers are shared with the contraction's
// accumulators.

// ------------------------------------------------------------- tile row passes
// Orbit pass K (tile -> tile) over NR rows of the tile, the r-th being tile row rowmap(r)
// (consecutive rows, [0, NR), for tile_orbit_pass): every thread runs the generic orbits of
// its rows, then the NR * NB merged orbits are spread one per thread. Rows that share a
// warp must map to consecutive tile rows in aligned groups of RW.
template <int P, int NT, int K, bool INV, typename T, typename RowMap>
__device__ __forceinline__ void tile_orbit_pass_mapped(float* tile, int NR, RowMap rowmap) {
  using G = LayerGeo<P>;
  constexpr int TPR = G::TPR, RPR = NT / TPR;
  constexpr int NB = PassShape<G, K>::NB;
  const int v = threadIdx.x % TPR;
  for (int r = threadIdx.x / TPR; r < NR; r += RPR)
    generic_pass<G, K, INV, 0, 0>(tile, rowmap(r), v, (T*)nullptr, false);
  for (int mu = threadIdx.x; mu < NR * NB; mu += NT)
    merged_orbit<G, K, INV, 0, 0>(tile, rowmap(mu / NB), mu % NB, (T*)nullptr, false);
}

template <int P, int NT, int K, bool INV, typename T>
__device__ __forceinline__ void tile_orbit_pass(float* tile, int NR) {
  tile_orbit_pass_mapped<P, NT, K, INV, T>(tile, NR, [](int r) { return r; });
}

// Forward rdFFT of tile rows [0, NR): row r reads its input from src(r) (nullptr
// means a row of zeros), the spectrum stays in the tile.
template <int P, int NT, typename T, int K, typename SrcFn>
__device__ __forceinline__ void fft_rows_rest(float* tile, int NR, SrcFn src) {
  if constexpr (K < LayerGeo<P>::NPASS) {
    __syncthreads();
    tile_orbit_pass<P, NT, K, false, T>(tile, NR);
    fft_rows_rest<P, NT, T, K + 1>(tile, NR, src);
  }
}

// Passes K.. of the forward rdFFT of NR rows mapped to tile rows by rowmap (see
// tile_orbit_pass_mapped); pass 0 is the caller's.
template <int P, int NT, typename T, int K, typename RowMap>
__device__ __forceinline__ void fft_rows_rest_mapped(float* tile, int NR, RowMap rowmap) {
  if constexpr (K < LayerGeo<P>::NPASS) {
    __syncthreads();
    tile_orbit_pass_mapped<P, NT, K, false, T>(tile, NR, rowmap);
    fft_rows_rest_mapped<P, NT, T, K + 1>(tile, NR, rowmap);
  }
}

template <int P, int NT, typename T, typename SrcFn>
__device__ __forceinline__ void fft_rows(float* tile, int NR, SrcFn src) {
  constexpr int TPR = LayerGeo<P>::TPR, RPR = NT / TPR;
  static_assert(NT % TPR == 0, "threads per CTA must cover whole rows");
  const int v = threadIdx.x % TPR;
  for (int r = threadIdx.x / TPR; r < NR; r += RPR) {
    const T* g = src(r);
    fwd_pass0<LayerGeo<P>, T>(tile, r, v, g, g != nullptr);
  }
  fft_rows_rest<P, NT, T, 1>(tile, NR, src);
}

// Last pass of a forward transform over tile rows [0, NR), written to global rows
// dst(r) (nullptr: dropped) with the mirror epilogue: the Hartley form of the inverse.
template <int P, int NT, typename T, typename DstFn>
__device__ __forceinline__ void last_pass_mirror_to_global(float* tile, int NR, DstFn dst) {
  using G = LayerGeo<P>;
  constexpr int K = G::NPASS - 1;
  constexpr int TPR = G::TPR, RPR = NT / TPR;
  static_assert(PassShape<G, K>::NB == 1, "the last pass covers whole rows");
  const int v = threadIdx.x % TPR;
  for (int r = threadIdx.x / TPR; r < NR; r += RPR) {
    T* g = dst(r);
    generic_pass<G, K, false, 0, 1, T, 1>(tile, r, v, g, g != nullptr);
  }
  for (int r = threadIdx.x; r < NR; r += NT) {
    T* g = dst(r);
    merged_orbit<G, K, false, 0, 1, T, 1>(tile, r, 0, g, g != nullptr);
  }
}

template <int P, int NT, typename T, int K, typename DstFn>
__device__ __forceinline__ void fwd_tile_passes_then_mirror(float* tile, int NR, DstFn dst) {
  using G = LayerGeo<P>;
  __syncthreads();
  if constexpr (K < G::NPASS - 1) {
    tile_orbit_pass<P, NT, K, false, T>(tile, NR);
    fwd_tile_passes_then_mirror<P, NT, T, K + 1>(tile, NR, dst);
  } else {
    last_pass_mirror_to_global<P, NT, T>(tile, NR, dst);
  }
}

// Inverse rdFFT of tile rows [0, NR) whose spectra were stored in mirrored form
// (slot k = Re - Im, slot p-k = Re + Im of bin k; the caller has synchronised the
// tile): by rdIFFT = (1/p) M rdFFT M, with M that mirror, this is a forward transform
// of the tile rows with the mirror and the 1/p applied as the last pass writes row r
// to dst(r). The forward butterflies cost 6 FP instructions per group against the
// inverse's 8.
template <int P, int NT, typename T, typename DstFn>
__device__ __forceinline__ void ifft_rows_mirrored(float* tile, int NR, DstFn dst) {
  using G = LayerGeo<P>;
  constexpr int TPR = G::TPR, RPR = NT / TPR;
  const int v = threadIdx.x % TPR;
  // pass 0 in place in the tile: gather every row of a round, barrier, scatter
  for (int r0 = 0; r0 < NR; r0 += RPR) {
    const int r = r0 + threadIdx.x / TPR;
    float a[G::E];
    if (r < NR) fwd_pass0_load_tile<G>(a, v, tile + G::row_base(r));
    __syncthreads();
    if (r < NR) fwd_pass0_finish<G>(a, v, tile + G::row_base(r));
  }
  fwd_tile_passes_then_mirror<P, NT, T, 1>(tile, NR, dst);
}

// Packed-bin view of a row: bin 0 is the real pair (slot 0, slot p/2); bin k > 0 is
// the complex value (slot k, slot p - k).
template <int P>
__device__ __forceinline__ int bin_im_slot(int k) { return k == 0 ? P / 2 : P - k; }

// --------------------------------------------------------------- forward, grad_x
// BWDX = false: in = x, out = y; the CTA's QI output blocks are i, summed over j.
// BWDX = true : in = g, out = grad_x; the CTA's QI output blocks are j, summed over i,
//               against conj(c_hat).
template <int P, typename T, int NT, int TT, int NS, bool BWDX>
// 256-thread CTAs are declared for two per SM (<= 128 registers), 512-thread ones for one
__global__ void __launch_bounds__(NT, NT >= 512 ? 1 : (NT >= 256 ? 2 : 1))
k_circ_x(const T* __restrict__ in, const float* __restrict__ chat, T* __restrict__ out,
         int64_t B, int q, int QI) {
  extern __shared__ float tile[];
  const int D = q * P;
  const int64_t tok0 = (int64_t)blockIdx.x * TT;
  const int ntok = (int)((B - tok0) < TT ? (B - tok0) : TT);
  const int o0 = blockIdx.y * QI;            // first output block of this CTA
  griddep_wait();                            // earlier work in the stream (c_hat, the input) is done

  // 1. rdFFT of the TT*q input rows (row r = t*q + b)
  fft_rows<P, NT, T>(tile, TT * q, [&](int r) -> const T* {
    const int t = r / q, b = r - t * q;
    return t < ntok ? in + (tok0 + t) * (int64_t)D + (int64_t)b * P : nullptr;
  });
  __syncthreads();

  // 2.-3. contraction and output spectra. When all of a thread's slots share one bin
  // (NT a multiple of p/2, i.e. p <= 512), slot pairs run on packed fp32 pairs; with a
  // bin per slot (p >= 1024) pairing saves no loads and costs registers, so it is scalar.
  if constexpr (NT % (P / 2) == 0 && NS >= 2) {
    // 2. contraction: thread slot s covers bin k = tid % (p/2) and output block
    // ol = w + G s (w = tid / (p/2), G = NT / (p/2) slot groups) of all TT tokens. Slots
    // are taken in pairs (s, s + 1) on packed fp32 pairs: each pair accumulates two output
    // blocks of one token in one FFMA2 per term.
    constexpr int HB = P / 2;
    constexpr int G = NT / HB;
    constexpr int NP = (NS + 1) / 2;              // slot pairs (an odd last slot pairs with a zero slot)
    const int w = threadIdx.x / HB, k = threadIdx.x % HB;
    const int kr = LayerGeo<P>::at(k), ki = LayerGeo<P>::at(bin_im_slot<P>(k));
    f2 acc_r[NP][TT], acc_i[NP][TT];
  #pragma unroll
    for (int u = 0; u < NP; ++u)
  #pragma unroll
      for (int t = 0; t < TT; ++t) acc_r[u][t] = acc_i[u][t] = f2_bc(0.0f);

    auto load_c = [&](int j, float (&cr)[2 * NP], float (&ci)[2 * NP]) {
  #pragma unroll
      for (int s = 0; s < 2 * NP; ++s) {
        const int ol = w + G * s;
        if (s < NS && ol < QI) {
          const int ob = o0 + ol;
          const float* crow = chat + (int64_t)(BWDX ? (j * q + ob) : (ob * q + j)) * P;
          cr[s] = __ldg(crow + k);
          ci[s] = __ldg(crow + bin_im_slot<P>(k));
        } else {
          cr[s] = ci[s] = 0.0f;
        }
      }
    };
    // no guard on the slot here: a slot beyond the CTA's blocks has c = 0 (load_c), so
    // its accumulators stay 0 and are never stored; all slots share the loads of X.
    // The packed product as acc_r += cr xa + ci xb, acc_i += cr xc + ci xd, with the
    // token's x terms chosen once for all slots:
    //   forward, complex bin : xa = xr, xb = -xi, xc = xi, xd =  xr   (c x)
    //   grad_x,  complex bin : xa = xr, xb =  xi, xc = xi, xd = -xr   (conj(c) x)
    //   bin 0 (real pair)    : xa = xr, xb =   0, xc =  0, xd =  xi   (component-wise)
    // bin0 = false (a warp with no bin-0 lane) drops the bin-0 selects.
    auto contract = [&](bool bin0, int j, const float (&cr_c)[2 * NP], const float (&ci_c)[2 * NP]) {
      f2 cr[NP], ci[NP];
  #pragma unroll
      for (int u = 0; u < NP; ++u) {
        cr[u] = f2_mk(cr_c[2 * u], cr_c[2 * u + 1]);
        ci[u] = f2_mk(ci_c[2 * u], ci_c[2 * u + 1]);
      }
      const bool z = bin0 && (k == 0);
  #pragma unroll
      for (int t = 0; t < TT; ++t) {
        const int rb = LayerGeo<P>::row_base(t * q + j);
        const float vr = tile[rb + kr], vi = tile[rb + ki];
        const f2 xa = f2_bc(vr);
        const f2 xb = f2_bc(z ? 0.0f : (BWDX ? vi : -vi));
        const f2 xc = f2_bc(z ? 0.0f : vi);
        const f2 xd = f2_bc(z ? vi : (BWDX ? -vr : vr));
  #pragma unroll
        for (int u = 0; u < NP; ++u) {
          acc_r[u][t] = f2_fma(cr[u], xa, f2_fma(ci[u], xb, acc_r[u][t]));
          acc_i[u][t] = f2_fma(cr[u], xc, f2_fma(ci[u], xd, acc_i[u][t]));
        }
      }
    };
    // a block's contraction is too short to hide an L2 round trip, so the c_hat of KB
    // summed blocks is requested at once (at most 32 floats), then contracted
    constexpr int KB = 8 / NP < 8 ? 8 / NP : 8;
    auto contract_all = [&](bool bin0) {
      if constexpr (KB > 1) {
        for (int j0 = 0; j0 < q; j0 += KB) {
          float crb[KB][2 * NP], cib[KB][2 * NP];
  #pragma unroll
          for (int d = 0; d < KB; ++d)
            if (j0 + d < q) load_c(j0 + d, crb[d], cib[d]);
  #pragma unroll
          for (int d = 0; d < KB; ++d)
            if (j0 + d < q) contract(bin0, j0 + d, crb[d], cib[d]);
        }
      } else {
        // c_hat of the summed block j + 1 is loaded while block j is contracted
        float cr_n[2 * NP], ci_n[2 * NP];
        load_c(0, cr_n, ci_n);
        for (int j = 0; j < q; ++j) {             // j: summed block (input j for fwd, output i for grad_x)
          float cr_c[2 * NP], ci_c[2 * NP];
  #pragma unroll
          for (int sl = 0; sl < 2 * NP; ++sl) {
            cr_c[sl] = cr_n[sl];
            ci_c[sl] = ci_n[sl];
          }
          if (j + 1 < q) load_c(j + 1, cr_n, ci_n);
          contract(bin0, j, cr_c, ci_c);
        }
      }
    };
    // a warp holds bin 0 when its first lane does (p/2 >= 32); a warp-uniform branch, so
    // each side is specialised
    if ((threadIdx.x & ~31u) % HB == 0) contract_all(true);
    else contract_all(false);
    __syncthreads();

    // 3. output spectra over the tile: row t*QI + ol
  #pragma unroll
    for (int s = 0; s < NS; ++s) {
      const int ol = w + G * s;
      if (ol < QI) {
  #pragma unroll
        for (int t = 0; t < TT; ++t) {
          // stored mirrored (slot k = Re - Im, slot p-k = Re + Im) for the Hartley-form
          // inverse below; bin 0 keeps its real pair
          const float ar = (s & 1) ? acc_r[s / 2][t].y : acc_r[s / 2][t].x;
          const float ai = (s & 1) ? acc_i[s / 2][t].y : acc_i[s / 2][t].x;
          const int rb = LayerGeo<P>::row_base(t * QI + ol);
          tile[rb + kr] = k == 0 ? ar : ar - ai;
          tile[rb + ki] = k == 0 ? ai : ar + ai;
        }
      }
    }
    __syncthreads();

  } else {
    // 2. contraction: thread slot s covers bin k and output block ol of all TT tokens
    constexpr int HB = P / 2;
    float acc_r[NS][TT], acc_i[NS][TT];
  #pragma unroll
    for (int s = 0; s < NS; ++s)
  #pragma unroll
      for (int t = 0; t < TT; ++t) acc_r[s][t] = acc_i[s][t] = 0.0f;

    // c_hat of the summed block j + 1 is loaded (through L2) while block j is
    // contracted, so the L2 latency overlaps the FMA work.
    float cr_n[NS], ci_n[NS];
    auto load_c = [&](int j, float (&cr)[NS], float (&ci)[NS]) {
  #pragma unroll
      for (int s = 0; s < NS; ++s) {
        const int pi = threadIdx.x + NT * s;
        const int ol = pi / HB, k = pi % HB;
        if (ol < QI) {
          const int ob = o0 + ol;
          const float* crow = chat + (int64_t)(BWDX ? (j * q + ob) : (ob * q + j)) * P;
          cr[s] = __ldg(crow + k);
          ci[s] = __ldg(crow + bin_im_slot<P>(k));
        } else {
          cr[s] = ci[s] = 0.0f;
        }
      }
    };
    // no guard on the slot here: a slot beyond the CTA's blocks has c = 0 (load_c), so
    // its accumulators stay 0 and are never stored; without a branch, slots that share
    // a bin (all of them when NT >= p/2) share the loads of X.
    auto contract = [&](int j, const float (&cr_c)[NS], const float (&ci_c)[NS]) {
  #pragma unroll
      for (int t = 0; t < TT; ++t) {
        const int rb = LayerGeo<P>::row_base(t * q + j);
  #pragma unroll
        for (int s = 0; s < NS; ++s) {
          const int k = (threadIdx.x + NT * s) % HB;
          const float cr = cr_c[s], ci = ci_c[s];
          // packed product: bin 0 multiplies the real pair component-wise, other bins
          // are complex products (conjugated c for grad_x)
          const bool z = (k == 0);
          const float a2 = z ? 0.0f : (BWDX ? ci : -ci);
          const float a3 = z ? ci : cr;
          const float a4 = z ? 0.0f : (BWDX ? -ci : ci);
          const float xr = tile[rb + LayerGeo<P>::at(k)];
          const float xi = tile[rb + LayerGeo<P>::at(bin_im_slot<P>(k))];
          acc_r[s][t] = fmaf(cr, xr, fmaf(a2, xi, acc_r[s][t]));
          acc_i[s][t] = fmaf(a3, xi, fmaf(a4, xr, acc_i[s][t]));
        }
      }
    };
    // c_hat of KB summed blocks requested at once (at most 32 floats), then contracted;
    // the 128-thread multi-token shapes (p >= 1024) are register-heavy and keep one
    // block ahead
    constexpr int KB = (P <= 512 || TT == 1) ? (16 / NS < 8 ? 16 / NS : 8) : 1;
    if constexpr (KB > 1) {
      for (int j0 = 0; j0 < q; j0 += KB) {
        float crb[KB][NS], cib[KB][NS];
  #pragma unroll
        for (int d = 0; d < KB; ++d)
          if (j0 + d < q) load_c(j0 + d, crb[d], cib[d]);
  #pragma unroll
        for (int d = 0; d < KB; ++d)
          if (j0 + d < q) contract(j0 + d, crb[d], cib[d]);
      }
    } else {
      load_c(0, cr_n, ci_n);
      for (int j = 0; j < q; ++j) {               // j: summed block (input j for fwd, output i for grad_x)
        float cr_c[NS], ci_c[NS];
  #pragma unroll
        for (int s = 0; s < NS; ++s) {
          cr_c[s] = cr_n[s];
          ci_c[s] = ci_n[s];
        }
        if (j + 1 < q) load_c(j + 1, cr_n, ci_n);
        contract(j, cr_c, ci_c);
      }
    }
    __syncthreads();

    // 3. output spectra over the tile: row t*QI + ol
  #pragma unroll
    for (int s = 0; s < NS; ++s) {
      const int pi = threadIdx.x + NT * s;
      const int ol = pi / HB, k = pi % HB;
      if (ol < QI) {
        const int kr = LayerGeo<P>::at(k), ki = LayerGeo<P>::at(bin_im_slot<P>(k));
  #pragma unroll
        for (int t = 0; t < TT; ++t) {
          // stored mirrored (slot k = Re - Im, slot p-k = Re + Im) for the Hartley-form
          // inverse below; bin 0 keeps its real pair
          const int rb = LayerGeo<P>::row_base(t * QI + ol);
          tile[rb + kr] = k == 0 ? acc_r[s][t] : acc_r[s][t] - acc_i[s][t];
          tile[rb + ki] = k == 0 ? acc_i[s][t] : acc_r[s][t] + acc_i[s][t];
        }
      }
    }
    __syncthreads();

  }

  // 4. rdIFFT of the TT*QI output rows straight to HBM; the next launch in the stream
  // may be scheduled meanwhile (it waits for this grid before touching memory)
  griddep_launch_dependents();
  ifft_rows_mirrored<P, NT, T>(tile, TT * QI, [&](int r) -> T* {
    const int t = r / QI, ol = r - t * QI;
    return t < ntok ? out + (tok0 + t) * (int64_t)D + (int64_t)(o0 + ol) * P : nullptr;
  });
}

// ---------------------------------------------------------------------- grad_c
// Thread group gamma = (k, ib, jb): bin k, output blocks i = ib*RI .. +RI, input
// blocks jl = jb*RJ .. +RJ of the CTA's QJ-block group. The tile holds, per tile of
// ntok <= TT tokens, G for rows t*q + i and X for rows ntok*q + t*QJ + jl.
template <int P, typename T, int NT, int TT, int NG, int RI, int RJ>
__global__ void __launch_bounds__(NT, 1)
k_circ_gc(const T* __restrict__ g, const T* __restrict__ x, float* __restrict__ grad_c,
          float* __restrict__ partial, int64_t B, int q, int QJ, int64_t tok_per_cta, int ifft_here) {
  extern __shared__ float tile[];
  constexpr int HB = P / 2;
  const int D = q * P;
  const int j0 = blockIdx.y * QJ;
  const int64_t tbeg = (int64_t)blockIdx.x * tok_per_cta;
  const int64_t tend = (tbeg + tok_per_cta < B) ? tbeg + tok_per_cta : B;
  const int nib = q / RI, njb = QJ / RJ;
  const int ngroups = HB * nib * njb;
  // the only token slice: this CTA's sums are final and every (bin, i, j) of its group
  // is one thread-group's, so it stores them instead of adding into a zeroed grad_c; with
  // per-slice sums (partial), each slice stores its own q x q x p spectrum the same way
  const bool store = (gridDim.x == 1) || partial != nullptr;
  float* const gc_base = partial != nullptr ? partial + (int64_t)blockIdx.x * q * q * P : grad_c;
  griddep_wait();                            // earlier work in the stream (g, x, zeroed grad_c) is done

  if constexpr (RJ % 2 == 0) {
    // S accumulators: input blocks b and b + 1 of a group on packed fp32 pairs (RJ even),
    // the G value they share broadcast to both halves.
    constexpr int RJP = (RJ + 1) / 2;
    f2 s_r[NG][RI][RJP], s_i[NG][RI][RJP];
  #pragma unroll
    for (int n = 0; n < NG; ++n)
  #pragma unroll
      for (int a = 0; a < RI; ++a)
  #pragma unroll
        for (int b = 0; b < RJP; ++b) s_r[n][a][b] = s_i[n][a][b] = f2_bc(0.0f);

    for (int64_t tok0 = tbeg; tok0 < tend; tok0 += TT) {
      const int ntok = (int)((tend - tok0) < TT ? (tend - tok0) : TT);
      if (tok0 != tbeg) __syncthreads();          // previous tile fully consumed
      // rows [0, ntok*q): G; rows [ntok*q, ntok*(q + QJ)): X of the CTA's blocks. A
      // partial tile (a ragged tail, a handful of tokens) transforms only its rows.
      const int xrow0 = ntok * q;
      fft_rows<P, NT, T>(tile, ntok * (q + QJ), [&](int r) -> const T* {
        if (r < xrow0) {
          const int t = r / q, b = r - t * q;
          return g + (tok0 + t) * (int64_t)D + (int64_t)b * P;
        }
        const int rr = r - xrow0;
        const int t = rr / QJ, jl = rr - t * QJ;
        return x + (tok0 + t) * (int64_t)D + (int64_t)(j0 + jl) * P;
      });
      __syncthreads();
      // bin0 = false (warps with no bin-0 group) drops the real-pair selects
      auto accumulate = [&](bool bin0) {
    #pragma unroll
        for (int n = 0; n < NG; ++n) {
          const int gam = threadIdx.x + NT * n;
          if (gam < ngroups) {
            const int k = gam % HB;
            const int rest = gam / HB;
            const int ib = rest % nib, jb = rest / nib;
            const bool z = bin0 && (k == 0);
            const int kr = LayerGeo<P>::at(k), ki = LayerGeo<P>::at(bin_im_slot<P>(k));
            for (int t = 0; t < ntok; ++t) {
              float gr[RI], gi[RI];
    #pragma unroll
              for (int a = 0; a < RI; ++a) {
                const int rb = LayerGeo<P>::row_base(t * q + ib * RI + a);
                gr[a] = tile[rb + kr];
                gi[a] = tile[rb + ki];
              }
    #pragma unroll
              for (int bp = 0; bp < RJP; ++bp) {
                float xr[2], xi[2];
    #pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const int b = 2 * bp + h < RJ ? 2 * bp + h : RJ - 1;   // odd RJ: the spare half repeats b
                  const int rb = LayerGeo<P>::row_base(xrow0 + t * QJ + jb * RJ + b);
                  xr[h] = tile[rb + kr];
                  xi[h] = tile[rb + ki];
                }
                // G conj(X): re = gr xr + gi xi, im = gi xr - gr xi; bin 0: (gr xr, gi xi)
                const f2 vxr = f2_mk(xr[0], xr[1]);
                const f2 vxi_re = z ? f2_bc(0.0f) : f2_mk(xi[0], xi[1]);
                const f2 vx_im = z ? f2_mk(xi[0], xi[1]) : f2_mk(xr[0], xr[1]);
                const f2 vxi_im = z ? f2_bc(0.0f) : f2_mk(-xi[0], -xi[1]);
    #pragma unroll
                for (int a = 0; a < RI; ++a) {
                  const f2 vgr = f2_bc(gr[a]), vgi = f2_bc(gi[a]);
                  s_r[n][a][bp] = f2_fma(vgr, vxr, f2_fma(vgi, vxi_re, s_r[n][a][bp]));
                  s_i[n][a][bp] = f2_fma(vgi, vx_im, f2_fma(vgr, vxi_im, s_i[n][a][bp]));
                }
              }
            }
          }
        }
      };
      // a warp holds a bin-0 group only if its first lane does (gamma = tid + NT n with
      // NT and p/2 multiples of 32, and p/2 a multiple of NT when larger); a warp-uniform
      // branch, so each side is specialised
      if ((threadIdx.x & ~31u) % HB == 0) accumulate(true);
      else accumulate(false);
    }
    // add this CTA's partial packed cross-spectrum into grad_c, or, when it owns its rows
    // of grad_c outright, write them mirrored into the tile for the inverse below
    griddep_launch_dependents();
    if (ifft_here) __syncthreads();                 // the last token tile is fully consumed
  #pragma unroll
    for (int n = 0; n < NG; ++n) {
      const int gam = threadIdx.x + NT * n;
      if (gam < ngroups) {
        const int k = gam % HB;
        const int rest = gam / HB;
        const int ib = rest % nib, jb = rest / nib;
        const int kim = bin_im_slot<P>(k);
  #pragma unroll
        for (int a = 0; a < RI; ++a)
  #pragma unroll
          for (int b = 0; b < RJ; ++b) {
            float* dst = gc_base + ((int64_t)(ib * RI + a) * q + (j0 + jb * RJ + b)) * P;
            const float vr = (b & 1) ? s_r[n][a][b / 2].y : s_r[n][a][b / 2].x;
            const float vi = (b & 1) ? s_i[n][a][b / 2].y : s_i[n][a][b / 2].x;
            if (ifft_here) {
              const int rb = LayerGeo<P>::row_base((ib * RI + a) * QJ + jb * RJ + b);
              tile[rb + LayerGeo<P>::at(k)] = k == 0 ? vr : vr - vi;
              tile[rb + LayerGeo<P>::at(kim)] = k == 0 ? vi : vr + vi;
            } else if (store) {
              dst[k] = vr;
              dst[kim] = vi;
            } else {
              atomicAdd(dst + k, vr);
              atomicAdd(dst + kim, vi);
            }
          }
      }
    }
  } else {
    float s_r[NG][RI][RJ], s_i[NG][RI][RJ];
  #pragma unroll
    for (int n = 0; n < NG; ++n)
  #pragma unroll
      for (int a = 0; a < RI; ++a)
  #pragma unroll
        for (int b = 0; b < RJ; ++b) s_r[n][a][b] = s_i[n][a][b] = 0.0f;

    for (int64_t tok0 = tbeg; tok0 < tend; tok0 += TT) {
      const int ntok = (int)((tend - tok0) < TT ? (tend - tok0) : TT);
      if (tok0 != tbeg) __syncthreads();          // previous tile fully consumed
      // rows [0, ntok*q): G; rows [ntok*q, ntok*(q + QJ)): X of the CTA's blocks. A
      // partial tile (a ragged tail, a handful of tokens) transforms only its rows.
      const int xrow0 = ntok * q;
      fft_rows<P, NT, T>(tile, ntok * (q + QJ), [&](int r) -> const T* {
        if (r < xrow0) {
          const int t = r / q, b = r - t * q;
          return g + (tok0 + t) * (int64_t)D + (int64_t)b * P;
        }
        const int rr = r - xrow0;
        const int t = rr / QJ, jl = rr - t * QJ;
        return x + (tok0 + t) * (int64_t)D + (int64_t)(j0 + jl) * P;
      });
      __syncthreads();
  #pragma unroll
      for (int n = 0; n < NG; ++n) {
        const int gam = threadIdx.x + NT * n;
        if (gam < ngroups) {
          const int k = gam % HB;
          const int rest = gam / HB;
          const int ib = rest % nib, jb = rest / nib;
          const bool z = (k == 0);
          const int kr = LayerGeo<P>::at(k), ki = LayerGeo<P>::at(bin_im_slot<P>(k));
          for (int t = 0; t < ntok; ++t) {
            float gr[RI], gi[RI];
  #pragma unroll
            for (int a = 0; a < RI; ++a) {
              const int rb = LayerGeo<P>::row_base(t * q + ib * RI + a);
              gr[a] = tile[rb + kr];
              gi[a] = tile[rb + ki];
            }
  #pragma unroll
            for (int b = 0; b < RJ; ++b) {
              const int rb = LayerGeo<P>::row_base(xrow0 + t * QJ + jb * RJ + b);
              const float xr = tile[rb + kr];
              const float xi = tile[rb + ki];
              // G conj(X): re = gr xr + gi xi, im = gi xr - gr xi; bin 0: (gr xr, gi xi)
              const float xi_re = z ? 0.0f : xi;
              const float x_im = z ? xi : xr;
              const float xi_im = z ? 0.0f : -xi;
  #pragma unroll
              for (int a = 0; a < RI; ++a) {
                s_r[n][a][b] = fmaf(gr[a], xr, fmaf(gi[a], xi_re, s_r[n][a][b]));
                s_i[n][a][b] = fmaf(gi[a], x_im, fmaf(gr[a], xi_im, s_i[n][a][b]));
              }
            }
          }
        }
      }
    }
    // add this CTA's partial packed cross-spectrum into grad_c, or write it mirrored into
    // the tile for the inverse below
    griddep_launch_dependents();
    if (ifft_here) __syncthreads();                 // the last token tile is fully consumed
  #pragma unroll
    for (int n = 0; n < NG; ++n) {
      const int gam = threadIdx.x + NT * n;
      if (gam < ngroups) {
        const int k = gam % HB;
        const int rest = gam / HB;
        const int ib = rest % nib, jb = rest / nib;
        const int kim = bin_im_slot<P>(k);
  #pragma unroll
        for (int a = 0; a < RI; ++a)
  #pragma unroll
          for (int b = 0; b < RJ; ++b) {
            float* dst = gc_base + ((int64_t)(ib * RI + a) * q + (j0 + jb * RJ + b)) * P;
            if (ifft_here) {
              const int rb = LayerGeo<P>::row_base((ib * RI + a) * QJ + jb * RJ + b);
              const float vr = s_r[n][a][b], vi = s_i[n][a][b];
              tile[rb + LayerGeo<P>::at(k)] = k == 0 ? vr : vr - vi;
              tile[rb + LayerGeo<P>::at(kim)] = k == 0 ? vi : vr + vi;
            } else if (store) {
              dst[k] = s_r[n][a][b];
              dst[kim] = s_i[n][a][b];
            } else {
              atomicAdd(dst + k, s_r[n][a][b]);
              atomicAdd(dst + kim, s_i[n][a][b]);
            }
          }
      }
    }
  }
  if (ifft_here) {
    // a CTA that covered every token owns its q x QJ rows of grad_c: their rdIFFT (Hartley
    // form, the rows stored mirrored above) straight to grad_c, in place of a separate launch
    __syncthreads();
    ifft_rows_mirrored<P, NT, float>(tile, q * QJ, [&](int r) -> float* {
      return grad_c + ((int64_t)(r / QJ) * q + j0 + r % QJ) * P;
    });
  }
}

// ------------------------------------------------------------------ launchers
static int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
    return n;
  return 148;
}

template <typename KernelT>
static cudaError_t set_smem(KernelT kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Forward / grad_x: NT threads, TT tokens per CTA, NS bins per thread, so a CTA
// covers up to NS*NT/(P/2) output blocks.
template <int P, typename T, int NT, int TT, int NS, bool BWDX>
static cudaError_t launch_x_cfg(const void* in, const float* chat, void* out, int64_t B, int q,
                                cudaStream_t s) {
  constexpr int QI_MAX = NS * NT / (P / 2);
  static_assert(QI_MAX >= 1, "slots must cover one block");
  const int64_t gx = (B + TT - 1) / TT;
  if (gx > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int QI = layer_qi(q, QI_MAX, gx, num_sms());
  const size_t smem = sizeof(float) * (size_t)LayerGeo<P>::words(TT * q);
  auto kern = k_circ_x<P, T, NT, TT, NS, BWDX>;
  cudaError_t e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)gx, (unsigned)(q / QI));
  return launch_pdl(kern, grid, dim3(NT), smem, s, static_cast<const T*>(in), chat, static_cast<T*>(out), B, q,
                    QI);
}

// Launch policy (at most 32 complex accumulators per thread, NS * TT <= 32):
//  p <= 512 : 256 threads, up to 8 output blocks per CTA (16 at p = 128 from B = 256),
//             up to 4 tokens per CTA from B = 256, 2 from B = 32, fewer when the grid would
//             otherwise split a token's output blocks over CTAs (layer_x_tokens);
//  p >= 1024: 128 threads, one token per CTA (4 for the q = 1, p = 1024 layer; one
//             output block per CTA for q = 1 at p >= 2048).
template <int P, typename T, bool BWDX>
static cudaError_t launch_x_p(const void* in, const float* chat, void* out, int64_t B, int q,
                              cudaStream_t s) {
  if constexpr (P <= 512) {
    constexpr int NT = 256;
    // up to 8 output blocks per CTA; at p = 128 from B = 256 on, 16 (fewer CTA groups
    // transforming the same input rows: 7% faster at D = 4096, B = 256), and with q >= 16
    // CTAs of 512 threads over 2 tokens and up to 32 output blocks, so each input row is
    // transformed once (18.3 against 19.3 us at D = 4096, B = 256); at B = 1 the 8-block
    // CTAs, more of them, are 11% faster
    constexpr int NS = (8 * (P / 2)) / NT > 0 ? (8 * (P / 2)) / NT : 1;
    if constexpr (P == 128) {
      if (B >= 256 && q >= 16) return launch_x_cfg<P, T, 512, 2, 4, BWDX>(in, chat, out, B, q, s);
      if (B >= 256) return launch_x_cfg<P, T, NT, 4, 2 * NS, BWDX>(in, chat, out, B, q, s);
    }
    const int tt_max = (B >= 256 && NS * 4 <= 32) ? 4 : (B >= 32 ? 2 : 1);
    const int tt = layer_x_tokens(B, q, NS * NT / (P / 2), num_sms(), tt_max);
    if constexpr (NS * 4 <= 32) {
      if (tt == 4) return launch_x_cfg<P, T, NT, 4, NS, BWDX>(in, chat, out, B, q, s);
    }
    if (tt == 2) return launch_x_cfg<P, T, NT, 2, NS, BWDX>(in, chat, out, B, q, s);
    return launch_x_cfg<P, T, NT, 1, NS, BWDX>(in, chat, out, B, q, s);
  } else {
    constexpr int NT = 128;
    constexpr int NS1 = (P / 2) / NT;                       // one output block per CTA
    // up to 4 output blocks (p = 1024), 2 (p = 2048, 4096); <= 32 slots, 16 at p = 2048
    constexpr int NSM = P == 2048 ? 16 : (NS1 * 4 <= 32 ? NS1 * 4 : 32);
    if constexpr (P == 1024) {
      if (q == 1 && B >= 64) return launch_x_cfg<P, T, NT, 4, NS1, BWDX>(in, chat, out, B, q, s);
    } else {
      // one block (q = 1): wider slot groups would only add idle slots and registers
      // (measured 18% faster at p = 4096, B = 256)
      if (q == 1) return launch_x_cfg<P, T, NT, 1, NS1, BWDX>(in, chat, out, B, q, s);
    }
    return launch_x_cfg<P, T, NT, 1, NSM, BWDX>(in, chat, out, B, q, s);
  }
}

// grad_c := 0 before several token slices add into it. A kernel rather than a memset, so the
// launch chains with programmatic dependent launch like the kernels around it (in a CUDA
// graph a memset node does not). n is q^2 p, a multiple of 64; p is 16-byte aligned.
static __global__ void __launch_bounds__(256) k_zero_f4(float4* __restrict__ p, int64_t n4) {
  griddep_wait();                                  // earlier readers of the buffer are done
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n4; i += (int64_t)gridDim.x * 256)
    p[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  griddep_launch_dependents();
}

static cudaError_t launch_zero_f32(float* p, int64_t n, cudaStream_t s) {
  const int64_t n4 = n / 4;
  int64_t blocks = (n4 + 255) / 256;
  if (blocks > 4 * 148) blocks = 4 * 148;
  return launch_pdl(k_zero_f4, dim3((unsigned)blocks), dim3(256), 0, s, reinterpret_cast<float4*>(p), n4);
}

// Records the launch shape in the sink and picks where the slices' sums go: the sink's
// partial buffer when there are several slices and one was given (its capacity checked),
// else nothing (the kernel stores into grad_c with one slice, or adds into it).
static cudaError_t sink_plan(GcSink* sink, int slices, int64_t floats_per_slice, float** partial) {
  *partial = nullptr;
  if (sink == nullptr) return cudaSuccess;
  sink->slices = slices;
  sink->ifft_done = false;
  if (sink->plan_only || slices <= 1 || sink->partial == nullptr) return cudaSuccess;
  if ((int64_t)slices * floats_per_slice > sink->partial_floats) return cudaErrorInvalidValue;
  *partial = sink->partial;
  return cudaSuccess;
}

template <int P, typename T, int NT, int TT, int NG, int RI, int RJ>
static cudaError_t run_gc(const void* g, const void* x, float* grad_c, int64_t B, int q, int QJ,
                          cudaStream_t s, GcSink* sink) {
  auto kern = k_circ_gc<P, T, NT, TT, NG, RI, RJ>;
  const size_t smem = sizeof(float) * (size_t)LayerGeo<P>::words(TT * (q + QJ));
  const int njgroups = q / QJ;
  int64_t tiles_per = 1;
  const int slices = layer_gc_slices(njgroups, (B + TT - 1) / TT, num_sms(), &tiles_per);
  // one token slice: each CTA owns its rows of grad_c and inverse-transforms them itself
  // (its tile holds TT (q + QJ) rows, enough for the q QJ rows of grad_c it owns)
  const bool here = slices == 1 && (int64_t)q * QJ <= (int64_t)TT * (q + QJ);
  float* partial = nullptr;
  cudaError_t e = sink_plan(sink, slices, (int64_t)q * q * P, &partial);
  if (sink) sink->ifft_done = here;
  if (e != cudaSuccess || (sink && sink->plan_only)) return e;
  e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  if (slices > 1 && !partial) {
    // several token slices add their partial sums into grad_c; one slice stores them
    e = launch_zero_f32(grad_c, (int64_t)q * q * P, s);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((unsigned)slices, (unsigned)njgroups);
  return launch_pdl(kern, grid, dim3(NT), smem, s, static_cast<const T*>(g), static_cast<const T*>(x), grad_c,
                    partial, B, q, QJ, (int64_t)(tiles_per * TT), here ? 1 : 0);
}

// grad_c launcher: a CTA of 512 threads keeps S for QJ input blocks in registers,
// RI x RJ (output, input) blocks of one bin per thread-slot, NG slots per thread,
// at most 32 complex accumulators per thread.
template <int P, typename T, int TT>
static cudaError_t launch_gc_tt(const void* g, const void* x, float* grad_c, int64_t B, int q,
                                cudaStream_t s, GcSink* sink) {
  constexpr int NT = 512;
  constexpr int HB = P / 2;
  const int QJ = layer_qj(q, HB, 32LL * NT, (B + TT - 1) / TT, num_sms());
  if ((int64_t)HB * q * QJ > 32LL * NT) return cudaErrorInvalidConfiguration;
  const int64_t slots = (int64_t)HB * q * QJ;                // complex accumulators per CTA
  if (q % 4 == 0 && QJ % 8 == 0 && slots <= 32LL * NT) return run_gc<P, T, NT, TT, 1, 4, 8>(g, x, grad_c, B, q, QJ, s, sink);
  if (q % 4 == 0 && QJ % 4 == 0) {
    if (slots <= 16LL * NT) return run_gc<P, T, NT, TT, 1, 4, 4>(g, x, grad_c, B, q, QJ, s, sink);
    return run_gc<P, T, NT, TT, 2, 4, 4>(g, x, grad_c, B, q, QJ, s, sink);
  }
  if (q % 2 == 0 && QJ % 2 == 0) {
    if (slots <= 4LL * NT) return run_gc<P, T, NT, TT, 1, 2, 2>(g, x, grad_c, B, q, QJ, s, sink);
    if (slots <= 8LL * NT) return run_gc<P, T, NT, TT, 2, 2, 2>(g, x, grad_c, B, q, QJ, s, sink);
    if (slots <= 16LL * NT) return run_gc<P, T, NT, TT, 4, 2, 2>(g, x, grad_c, B, q, QJ, s, sink);
    return run_gc<P, T, NT, TT, 8, 2, 2>(g, x, grad_c, B, q, QJ, s, sink);
  }
  if (slots <= 1LL * NT) return run_gc<P, T, NT, TT, 1, 1, 1>(g, x, grad_c, B, q, QJ, s, sink);
  if (slots <= 4LL * NT) return run_gc<P, T, NT, TT, 4, 1, 1>(g, x, grad_c, B, q, QJ, s, sink);
  if (slots <= 8LL * NT) return run_gc<P, T, NT, TT, 8, 1, 1>(g, x, grad_c, B, q, QJ, s, sink);
  if (slots <= 16LL * NT) return run_gc<P, T, NT, TT, 16, 1, 1>(g, x, grad_c, B, q, QJ, s, sink);
  return run_gc<P, T, NT, TT, 32, 1, 1>(g, x, grad_c, B, q, QJ, s, sink);
}

// Token tiles of 4 (p <= 512), 2 (p = 1024) or 1 token, or half of that while a handful of
// tokens leaves the SMs idle (layer_gc_half_tiles: grad_c alone at D=4096, B=16: 11.3 against
// 14.2 us at p = 128, 10.3 against 12.3 at p = 512, 10.2 against 11.4 at p = 1024).
template <int P, typename T>
static cudaError_t launch_gc_p(const void* g, const void* x, float* grad_c, int64_t B, int q,
                               cudaStream_t s, GcSink* sink) {
  constexpr int TT = (P >= 2048) ? 1 : (P >= 1024 ? 2 : 4);
  if constexpr (TT > 1) {
    if (layer_gc_half_tiles(B, TT, q, P / 2, 32LL * 512, num_sms()))
      return launch_gc_tt<P, T, TT / 2>(g, x, grad_c, B, q, s, sink);
  }
  return launch_gc_tt<P, T, TT>(g, x, grad_c, B, q, s, sink);
}

// Per-p entry of the layer, instantiated once per translation unit (circ_p*.cu):
// op 0 = forward (a = x, out = y); op 1 = grad_x (a = g, out = grad_x);
// op 2 = grad_c accumulation (a = g, b = x, gc = grad_c; zeroed here when several
// token slices add into it). For op 2, the sink (if given) receives the slice count and
// whether the kernel also ran grad_c's rdIFFT (one token slice), so the caller must not; its
// partial buffer, if set, takes the slices' sums instead of atomics into grad_c.
template <int P>
cudaError_t circ_layer_p(int op, const void* a, const void* b, const float* chat, void* out, float* gc,
                         int64_t B, int q, int dtype, cudaStream_t s, GcSink* sink) {
  if (dtype == 0) {
    if (op == 0) return launch_x_p<P, float, false>(a, chat, out, B, q, s);
    if (op == 1) return launch_x_p<P, float, true>(a, chat, out, B, q, s);
    return launch_gc_p<P, float>(a, b, gc, B, q, s, sink);
  }
  if (op == 0) return launch_x_p<P, bf16_t, false>(a, chat, out, B, q, s);
  if (op == 1) return launch_x_p<P, bf16_t, true>(a, chat, out, B, q, s);
  return launch_gc_p<P, bf16_t>(a, b, gc, B, q, s, sink);
}

#define RDFFT_CIRC_INSTANCE(PP)                                                                  \
  cudaError_t circ_layer_##PP(int op, const void* a, const void* b, const float* chat, void* out, \
                              float* gc, int64_t B, int q, int dtype, cudaStream_t s,             \
                              GcSink* sink) {                                                     \
    return circ_layer_p<PP>(op, a, b, chat, out, gc, B, q, dtype, s, sink);                       \
  }

}  // namespace rdfft
