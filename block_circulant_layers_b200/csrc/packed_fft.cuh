// Packed real-domain FFT building blocks (rdFFT) for sm_100a kernels.
//
// Method: "Memory-Efficient Training with In-Place FFT Implementation"
// (paper-notes page, method section):
//   * "Squeeze N+2 -> N": a length-p real row and its spectrum share one buffer;
//     y_0 at 0, y_{p/2} at p/2, Re y_k at k, Im y_k at p-k.
//   * "Proposition 1": radix-2 Cooley-Tukey (decimation in time, bit-reversed input)
//     whose butterflies act on four-element groups {k, M/2-k, M/2+k, M-k} of a
//     block of size M, symmetric about the centre M/2.
//   * "In-place IFFT design": the inverse walks the same graph backwards, splitting
//     each conjugate pair into symmetric and antisymmetric parts.
//
// Stage M on a block b (all indices relative to b):
//   k = 0      : (a[0], a[M/2]) <- (a[0] + a[M/2], a[0] - a[M/2])
//   k = M/4    : a[3M/4] <- -a[3M/4]
//   0 < k < M/4: E = a[k] + i a[M/2-k], O = a[M/2+k] + i a[M-k], t = W_M^k O,
//                a[k] = Re(E+t), a[M-k] = Im(E+t), a[M/2-k] = Re(E-t), a[M/2+k] = -Im(E-t)
// The inverse stage undoes it without the factor 1/2 (so the k = M/4 pair is doubled);
// the whole inverse is scaled by 1/p once at the end, which is exact in binary
// floating point.
//
// GPU decomposition (ours). After the stages up to block size H (M/2 = H at the next
// stage), the positions {m*H + r, m*H + H - r} of a larger block form an "orbit" that
// the later stages never mix with other positions (0 < r < H/2); positions that are
// multiples of H/2 form one more orbit ("merged"). So a row is transformed in passes:
// pass 0 runs stages 2..E on contiguous blocks of E = 32 bit-reversed elements held
// in registers by one thread; every later pass gathers one orbit per thread into
// registers, runs up to log2(E)-1 stages there, and scatters it back. Only the passes
// exchange data, through shared memory (or straight from / to global memory for the
// first and last pass), so a row of 4096 needs two exchanges and a row of 512 one.
//
// Everything here is __host__ __device__ so the same per-thread pass functions run
// on the GPU and in the host emulator used by the CPU tests.
#pragma once

#include <math.h>
#include <stdint.h>

#if defined(__CUDACC__)
#include <cuda_bf16.h>
#define RD_HD __host__ __device__ __forceinline__
#define RD_DEV __device__ __forceinline__
#else
#define RD_HD inline
#define RD_DEV inline
#endif

#include "twiddles.inc"

namespace rdfft {

// --------------------------------------------------------------------------- basics
constexpr int kMaxP = 4096;
constexpr int kEPT = 32;            // elements per thread in the multi-pass kernels

RD_HD constexpr int ilog2(int n) { return n <= 1 ? 0 : 1 + ilog2(n >> 1); }

RD_HD constexpr int bitrev(int v, int bits) {
  int r = 0;
  for (int i = 0; i < bits; ++i) r = (r << 1) | ((v >> i) & 1);
  return r;
}

struct Tw { float c, s; };          // W = c - i s

// Per-stage twiddle tables: W_M^k at index M/4 - 1 + k, k < M/4, M = 4..4096.
// The constant-bank copy serves compile-time indices (pass 0 and merged orbits,
// folded into instruction operands); the global copy serves lane-dependent indices.
#if defined(__CUDACC__)
static __constant__ Tw c_tw[RDFFT_TWIDDLE_COUNT] = {RDFFT_TWIDDLE_VALUES};
static __device__ Tw g_tw[RDFFT_TWIDDLE_COUNT] = {RDFFT_TWIDDLE_VALUES};
#endif
static const Tw h_tw[RDFFT_TWIDDLE_COUNT] = {RDFFT_TWIDDLE_VALUES};

RD_HD constexpr int tw_index(int M, int k) { return M / 4 - 1 + k; }

RD_HD Tw tw_const(int idx) {
#if defined(__CUDA_ARCH__)
  return c_tw[idx];
#else
  return h_tw[idx];
#endif
}

RD_HD Tw tw_lane(int idx) {
#if defined(__CUDA_ARCH__)
  const float2 v = __ldg(reinterpret_cast<const float2*>(g_tw) + idx);
  return Tw{v.x, v.y};
#else
  return h_tw[idx];
#endif
}

// ------------------------------------------------------------------ storage types
// bf16 is carried as its raw 16-bit pattern; arithmetic is always fp32.
typedef uint16_t bf16_t;

RD_HD float to_f32(float v) { return v; }
RD_HD float to_f32(bf16_t v) {
#if defined(__CUDA_ARCH__)
  return __bfloat162float(__ushort_as_bfloat16(v));
#else
  uint32_t u = (uint32_t)v << 16;
  float f;
  __builtin_memcpy(&f, &u, 4);
  return f;
#endif
}

template <typename T> RD_HD T from_f32(float v);
template <> RD_HD float from_f32<float>(float v) { return v; }
template <> RD_HD bf16_t from_f32<bf16_t>(float v) {
#if defined(__CUDA_ARCH__)
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
#else
  // round to nearest, ties to even, on the bit pattern
  uint32_t u;
  __builtin_memcpy(&u, &v, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (bf16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (bf16_t)(u >> 16);
#endif
}

// Load of transform data. A plain (coherent) load on purpose: the transforms are in
// place, and a read-only (non-coherent) load may legally be repeated by the compiler
// after the same thread has overwritten the row.
template <typename T> RD_HD float ld(const T* p) { return to_f32(*p); }

// ------------------------------------------------------------------- butterflies
// Forward group at (k, M/2-k, M/2+k, M-k) with twiddle W = wr + i wi.
// Six FP instructions: A = E + W O by two FMA chains, B = 2E - A.
RD_HD void bfly_fwd(float& pk, float& pmk, float& pHk, float& pMk, float wr, float wi) {
  const float er = pk, ei = pmk, orr = pHk, oi = pMk;
  const float ar = fmaf(wr, orr, fmaf(-wi, oi, er));
  const float ai = fmaf(wr, oi, fmaf(wi, orr, ei));
  pk = ar;
  pMk = ai;
  pmk = fmaf(2.0f, er, -ar);        //  Re(E - t)
  pHk = fmaf(-2.0f, ei, ai);        // -Im(E - t)
}

// Inverse group (without the 1/2): A = a[k] + i a[M-k], B = a[M/2-k] - i a[M/2+k],
// a[k], a[M/2-k] <- A + B;  a[M/2+k], a[M-k] <- (A - B) conj(W).
RD_HD void bfly_inv(float& pk, float& pmk, float& pHk, float& pMk, float wr, float wi) {
  const float a = pk, b = pMk, c = pmk, d = pHk;
  const float dr = a - c, di = b + d;
  pk = a + c;
  pmk = b - d;
  pHk = fmaf(dr, wr, di * wi);
  pMk = fmaf(di, wr, -(dr * wi));
}

template <bool INV>
RD_HD void bfly(float& pk, float& pmk, float& pHk, float& pMk, Tw w) {
  if (INV) bfly_inv(pk, pmk, pHk, pMk, w.c, -w.s);
  else bfly_fwd(pk, pmk, pHk, pMk, w.c, -w.s);
}

// One stage of size M over the contiguous register range a[OFF, OFF + NB).
// The positions are the algorithm's own; twiddles are compile-time.
template <int M, int NB, int OFF, bool INV, int E>
RD_HD void stage_contig(float (&a)[E]) {
  static_assert(NB % M == 0 && OFF + NB <= E, "stage range");
#pragma unroll
  for (int b = OFF; b < OFF + NB; b += M) {
    const float x0 = a[b], x1 = a[b + M / 2];
    a[b] = x0 + x1;
    a[b + M / 2] = x0 - x1;
    if (M >= 4) {
      if (INV) {
        a[b + M / 4] = 2.0f * a[b + M / 4];
        a[b + 3 * M / 4] = -2.0f * a[b + 3 * M / 4];
      } else {
        a[b + 3 * M / 4] = -a[b + 3 * M / 4];
      }
    }
#pragma unroll
    for (int k = 1; k < M / 4; ++k)
      bfly<INV>(a[b + k], a[b + M / 2 - k], a[b + M / 2 + k], a[b + M - k], tw_const(tw_index(M, k)));
  }
}

// Stages MLO..MHI (powers of two) on a[OFF, OFF+NB): ascending for the forward
// transform, descending for the inverse.
template <int MLO, int MHI, int NB, int OFF, bool INV, int E>
RD_HD void stages_contig(float (&a)[E]) {
  if constexpr (MLO <= MHI) {
    if constexpr (!INV) {
      stage_contig<MLO, NB, OFF, false>(a);
      stages_contig<MLO * 2, MHI, NB, OFF, false>(a);
    } else {
      stage_contig<MHI, NB, OFF, true>(a);
      stages_contig<MLO, MHI / 2, NB, OFF, true>(a);
    }
  }
}

// Generic orbit: a[OFF + 2m] <-> position m*H + r, a[OFF + 2m + 1] <-> (m+1)*H - r,
// m < UMAX. Stage M' = U*H (U = 2..UMAX) acts on the groups with k' = s*H + r and
// k' = (s+1)*H - r (s < U/4), or k' = r alone when U = 2.
template <int H, int UMAX, int U, int OFF, bool INV, int E>
RD_HD void orbit_stage(float (&a)[E], int r) {
  constexpr int MP = U * H;
  constexpr int U2 = U / 2;
  if constexpr (U == 2) {
    const Tw w = tw_lane(tw_index(MP, 0) + r);
#pragma unroll
    for (int m0 = 0; m0 < UMAX; m0 += 2)
      bfly<INV>(a[OFF + 2 * m0], a[OFF + 2 * m0 + 1], a[OFF + 2 * m0 + 2], a[OFF + 2 * m0 + 3], w);
  } else {
#pragma unroll
    for (int s = 0; s < U / 4; ++s) {
      const Tw w1 = tw_lane(tw_index(MP, s * H) + r);
      const Tw w2 = tw_lane(tw_index(MP, (s + 1) * H) - r);
#pragma unroll
      for (int m0 = 0; m0 < UMAX; m0 += U) {
        bfly<INV>(a[OFF + 2 * (m0 + s)], a[OFF + 2 * (m0 + U2 - s - 1) + 1],
                  a[OFF + 2 * (m0 + U2 + s)], a[OFF + 2 * (m0 + U - s - 1) + 1], w1);
        bfly<INV>(a[OFF + 2 * (m0 + s) + 1], a[OFF + 2 * (m0 + U2 - s - 1)],
                  a[OFF + 2 * (m0 + U2 + s) + 1], a[OFF + 2 * (m0 + U - s - 1)], w2);
      }
    }
  }
}

template <int H, int UMAX, int U, int OFF, bool INV, int E>
RD_HD void orbit_stages(float (&a)[E], int r) {
  if constexpr (U <= UMAX) {
    if constexpr (!INV) {
      orbit_stage<H, UMAX, U, OFF, false>(a, r);
      orbit_stages<H, UMAX, U * 2, OFF, false>(a, r);
    } else {
      orbit_stages<H, UMAX, U * 2, OFF, true>(a, r);
      orbit_stage<H, UMAX, U, OFF, true>(a, r);
    }
  }
}

// ------------------------------------------------------------------------ plan
// Pass 0 covers stages 1..e (blocks of E = 2^e); pass k >= 1 covers stages
// s0+1..s1 with s0 = e + (k-1)(e-1), s1 = min(s0 + e - 1, L).
template <int P>
struct Plan {
  static_assert(P >= 2 && P <= kMaxP && (P & (P - 1)) == 0, "p must be a power of two in [2, 4096]");
  static constexpr int L = ilog2(P);
  static constexpr int E = P < kEPT ? P : kEPT;
  static constexpr int e = ilog2(E);
  static constexpr int TPR = P / E;               // threads per row
  static constexpr int LOG_TPR = ilog2(TPR);
  static constexpr int NPASS = (L <= e) ? 1 : 1 + (L - e + (e - 2)) / (e - 1);
  RD_HD static constexpr int s0(int k) { return e + (k - 1) * (e - 1); }
  RD_HD static constexpr int s1(int k) { return s0(k) + e - 1 < L ? s0(k) + e - 1 : L; }
};

template <int P, int K>
struct PassShape {
  static constexpr int H = 1 << Plan<P>::s0(K);
  static constexpr int LB = 1 << Plan<P>::s1(K);
  static constexpr int UMAX = LB / H;
  static constexpr int N = 2 * UMAX;              // elements per orbit
  static constexpr int C = Plan<P>::E / N;        // orbits per thread
  static constexpr int HH = H / 2;                // orbits per block of LB
};

// Shared-memory swizzle of the row tile: XOR the low 5 bits of the word index with
// a function of its higher bits, chosen per p so that the pass-0 scatter and the
// orbit gathers/scatters of 32 lanes fall in distinct banks.
template <int P>
struct Swz {
  static constexpr int A = P >= 4096 ? 2 : (P >= 2048 ? 1 : 0);
  static constexpr int B = P >= 2048 ? 4 : -1;
  RD_HD static int at(int G) {
    const int g = G >> 5;
    int f = (g >> A) & 31;
    if (B >= 0) f ^= ((g >> (B < 0 ? 0 : B)) & 1) << 4;
    return G ^ f;
  }
};

// ------------------------------------------------------------- per-thread passes
// `tile` is the CTA's shared (or, in the emulator, host) fp32 row tile of ROWS*P
// words; `lrow` the thread's row in the tile, `v` its index within the row's
// TPR threads; `g` the row in global memory (valid only when `active`).

// Forward pass 0: bit-reversed gather straight from global memory (coalesced:
// lane v reads v + TPR*j'), stages 2..E in registers, scatter of block
// t = bitrev(v) to the tile.
template <int P, typename T>
RD_HD void fwd_pass0(float* tile, int lrow, int v, const T* g, bool active) {
  using PL = Plan<P>;
  float a[PL::E];
#pragma unroll
  for (int jp = 0; jp < PL::E; ++jp) a[bitrev(jp, PL::e)] = active ? ld(g + v + PL::TPR * jp) : 0.0f;
  stages_contig<2, PL::E, PL::E, 0, false>(a);
  const int t = bitrev(v, PL::LOG_TPR);
#pragma unroll
  for (int j = 0; j < PL::E; ++j) tile[Swz<P>::at(lrow * P + t * PL::E + j)] = a[j];
}

// Inverse pass 0 (the last inverse step): gather block t from the tile, inverse
// stages E..2, scale by 1/P, scatter to global at the bit-reversed positions.
template <int P, typename T>
RD_HD void inv_pass0(const float* tile, int lrow, int v, T* g, bool active) {
  using PL = Plan<P>;
  float a[PL::E];
  const int t = bitrev(v, PL::LOG_TPR);
#pragma unroll
  for (int j = 0; j < PL::E; ++j) a[j] = tile[Swz<P>::at(lrow * P + t * PL::E + j)];
  stages_contig<2, PL::E, PL::E, 0, true>(a);
  constexpr float scale = 1.0f / P;
  if (active) {
#pragma unroll
    for (int j = 0; j < PL::E; ++j) g[v + PL::TPR * bitrev(j, PL::e)] = from_f32<T>(a[j] * scale);
  }
}

// Position (within its block of size LB) of element i of the generic orbit with
// residue r of a pass that starts at block size H: even i = 2m -> m*H + r, odd
// i = 2m+1 -> (m+1)*H - r. For H = 8, r = 2 the first four are 2, 6, 10, 14: the
// conjugate pair (2, 6) of the 8-point stage and its partner (10, 14) in the
// 16-point stage ("Proposition 1" on the paper-notes page).
RD_HD constexpr int orbit_pos(int H, int i, int r) {
  return (i & 1) ? ((i >> 1) + 1) * H - r : (i >> 1) * H + r;
}

// Slot CI of a middle/last pass K >= 1, then the following slots.
// SRC/DST: 0 = tile, 1 = global row (natural order). Each of the thread's C orbits
// is gathered, transformed and written back to the same positions, so a pass needs
// no synchronisation inside itself.
template <int P, int K, bool INV, int SRC, int DST, int CI, typename T, int E>
RD_HD void orbit_slots(float (&a)[E], float* tile, int tb, int v, T* g, bool active) {
  using PL = Plan<P>;
  using S = PassShape<P, K>;
  if constexpr (CI < S::C) {
    constexpr int OFF = CI * S::N;
    const int o = v + PL::TPR * CI;
    const int beta = o / S::HH;
    const int rho = o % S::HH;
    const int base = beta * S::LB;
    if (rho == 0) {
      // merged orbit: positions base + l*H/2 form a packed real transform of N
      // points whose first stage (M = 2) is already done.
#pragma unroll
      for (int l = 0; l < S::N; ++l) {
        const int n = base + l * S::HH;
        a[OFF + l] = SRC == 0 ? tile[Swz<P>::at(tb + n)] : (active ? ld(g + n) : 0.0f);
      }
      stages_contig<4, S::N, S::N, OFF, INV>(a);
#pragma unroll
      for (int l = 0; l < S::N; ++l) {
        const int n = base + l * S::HH;
        if (DST == 0) tile[Swz<P>::at(tb + n)] = a[OFF + l];
        else if (active) g[n] = from_f32<T>(a[OFF + l]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < S::N; ++i) {
        const int n = base + orbit_pos(S::H, i, rho);
        a[OFF + i] = SRC == 0 ? tile[Swz<P>::at(tb + n)] : (active ? ld(g + n) : 0.0f);
      }
      orbit_stages<S::H, S::UMAX, 2, OFF, INV>(a, rho);
#pragma unroll
      for (int i = 0; i < S::N; ++i) {
        const int n = base + orbit_pos(S::H, i, rho);
        if (DST == 0) tile[Swz<P>::at(tb + n)] = a[OFF + i];
        else if (active) g[n] = from_f32<T>(a[OFF + i]);
      }
    }
    orbit_slots<P, K, INV, SRC, DST, CI + 1>(a, tile, tb, v, g, active);
  }
}

template <int P, int K, bool INV, int SRC, int DST, typename T>
RD_HD void orbit_pass(float* tile, int lrow, int v, T* g, bool active) {
  float a[Plan<P>::E];
  orbit_slots<P, K, INV, SRC, DST, 0>(a, tile, lrow * P, v, g, active);
}

}  // namespace rdfft
