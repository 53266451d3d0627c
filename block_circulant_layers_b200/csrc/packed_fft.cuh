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
// exchange data, through an fp32 shared-memory tile (the first pass reads the row
// where the caller staged it, the last writes it there), so a row of 4096 needs two
// exchanges and a row of 512 one.
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
constexpr int kEPT = 32;            // elements per thread of the multi-pass kernels

// Elements per thread of the standalone transforms. 32 for every p: wider rows per
// thread (64 at p = 1024/2048, 128 at p = 4096) save a shared-memory exchange but
// measured slower on B200, the register cost lowering occupancy more than the saved
// exchange gains. At p = 4096 with bulk-copy staging, 128 elements per thread (two
// passes, one warp and about 25 KB of shared memory per row) cut the shared-memory
// wavefronts by 31%, but only 8 warps fit per SM and the kernel turned latency-bound
// (inverse over 160 MiB: 151.6 against 111.6 us).
RD_HD constexpr int ept_for(int) { return kEPT; }

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

// ------------------------------------------------------------------ paired stages
// sm_100 executes two fp32 FMAs, adds or multiplies in one instruction on a float2
// register pair. Every stage but the last of a register block applies the same
// operations and twiddles to both halves of the block, so those stages run on pairs
// (a[i], a[i + HALF]). Each packed operation rounds exactly like the scalar one it
// replaces (a - b is fma(b, -1, a); 2e - a is fma(a, -1, e + e)), so the results are
// bit-identical to the scalar butterflies above.
#if defined(__CUDA_ARCH__)
typedef float2 f2;
RD_HD f2 f2_mk(float x, float y) { return make_float2(x, y); }
RD_HD f2 f2_fma(f2 a, f2 b, f2 c) { return __ffma2_rn(a, b, c); }
RD_HD f2 f2_add(f2 a, f2 b) { return __fadd2_rn(a, b); }
RD_HD f2 f2_mul(f2 a, f2 b) { return __fmul2_rn(a, b); }
#else
struct f2 { float x, y; };
RD_HD f2 f2_mk(float x, float y) { return f2{x, y}; }
RD_HD f2 f2_fma(f2 a, f2 b, f2 c) { return f2{fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y)}; }
RD_HD f2 f2_add(f2 a, f2 b) { return f2{a.x + b.x, a.y + b.y}; }
RD_HD f2 f2_mul(f2 a, f2 b) { return f2{a.x * b.x, a.y * b.y}; }
#endif
RD_HD f2 f2_bc(float v) { return f2_mk(v, v); }
RD_HD f2 f2_sub(f2 a, f2 b) { return f2_fma(b, f2_bc(-1.0f), a); }

// bfly_fwd on two groups at once (nwi = -wi).
RD_HD void bfly_fwd2(f2& pk, f2& pmk, f2& pHk, f2& pMk, f2 wr, f2 wi, f2 nwi) {
  const f2 er = pk, ei = pmk, orr = pHk, oi = pMk;
  const f2 ar = f2_fma(wr, orr, f2_fma(nwi, oi, er));
  const f2 ai = f2_fma(wr, oi, f2_fma(wi, orr, ei));
  pk = ar;
  pMk = ai;
  pmk = f2_fma(ar, f2_bc(-1.0f), f2_add(er, er));
  pHk = f2_fma(f2_bc(-2.0f), ei, ai);
}

// bfly_inv on two groups at once (nwi = -wi).
RD_HD void bfly_inv2(f2& pk, f2& pmk, f2& pHk, f2& pMk, f2 wr, f2 wi, f2 nwi) {
  const f2 a = pk, b = pMk, c = pmk, d = pHk;
  const f2 dr = f2_sub(a, c), di = f2_add(b, d);
  pk = f2_add(a, c);
  pmk = f2_sub(b, d);
  pHk = f2_fma(dr, wr, f2_mul(di, wi));
  pMk = f2_fma(di, wr, f2_mul(dr, nwi));
}

// The group (i0, i1, i2, i3) of the lower half and the same group of the upper half
// (+HALF) as one paired butterfly with twiddle w.
template <bool INV, int HALF, int E>
RD_HD void bfly_pair(float (&a)[E], int i0, int i1, int i2, int i3, Tw w) {
  f2 x0 = f2_mk(a[i0], a[i0 + HALF]), x1 = f2_mk(a[i1], a[i1 + HALF]);
  f2 x2 = f2_mk(a[i2], a[i2 + HALF]), x3 = f2_mk(a[i3], a[i3 + HALF]);
  const f2 wr = f2_bc(w.c), wi = f2_bc(-w.s), nwi = f2_bc(w.s);
  if (INV) bfly_inv2(x0, x1, x2, x3, wr, wi, nwi);
  else bfly_fwd2(x0, x1, x2, x3, wr, wi, nwi);
  a[i0] = x0.x; a[i0 + HALF] = x0.y;
  a[i1] = x1.x; a[i1 + HALF] = x1.y;
  a[i2] = x2.x; a[i2 + HALF] = x2.y;
  a[i3] = x3.x; a[i3 + HALF] = x3.y;
}

// Stage M on the blocks of a[OFF, OFF + HALF) and, identically, of the upper half.
template <int M, int HALF, int OFF, bool INV, int E>
RD_HD void stage_paired(float (&a)[E]) {
  static_assert(HALF % M == 0 && OFF + 2 * HALF <= E, "paired stage range");
#pragma unroll
  for (int b = OFF; b < OFF + HALF; b += M) {
    const f2 x0 = f2_mk(a[b], a[b + HALF]), x1 = f2_mk(a[b + M / 2], a[b + M / 2 + HALF]);
    const f2 s = f2_add(x0, x1), d = f2_sub(x0, x1);
    a[b] = s.x; a[b + HALF] = s.y;
    a[b + M / 2] = d.x; a[b + M / 2 + HALF] = d.y;
    if (M >= 4) {
      constexpr int q1 = M / 4, q3 = 3 * M / 4;
      if (INV) {
        const f2 y1 = f2_mul(f2_mk(a[b + q1], a[b + q1 + HALF]), f2_bc(2.0f));
        const f2 y3 = f2_mul(f2_mk(a[b + q3], a[b + q3 + HALF]), f2_bc(-2.0f));
        a[b + q1] = y1.x; a[b + q1 + HALF] = y1.y;
        a[b + q3] = y3.x; a[b + q3 + HALF] = y3.y;
      } else {
        const f2 y3 = f2_mul(f2_mk(a[b + q3], a[b + q3 + HALF]), f2_bc(-1.0f));
        a[b + q3] = y3.x; a[b + q3 + HALF] = y3.y;
      }
    }
#pragma unroll
    for (int k = 1; k < M / 4; ++k)
      bfly_pair<INV, HALF>(a, b + k, b + M / 2 - k, b + M / 2 + k, b + M - k, tw_const(tw_index(M, k)));
  }
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
// Stage M of a block of NB registers: on pairs while M <= NB/2, else scalar.
template <int M, int NB, int OFF, bool INV, int E>
RD_HD void stage_block(float (&a)[E]) {
  if constexpr (M <= NB / 2) stage_paired<M, NB / 2, OFF, INV>(a);
  else stage_contig<M, NB, OFF, INV>(a);
}

template <int MLO, int MHI, int NB, int OFF, bool INV, int E>
RD_HD void stages_contig(float (&a)[E]) {
  if constexpr (MLO <= MHI) {
    if constexpr (!INV) {
      stage_block<MLO, NB, OFF, false>(a);
      stages_contig<MLO * 2, MHI, NB, OFF, false>(a);
    } else {
      stage_block<MHI, NB, OFF, true>(a);
      stages_contig<MLO, MHI / 2, NB, OFF, true>(a);
    }
  }
}

// Twiddles of orbit stage U (M' = U*H) for s < U/4 from one loaded value
// B = W_M'^r: W_M'^(s*H + r) = W_U^s * B and W_M'^((s+1)*H - r) = W_U^(s+1) * conj(B),
// with W_U^s compile-time; W_U^0 = 1 and W_U^(U/4) = -i make those cases exact. So a
// stage loads one lane-dependent twiddle instead of U/2 (Tw {c, s} is c - i s).
template <int U, int S>
RD_HD void orbit_twiddles(Tw B, Tw& w1, Tw& w2) {
  if constexpr (S == 0) {
    w1 = B;
  } else {
    const Tw c = tw_const(tw_index(U, S));
    w1 = Tw{fmaf(c.c, B.c, -(c.s * B.s)), fmaf(c.c, B.s, c.s * B.c)};
  }
  if constexpr (S + 1 == U / 4) {
    w2 = Tw{B.s, B.c};
  } else {
    const Tw d = tw_const(tw_index(U, S + 1));
    w2 = Tw{fmaf(d.c, B.c, d.s * B.s), fmaf(d.s, B.c, -(d.c * B.s))};
  }
}

template <int U, int S = 0>
RD_HD void orbit_stage_twiddles(int s, Tw B, Tw& w1, Tw& w2) {
  if constexpr (S < U / 4) {
    if (s == S) orbit_twiddles<U, S>(B, w1, w2);
    else orbit_stage_twiddles<U, S + 1>(s, B, w1, w2);
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
    const Tw B = tw_lane(tw_index(MP, 0) + r);
#pragma unroll
    for (int s = 0; s < U / 4; ++s) {
      Tw w1, w2;
      orbit_stage_twiddles<U>(s, B, w1, w2);
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

// Stage U <= UMAX/2 of a generic orbit on pairs: block m0 of the lower half of the
// orbit (m < UMAX/2, elements OFF .. OFF + UMAX) with block m0 + UMAX/2 (elements
// + UMAX), which takes the same twiddles.
template <int H, int UMAX, int U, int OFF, bool INV, int E>
RD_HD void orbit_stage_paired(float (&a)[E], int r) {
  constexpr int MP = U * H;
  constexpr int U2 = U / 2;
  constexpr int HALF = UMAX;
  if constexpr (U == 2) {
    const Tw w = tw_lane(tw_index(MP, 0) + r);
#pragma unroll
    for (int m0 = 0; m0 < UMAX / 2; m0 += 2)
      bfly_pair<INV, HALF>(a, OFF + 2 * m0, OFF + 2 * m0 + 1, OFF + 2 * m0 + 2, OFF + 2 * m0 + 3, w);
  } else {
    const Tw B = tw_lane(tw_index(MP, 0) + r);
#pragma unroll
    for (int s = 0; s < U / 4; ++s) {
      Tw w1, w2;
      orbit_stage_twiddles<U>(s, B, w1, w2);
#pragma unroll
      for (int m0 = 0; m0 < UMAX / 2; m0 += U) {
        bfly_pair<INV, HALF>(a, OFF + 2 * (m0 + s), OFF + 2 * (m0 + U2 - s - 1) + 1, OFF + 2 * (m0 + U2 + s),
                             OFF + 2 * (m0 + U - s - 1) + 1, w1);
        bfly_pair<INV, HALF>(a, OFF + 2 * (m0 + s) + 1, OFF + 2 * (m0 + U2 - s - 1), OFF + 2 * (m0 + U2 + s) + 1,
                             OFF + 2 * (m0 + U - s - 1), w2);
      }
    }
  }
}

template <int H, int UMAX, int U, int OFF, bool INV, int E>
RD_HD void orbit_stage_any(float (&a)[E], int r) {
  if constexpr (U <= UMAX / 2) orbit_stage_paired<H, UMAX, U, OFF, INV>(a, r);
  else orbit_stage<H, UMAX, U, OFF, INV>(a, r);
}

template <int H, int UMAX, int U, int OFF, bool INV, int E>
RD_HD void orbit_stages(float (&a)[E], int r) {
  if constexpr (U <= UMAX) {
    if constexpr (!INV) {
      orbit_stage_any<H, UMAX, U, OFF, false>(a, r);
      orbit_stages<H, UMAX, U * 2, OFF, false>(a, r);
    } else {
      orbit_stages<H, UMAX, U * 2, OFF, true>(a, r);
      orbit_stage_any<H, UMAX, U, OFF, true>(a, r);
    }
  }
}

// ------------------------------------------------------------------------ plan
// Geometry of a row transform: row length P and elements per thread E (pass 0 runs
// stages 1..e on contiguous blocks of E = 2^e; pass k >= 1 covers stages s0+1..s1
// with s0 = e + (k-1)(e-1), s1 = min(s0 + e - 1, L)), and the padded tile layout:
// word G (row lrow, element n at G = lrow*P + n) lives at G + (G >> S), one pad word
// per 2^S words. S is chosen per geometry so that the 32 lanes of every pass-0
// scatter and orbit gather/scatter fall in distinct banks (checked by a bank model),
// and because every row/block base is a multiple of 2^S, each access is a per-thread
// base register plus a compile-time offset.
template <int P_, int EPT_, int SKEW_ = 0>
struct Geo {
  static constexpr int P = P_;
  static_assert(P >= 2 && P <= kMaxP && (P & (P - 1)) == 0, "p must be a power of two in [2, 4096]");
  static constexpr int L = ilog2(P);
  static constexpr int E = P < EPT_ ? P : EPT_;
  static constexpr int e = ilog2(E);
  static constexpr int TPR = P / E;               // threads per row
  static constexpr int LOG_TPR = ilog2(TPR);
  static constexpr int NPASS = (L <= e) ? 1 : 1 + (L - e + (e - 2)) / (e - 1);
  RD_HD static constexpr int s0(int k) { return e + (k - 1) * (e - 1); }
  RD_HD static constexpr int s1(int k) { return s0(k) + e - 1 < L ? s0(k) + e - 1 : L; }
  static constexpr int S = (E <= 32) ? (P >= 4096 ? 7 : (P >= 2048 ? 6 : 5)) : e;
  // offset of element n within its row (n + one pad word per 2^S)
  RD_HD static constexpr int at(int n) { return n + (n >> S); }
  // Row r starts at r * RS plus one extra word per RW rows, RW being the rows that
  // share a warp (32 / TPR, or 1): rows of one warp keep the bank pattern above, and
  // the 32 rows whose merged orbits one warp processes get 32 distinct bank offsets.
  // When a warp never spans two rows (RW = 1), row r is shifted by SKEW_ * r words
  // instead; that moves no access of a warp relative to another, only the merged
  // orbits of different rows, which one warp processes together.
  static constexpr int RS = P + (P >> S);
  static constexpr int RW = TPR < 32 ? 32 / TPR : 1;
  RD_HD static constexpr int row_base(int r) { return r * RS + (RW > 1 ? r / RW : SKEW_ * r); }
  // words of a tile of `rows` rows (plus one spare word)
  RD_HD static constexpr int words(int rows) { return row_base(rows) + 1; }
};

// The geometry of the standalone transforms. Rows of p >= 1024 (one warp or more per
// row) are skewed by 4 words: the merged orbits of pass 1, one per (row, block), then
// fall in distinct banks (at p = 1024 they were 4-way conflicts, 18% of the kernel's
// shared-memory wavefronts in a bank model of all its accesses).
template <int P>
using RowGeo = Geo<P, ept_for(P), 4>;

// The geometry of the layer kernels' tiles: 32 elements per thread. Their tiles hold up
// to 16 rows at p >= 1024 (grad_c), so rows are skewed by one word: one warp's merged
// orbits, (row, block) pairs, then cover 32 distinct banks.
template <int P>
using LayerGeo = Geo<P, kEPT, 1>;

template <class G, int K>
struct PassShape {
  static constexpr int H = 1 << G::s0(K);
  static constexpr int LB = 1 << G::s1(K);
  static constexpr int UMAX = LB / H;
  static constexpr int N = 2 * UMAX;              // elements per orbit
  static constexpr int C = G::E / N;              // orbits per thread
  static constexpr int HH = H / 2;                // orbits per block of LB
  static constexpr int NB = G::P / LB;            // blocks (merged orbits) per row
};

// ------------------------------------------------------------- per-thread passes
// `tile` is the CTA's shared (or, in the emulator, host) fp32 row tile; `lrow` the
// thread's row in the tile, `v` its index within the row's TPR threads; `g` the row
// in global memory (valid only when `active`).

// Forward pass 0: bit-reversed gather (lane v reads v + TPR*j', coalesced), stages
// 2..E in registers, scatter of block t = bitrev(v) to the tile row.
template <class G, typename T>
RD_HD void fwd_pass0_load(float (&a)[G::E], int v, const T* g, bool active) {
#pragma unroll
  for (int jp = 0; jp < G::E; ++jp) a[bitrev(jp, G::e)] = active ? ld(g + v + G::TPR * jp) : 0.0f;
}

// The same gather from a tile row (for a transform whose input already sits in
// shared memory); the caller puts a barrier between this and fwd_pass0_finish, as
// the scatter overwrites positions other threads gather.
// Element TPR*j' + v sits at [v + (v>>S)] + [TPR*j' + ((TPR*j')>>S)]: TPR*j' is a
// multiple of TPR and, when TPR < 2^S, TPR*j' mod 2^S + v < 2^S.
template <class G>
RD_HD void fwd_pass0_load_tile(float (&a)[G::E], int v, const float* trow) {
  const float* src = trow + v + (v >> G::S);
#pragma unroll
  for (int jp = 0; jp < G::E; ++jp) {
    const int n = G::TPR * jp;
    a[bitrev(jp, G::e)] = src[n + (n >> G::S)];
  }
}

template <class G>
RD_HD void fwd_pass0_finish(float (&a)[G::E], int v, float* trow) {
  stages_contig<2, G::E, G::E, 0, false>(a);
  const int t = bitrev(v, G::LOG_TPR);
  float* dst = trow + G::at(t * G::E);          // block start, a multiple of 2^S
#pragma unroll
  for (int j = 0; j < G::E; ++j) dst[j + (j >> G::S)] = a[j];
}

template <class G, typename T>
RD_HD void fwd_pass0(float* tile, int lrow, int v, const T* g, bool active) {
  float a[G::E];
  fwd_pass0_load<G, T>(a, v, g, active);
  fwd_pass0_finish<G>(a, v, tile + G::row_base(lrow));
}

// Inverse pass 0 (the last inverse step): gather block t from the tile, inverse
// stages E..2, scale by 1/P, scatter to global at the bit-reversed positions.
template <class G, typename T>
RD_HD void inv_pass0(const float* tile, int lrow, int v, T* g, bool active) {
  float a[G::E];
  const int t = bitrev(v, G::LOG_TPR);
  const float* src = tile + G::row_base(lrow) + G::at(t * G::E);
#pragma unroll
  for (int j = 0; j < G::E; ++j) a[j] = src[j + (j >> G::S)];
  stages_contig<2, G::E, G::E, 0, true>(a);
  constexpr float scale = 1.0f / G::P;
  if (active) {
#pragma unroll
    for (int j = 0; j < G::E; ++j) g[v + G::TPR * bitrev(j, G::e)] = from_f32<T>(a[j] * scale);
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

// Orbit assignment of slot CI of pass K to thread v of its row: o = v + TPR*CI,
// block beta = o / (H/2), residue rho = o % (H/2) (rho = 0: the merged orbit). In
// pass 1 of rows with >= 32 threads and 16 residues per block, the two half-warps
// take blocks NB/2 apart, so that their residues fall in opposite halves of the banks.
template <class G, int K>
RD_HD void orbit_of(int v, int CI, int& beta, int& rho) {
  using S = PassShape<G, K>;
  if constexpr (K == 1 && G::TPR >= 32 && S::HH == 16 && S::C == 1 && S::NB >= 2) {
    const int lane = v & 31;
    beta = (v >> 5) + (lane >> 4) * (S::NB / 2);
    rho = lane & 15;
  } else {
    const int o = v + G::TPR * CI;
    beta = o / S::HH;
    rho = o % S::HH;
  }
}

// Mirror epilogue of the last pass (Hartley form of the inverse): with P the packed
// forward transform of the mirrored spectrum, x_n = (P[n] - P[N-n]) / N and
// x_{N-n} = (P[n] + P[N-n]) / N for 0 < n < N/2, x_0 = P[0] / N, x_{N/2} = P[N/2] / N.
// `lo` and `hi` hold P at n < N/2 and N - n.
RD_HD void mirror_pair(float& lo, float& hi, float scale) {
  const float a = lo, b = hi;
  lo = (a - b) * scale;
  hi = (a + b) * scale;
}

// Generic slots CI.. of a middle/last pass K >= 1 for thread v of the tile row at
// `trow` (global row g). SRC/DST: 0 = tile, 1 = global row (natural order). Each
// generic orbit is gathered, transformed and written back to the same positions, so
// a pass needs no synchronisation inside itself. A slot whose residue is 0 (the
// merged orbit) is skipped here: the merged orbits of all rows are done by
// merged_orbit() below, one per thread, so that no warp runs both code paths.
// EPI = 1 (last pass only, LB = P) applies the mirror epilogue before the store:
// the mirror of element 2m (position mH + r) is element 2(U-1-m)+1, in the same orbit.
// Tile addresses: with R0 = block base (a multiple of 2^S) and c a compile-time
// multiple of 32, the element at R0 + c + r sits at [R0 + (R0>>S) + r + (r>>S)] +
// [c + (c>>S)] and the one at R0 + c - r (1 <= r) at [R0 + (R0>>S) - r - ((r-1)>>S)] +
// [c + ((c-1)>>S)]: a per-thread base plus an immediate.
template <class G, int K, bool INV, int SRC, int DST, int EPI, int CI, typename T, int E>
RD_HD void generic_slots(float (&a)[E], float* trow, int v, T* g, bool active) {
  using S = PassShape<G, K>;
  constexpr int SH = G::S;
  if constexpr (CI < S::C) {
    constexpr int OFF = CI * S::N;
    int beta, rho;
    orbit_of<G, K>(v, CI, beta, rho);
    if (rho != 0) {
      const int base = beta * S::LB;
      float* tbase = trow + G::at(base);
      float* tp = tbase + rho + (rho >> SH);
      float* tm = tbase - rho - ((rho - 1) >> SH);
      T* gp = g + base + rho;
      T* gm = g + base - rho;
#pragma unroll
      for (int m = 0; m < S::UMAX; ++m) {
        const int cp = m * S::H, cm = (m + 1) * S::H;
        a[OFF + 2 * m] = SRC == 0 ? tp[cp + (cp >> SH)] : (active ? ld(gp + cp) : 0.0f);
        a[OFF + 2 * m + 1] = SRC == 0 ? tm[cm + ((cm - 1) >> SH)] : (active ? ld(gm + cm) : 0.0f);
      }
      orbit_stages<S::H, S::UMAX, 2, OFF, INV>(a, rho);
      if constexpr (EPI == 1) {
        static_assert(S::LB == G::P && DST == 1, "mirror epilogue: last pass to global");
        constexpr float scale = 1.0f / G::P;
#pragma unroll
        for (int m = 0; m < S::UMAX / 2; ++m)
          mirror_pair(a[OFF + 2 * m], a[OFF + 2 * (S::UMAX - 1 - m) + 1], scale);
#pragma unroll
        for (int m = S::UMAX / 2; m < S::UMAX; ++m)
          mirror_pair(a[OFF + 2 * (S::UMAX - 1 - m) + 1], a[OFF + 2 * m], scale);
      }
#pragma unroll
      for (int m = 0; m < S::UMAX; ++m) {
        const int cp = m * S::H, cm = (m + 1) * S::H;
        if (DST == 0) {
          tp[cp + (cp >> SH)] = a[OFF + 2 * m];
          tm[cm + ((cm - 1) >> SH)] = a[OFF + 2 * m + 1];
        } else if (active) {
          gp[cp] = from_f32<T>(a[OFF + 2 * m]);
          gm[cm] = from_f32<T>(a[OFF + 2 * m + 1]);
        }
      }
    }
    generic_slots<G, K, INV, SRC, DST, EPI, CI + 1>(a, trow, v, g, active);
  }
}

template <class G, int K, bool INV, int SRC, int DST, typename T, int EPI = 0>
RD_HD void generic_pass(float* tile, int lrow, int v, T* g, bool active) {
  float a[G::E];
  generic_slots<G, K, INV, SRC, DST, EPI, 0>(a, tile + G::row_base(lrow), v, g, active);
}

// The merged orbit of block beta of the row at tile row lrow in pass K: positions
// base + l*H/2 (l < N) form a packed real transform of N points whose first stage
// (M = 2) is already done; run its stages 4..N (or N..4 inverse). EPI = 1 applies the
// mirror epilogue (pairs l, N - l; l = 0 and N/2 are their own mirrors).
template <class G, int K, bool INV, int SRC, int DST, typename T, int EPI = 0>
RD_HD void merged_orbit(float* tile, int lrow, int beta, T* g, bool active) {
  using S = PassShape<G, K>;
  constexpr int SH = G::S;
  float a[S::N];
  const int base = beta * S::LB;
  float* tbase = tile + G::row_base(lrow) + G::at(base);
#pragma unroll
  for (int l = 0; l < S::N; ++l) {
    const int c = l * S::HH;
    a[l] = SRC == 0 ? tbase[c + (c >> SH)] : (active ? ld(g + base + c) : 0.0f);
  }
  stages_contig<4, S::N, S::N, 0, INV>(a);
  if constexpr (EPI == 1) {
    static_assert(S::LB == G::P && DST == 1, "mirror epilogue: last pass to global");
    constexpr float scale = 1.0f / G::P;
    a[0] *= scale;
    a[S::N / 2] *= scale;
#pragma unroll
    for (int l = 1; l < S::N / 2; ++l) mirror_pair(a[l], a[S::N - l], scale);
  }
#pragma unroll
  for (int l = 0; l < S::N; ++l) {
    const int c = l * S::HH;
    if (DST == 0) tbase[c + (c >> SH)] = a[l];
    else if (active) g[base + c] = from_f32<T>(a[l]);
  }
}

}  // namespace rdfft
