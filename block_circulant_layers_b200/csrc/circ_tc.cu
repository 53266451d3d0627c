// Block-circulant layer forward and grad_x with the per-bin contraction on the
// fifth-generation tensor cores (tcgen05.mma, kind::tf32, fp32 accumulation in tensor
// memory), for D = 4096 split into q = 32 blocks of p = 128, bf16 activations.
//
// "Memory-Efficient Training with In-Place FFT Implementation", paper-notes page,
// "Circulant matrix training adaptation": y_i = IFFT( sum_j FFT(c_ij) (.) FFT(x_j) ).
// For one frequency bin k of the packed spectra this sum is a complex q x q matrix
// times a q-vector per token, i.e. for TT tokens at once a small complex GEMM:
//     [Yr; Yi] = [Cr; Ci] Xr + [-Ci; Cr] Xi       (64 x N, K = 32 each)
// with Cr, Ci the real and imaginary parts of c_hat at bin k (i rows, j columns), and
// Xr, Xi those of the tokens' input spectra (N = 8 token columns, TT of them real).
// grad_x uses conj(c_hat) transposed: [Yr; Yi] = [Cr^T; -Ci^T] Gr + [Ci^T; Cr^T] Gi.
// Both A operands are windows of one 96 x 32 stack S = [s0 Ci; Cr; s2 Ci] (signs and
// transposition by direction): A2 = rows 0..63 and A1 = rows 32..95, so a bin takes
// 12 KB of shared memory instead of 16.
//
// A CTA owns TT = 4 tokens and all 32 output blocks:
//   1. rdFFT of the TT x 32 input rows from HBM into an fp32 tile (packed_fft.cuh);
//   2. bins 0 and p/2 (real) on CUDA cores, kept in registers;
//   3. bins 1..63 in chunks of 4 through a two-slot shared-memory ring: every thread
//      builds the chunk's A stacks from c_hat (L2) and copies the chunk's X columns
//      from the tile into B operands; one thread issues 8 MMAs per bin and commits
//      them to the slot's mbarrier, which the builders wait on before reusing the slot;
//   4. the accumulators (63 bins x 8 columns of tensor memory) are read back, written
//      over the tile as the output spectra, and rdIFFT'd (Hartley form) to HBM.
// tf32 keeps 10 mantissa bits of each operand (A and B are rounded to nearest), which
// stays far inside the bf16 I/O tolerance; fp32 I/O keeps the CUDA-core kernel.
#include <cuda_runtime.h>

#include "bulk_copy.cuh"
#include "circ_kernels.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace rdfft {
namespace {

constexpr int TC_P = 128;
constexpr int TC_Q = 32;
constexpr int TC_D = TC_P * TC_Q;
constexpr int TC_TT = 4;                     // tokens per CTA
constexpr int TC_N = 8;                      // MMA N (token columns; TT of them real)
constexpr int TC_NT = 256;
constexpr int TC_CB = 4;                     // bins per ring slot
constexpr int TC_NCHUNK = (TC_P / 2 - 1 + TC_CB - 1) / TC_CB;   // 63 complex bins -> 16 chunks
constexpr int TC_A_BYTES = 96 * TC_Q * 4;    // one bin's stack S: 96 rows x 32 tf32
constexpr int TC_B_BYTES = TC_N * TC_Q * 4;  // one of Xr / Xi: 8 x 32 tf32
constexpr int TC_BIN_BYTES = TC_A_BYTES + 2 * TC_B_BYTES;
constexpr int TC_SLOT_BYTES = TC_CB * TC_BIN_BYTES;
constexpr int TC_LBO = 128;                  // core matrices along K: adjacent
constexpr int TC_SBO = (TC_Q / 4) * 128;     // 8-row groups: one K row of 8 core matrices apart
constexpr int TC_TMEM_COLS = 512;            // 63 bins x 8 columns

using TG = LayerGeo<TC_P>;
constexpr int TC_TILE_BYTES = ((TG::words(TC_TT * TC_Q) * 4 + 127) / 128) * 128;
constexpr int TC_RING_OFF = TC_TILE_BYTES;
constexpr int TC_MBAR_OFF = TC_RING_OFF + 2 * TC_SLOT_BYTES;
constexpr int TC_SMEM_BYTES = TC_MBAR_OFF + 32;
static_assert(TC_SMEM_BYTES <= 227 * 1024, "shared memory of the tensor-core layer kernel");
static_assert(TC_RING_OFF % 128 == 0 && TC_SLOT_BYTES % 128 == 0 && TC_BIN_BYTES % 16 == 0, "16-byte operands");

// byte offset of element (row, kappa) of a K-major no-swizzle operand with 32 K columns
__device__ __forceinline__ int canon(int row, int kappa) {
  return (row >> 3) * TC_SBO + (kappa >> 2) * TC_LBO + (row & 7) * 16 + (kappa & 3) * 4;
}

// c_hat values of one chunk for this thread: per block `it`, Cr at slots k0 .. k0+3
// (k0 = 4c + 1: two aligned float4 from 4c) and Ci at slots p - k0 - 3 .. p - k0
// (= 124 - 4c .. 127 - 4c: one aligned float4). Thread lane l of warp w covers (row
// index r, column kappa) = (8 rh + l / 4, 4 kh + l % 4) with (rh, kh) = block w + 8 it:
// the 32 lanes of each shared-memory store then hit 32 distinct banks.
struct AChunk {
  float4 ca[4], cb[4], ci[4];
};

template <bool BWDX>
__device__ __forceinline__ void load_a(AChunk& a, const float* __restrict__ chat, int k0) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rl = lane >> 2, kl = lane & 3;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int blk = warp + 8 * it;            // 32 blocks of 8 x 4
    const int r = 8 * (blk >> 3) + rl, kap = 4 * (blk & 7) + kl;
    const int i = BWDX ? kap : r, j = BWDX ? r : kap;
    const float* crow = chat + (int64_t)(i * TC_Q + j) * TC_P;
    a.ca[it] = __ldg(reinterpret_cast<const float4*>(crow + (k0 - 1)));
    a.cb[it] = __ldg(reinterpret_cast<const float4*>(crow + (k0 + 3)));
    a.ci[it] = __ldg(reinterpret_cast<const float4*>(crow + (TC_P - k0 - 3)));
  }
}

// Writes the A stacks of the chunk's bins k0..k0+nb-1 into slot `ring` from the loaded
// values: forward S = [-Ci; Cr; Ci] with rows i, columns j; grad_x [Ci^T; Cr^T; -Ci^T].
template <bool BWDX>
__device__ __forceinline__ void store_a(unsigned char* ring, const AChunk& a, int nb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rl = lane >> 2, kl = lane & 3;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int blk = warp + 8 * it;
    const int r = 8 * (blk >> 3) + rl, kap = 4 * (blk & 7) + kl;
    const float crv[4] = {a.ca[it].y, a.ca[it].z, a.ca[it].w, a.cb[it].x};
    const float civ[4] = {a.ci[it].w, a.ci[it].z, a.ci[it].y, a.ci[it].x};
#pragma unroll
    for (int u = 0; u < TC_CB; ++u) {
      if (u < nb) {
        unsigned char* S = ring + u * TC_BIN_BYTES;
        const float cr = tc::to_tf32(crv[u]), cim = tc::to_tf32(civ[u]);
        *reinterpret_cast<float*>(S + canon(r, kap)) = BWDX ? cim : -cim;
        *reinterpret_cast<float*>(S + canon(32 + r, kap)) = cr;
        *reinterpret_cast<float*>(S + canon(64 + r, kap)) = BWDX ? -cim : cim;
      }
    }
  }
}

// Copies the chunk's input spectra (bins k0..k0+nb-1, the CTA's TT tokens, 32 blocks)
// from the tile into the slot's B operands (Xr then Xi, token t = row n, block = K).
__device__ __forceinline__ void build_b(unsigned char* ring, const float* tile, int k0, int nb) {
  for (int e = threadIdx.x; e < TC_CB * TC_TT * TC_Q; e += TC_NT) {
    const int u = e / (TC_TT * TC_Q);
    const int rem = e - u * (TC_TT * TC_Q);
    const int t = rem / TC_Q, j = rem - t * TC_Q;
    if (u < nb) {
      const int k = k0 + u;
      const int rb = TG::row_base(t * TC_Q + j);
      unsigned char* Bp = ring + u * TC_BIN_BYTES + TC_A_BYTES;
      *reinterpret_cast<float*>(Bp + canon(t, j)) = tc::to_tf32(tile[rb + TG::at(k)]);
      *reinterpret_cast<float*>(Bp + TC_B_BYTES + canon(t, j)) = tc::to_tf32(tile[rb + TG::at(TC_P - k)]);
    }
  }
}

template <bool BWDX>
__global__ void __launch_bounds__(TC_NT, 1)
k_circ_x_tc(const bf16_t* __restrict__ in, const float* __restrict__ chat, bf16_t* __restrict__ out, int64_t B) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float* tile = reinterpret_cast<float*>(smem);
  unsigned char* ring0 = smem + TC_RING_OFF;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + TC_MBAR_OFF);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + TC_MBAR_OFF + 16);
  const int64_t tok0 = (int64_t)blockIdx.x * TC_TT;
  const int ntok = (int)((B - tok0) < TC_TT ? (B - tok0) : TC_TT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  griddep_wait();                              // earlier work in the stream is done
  if (warp == 0) tc::tmem_alloc(tmem_holder, TC_TMEM_COLS);
  if (threadIdx.x == 0) {
    mbar_init(&mbar[0], 1);
    mbar_init(&mbar[1], 1);
  }
  // token columns TT..N-1 of every B operand stay zero
  for (int e = threadIdx.x; e < 2 * TC_CB * 2 * (TC_N - TC_TT) * TC_Q; e += TC_NT) {
    const int q2 = e / ((TC_N - TC_TT) * TC_Q);
    const int rem = e - q2 * ((TC_N - TC_TT) * TC_Q);
    const int t = TC_TT + rem / TC_Q, j = rem % TC_Q;
    const int slot = q2 / (2 * TC_CB), u = (q2 / 2) % TC_CB, part = q2 & 1;
    *reinterpret_cast<float*>(ring0 + slot * TC_SLOT_BYTES + u * TC_BIN_BYTES + TC_A_BYTES + part * TC_B_BYTES +
                              canon(t, j)) = 0.0f;
  }

  // 1. rdFFT of the TT x 32 input rows into the tile (rows of absent tokens are zero)
  fft_rows<TC_P, TC_NT, bf16_t>(tile, TC_TT * TC_Q, [&](int r) -> const bf16_t* {
    const int t = r / TC_Q, b = r - t * TC_Q;
    return t < ntok ? in + (tok0 + t) * (int64_t)TC_D + (int64_t)b * TC_P : nullptr;
  });
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  // 2. bins 0 and p/2: one (output block, slot, token) per thread, kept until the end
  float y_real;
  {
    const int o = threadIdx.x & 31, part = (threadIdx.x >> 5) & 1, t = threadIdx.x >> 6;
    const int slot = part ? TC_P / 2 : 0;
    float acc = 0.0f;
#pragma unroll
    for (int s = 0; s < TC_Q; ++s) {
      const int i = BWDX ? s : o, j = BWDX ? o : s;
      acc = fmaf(__ldg(chat + (int64_t)(i * TC_Q + j) * TC_P + slot), tile[TG::row_base(t * TC_Q + s) + TG::at(slot)],
                 acc);
    }
    y_real = acc;
  }

  // 3. bins 1..63 through the ring; the c_hat values of chunk c + 1 are requested
  // before chunk c is stored, so their L2 latency overlaps a whole chunk
  const uint32_t idesc = tc::idesc_tf32(64, TC_N);
  bool ok = true;
  AChunk pre;
  load_a<BWDX>(pre, chat, 1);
  for (int c = 0; c < TC_NCHUNK; ++c) {
    const int slot = c & 1;
    unsigned char* ring = ring0 + slot * TC_SLOT_BYTES;
    const int k0 = TC_CB * c + 1;
    const int nb = (TC_P / 2 - k0) < TC_CB ? (TC_P / 2 - k0) : TC_CB;
    const AChunk cur = pre;
    if (c + 1 < TC_NCHUNK) load_a<BWDX>(pre, chat, k0 + TC_CB);
    if (c >= 2) {
      // the MMAs that read this slot two chunks ago have completed
      ok = ok && mbar_wait_bounded(&mbar[slot], ((c - 2) >> 1) & 1);
      tc::fence_after_sync();
    }
    store_a<BWDX>(ring, cur, nb);
    build_b(ring, tile, k0, nb);
    fence_smem_to_async();                    // generic-proxy stores -> tensor-core reads
    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc::fence_after_sync();
      for (int u = 0; u < nb; ++u) {
        const uint32_t sa = tc::smem_u32(ring + u * TC_BIN_BYTES);
        const uint32_t sb = sa + TC_A_BYTES;
        const uint32_t d = tmem + (uint32_t)((k0 + u - 1) * TC_N);
#pragma unroll
        for (int ks = 0; ks < TC_Q / 8; ++ks)   // [Cr; Ci] (rows 32..95) x Xr
          tc::mma_tf32(d, tc::smem_desc(sa + 4 * TC_SBO + ks * 2 * TC_LBO, TC_LBO, TC_SBO),
                       tc::smem_desc(sb + ks * 2 * TC_LBO, TC_LBO, TC_SBO), idesc, ks > 0);
#pragma unroll
        for (int ks = 0; ks < TC_Q / 8; ++ks)   // [-Ci; Cr] (rows 0..63) x Xi
          tc::mma_tf32(d, tc::smem_desc(sa + ks * 2 * TC_LBO, TC_LBO, TC_SBO),
                       tc::smem_desc(sb + TC_B_BYTES + ks * 2 * TC_LBO, TC_LBO, TC_SBO), idesc, 1u);
      }
      tc::mma_commit(&mbar[slot]);
    }
  }
  // the last commit covers every MMA issued before it
  constexpr int LAST = TC_NCHUNK - 1;
  ok = ok && mbar_wait_bounded(&mbar[LAST & 1], (LAST >> 1) & 1);
  if (!__syncthreads_and(ok)) {
    // a wait gave up (error word set): wait once more for the MMAs, free the tensor
    // memory and leave the outputs unwritten
    mbar_wait_bounded(&mbar[LAST & 1], (LAST >> 1) & 1);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, TC_TMEM_COLS);
    return;
  }
  tc::fence_after_sync();

  // 4. accumulators -> output spectra over the tile. Warp w reads lane quarter w % 4,
  // i.e. rows 16 (w % 4) .. + 15 of every bin (lanes 0..15): Yr of output blocks
  // 0..31 for quarters 0, 1 and Yi for quarters 2, 3; warps w and w + 4 split the bins.
  {
    const int quarter = warp & 3, half = warp >> 2;
    const int m = 16 * quarter + lane;        // accumulator row (valid for lane < 16)
    const int o = m & 31;
    const bool im = m >= 32;
    // 32 bins per half (the last half has 31): four bins per batch of loads, one wait
    const int kb = half ? 33 : 1;
    const int nbin = half ? TC_P / 2 - 33 : 32;
    for (int k4 = 0; k4 < nbin; k4 += 4) {
      float v[4][8];
      const uint32_t base = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)((kb + k4 - 1) * TC_N);
      tc::tmem_ld8x4(base, v);
      if (lane < 16) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = kb + k4 + u;
          if (k4 + u < nbin) {
            const int slot = im ? TC_P - k : k;
#pragma unroll
            for (int t = 0; t < TC_TT; ++t) tile[TG::row_base(t * TC_Q + o) + TG::at(slot)] = v[u][t];
          }
        }
      }
    }
    // bins 0 and p/2 from registers
    {
      const int o2 = threadIdx.x & 31, part = (threadIdx.x >> 5) & 1, t = threadIdx.x >> 6;
      tile[TG::row_base(t * TC_Q + o2) + TG::at(part ? TC_P / 2 : 0)] = y_real;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, TC_TMEM_COLS);
  // mirrored form for the Hartley-form inverse: slot k = Re - Im, slot p - k = Re + Im
  for (int e = threadIdx.x; e < TC_TT * TC_Q * (TC_P / 2 - 1); e += TC_NT) {
    const int r = e / (TC_P / 2 - 1), k = 1 + e % (TC_P / 2 - 1);
    float* row = tile + TG::row_base(r);
    const float re = row[TG::at(k)], imv = row[TG::at(TC_P - k)];
    row[TG::at(k)] = re - imv;
    row[TG::at(TC_P - k)] = re + imv;
  }
  __syncthreads();
  griddep_launch_dependents();
  ifft_rows_mirrored<TC_P, TC_NT, bf16_t>(tile, TC_TT * TC_Q, [&](int r) -> bf16_t* {
    const int t = r / TC_Q, ob = r - t * TC_Q;
    return t < ntok ? out + (tok0 + t) * (int64_t)TC_D + (int64_t)ob * TC_P : nullptr;
  });
}

}  // namespace

bool circ_tc_supported(int p, int D, int dtype) { return p == TC_P && D == TC_D && dtype == 1; }

cudaError_t launch_circ_x_tc(const void* in, const float* chat, void* out, int64_t B, bool bwdx, cudaStream_t s) {
  const int64_t grid = (B + TC_TT - 1) / TC_TT;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  auto kern = bwdx ? k_circ_x_tc<true> : k_circ_x_tc<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TC_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3((unsigned)grid), dim3(TC_NT), (size_t)TC_SMEM_BYTES, s,
                    static_cast<const bf16_t*>(in), chat, static_cast<bf16_t*>(out), B);
}

cudaError_t take_tc_device_error(unsigned int* flags) {
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  *flags = v;
  return e;
}

}  // namespace rdfft
