// 2-D rdFFT of R x C images in place (sm_100a): the standalone row kernel over the
// image rows, and the column kernels of rdfft2d_steps.cuh (the forward runs rows
// then columns, the inverse columns then rows). Each half reads and writes every
// element once.
#include <cuda_runtime.h>

#include "internal.h"
#include "rdfft2d_steps.cuh"

namespace rdfft {

// Orbit passes K.. of the forward column transform, a barrier before each.
template <class G, int W, int NT, int K>
__device__ __forceinline__ void run_col_passes(float* tile, int tid) {
  if constexpr (K < G::NPASS) {
    __syncthreads();
    cols_orbit_pass<G, K>(tile, W, tid, NT);
    run_col_passes<G, W, NT, K + 1>(tile, tid);
  }
}

// One CTA per strip pair of one image (R >= 64). INV: un-combine + mirror, forward
// column transform, mirror + 1/R on the store; else forward transform and combine.
template <int R, bool INV, typename T>
__global__ void __launch_bounds__(ColTiling<R>::NT)
k_cols(T* __restrict__ data, int C, int ngroups) {
  using CT = ColTiling<R>;
  constexpr int W = CT::W, NT = CT::NT;
  using G = ColGeo<R, W>;
  constexpr int TPR = G::TPR;
  extern __shared__ float tile[];
  const int64_t img = blockIdx.x / ngroups;
  const int k0 = (int)(blockIdx.x - img * ngroups) * (W / 2);
  T* base = data + img * (int64_t)R * C;
  const int tid = threadIdx.x;

  if constexpr (INV) cols_load_unpair<G, W, NT, T>(tile, base, C, k0, tid);
  else cols_load<G, W, NT, T>(tile, base, C, k0, tid);
  __syncthreads();
  // pass 0 in place in the tile: every row of a round gathers, barrier, scatters
  const int v = tid % TPR;
  for (int r0 = 0; r0 < W; r0 += NT / TPR) {
    const int r = r0 + tid / TPR;
    float a[G::E];
    if (r < W) fwd_pass0_load_tile<G>(a, v, tile + G::row_base(r));
    __syncthreads();
    if (r < W) fwd_pass0_finish<G>(a, v, tile + G::row_base(r));
  }
  run_col_passes<G, W, NT, 1>(tile, tid);
  __syncthreads();
  if constexpr (INV) cols_store_inv<G, W, NT, T>(tile, base, C, k0, tid);
  else cols_store_fwd<G, W, NT, T>(tile, base, C, k0, tid);
}

// Columns of R <= 32: one thread per (image, left column k <= C/2).
template <int R, bool INV, typename T>
__global__ void __launch_bounds__(128) k_cols_small(T* __restrict__ data, int64_t images, int C) {
  const int nk = C / 2 + 1;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= images * nk) return;
  const int64_t img = t / nk;
  col_small<R, INV, T>(data + img * (int64_t)R * C, C, (int)(t - img * nk));
}

template <int R, bool INV, typename T>
static cudaError_t launch_cols_r(T* data, int64_t images, int C, cudaStream_t s) {
  if constexpr (R <= 32) {
    const int64_t threads = images * (C / 2 + 1);
    const int64_t grid = (threads + 127) / 128;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    k_cols_small<R, INV, T><<<(unsigned)grid, 128, 0, s>>>(data, images, C);
  } else {
    using CT = ColTiling<R>;
    using G = ColGeo<R, CT::W>;
    const int ngroups = col_groups(C, CT::W / 2);
    const int64_t grid = images * ngroups;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const size_t smem = sizeof(float) * (size_t)G::words(CT::W);
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(k_cols<R, INV, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
      if (e != cudaSuccess) return e;
    }
    k_cols<R, INV, T><<<(unsigned)grid, CT::NT, smem, s>>>(data, C, ngroups);
  }
  return cudaGetLastError();
}

template <bool INV, typename T>
static cudaError_t launch_cols_t(T* data, int64_t images, int R, int C, cudaStream_t s) {
  switch (R) {
    case 2: return launch_cols_r<2, INV, T>(data, images, C, s);
    case 4: return launch_cols_r<4, INV, T>(data, images, C, s);
    case 8: return launch_cols_r<8, INV, T>(data, images, C, s);
    case 16: return launch_cols_r<16, INV, T>(data, images, C, s);
    case 32: return launch_cols_r<32, INV, T>(data, images, C, s);
    case 64: return launch_cols_r<64, INV, T>(data, images, C, s);
    case 128: return launch_cols_r<128, INV, T>(data, images, C, s);
    case 256: return launch_cols_r<256, INV, T>(data, images, C, s);
    case 512: return launch_cols_r<512, INV, T>(data, images, C, s);
    case 1024: return launch_cols_r<1024, INV, T>(data, images, C, s);
    case 2048: return launch_cols_r<2048, INV, T>(data, images, C, s);
    case 4096: return launch_cols_r<4096, INV, T>(data, images, C, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_cols(void* data, int64_t images, int R, int C, int dtype, bool inverse, cudaStream_t s) {
  if (dtype == 0) {
    float* d = static_cast<float*>(data);
    return inverse ? launch_cols_t<true>(d, images, R, C, s) : launch_cols_t<false>(d, images, R, C, s);
  }
  bf16_t* d = static_cast<bf16_t*>(data);
  return inverse ? launch_cols_t<true>(d, images, R, C, s) : launch_cols_t<false>(d, images, R, C, s);
}

}  // namespace rdfft
