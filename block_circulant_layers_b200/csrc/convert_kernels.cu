// Conversions between the packed real layout of rdFFT and the rFFT complex layout.
//
// "Memory-Efficient Training with In-Place FFT Implementation", summary page,
// "Limitations": the frequency-domain information is encoded implicitly, so explicit
// access to the complex spectrum needs a cast that cannot stay in place (p reals vs
// p/2 + 1 complex values). These kernels are that cast, out of place into buffers the
// caller owns: packed row of p reals <-> p/2 + 1 interleaved (re, im) pairs.
#include <cuda_runtime.h>

#include "internal.h"
#include "packed_fft.cuh"

namespace rdfft {

// One thread per complex bin k of one row: reads slots k and p-k (bin 0: 0 and p/2).
template <typename T>
__global__ void k_packed_to_complex(const T* __restrict__ packed, T* __restrict__ cplx, int64_t rows, int p) {
  const int nb = p / 2 + 1;
  const int64_t total = rows * nb;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / nb;
    const int k = (int)(idx - row * nb);
    const T* src = packed + row * p;
    T* dst = cplx + 2 * idx;
    float re, im;
    if (k == 0) {
      re = to_f32(src[0]);
      im = 0.0f;
    } else if (k == p / 2) {
      re = to_f32(src[p / 2]);
      im = 0.0f;
    } else {
      re = to_f32(src[k]);
      im = to_f32(src[p - k]);
    }
    dst[0] = from_f32<T>(re);
    dst[1] = from_f32<T>(im);
  }
}

// One thread per packed slot n of one row: slot k <- Re Y_k, slot p-k <- Im Y_k; the
// imaginary parts of Y_0 and Y_{p/2} are not read (zero for a real signal).
template <typename T>
__global__ void k_complex_to_packed(const T* __restrict__ cplx, T* __restrict__ packed, int64_t rows, int p) {
  const int64_t total = rows * p;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / p;
    const int n = (int)(idx - row * p);
    const T* src = cplx + row * (int64_t)(p + 2);
    packed[idx] = n <= p / 2 ? src[2 * n] : src[2 * (p - n) + 1];
  }
}

static unsigned grid_for(int64_t work) {
  int64_t g = (work + 255) / 256;
  if (g > 148 * 32) g = 148 * 32;          // grid-stride beyond 32 CTAs per SM
  return (unsigned)(g > 0 ? g : 1);
}

cudaError_t launch_convert(const void* in, void* out, int64_t rows, int p, int dtype, bool to_complex,
                           cudaStream_t s) {
  if (to_complex) {
    const unsigned g = grid_for(rows * (p / 2 + 1));
    if (dtype == 0) k_packed_to_complex<float><<<g, 256, 0, s>>>((const float*)in, (float*)out, rows, p);
    else k_packed_to_complex<bf16_t><<<g, 256, 0, s>>>((const bf16_t*)in, (bf16_t*)out, rows, p);
  } else {
    const unsigned g = grid_for(rows * p);
    if (dtype == 0) k_complex_to_packed<float><<<g, 256, 0, s>>>((const float*)in, (float*)out, rows, p);
    else k_complex_to_packed<bf16_t><<<g, 256, 0, s>>>((const bf16_t*)in, (bf16_t*)out, rows, p);
  }
  return cudaGetLastError();
}

}  // namespace rdfft
