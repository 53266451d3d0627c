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

// Both casts are bit copies. A CTA of 256 threads owns 256 / TPR rows at a time (grid-stride
// over row groups), TPR = p / (2 U) threads per row, at least MINT (and at most p/2 and 256);
// a thread handles the bins k = v + j TPR below p/2 in groups of U, issuing a group's loads
// before its stores (one 2-byte element per bin and thread keeps too few bytes in flight to
// cover the DRAM latency), and thread v = 0 also bin p/2. Across a warp the packed slots k
// and p - k run ascending and descending (coalesced), and a bin's (re, im) pair moves as one
// 32-bit (16-bit elements) or 64-bit (fp32) access: complex rows of p + 2 elements keep every
// pair aligned.
template <typename T> struct Pair;
template <> struct Pair<float> {
  typedef float2 V;
  static __device__ __forceinline__ V make(float re, float im) { return make_float2(re, im); }
  static __device__ __forceinline__ float re(V v) { return v.x; }
  static __device__ __forceinline__ float im(V v) { return v.y; }
};
template <> struct Pair<bf16_t> {
  typedef uint32_t V;
  static __device__ __forceinline__ V make(bf16_t re, bf16_t im) { return (uint32_t)re | ((uint32_t)im << 16); }
  static __device__ __forceinline__ bf16_t re(V v) { return (bf16_t)(v & 0xffffu); }
  static __device__ __forceinline__ bf16_t im(V v) { return (bf16_t)(v >> 16); }
};

struct CastShape {
  int tpr, rpc;                                 // threads per row, rows per CTA pass
  __host__ __device__ CastShape(int p, int U, int MINT) {
    int t = p / (2 * U);
    if (t < MINT) t = MINT;
    if (t > p / 2) t = p / 2;
    tpr = t < 1 ? 1 : (t > 256 ? 256 : t);
    rpc = 256 / tpr;
  }
};

// packed row of p reals -> p/2 + 1 (re, im) pairs; Im of bins 0 and p/2 is zero
template <typename T, int U, int MINT>
__global__ void __launch_bounds__(256) k_packed_to_complex(const T* __restrict__ packed, T* __restrict__ cplx,
                                                           int64_t rows, int p) {
  typedef typename Pair<T>::V V;
  const CastShape sh(p, U, MINT);
  const int v = threadIdx.x % sh.tpr;
  const int64_t r0 = threadIdx.x / sh.tpr;
  const int hb = p / 2;
  const T zero = T(0);
  for (int64_t row = (int64_t)blockIdx.x * sh.rpc + r0; row < rows; row += (int64_t)gridDim.x * sh.rpc) {
    const T* src = packed + row * p;
    V* dst = reinterpret_cast<V*>(cplx + row * (int64_t)(p + 2));
    for (int k0 = v; k0 < hb; k0 += U * sh.tpr) {
      T re[U], im[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int k = k0 + u * sh.tpr;
        if (k < hb) {
          re[u] = src[k];
          im[u] = k == 0 ? zero : src[p - k];
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int k = k0 + u * sh.tpr;
        if (k < hb) dst[k] = Pair<T>::make(re[u], im[u]);
      }
    }
    if (v == 0) dst[hb] = Pair<T>::make(src[hb], zero);
  }
}

// The same for short rows (p < 64), where a row has too few bins for a thread group: one
// thread per bin over the flat (row, bin) index, the pair as one access.
template <typename T>
__global__ void __launch_bounds__(256) k_packed_to_complex_flat(const T* __restrict__ packed,
                                                                T* __restrict__ cplx, int64_t rows, int p) {
  typedef typename Pair<T>::V V;
  const int nb = p / 2 + 1;
  const int64_t total = rows * nb;
  V* dst = reinterpret_cast<V*>(cplx);
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / nb;
    const int k = (int)(idx - row * nb);
    const T* src = packed + row * p;
    dst[idx] = Pair<T>::make(src[k], (k == 0 || k == p / 2) ? T(0) : src[p - k]);
  }
}

// p/2 + 1 (re, im) pairs -> packed row: slot k <- Re Y_k, slot p - k <- Im Y_k; the imaginary
// parts of Y_0 and Y_{p/2} are not read (zero for a real signal)
template <typename T, int U, int MINT>
__global__ void __launch_bounds__(256) k_complex_to_packed(const T* __restrict__ cplx, T* __restrict__ packed,
                                                           int64_t rows, int p) {
  typedef typename Pair<T>::V V;
  const CastShape sh(p, U, MINT);
  const int v = threadIdx.x % sh.tpr;
  const int64_t r0 = threadIdx.x / sh.tpr;
  const int hb = p / 2;
  for (int64_t row = (int64_t)blockIdx.x * sh.rpc + r0; row < rows; row += (int64_t)gridDim.x * sh.rpc) {
    const V* src = reinterpret_cast<const V*>(cplx + row * (int64_t)(p + 2));
    T* dst = packed + row * p;
    for (int k0 = v; k0 < hb; k0 += U * sh.tpr) {
      V y[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int k = k0 + u * sh.tpr;
        if (k < hb) y[u] = src[k];
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int k = k0 + u * sh.tpr;
        if (k < hb) {
          dst[k] = Pair<T>::re(y[u]);
          if (k != 0) dst[p - k] = Pair<T>::im(y[u]);
        }
      }
    }
    if (v == 0) dst[hb] = Pair<T>::re(src[hb]);
  }
}

static unsigned grid_for(int64_t rows, const CastShape& sh) {
  int64_t g = (rows + sh.rpc - 1) / sh.rpc;
  if (g > 148 * 8) g = 148 * 8;             // grid-stride beyond 8 CTAs of 256 threads per SM
  return (unsigned)(g > 0 ? g : 1);
}

template <typename T, int U, int MINT>
static void cast_to(const void* in, void* out, int64_t rows, int p, cudaStream_t s) {
  k_packed_to_complex<T, U, MINT><<<grid_for(rows, CastShape(p, U, MINT)), 256, 0, s>>>(
      static_cast<const T*>(in), static_cast<T*>(out), rows, p);
}

template <typename T, int U, int MINT>
static void cast_from(const void* in, void* out, int64_t rows, int p, cudaStream_t s) {
  k_complex_to_packed<T, U, MINT><<<grid_for(rows, CastShape(p, U, MINT)), 256, 0, s>>>(
      static_cast<const T*>(in), static_cast<T*>(out), rows, p);
}

// Shapes measured on B200 (128 MiB of packed rows, CUDA graphs, bit-identical outputs): to
// complex 8 bins per thread from p = 64 on (bf16 p = 512: 4239 against 2671 GB/s for one bin per
// thread over a flat index, which short rows keep); from complex 4 bins per thread with at
// least 32 threads per row (bf16 p = 512: 5050 against 1715 GB/s).
template <typename T>
static void cast_t(const void* in, void* out, int64_t rows, int p, bool to_complex, cudaStream_t s) {
  if (to_complex) {
    if (p < 64) {
      int64_t g = (rows * (p / 2 + 1) + 255) / 256;
      if (g > 148 * 32) g = 148 * 32;
      k_packed_to_complex_flat<T><<<(unsigned)(g > 0 ? g : 1), 256, 0, s>>>(static_cast<const T*>(in),
                                                                          static_cast<T*>(out), rows, p);
    } else {
      cast_to<T, 8, 8>(in, out, rows, p, s);
    }
  } else {
    cast_from<T, 4, 32>(in, out, rows, p, s);
  }
}

cudaError_t launch_convert(const void* in, void* out, int64_t rows, int p, int dtype, bool to_complex,
                           cudaStream_t s) {
  if (dtype == 0) cast_t<float>(in, out, rows, p, to_complex, s);
  else cast_t<bf16_t>(in, out, rows, p, to_complex, s);
  return cudaGetLastError();
}

}  // namespace rdfft
