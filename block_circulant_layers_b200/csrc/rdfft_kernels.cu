// Standalone batched rdFFT / rdIFFT kernels (sm_100a) and their launcher.
//
// One CTA of 128 threads owns a run of consecutive rows: for p >= 64 it owns
// 128 / (p/32) rows with p/32 threads per row, a staging buffer holding the rows as
// they are in HBM and an fp32 shared tile of about 16.5 KiB; for p <= 32 one thread
// owns one row. Every element is read once from HBM and written once, in place; no
// other global memory is touched apart from the twiddle tables (constant bank and an
// L1-cached global copy).
#include <cuda_runtime.h>

#include "bulk_copy.cuh"
#include "internal.h"
#include "rdfft_steps.cuh"

namespace rdfft {

template <class G, bool INV, int K, int ROWS, typename T, typename RowPtr, typename RowOk>
__device__ __forceinline__ void run_steps(float* tile, int lrow, int v, RowPtr rowptr, RowOk rowok) {
  if constexpr (K < G::NPASS) {
    if constexpr (K > 0) __syncthreads();
    row_step<G, INV, K, ROWS, T>(tile, lrow, v, rowptr, rowok);
    run_steps<G, INV, K + 1, ROWS, T>(tile, lrow, v, rowptr, rowok);
  }
}

// One CTA: ROWS consecutive rows, read from src and written to dst (the same rows for
// the in-place transforms; src and dst are therefore not restrict). For p >= 64 the
// rows travel between HBM and the staging buffer by bulk copies (the TMA engine, no
// per-element load or store instructions), and the passes read their first input from
// and write their last output to that buffer.
template <int P, bool INV, typename T>
__global__ void __launch_bounds__(RowTiling<P>::THREADS)
k_rows(const T* src, T* dst, int64_t rows) {
  constexpr int ROWS = RowTiling<P>::ROWS;
  griddep_wait();                                     // earlier work on these rows is done
  if constexpr (P <= 32) {
    const int64_t row = (int64_t)blockIdx.x * ROWS + threadIdx.x;
    if (row < rows) row_small<P, INV, T>(src + row * P, dst + row * P);
    griddep_launch_dependents();
  } else {
    using G = RowGeo<P>;
    using SM = RowSmem<P, T>;
    constexpr int TPR = G::TPR;
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* raw = smem;
    float* tile = reinterpret_cast<float*>(smem + SM::TILE_OFF);
    uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + SM::MBAR_OFF);
    const int64_t row0 = (int64_t)blockIdx.x * ROWS;
    const int nr = (int)((rows - row0) < ROWS ? (rows - row0) : ROWS);
    if (threadIdx.x == 0) {
      mbar_init(mbar, 1);
      mbar_arrive_expect_tx(mbar, (unsigned)(nr * SM::RAW_ROW));
      for (int r = 0; r < nr; ++r)
        bulk_load(raw + SM::raw_off(r), src + (row0 + r) * P, SM::RAW_ROW, mbar);
    }
    __syncthreads();                                  // the barrier exists before anyone waits
    const bool arrived = mbar_wait_bounded(mbar, 0);
    if (!__syncthreads_and(arrived)) {
      mbar_wait_bounded(mbar, 0);                     // give copies in flight a last chance
      return;
    }
    const int lrow = threadIdx.x / TPR;
    const int v = threadIdx.x % TPR;
    auto rowok = [&](int r) { return r < nr; };
    auto rowptr = [&](int r) { return reinterpret_cast<T*>(raw + SM::raw_off(r)); };
    run_steps<G, INV, 0, ROWS, T>(tile, lrow, v, rowptr, rowok);
    fence_smem_to_async();
    __syncthreads();
    griddep_launch_dependents();                      // the next launch may be scheduled
    if (threadIdx.x == 0) {
      for (int r = 0; r < nr; ++r) bulk_store(dst + (row0 + r) * P, raw + SM::raw_off(r), SM::RAW_ROW);
      bulk_commit();
      bulk_wait_read();
    }
  }
}

// Self-test of the bounded wait: an mbarrier that expects 16 bytes nobody sends.
__global__ void k_wait_selftest(long long limit_cycles) {
  __shared__ __align__(8) uint64_t mbar;
  mbar_init(&mbar, 1);
  mbar_arrive_expect_tx(&mbar, 16);
  mbar_wait_bounded(&mbar, 0, limit_cycles);
}

cudaError_t take_rows_device_error(unsigned int* flags) {
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  *flags = v;
  return e;
}

cudaError_t launch_wait_selftest(cudaStream_t s) {
  k_wait_selftest<<<1, 1, 0, s>>>(2000000LL);          // about a millisecond
  return cudaGetLastError();
}

template <int P, bool INV, typename T>
static cudaError_t launch_pi(const T* src, T* d, int64_t rows, cudaStream_t s) {
  constexpr int ROWS = RowTiling<P>::ROWS;
  const int64_t grid = (rows + ROWS - 1) / ROWS;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  size_t smem = 0;
  if constexpr (P > 32) {
    smem = RowSmem<P, T>::BYTES;
    if (smem > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(k_rows<P, INV, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
      if (e != cudaSuccess) return e;
    }
  }
  // programmatic stream serialization: the next rows launch in the stream can be
  // scheduled while this one drains; each CTA waits (griddep_wait) before touching data
  return launch_pdl(k_rows<P, INV, T>, dim3((unsigned)grid), dim3(RowTiling<P>::THREADS), smem, s, src, d, rows);
}

template <int P, typename T>
static cudaError_t launch_p(const void* src, void* data, int64_t rows, bool inverse, cudaStream_t s) {
  const T* x = static_cast<const T*>(src);
  T* d = static_cast<T*>(data);
  return inverse ? launch_pi<P, true, T>(x, d, rows, s) : launch_pi<P, false, T>(x, d, rows, s);
}

template <typename T>
static cudaError_t launch_t(const void* src, void* data, int64_t rows, int p, bool inverse, cudaStream_t s) {
  switch (p) {
    case 2: return launch_p<2, T>(src, data, rows, inverse, s);
    case 4: return launch_p<4, T>(src, data, rows, inverse, s);
    case 8: return launch_p<8, T>(src, data, rows, inverse, s);
    case 16: return launch_p<16, T>(src, data, rows, inverse, s);
    case 32: return launch_p<32, T>(src, data, rows, inverse, s);
    case 64: return launch_p<64, T>(src, data, rows, inverse, s);
    case 128: return launch_p<128, T>(src, data, rows, inverse, s);
    case 256: return launch_p<256, T>(src, data, rows, inverse, s);
    case 512: return launch_p<512, T>(src, data, rows, inverse, s);
    case 1024: return launch_p<1024, T>(src, data, rows, inverse, s);
    case 2048: return launch_p<2048, T>(src, data, rows, inverse, s);
    case 4096: return launch_p<4096, T>(src, data, rows, inverse, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_rows_to(const void* src, void* dst, int64_t rows, int p, int dtype, bool inverse, cudaStream_t s) {
  if (dtype == 0) return launch_t<float>(src, dst, rows, p, inverse, s);
  return launch_t<bf16_t>(src, dst, rows, p, inverse, s);
}

cudaError_t launch_rows(void* data, int64_t rows, int p, int dtype, bool inverse, cudaStream_t s) {
  return launch_rows_to(data, data, rows, p, dtype, inverse, s);
}

}  // namespace rdfft
