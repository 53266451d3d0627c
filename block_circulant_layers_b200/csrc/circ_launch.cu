// Block-circulant layer: dispatch on the block size p and the backward sequence.
#include <cuda_runtime.h>

#include "internal.h"
#include "pdl.cuh"

namespace rdfft {

cudaError_t circ_layer_64(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             GcSink*);
cudaError_t circ_layer_128(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             GcSink*);
cudaError_t circ_layer_256(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             GcSink*);
cudaError_t circ_layer_512(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             GcSink*);
cudaError_t circ_layer_1024(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             GcSink*);
cudaError_t circ_layer_2048(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             GcSink*);
cudaError_t circ_layer_4096(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             GcSink*);

static cudaError_t circ_layer(int p, int op, const void* a, const void* b, const float* chat, void* out,
                              float* gc, int64_t B, int q, int dtype, cudaStream_t s, GcSink* sink = nullptr) {
  switch (p) {
    case 64: return circ_layer_64(op, a, b, chat, out, gc, B, q, dtype, s, sink);
    case 128: return circ_layer_128(op, a, b, chat, out, gc, B, q, dtype, s, sink);
    case 256: return circ_layer_256(op, a, b, chat, out, gc, B, q, dtype, s, sink);
    case 512: return circ_layer_512(op, a, b, chat, out, gc, B, q, dtype, s, sink);
    case 1024: return circ_layer_1024(op, a, b, chat, out, gc, B, q, dtype, s, sink);
    case 2048: return circ_layer_2048(op, a, b, chat, out, gc, B, q, dtype, s, sink);
    case 4096: return circ_layer_4096(op, a, b, chat, out, gc, B, q, dtype, s, sink);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_circ_fwd(const void* x, const float* c_hat, void* y, int64_t B, int D, int p,
                            int dtype, cudaStream_t s) {
  return circ_layer(p, 0, x, nullptr, c_hat, y, nullptr, B, D / p, dtype, s);
}

// grad_c = sum over the token slices of their packed sums, in an order that depends on the
// slice count alone, so the result does not depend on which CTA finished first: for each
// float4 element, thread group r (of SPLIT) adds slices r, r + SPLIT, r + 2 SPLIT, ... in that
// order, then the SPLIT group sums are added in order r = 0, 1, ..., SPLIT - 1 (groups with no
// slice add an exact zero). Reads slices x n4 x 16 bytes once; SPLIT threads per element keep
// enough loads in flight when there are few elements and many slices.
constexpr int kSumSplit = 32;
constexpr int kSumThreads = 256;

__global__ void __launch_bounds__(kSumThreads) k_sum_slices(const float4* __restrict__ part, int64_t n4,
                                                            int slices, float4* __restrict__ out) {
  constexpr int EPB = kSumThreads / kSumSplit;     // elements per CTA
  __shared__ float4 group_sum[kSumSplit][EPB];
  griddep_wait();                                  // the slices' sums are complete
  const int el = threadIdx.x % EPB, r = threadIdx.x / EPB;
  const int64_t e = (int64_t)blockIdx.x * EPB + el;
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  if (e < n4) {
    for (int sl = r; sl < slices; sl += kSumSplit) {
      const float4 v = part[(int64_t)sl * n4 + e];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
  }
  group_sum[r][el] = acc;
  __syncthreads();
  griddep_launch_dependents();
  if (r == 0 && e < n4) {
    float4 t = group_sum[0][el];
#pragma unroll
    for (int j = 1; j < kSumSplit; ++j) {
      t.x += group_sum[j][el].x;
      t.y += group_sum[j][el].y;
      t.z += group_sum[j][el].z;
      t.w += group_sum[j][el].w;
    }
    out[e] = t;
  }
}

static cudaError_t launch_sum_slices(const float* part, int slices, int64_t n, float* out, cudaStream_t s) {
  const int64_t n4 = n / 4;                        // n = q^2 p, a multiple of 64
  constexpr int EPB = kSumThreads / kSumSplit;
  const int64_t blocks = (n4 + EPB - 1) / EPB;
  return launch_pdl(k_sum_slices, dim3((unsigned)blocks), dim3(kSumThreads), 0, s,
                    reinterpret_cast<const float4*>(part), n4, slices, reinterpret_cast<float4*>(out));
}

cudaError_t launch_circ_bwd(const void* g, const void* x, const float* c_hat, void* grad_x,
                            float* grad_c, int64_t B, int D, int p, int dtype, cudaStream_t s, GcSink* sink) {
  const int q = D / p;
  cudaError_t e = cudaSuccess;
  // after the grad_c kernel: the ordered sum of the slices (deterministic mode), then the
  // in-place rdIFFT unless the kernel ran it itself
  auto finish_gc = [&](bool ifft_done) -> cudaError_t {
    cudaError_t r = cudaSuccess;
    if (sink != nullptr && sink->partial != nullptr && sink->slices > 1)
      r = launch_sum_slices(sink->partial, sink->slices, (int64_t)q * q * p, grad_c, s);
    if (r == cudaSuccess && !ifft_done) r = launch_rows(grad_c, (int64_t)q * q, p, 0, true, s);
    return r;
  };
  if (grad_c != nullptr && grad_x != nullptr && circ_bwd_fused_supported(p, D, B)) {
    // both gradients from one transform of g and x (circ_bwd_fused.cu), then grad_c's rdIFFT
    e = launch_circ_bwd_fused(g, x, c_hat, grad_x, grad_c, B, D, p, dtype, s, sink);
    if (e != cudaSuccess) return e;
    return finish_gc(false);
  }
  if (grad_c != nullptr) {
    // the packed cross-spectrum summed over all tokens (the launcher zeroes grad_c
    // first when several CTAs add into it), then rdIFFT in place, unless one token slice
    // let the kernel invert its own rows
    GcSink local;
    GcSink* sk = sink != nullptr ? sink : &local;
    e = circ_layer(p, 2, g, x, c_hat, nullptr, grad_c, B, q, dtype, s, sk);
    if (e != cudaSuccess) return e;
    e = finish_gc(sk->ifft_done);
    if (e != cudaSuccess) return e;
  }
  if (grad_x != nullptr) e = circ_layer(p, 1, g, nullptr, c_hat, grad_x, nullptr, B, q, dtype, s);
  return e;
}

cudaError_t plan_circ_bwd(int64_t B, int D, int p, int dtype, bool with_grad_x, int* slices) {
  // the same path choice as launch_circ_bwd with grad_c requested; a plan-only sink makes
  // the launcher stop after working out its grid, before it touches a pointer
  GcSink plan;
  plan.plan_only = true;
  const cudaError_t e =
      (with_grad_x && circ_bwd_fused_supported(p, D, B))
          ? launch_circ_bwd_fused(nullptr, nullptr, nullptr, nullptr, nullptr, B, D, p, dtype, nullptr, &plan)
          : circ_layer(p, 2, nullptr, nullptr, nullptr, nullptr, nullptr, B, D / p, dtype, nullptr, &plan);
  *slices = plan.slices;
  return e;
}

}  // namespace rdfft
