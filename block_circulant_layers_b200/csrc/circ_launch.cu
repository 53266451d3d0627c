// Block-circulant layer: dispatch on the block size p and the backward sequence.
#include <cuda_runtime.h>

#include "internal.h"

namespace rdfft {

cudaError_t circ_layer_64(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             bool*);
cudaError_t circ_layer_128(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             bool*);
cudaError_t circ_layer_256(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             bool*);
cudaError_t circ_layer_512(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             bool*);
cudaError_t circ_layer_1024(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             bool*);
cudaError_t circ_layer_2048(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             bool*);
cudaError_t circ_layer_4096(int, const void*, const void*, const float*, void*, float*, int64_t, int, int, cudaStream_t,
                             bool*);

static cudaError_t circ_layer(int p, int op, const void* a, const void* b, const float* chat, void* out,
                              float* gc, int64_t B, int q, int dtype, cudaStream_t s, bool* ifft_done = nullptr) {
  switch (p) {
    case 64: return circ_layer_64(op, a, b, chat, out, gc, B, q, dtype, s, ifft_done);
    case 128: return circ_layer_128(op, a, b, chat, out, gc, B, q, dtype, s, ifft_done);
    case 256: return circ_layer_256(op, a, b, chat, out, gc, B, q, dtype, s, ifft_done);
    case 512: return circ_layer_512(op, a, b, chat, out, gc, B, q, dtype, s, ifft_done);
    case 1024: return circ_layer_1024(op, a, b, chat, out, gc, B, q, dtype, s, ifft_done);
    case 2048: return circ_layer_2048(op, a, b, chat, out, gc, B, q, dtype, s, ifft_done);
    case 4096: return circ_layer_4096(op, a, b, chat, out, gc, B, q, dtype, s, ifft_done);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_circ_fwd(const void* x, const float* c_hat, void* y, int64_t B, int D, int p,
                            int dtype, cudaStream_t s) {
  return circ_layer(p, 0, x, nullptr, c_hat, y, nullptr, B, D / p, dtype, s);
}

cudaError_t launch_circ_bwd(const void* g, const void* x, const float* c_hat, void* grad_x,
                            float* grad_c, int64_t B, int D, int p, int dtype, cudaStream_t s) {
  const int q = D / p;
  cudaError_t e = cudaSuccess;
  if (grad_c != nullptr && grad_x != nullptr && circ_bwd_fused_supported(p, D, B)) {
    // both gradients from one transform of g and x (circ_bwd_fused.cu), then grad_c's rdIFFT
    e = launch_circ_bwd_fused(g, x, c_hat, grad_x, grad_c, B, D, p, dtype, s);
    if (e == cudaSuccess) e = launch_rows(grad_c, (int64_t)q * q, p, 0, true, s);
    return e;
  }
  if (grad_c != nullptr) {
    // the packed cross-spectrum summed over all tokens (the launcher zeroes grad_c
    // first when several CTAs add into it), then rdIFFT in place, unless one token slice
    // let the kernel invert its own rows
    bool done = false;
    e = circ_layer(p, 2, g, x, c_hat, nullptr, grad_c, B, q, dtype, s, &done);
    if (e == cudaSuccess && !done) e = launch_rows(grad_c, (int64_t)q * q, p, 0, true, s);
    if (e != cudaSuccess) return e;
  }
  if (grad_x != nullptr) e = circ_layer(p, 1, g, nullptr, c_hat, grad_x, nullptr, B, q, dtype, s);
  return e;
}

}  // namespace rdfft
