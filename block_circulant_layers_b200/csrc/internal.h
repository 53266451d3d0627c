// Launchers shared between the C ABI layer and the kernel translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace rdfft {

// Batched in-place rdFFT (inverse = false) or rdIFFT (inverse = true) of `rows`
// rows of length p; dtype 0 = fp32, 1 = bf16. Arguments are already validated.
cudaError_t launch_rows(void* data, int64_t rows, int p, int dtype, bool inverse, cudaStream_t s);

// The same transform out of place: rows read from src, written to dst (dst == src is the
// in-place transform; any other overlap is the caller's to avoid).
cudaError_t launch_rows_to(const void* src, void* dst, int64_t rows, int p, int dtype, bool inverse, cudaStream_t s);

// Reads and clears the error word of the rows kernels (bit 0: a bounded wait timed out).
cudaError_t take_rows_device_error(unsigned int* flags);

// Launches a kernel whose bounded wait must time out (self-test of the error path).
cudaError_t launch_wait_selftest(cudaStream_t s);

// Packed <-> rFFT complex layout conversion (see rdfft_to_complex / rdfft_from_complex).
cudaError_t launch_convert(const void* in, void* out, int64_t rows, int p, int dtype, bool to_complex,
                           cudaStream_t s);

// Column half of the 2-D rdFFT of `images` images of R x C (see rdfft2_fwd / rdfft2_inv):
// forward column transform with the pair combine, or its inverse.
cudaError_t launch_cols(void* data, int64_t images, int R, int C, int dtype, bool inverse, cudaStream_t s);

// Tensor-core (tcgen05) forward / grad_x of the layer for the shape it covers
// (circ_tc_supported: p = 128, D = 4096, bf16; circ_fwd_tc / circ_bwd_x_tc in rdfft.h),
// and the error word of its bounded waits.
bool circ_tc_supported(int p, int D, int dtype);
cudaError_t launch_circ_x_tc(const void* in, const float* chat, void* out, int64_t B, bool bwdx, cudaStream_t s);
cudaError_t take_tc_device_error(unsigned int* flags);

// Where a grad_c launch puts its token slices' sums, and what it reports back. Without a
// sink (or with partial == nullptr) several slices add into a zeroed grad_c with fp32
// atomics; with partial, slice s stores its packed sums at partial + s q^2 p (the whole
// q x q x p spectrum over the slice's block groups) and the caller sums the slices in order.
struct GcSink {
  float* partial = nullptr;      // in: per-slice sums (deterministic mode), or nullptr
  int64_t partial_floats = 0;    // in: capacity of partial
  bool plan_only = false;        // in: work out the launch shape, enqueue nothing
  int slices = 0;                // out: token slices of the grad_c launch
  bool ifft_done = false;        // out: the kernel also ran grad_c's rdIFFT (one slice)
};

// Backward in one kernel (grad_x and the grad_c cross-spectrum from one transform of g
// and x per input-block group) for the shapes it covers (circ_bwd_fused_supported: D = 4096
// at p = 128, 512 or 1024, and layers of one or two blocks, D in {p, 2p},
// p >= 512); the caller runs the in-place rdIFFT of grad_c after it.
bool circ_bwd_fused_supported(int p, int D, int64_t B);
// Reads and clears the error word of the fused backward (bit 0: a bounded wait for its staged
// rows timed out).
cudaError_t take_fused_device_error(unsigned int* flags);
cudaError_t launch_circ_bwd_fused(const void* g, const void* x, const float* chat, void* grad_x, float* grad_c,
                                  int64_t B, int D, int p, int dtype, cudaStream_t s, GcSink* sink);

// Block-circulant layer forward: y = W x (see circ_fwd in rdfft.h).
cudaError_t launch_circ_fwd(const void* x, const float* c_hat, void* y, int64_t B, int D, int p,
                            int dtype, cudaStream_t s);

// Block-circulant layer backward (see circ_bwd in rdfft.h). grad_x / grad_c may be null.
// With a sink whose partial is set, grad_c's token slices are summed in slice order (see
// circ_bwd_deterministic).
cudaError_t launch_circ_bwd(const void* g, const void* x, const float* c_hat, void* grad_x,
                            float* grad_c, int64_t B, int D, int p, int dtype, cudaStream_t s,
                            GcSink* sink = nullptr);

// Token slices of the grad_c launch that launch_circ_bwd would make for these sizes with
// grad_c requested (and grad_x too if with_grad_x); enqueues nothing.
cudaError_t plan_circ_bwd(int64_t B, int D, int p, int dtype, bool with_grad_x, int* slices);

}  // namespace rdfft
