// C ABI of the library: argument validation and dispatch (declared in rdfft.h).
// Every argument check happens before any CUDA call, so invalid calls enqueue
// nothing and need no GPU.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "rdfft.h"
#include "internal.h"

namespace {

thread_local cudaError_t t_last_cuda = cudaSuccess;
thread_local char t_msg[256];

bool pow2_in_range(int p) { return p >= 2 && p <= 4096 && (p & (p - 1)) == 0; }
bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }
bool dtype_ok(int dtype) { return dtype == RDFFT_F32 || dtype == RDFFT_BF16; }

int finish(cudaError_t e) {
  if (e == cudaSuccess) return RDFFT_OK;
  t_last_cuda = e;
  return RDFFT_ECUDA;
}

int rows_call(void* data, int64_t rows, int p, int dtype, rdfft_stream_t stream, bool inverse) {
  if (!dtype_ok(dtype)) return RDFFT_EDTYPE;
  if (!pow2_in_range(p) || rows < 0) return RDFFT_EINVAL;
  if (rows == 0) return RDFFT_OK;
  if (data == nullptr) return RDFFT_ENULL;
  if (!aligned16(data)) return RDFFT_EALIGN;
  return finish(rdfft::launch_rows(data, rows, p, dtype, inverse, reinterpret_cast<cudaStream_t>(stream)));
}

int layer_shape_ok(int64_t B, int D, int p) {
  if (!pow2_in_range(p) || p < 64 || B < 0 || D < p || D > RDFFT_MAX_D || D % p != 0) return 0;
  return 1;
}

// Byte ranges [a, a + na) and [b, b + nb) intersect (null pointers never do).
bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int convert_call(const void* in, void* out, int64_t rows, int p, int dtype, bool to_complex,
                 rdfft_stream_t stream) {
  if (!dtype_ok(dtype)) return RDFFT_EDTYPE;
  if (!pow2_in_range(p) || rows < 0) return RDFFT_EINVAL;
  if (rows == 0) return RDFFT_OK;
  if (in == nullptr || out == nullptr) return RDFFT_ENULL;
  if (!aligned16(in) || !aligned16(out)) return RDFFT_EALIGN;
  const size_t es = dtype == RDFFT_F32 ? 4 : 2;
  const size_t packed_bytes = (size_t)rows * p * es, cplx_bytes = (size_t)rows * (p + 2) * es;
  if (overlap(in, to_complex ? packed_bytes : cplx_bytes, out, to_complex ? cplx_bytes : packed_bytes))
    return RDFFT_EOVERLAP;
  return finish(rdfft::launch_convert(in, out, rows, p, dtype, to_complex, reinterpret_cast<cudaStream_t>(stream)));
}

// The 2-D transform: rows then columns (forward), columns then rows (inverse), in
// place; both halves are enqueued on the same stream.
int image_call(void* data, int64_t images, int R, int C, int dtype, rdfft_stream_t stream, bool inverse) {
  if (!dtype_ok(dtype)) return RDFFT_EDTYPE;
  if (!pow2_in_range(R) || !pow2_in_range(C) || images < 0) return RDFFT_EINVAL;
  if (images > INT64_MAX / ((int64_t)R * C)) return RDFFT_EINVAL;
  if (images == 0) return RDFFT_OK;
  if (data == nullptr) return RDFFT_ENULL;
  if (!aligned16(data)) return RDFFT_EALIGN;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t rows = images * R;
  if (!inverse) {
    const cudaError_t e = rdfft::launch_rows(data, rows, C, dtype, false, s);
    if (e != cudaSuccess) return finish(e);
    return finish(rdfft::launch_cols(data, images, R, C, dtype, false, s));
  }
  const cudaError_t e = rdfft::launch_cols(data, images, R, C, dtype, true, s);
  if (e != cudaSuccess) return finish(e);
  return finish(rdfft::launch_rows(data, rows, C, dtype, true, s));
}

// Bytes of c_hat or grad_c: q x q x p fp32.
size_t gc_bytes(int D, int p) { return sizeof(float) * (size_t)(D / p) * (D / p) * p; }

// Argument checks of the layer backward (circ_bwd, circ_bwd_deterministic). Returns
// kEnqueue when the call has work to enqueue, else the call's return code (an error, or
// RDFFT_OK when there is nothing to do or an empty batch only zeroed grad_c).
constexpr int kEnqueue = -1;
int bwd_args(const void* g, const void* x, const float* c_hat, void* grad_x, float* grad_c, int64_t B, int D,
             int p, int dtype, rdfft_stream_t stream) {
  if (!dtype_ok(dtype)) return RDFFT_EDTYPE;
  if (!layer_shape_ok(B, D, p)) return RDFFT_EINVAL;
  if (grad_x == nullptr && grad_c == nullptr) return RDFFT_OK;
  const size_t cb = gc_bytes(D, p);
  if (B == 0) {
    // no tokens: grad_x is empty and grad_c is an empty sum
    if (grad_c == nullptr) return RDFFT_OK;
    if (!aligned16(grad_c)) return RDFFT_EALIGN;
    return finish(cudaMemsetAsync(grad_c, 0, cb, reinterpret_cast<cudaStream_t>(stream)));
  }
  if (g == nullptr || c_hat == nullptr) return RDFFT_ENULL;
  if (grad_c != nullptr && x == nullptr) return RDFFT_ENULL;
  if (!aligned16(g) || !aligned16(c_hat) || (x && !aligned16(x)) || (grad_x && !aligned16(grad_x)) ||
      (grad_c && !aligned16(grad_c)))
    return RDFFT_EALIGN;
  const size_t act = (size_t)B * D * (dtype == RDFFT_F32 ? 4 : 2);
  if (overlap(grad_x, act, g, act) || overlap(grad_x, act, x, act) || overlap(grad_x, act, c_hat, cb) ||
      overlap(grad_x, act, grad_c, cb) || overlap(grad_c, cb, g, act) || overlap(grad_c, cb, x, act) ||
      overlap(grad_c, cb, c_hat, cb))
    return RDFFT_EOVERLAP;
  return kEnqueue;
}

// Scratch of circ_bwd_deterministic_noalloc: its per-slice grad_c sums live here instead
// of in caller memory. Every device that loads the library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = RDFFT_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of g_noalloc_scratch on the current device. In host code the array's name
// is only a stand-in, so the address is looked up with cudaGetSymbolAddress, once per
// device with that device current, and kept (no host or device allocation).
constexpr int kMaxDevices = 64;
cudaError_t noalloc_scratch(float** ptr) {
  static std::mutex mu;
  static float* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<float*>(p);
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

int rdfft_fwd(void* data, int64_t rows, int p, int dtype, rdfft_stream_t stream) {
  return rows_call(data, rows, p, dtype, stream, false);
}

int rdfft_inv(void* data, int64_t rows, int p, int dtype, rdfft_stream_t stream) {
  return rows_call(data, rows, p, dtype, stream, true);
}

int rdfft_to_complex(const void* packed, void* cplx, int64_t rows, int p, int dtype, rdfft_stream_t stream) {
  return convert_call(packed, cplx, rows, p, dtype, true, stream);
}

int rdfft_from_complex(const void* cplx, void* packed, int64_t rows, int p, int dtype, rdfft_stream_t stream) {
  return convert_call(cplx, packed, rows, p, dtype, false, stream);
}

int rdfft2_fwd(void* data, int64_t images, int R, int C, int dtype, rdfft_stream_t stream) {
  return image_call(data, images, R, C, dtype, stream, false);
}

int rdfft2_inv(void* data, int64_t images, int R, int C, int dtype, rdfft_stream_t stream) {
  return image_call(data, images, R, C, dtype, stream, true);
}

int circ_prepare(const float* c, float* c_hat, int D, int p, rdfft_stream_t stream) {
  if (!layer_shape_ok(0, D, p)) return RDFFT_EINVAL;
  if (c == nullptr || c_hat == nullptr) return RDFFT_ENULL;
  if (!aligned16(c) || !aligned16(c_hat)) return RDFFT_EALIGN;
  const size_t cb = sizeof(float) * (size_t)(D / p) * (D / p) * p;
  if (c != c_hat && overlap(c, cb, c_hat, cb)) return RDFFT_EOVERLAP;
  const int64_t rows = (int64_t)(D / p) * (D / p);
  return finish(rdfft::launch_rows_to(c, c_hat, rows, p, RDFFT_F32, false, reinterpret_cast<cudaStream_t>(stream)));
}

int circ_fwd(const void* x, const float* c_hat, void* y, int64_t B, int D, int p, int dtype,
             rdfft_stream_t stream) {
  if (!dtype_ok(dtype)) return RDFFT_EDTYPE;
  if (!layer_shape_ok(B, D, p)) return RDFFT_EINVAL;
  if (B == 0) return RDFFT_OK;
  if (x == nullptr || c_hat == nullptr || y == nullptr) return RDFFT_ENULL;
  if (!aligned16(x) || !aligned16(c_hat) || !aligned16(y)) return RDFFT_EALIGN;
  const size_t act = (size_t)B * D * (dtype == RDFFT_F32 ? 4 : 2);
  const size_t cb = sizeof(float) * (size_t)(D / p) * (D / p) * p;
  if (overlap(y, act, x, act) || overlap(y, act, c_hat, cb)) return RDFFT_EOVERLAP;
  return finish(rdfft::launch_circ_fwd(x, c_hat, y, B, D, p, dtype, reinterpret_cast<cudaStream_t>(stream)));
}

int circ_bwd(const void* g, const void* x, const float* c_hat, void* grad_x, float* grad_c,
             int64_t B, int D, int p, int dtype, rdfft_stream_t stream) {
  const int chk = bwd_args(g, x, c_hat, grad_x, grad_c, B, D, p, dtype, stream);
  if (chk != kEnqueue) return chk;
  return finish(rdfft::launch_circ_bwd(g, x, c_hat, grad_x, grad_c, B, D, p, dtype,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

int circ_bwd_workspace_size(int64_t B, int D, int p, int dtype, int with_grad_x, size_t* bytes) {
  if (bytes == nullptr) return RDFFT_ENULL;
  *bytes = 0;
  if (!dtype_ok(dtype)) return RDFFT_EDTYPE;
  if (!layer_shape_ok(B, D, p)) return RDFFT_EINVAL;
  if (B == 0) return RDFFT_OK;
  int slices = 0;
  const cudaError_t e = rdfft::plan_circ_bwd(B, D, p, dtype, with_grad_x != 0, &slices);
  if (e != cudaSuccess) return finish(e);
  if (slices > 1) *bytes = (size_t)slices * gc_bytes(D, p);
  return RDFFT_OK;
}

int circ_bwd_deterministic(const void* g, const void* x, const float* c_hat, void* grad_x, float* grad_c,
                           int64_t B, int D, int p, int dtype, void* workspace, size_t workspace_bytes,
                           rdfft_stream_t stream) {
  const int chk = bwd_args(g, x, c_hat, grad_x, grad_c, B, D, p, dtype, stream);
  if (chk != kEnqueue) return chk;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (grad_c == nullptr) return finish(rdfft::launch_circ_bwd(g, x, c_hat, grad_x, grad_c, B, D, p, dtype, s));
  size_t need = 0;
  const int rc = circ_bwd_workspace_size(B, D, p, dtype, grad_x != nullptr, &need);
  if (rc != RDFFT_OK) return rc;
  rdfft::GcSink sink;
  if (need > 0) {
    if (workspace == nullptr) return RDFFT_ENULL;
    if (!aligned16(workspace)) return RDFFT_EALIGN;
    if (workspace_bytes < need) return RDFFT_ESPACE;
    const size_t act = (size_t)B * D * (dtype == RDFFT_F32 ? 4 : 2), cb = gc_bytes(D, p);
    if (overlap(workspace, need, g, act) || overlap(workspace, need, x, act) ||
        overlap(workspace, need, c_hat, cb) || overlap(workspace, need, grad_x, act) ||
        overlap(workspace, need, grad_c, cb))
      return RDFFT_EOVERLAP;
    sink.partial = static_cast<float*>(workspace);
    sink.partial_floats = (int64_t)(need / sizeof(float));
  }
  return finish(rdfft::launch_circ_bwd(g, x, c_hat, grad_x, grad_c, B, D, p, dtype, s, &sink));
}

int circ_bwd_deterministic_noalloc(const void* g, const void* x, const float* c_hat, void* grad_x, float* grad_c,
                                   int64_t B, int D, int p, int dtype, rdfft_stream_t stream) {
  const int chk = bwd_args(g, x, c_hat, grad_x, grad_c, B, D, p, dtype, stream);
  if (chk != kEnqueue) return chk;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (grad_c == nullptr) return finish(rdfft::launch_circ_bwd(g, x, c_hat, grad_x, grad_c, B, D, p, dtype, s));
  size_t need = 0;
  const int rc = circ_bwd_workspace_size(B, D, p, dtype, grad_x != nullptr, &need);
  if (rc != RDFFT_OK) return rc;
  if (need > kNoAllocScratchBytes) return RDFFT_ESPACE;
  rdfft::GcSink sink;
  if (need > 0) {
    float* scratch = nullptr;
    const cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return finish(e);
    sink.partial = scratch;
    sink.partial_floats = (int64_t)(need / sizeof(float));
  }
  return finish(rdfft::launch_circ_bwd(g, x, c_hat, grad_x, grad_c, B, D, p, dtype, s, &sink));
}

int circ_fwd_tc(const void* x, const float* c_hat, void* y, int64_t B, int D, int p, int dtype,
                rdfft_stream_t stream) {
  if (!dtype_ok(dtype)) return RDFFT_EDTYPE;
  if (!layer_shape_ok(B, D, p) || !rdfft::circ_tc_supported(p, D, dtype)) return RDFFT_EINVAL;
  if (B == 0) return RDFFT_OK;
  if (x == nullptr || c_hat == nullptr || y == nullptr) return RDFFT_ENULL;
  if (!aligned16(x) || !aligned16(c_hat) || !aligned16(y)) return RDFFT_EALIGN;
  const size_t act = (size_t)B * D * 2;
  const size_t cb = sizeof(float) * (size_t)(D / p) * (D / p) * p;
  if (overlap(y, act, x, act) || overlap(y, act, c_hat, cb)) return RDFFT_EOVERLAP;
  return finish(rdfft::launch_circ_x_tc(x, c_hat, y, B, false, reinterpret_cast<cudaStream_t>(stream)));
}

int circ_bwd_x_tc(const void* g, const float* c_hat, void* grad_x, int64_t B, int D, int p, int dtype,
                  rdfft_stream_t stream) {
  if (!dtype_ok(dtype)) return RDFFT_EDTYPE;
  if (!layer_shape_ok(B, D, p) || !rdfft::circ_tc_supported(p, D, dtype)) return RDFFT_EINVAL;
  if (B == 0) return RDFFT_OK;
  if (g == nullptr || c_hat == nullptr || grad_x == nullptr) return RDFFT_ENULL;
  if (!aligned16(g) || !aligned16(c_hat) || !aligned16(grad_x)) return RDFFT_EALIGN;
  const size_t act = (size_t)B * D * 2;
  const size_t cb = sizeof(float) * (size_t)(D / p) * (D / p) * p;
  if (overlap(grad_x, act, g, act) || overlap(grad_x, act, c_hat, cb)) return RDFFT_EOVERLAP;
  return finish(rdfft::launch_circ_x_tc(g, c_hat, grad_x, B, true, reinterpret_cast<cudaStream_t>(stream)));
}

const char* rdfft_strerror(int code) {
  switch (code) {
    case RDFFT_OK: return "ok";
    case RDFFT_EINVAL: return "invalid size: p must be a power of two in [2, 4096] (>= 64 for the layer), counts >= 0, D a multiple of p and <= RDFFT_MAX_D";
    case RDFFT_ENULL: return "a required pointer is NULL";
    case RDFFT_EALIGN: return "a pointer is not 16-byte aligned";
    case RDFFT_EDTYPE: return "dtype must be RDFFT_F32 (0) or RDFFT_BF16 (1)";
    case RDFFT_EOVERLAP: return "an output buffer overlaps an input buffer";
    case RDFFT_ETIMEOUT: return "a kernel's bounded wait for its data timed out; its rows were not transformed";
    case RDFFT_ESPACE:
      return "the workspace is smaller than circ_bwd_workspace_size reports for this call (for "
             "circ_bwd_deterministic_noalloc: the call needs more than its built-in 16 MiB of scratch)";
    case RDFFT_ECUDA:
      snprintf(t_msg, sizeof(t_msg), "CUDA error while enqueuing: %s (%d)", cudaGetErrorString(t_last_cuda),
               (int)t_last_cuda);
      return t_msg;
    default: return "unknown rdfft error code";
  }
}

int rdfft_take_device_error(void) {
  unsigned int flags = 0, tc_flags = 0, fused_flags = 0;
  cudaError_t e = rdfft::take_rows_device_error(&flags);
  if (e == cudaSuccess) e = rdfft::take_tc_device_error(&tc_flags);
  if (e == cudaSuccess) e = rdfft::take_fused_device_error(&fused_flags);
  if (e != cudaSuccess) return finish(e);
  return ((flags | tc_flags | fused_flags) & 1u) ? RDFFT_ETIMEOUT : RDFFT_OK;
}

int rdfft_selftest_wait_timeout(rdfft_stream_t stream) {
  return finish(rdfft::launch_wait_selftest(reinterpret_cast<cudaStream_t>(stream)));
}

int rdfft_version(void) { return 110; }

}  // extern "C"
