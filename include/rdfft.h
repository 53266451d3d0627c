/*
 * rdfft.h -- C ABI of the B200 (sm_100a) rdFFT library: a real-domain, fully
 * in-place FFT / IFFT over batched rows, and the block-circulant linear layer it
 * drives, forward and backward.
 *
 * Source of the method: "Memory-Efficient Training with In-Place FFT
 * Implementation" (arXiv 2511.01385). Citations below name the web page that
 * describes a step and its section:
 *   [summary]     the AI-written summary page, sections "Approach", "Problem" and
 *                 "Limitations";
 *   [notes]       the paper-notes page, method section, items "Squeeze N+2 -> N",
 *                 "Proposition 1", "In-place IFFT design" and "Circulant matrix
 *                 training adaptation", its "Training strategy" list and its
 *                 "Limitations and outlook".
 *
 * Packed layout of a row of length p (every transform buffer uses it)
 * ([summary] Approach; [notes] "Squeeze N+2 -> N"): the spectrum Y of a real row
 * is conjugate symmetric, so it is stored in the row's own p slots:
 *     slot 0     = Y_0            (real)
 *     slot p/2   = Y_{p/2}        (real)
 *     slot k     = Re Y_k         for 0 < k < p/2
 *     slot p - k = Im Y_k         for 0 < k < p/2
 * with Y_k = sum_n x_n exp(-2 pi i k n / p). For p = 2 the row is [Y_0, Y_1].
 *
 * Conventions shared by every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller, 16-byte aligned,
 *     to dense row-major arrays. The library allocates no memory of any kind; its
 *     only state is a read-only twiddle table built into the module image.
 *   - `dtype` is RDFFT_F32 (float) or RDFFT_BF16 (bfloat16 raw bits, uint16). The
 *     arithmetic is fp32 in both cases; bf16 results are rounded once, to nearest
 *     even, when they are stored.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream) of the current
 *     device. Calls are asynchronous on it: they validate their arguments, enqueue
 *     kernels and return. They keep no state between calls and may be made from
 *     several host threads at once.
 *   - Return value: RDFFT_OK, or an error code. Argument errors are reported before
 *     anything is enqueued. RDFFT_ECUDA means a CUDA call failed when enqueuing;
 *     rdfft_strerror() then includes the CUDA message, which is kept per host
 *     thread. Empty work (rows == 0, images == 0 or B == 0) returns RDFFT_OK and
 *     enqueues nothing.
 */
#ifndef RDFFT_H
#define RDFFT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* rdfft_stream_t;

enum {
  RDFFT_F32 = 0,
  RDFFT_BF16 = 1
};

enum {
  RDFFT_OK = 0,
  RDFFT_EINVAL = 1,   /* p not a power of two in [2, 4096] ([64, 4096] for the layer); negative count; D % p != 0; D too large */
  RDFFT_ENULL = 2,    /* a required pointer is NULL */
  RDFFT_EALIGN = 3,   /* a pointer is not 16-byte aligned */
  RDFFT_EDTYPE = 4,   /* dtype is neither RDFFT_F32 nor RDFFT_BF16 */
  RDFFT_ECUDA = 5,    /* a CUDA call failed while enqueuing work */
  RDFFT_EOVERLAP = 6, /* an output buffer overlaps an input buffer it may not alias */
  RDFFT_ETIMEOUT = 7, /* reported by rdfft_take_device_error(): a bounded device wait gave up */
  RDFFT_ESPACE = 8    /* the workspace is smaller than circ_bwd_workspace_size reports */
};

/* Largest feature size D accepted by circ_fwd / circ_bwd. */
#define RDFFT_MAX_D 8192

/*
 * rdfft_fwd -- forward rdFFT of `rows` rows of length p, in place.
 * [notes] "Squeeze N+2 -> N" and "Proposition 1": radix-2 Cooley-Tukey whose
 * butterflies act on four-element groups symmetric about a centre index, so the
 * spectrum of each row overwrites the row in the packed layout above.
 *   data  : rows x p elements of `dtype`; read as real rows, overwritten by their
 *           packed spectra (unnormalised).
 *   rows  : number of rows (>= 0).   p : row length, power of two in [2, 4096].
 */
int rdfft_fwd(void* data, int64_t rows, int p, int dtype, rdfft_stream_t stream);

/*
 * rdfft_inv -- inverse rdFFT (rdIFFT) of `rows` packed rows of length p, in place.
 * [notes] "In-place IFFT design": the forward graph run backwards, each conjugate
 * pair split into its symmetric and antisymmetric parts, x_a = (y_a + y_b)/2,
 * x_b = (y_a - y_b)/(2 W). The product of those halvings is the 1/p of the inverse
 * DFT, so rdfft_inv(rdfft_fwd(x)) = x up to rounding.
 *   data  : rows x p packed spectra of `dtype`, overwritten by the real rows.
 */
int rdfft_inv(void* data, int64_t rows, int p, int dtype, rdfft_stream_t stream);

/*
 * rdfft_to_complex -- explicit complex bins of packed rows, out of place.
 * [summary] "Limitations": the packed layout encodes the spectrum implicitly, and
 * reaching the complex values (for spectral filtering, say) takes a cast that cannot
 * stay in the same buffer, since p reals become p/2 + 1 complex values. This is that
 * cast; it only moves values (bf16 stays bf16, bit for bit).
 *   packed : rows x p of `dtype` in the packed layout above, read only.
 *   cplx   : rows x (p/2 + 1) interleaved (re, im) pairs of `dtype` (rows x (p + 2)
 *            elements), written: bin k = (slot k, slot p-k) for 0 < k < p/2, bins 0
 *            and p/2 = (slot 0 or p/2, 0). Must not overlap `packed` (RDFFT_EOVERLAP).
 *   rows >= 0; p a power of two in [2, 4096].
 */
int rdfft_to_complex(const void* packed, void* cplx, int64_t rows, int p, int dtype, rdfft_stream_t stream);

/*
 * rdfft_from_complex -- packed rows from complex bins, out of place (the reverse cast
 * of rdfft_to_complex). The imaginary parts of bins 0 and p/2 are not read: they are
 * zero for the spectrum of a real row, and the packed layout has no slot for them.
 *   cplx   : rows x (p/2 + 1) interleaved (re, im) pairs of `dtype`, read only.
 *   packed : rows x p of `dtype`, written. Must not overlap `cplx` (RDFFT_EOVERLAP).
 */
int rdfft_from_complex(const void* cplx, void* packed, int64_t rows, int p, int dtype, rdfft_stream_t stream);

/*
 * rdfft2_fwd -- 2-D rdFFT of `images` real images of R x C (row-major), in place.
 * [notes] "Limitations and outlook" leaves the 2-D transform open; this library takes
 * the packed layout per axis, so that every slot of the image holds one real number
 * of its 2-D spectrum Y[k1, k2] = sum_{r,c} x[r,c] exp(-2 pi i (k1 r/R + k2 c/C)):
 *   columns 0 < k2 < C/2 : slot [k1][k2] = Re Y[k1, k2], slot [k1][C-k2] = Im Y[k1, k2]
 *                          for every k1 < R;
 *   columns k2 = 0, C/2  : Y[., k2] is conjugate symmetric in k1 and is stored down
 *                          the column in the 1-D packed layout above.
 * Computed as rdfft_fwd of the R rows of each image, then an in-place column
 * transform that combines the columns k2 and C - k2 (two kernels, each reading and
 * writing the data once).
 *   data   : images x R x C of `dtype`, overwritten by the packed 2-D spectra.
 *   images >= 0; R, C powers of two in [2, 4096].
 */
int rdfft2_fwd(void* data, int64_t images, int R, int C, int dtype, rdfft_stream_t stream);

/*
 * rdfft2_inv -- inverse of rdfft2_fwd (with the 1/(R C) of the inverse DFT), in place:
 * the column inverse (in its Hartley form, (1/R) M rdFFT M with M the mirror of a
 * packed row) and then rdfft_inv of the rows.
 */
int rdfft2_inv(void* data, int64_t images, int R, int C, int dtype, rdfft_stream_t stream);

/*
 * circ_prepare -- c_hat for circ_fwd / circ_bwd: the packed rdFFT of each of the q x q
 * circulant vectors c[i][j][:] (fp32), in one launch, out of place or in place.
 * [notes] "Circulant matrix training adaptation": the layer multiplies by FFT(c) in the
 * frequency domain; this computes it once per call of the layer (c changes every step).
 *   c     : q x q x p fp32 (i = output block, j = input block), D = q p. Read only.
 *   c_hat : q x q x p fp32, written with the packed spectra. It may be c itself (in
 *           place); any other overlap with c returns RDFFT_EOVERLAP.
 *   D, p  : as for circ_fwd (p a power of two in [64, 4096], D a multiple of p, <= RDFFT_MAX_D).
 */
int circ_prepare(const float* c, float* c_hat, int D, int p, rdfft_stream_t stream);

/*
 * circ_fwd -- block-circulant linear layer, forward.
 * [notes] "Circulant matrix training adaptation": y = IFFT(FFT(c) (.) FFT(x)); the
 * product of two conjugate-symmetric spectra is conjugate symmetric, so the packed
 * layout carries it. With D = q p, block j of a token is x_j = x[j p, (j+1) p) and
 *     y_i = IFFT( sum_{j<q} FFT(c_ij) (.) FFT(x_j) ),   i < q,
 * i.e. y = W x where block (i, j) of W is the p x p circulant whose first column is
 * c_ij.
 *   x     : B x D of `dtype`, read only.
 *   c_hat : q x q x p fp32, the packed rdfft_fwd of the fp32 parameters c[i][j][:]
 *           (the caller runs rdfft_fwd on an fp32 copy of c; i = output block,
 *           j = input block). Read only.
 *   y     : B x D of `dtype`, written. y must not overlap x or c_hat
 *           (RDFFT_EOVERLAP): several CTAs read each token row of x while others
 *           already write output blocks of the same row.
 *   B     : tokens (>= 0).  D : features, a multiple of p, D <= RDFFT_MAX_D.
 *   p     : block size, power of two in [64, 4096] for the layer.
 */
int circ_fwd(const void* x, const float* c_hat, void* y, int64_t B, int D, int p, int dtype,
             rdfft_stream_t stream);

/*
 * circ_bwd -- block-circulant linear layer, backward, for upstream gradient g = dL/dy.
 * [notes] "Circulant matrix training adaptation" (gradients keep the symmetry) and
 * "Training strategy" (forward and backward both in the real domain):
 *     grad_x_j = IFFT( sum_i conj(FFT(c_ij)) (.) FFT(g_i) )            (= W^T g)
 *     grad_c_ij = IFFT( sum_b FFT(g_i^b) (.) conj(FFT(x_j^b)) )        (summed over B)
 *   g, x   : B x D of `dtype`, read only.
 *   c_hat  : as in circ_fwd.
 *   grad_x : B x D of `dtype`, written; may be NULL to skip it. Must not overlap
 *            g, x, c_hat or grad_c (RDFFT_EOVERLAP).
 *   grad_c : q x q x p fp32 in the spatial domain (same layout as c), overwritten
 *            with the gradient summed over all B tokens; may be NULL to skip it.
 *            The buffer is used in place: it receives the packed cross-spectrum and
 *            ends with an in-place rdIFFT of its q*q rows. Its prior contents never
 *            matter. Must not overlap g, x or c_hat (RDFFT_EOVERLAP).
 * When the tokens are split over several CTAs, the grad_c sum over tokens is
 * accumulated with fp32 atomic adds into a zeroed buffer, so its last bits may differ
 * between runs (circ_bwd_deterministic below does not). With a handful of tokens one CTA
 * per block group sums them all and stores the result, and grad_c is deterministic; grad_x
 * and the forward always are.
 */
int circ_bwd(const void* g, const void* x, const float* c_hat, void* grad_x, float* grad_c,
             int64_t B, int D, int p, int dtype, rdfft_stream_t stream);

/*
 * circ_bwd_workspace_size -- device workspace, in bytes, that circ_bwd_deterministic needs
 * for these sizes on the current device, with grad_c requested and grad_x too when
 * with_grad_x != 0 (the two requests can take different kernels). 0 when the tokens fit
 * one slice per block group, whose sums need no workspace. Otherwise slices x q x q x p x 4
 * bytes, the slice count being what the grad_c kernel's grid uses for B tokens on this
 * device's SM count (at most one slice per SM). Enqueues nothing; needs no GPU (without one
 * it assumes 148 SMs).
 *   bytes : written. NULL returns RDFFT_ENULL.
 * Returns RDFFT_OK, RDFFT_EINVAL / RDFFT_EDTYPE as circ_bwd, or RDFFT_ECUDA.
 */
int circ_bwd_workspace_size(int64_t B, int D, int p, int dtype, int with_grad_x, size_t* bytes);

/*
 * circ_bwd_deterministic -- circ_bwd with a grad_c that is the same bit for bit from run to
 * run on a given GPU model (the slice count follows the SM count). [notes] "Circulant matrix
 * training adaptation", as circ_bwd; the sum over tokens is the same, only its order is
 * fixed: each token slice stores its packed partial sum in the workspace (slice s at byte
 * offset s q^2 p 4), and one more kernel adds the slices in order 0, 1, 2, ... into grad_c
 * before the in-place rdIFFT. grad_x is computed exactly as by circ_bwd.
 *   g, x, c_hat, grad_x, grad_c, B, D, p, dtype : as circ_bwd.
 *   workspace       : device memory owned by the caller, at least circ_bwd_workspace_size
 *                     bytes (same B, D, p, dtype, with_grad_x = grad_x != NULL), 16-byte
 *                     aligned; overwritten, and may be NULL when that size is 0. Must not
 *                     overlap any other argument (RDFFT_EOVERLAP).
 *   workspace_bytes : its size; too small returns RDFFT_ESPACE before anything is enqueued.
 * Costs one extra pass over the workspace (slices x q^2 p x 4 bytes written and read once).
 * Calls that share a workspace must be ordered on one stream. As with circ_bwd, a CTA whose
 * bounded wait gives up (rdfft_take_device_error then returns RDFFT_ETIMEOUT) leaves its part
 * unwritten, and grad_c is then wrong.
 */
int circ_bwd_deterministic(const void* g, const void* x, const float* c_hat, void* grad_x, float* grad_c,
                           int64_t B, int D, int p, int dtype, void* workspace, size_t workspace_bytes,
                           rdfft_stream_t stream);

/*
 * circ_bwd_deterministic_noalloc -- circ_bwd_deterministic for callers that cannot allocate
 * device memory: the same kernels and the same result bit for bit, with the workspace taken
 * from a scratch array built into the library instead of from the caller. The paper has no
 * counterpart; this is an interface convenience.
 *   g, x, c_hat, grad_x, grad_c, B, D, p, dtype : as circ_bwd.
 * Scratch: a file-scope device array of 16 MiB (RDFFT_NOALLOC_SCRATCH_BYTES) that every GPU
 * loading the library holds until the process exits. A call whose workspace
 * (circ_bwd_workspace_size) would exceed it returns RDFFT_ESPACE before enqueuing anything.
 * At 148 SMs, D = 4096, p = 128, B = 256 needs 16 MiB and fits; D = 4096, p = 512, B = 4096
 * needs 18.4 MiB and is refused; no shape needs more than 20 MiB. Nothing in it has to
 * start at zero: each call stores every element of the slices it then reads.
 * Set-up: the first call on each device (with that device current) looks up the array's
 * device address (cudaGetSymbolAddress) and keeps it; make that first call before any
 * stream capture on the device. Later calls do no set-up.
 * Sharing: every call on a device uses the same array, which keeps the last call's
 * contents. Calls that overlap on the GPU (different streams without ordering between
 * them, or several host threads) race on it and may return wrong grad_c; order them on
 * one stream. Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
#define RDFFT_NOALLOC_SCRATCH_BYTES (16u << 20)
int circ_bwd_deterministic_noalloc(const void* g, const void* x, const float* c_hat, void* grad_x, float* grad_c,
                                   int64_t B, int D, int p, int dtype, rdfft_stream_t stream);

/*
 * circ_fwd_tc, circ_bwd_x_tc -- the layer's forward and grad_x (as circ_fwd, and circ_bwd
 * with grad_c = NULL) with the per-frequency-bin contraction on the fifth-generation
 * tensor cores: tcgen05.mma of kind::tf32 with fp32 accumulation in tensor memory.
 * [notes] "Circulant matrix training adaptation": at bin k the sum over input blocks is
 * a complex q x q matrix (the bin of c_hat) times each token's q-vector, i.e. a small
 * GEMM over the tokens. Covered shape: p = 128, D = 4096 (q = 32), dtype RDFFT_BF16
 * (tf32 operands keep 10 mantissa bits: inside the bf16 tolerance, not the fp32 one);
 * other shapes and fp32 return RDFFT_EINVAL. Arguments, layouts and overlap rules as
 * for circ_fwd and circ_bwd. On B200 these run slower than circ_fwd / circ_bwd at every
 * batch size measured: the tensor cores need c_hat (q^2 p fp32, 512 KB here) staged in
 * shared memory for every tile of four tokens, which costs more than the CUDA-core
 * contraction it replaces. They are kept as the measured alternative.
 */
int circ_fwd_tc(const void* x, const float* c_hat, void* y, int64_t B, int D, int p, int dtype,
                rdfft_stream_t stream);
int circ_bwd_x_tc(const void* g, const float* c_hat, void* grad_x, int64_t B, int D, int p, int dtype,
                  rdfft_stream_t stream);

/*
 * rdfft_take_device_error -- the device error state of the transform kernels, then cleared.
 * No page has this; it is the library's failure detection. The row kernels move rows
 * with bulk copies and wait for them on a barrier with a bounded wait (about one
 * second): a wait that gives up leaves its rows unchanged, and records the event in a
 * word of the module's device memory instead of hanging the GPU. The one-kernel layer
 * backward (D = 4096 at p >= 512, 16-bit) stages its token tiles the same way (a wait that
 * gives up leaves that CTA's remaining grad_x rows and its grad_c part unwritten, and frees
 * its tensor memory), and the tensor-core layer kernels bound their waits for the tensor
 * cores (their outputs are then left unwritten and their tensor memory is freed). This call
 * reads and clears that word for the current device. It synchronises with the device (a
 * cudaMemcpyFromSymbol), so call it between steps, not inside a captured graph.
 * Returns RDFFT_OK, RDFFT_ETIMEOUT, or RDFFT_ECUDA.
 * After RDFFT_ETIMEOUT the contents of the rows of the launch that timed out are
 * undefined, and so are those of later launches in the stream until the stream has
 * been synchronised: a CTA whose wait gave up waits once more (again bounded) for its
 * own copies and then exits, and a copy still in flight after that second wait may
 * land in shared memory that a later CTA has been given.
 */
int rdfft_take_device_error(void);

/*
 * rdfft_selftest_wait_timeout -- enqueues a one-thread kernel whose bounded wait (about
 * one millisecond) is made to run out, on a barrier that expects bytes nobody sends.
 * No page has this; it lets a test check the failure path without any fault: after it
 * completes, rdfft_take_device_error() returns RDFFT_ETIMEOUT.
 */
int rdfft_selftest_wait_timeout(rdfft_stream_t stream);

/* Human-readable message for a return code (per host thread for RDFFT_ECUDA). */
const char* rdfft_strerror(int code);

/* Library version as 10000*major + 100*minor + patch. */
int rdfft_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RDFFT_H */
