// Block-circulant layer backward in one kernel: grad_x and grad_c from one transform of
// each token's g and x per group of input blocks (one group for layers with few blocks,
// q <= 8; four at q = 32).
//
// "Memory-Efficient Training with In-Place FFT Implementation", paper-notes page,
// "Circulant matrix training adaptation" (gradients keep the conjugate symmetry):
//     grad_x_j  = IFFT( sum_i conj(C_ij) (.) G_i )
//     grad_c_ij = IFFT( sum_b G_i^b (.) conj(X_j^b) )
// with G = rdFFT(g), X = rdFFT(x) per block, C = c_hat. circ_bwd otherwise runs two
// kernels, each transforming g again (and grad_c also x): 32 row transforms per token
// at q = 8. Here a persistent CTA per SM walks its slice of the tokens in tiles and,
// per tile, transforms g and x once into its shared tile (2 q rows per token), adds
// G conj(X) into the CTA's part of the cross-spectrum, forms the grad_x spectra over
// the X rows, and inverse-transforms them to HBM: 24 row transforms per token.
//
// The cross-spectrum of the CTA (q^2 p/2 complex values, 32768 floats at p = 512,
// q = 8: 64 per thread) lives in tensor memory, not in registers: loaded and stored
// back (tcgen05.ld / tcgen05.st, 32x32b shape, each thread its own lane) around the
// accumulation of each tile, it leaves the registers to the transforms and the grad_x
// contraction. Beside it each thread keeps the c_hat values of its grad_x slots (one
// bin, NS output blocks, all q summed blocks: 64 floats at p = 512), read from HBM once
// per CTA instead of once per tile. At the end each CTA adds its part into grad_c (fp32
// red.add into a zeroed grad_c; a plain store when one CTA per group covers all tokens, or
// into its slice's part of the workspace in the deterministic mode), and the caller's
// stream runs the in-place rdIFFT of grad_c's q^2 rows after, as circ_bwd does. Layers
// of one or two blocks take k_circ_bwd_small below, with the cross-spectrum in registers.
#include <cuda_runtime.h>

#include "bulk_copy.cuh"
#include "circ_kernels.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace rdfft {
namespace {

#ifndef RDFFT_FUSED_STAGING
#define RDFFT_FUSED_STAGING 1
#endif

// Shared memory of the fused kernel: the fp32 tile of TT (q + QJ) rows; with staging (16-bit
// rows, p >= 512, where a warp's lanes span at most two rows of the staged tile) a buffer of
// the next tile's g and x rows as they are in HBM, filled by bulk copies (the TMA engine, no
// cluster multicast) while the current tile is processed, and its mbarrier.
template <int P, int Q, int QJ, typename T, int TT>
struct FusedSmem {
  static constexpr bool STG = RDFFT_FUSED_STAGING && sizeof(T) == 2 && P >= 512;
  static constexpr int TILE_WORDS = ((LayerGeo<P>::words(TT * (Q + QJ)) + 3) / 4) * 4;
  static constexpr int STAGE_G = TT * Q * P;                     // elements: TT tokens' g rows
  static constexpr int STAGE = STAGE_G + TT * QJ * P;            // and their x rows of the group
  static constexpr size_t MBAR_OFF = sizeof(float) * (size_t)TILE_WORDS + (STG ? ((sizeof(T) * STAGE + 15) / 16) * 16 : 0);
  static constexpr size_t BYTES = MBAR_OFF + (STG ? 16 : 0);
};

// QJ: the input blocks j of a CTA group (blockIdx.y): the CTA transforms g in full but x
// only for its group's blocks, keeps the cross-spectrum S_ij of its group (every i) and
// forms grad_x for its group's blocks. QJ = q for layers with few blocks; at q = 32 (p = 128)
// four groups keep each CTA's part within tensor memory, and g is transformed once per group
// (4 times a token, against 6 times for the separate grad_x and grad_c kernels).
template <int P, int Q, int QJ, typename T, int NT, int TT, int RI, int RJ>
__global__ void __launch_bounds__(NT, 1)
k_circ_bwd_fused(const T* __restrict__ g, const T* __restrict__ x, const float* __restrict__ chat,
                 T* __restrict__ grad_x, float* __restrict__ grad_c, float* __restrict__ partial, int64_t B,
                 int64_t tok_per_cta) {
  using G = LayerGeo<P>;
  constexpr int q = Q;
  constexpr int HB = P / 2;
  constexpr int RJP = RJ / 2;
  constexpr int ACC = RI * RJ * 2;                  // floats of cross-spectrum per thread
  constexpr int NS = QJ * HB / NT;                  // grad_x output blocks per thread (one bin)
  constexpr int CPI = 2 * NS;                       // c_hat floats per thread and summed block i
  constexpr int BPL = 16 / CPI;                     // summed blocks per 16-column tensor-memory load
  constexpr int CH = CPI * Q;                       // floats of c_hat per thread
  constexpr int PER = ACC + CH;                     // tensor-memory columns per thread
  constexpr int WQ = NT / 128;                      // warps per tensor-memory lane quarter
  constexpr int COLS = WQ * PER;
  static_assert(RJ % 2 == 0 && ACC % 16 == 0 && CH % 16 == 0, "accumulator layout");
  static_assert((COLS & (COLS - 1)) == 0 && COLS >= 32 && COLS <= 512, "tensor-memory allocation");
  static_assert(NT % HB == 0 && NS >= 1, "the grad_x slots of a thread share one bin");
  static_assert(Q % QJ == 0 && QJ % RJ == 0 && 16 % CPI == 0 && Q % BPL == 0, "block groups");
  static_assert(NS % 2 == 0 || (NS == 1 && TT % 2 == 0), "slot pairs, or token pairs for one slot");
  extern __shared__ float tile[];
  __shared__ uint32_t tmem_holder;
  const int D = q * P;
  const int64_t tbeg = (int64_t)blockIdx.x * tok_per_cta;
  const int64_t tend = (tbeg + tok_per_cta < B) ? tbeg + tok_per_cta : B;
  // one token slice stores its sums (they are final); with per-slice sums (partial) every
  // slice stores its own q x q x p spectrum the same way; otherwise the slices add
  const bool store = (gridDim.x == 1) || partial != nullptr;
  float* const gc_base = partial != nullptr ? partial + (int64_t)blockIdx.x * q * q * P : grad_c;
  const int warp = threadIdx.x >> 5;
  const int j0 = blockIdx.y * QJ;                   // the group's first input block
  const int nib = q / RI;
  const int ng = HB * nib * (QJ / RJ);              // cross-spectrum groups (one per thread)
  const int XR = TT * q;                            // first X row of the tile (a multiple of 32)
  using SM = FusedSmem<P, Q, QJ, T, TT>;
  T* stage = reinterpret_cast<T*>(tile + SM::TILE_WORDS);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(tile) + SM::MBAR_OFF);
  // the rows of the tile starting at token tk into the staging buffer (thread 0)
  auto fill = [&](int64_t tk) {
    const int nt = (int)((tend - tk) < TT ? (tend - tk) : TT);
    mbar_arrive_expect_tx(mbar, (unsigned)(nt * (D + QJ * P) * (int)sizeof(T)));
    for (int t = 0; t < nt; ++t) {
      bulk_load(stage + (size_t)t * D, g + (tk + t) * (int64_t)D, (unsigned)(D * sizeof(T)), mbar);
      bulk_load(stage + SM::STAGE_G + (size_t)t * QJ * P, x + (tk + t) * (int64_t)D + (int64_t)j0 * P,
                (unsigned)(QJ * P * sizeof(T)), mbar);
    }
  };

  griddep_wait();
  if constexpr (SM::STG) {
    if (threadIdx.x == 0) {
      mbar_init(mbar, 1);
      if (tbeg < tend) fill(tbeg);
    }
  }
  if (warp == 0) tc::tmem_alloc(&tmem_holder, COLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tacc = tmem_holder + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(PER * (warp >> 2));
  const uint32_t tch = tacc + ACC;
  float acc[ACC];
#pragma unroll
  for (int i = 0; i < ACC; ++i) acc[i] = 0.0f;
#pragma unroll
  for (int c = 0; c < ACC; c += 16) tc::tmem_st16(tacc + c, acc + c);

  // the thread's cross-spectrum group: bin k, output blocks ib*RI.., input blocks j0 + jb*RJ..
  const int gam = threadIdx.x;
  const int gk = gam % HB, gib = (gam / HB) % nib, gjb = gam / HB / nib;
  // a warp holds bin 0 (grad_c group or grad_x slot) only if its first lane does; such
  // warps take the real pair's component-wise products, the others the complex ones
  const bool warp_bin0 = (threadIdx.x & ~31u) % HB == 0;
  const int gkr = G::at(gk), gki = G::at(bin_im_slot<P>(gk));
  // the thread's grad_x slots: bin xk, output blocks j0 + o_u, o_u = xo0 + u NT / HB (u < NS).
  // Their c_hat values (for every summed block i) are the same for every token: read once
  // here and kept in tensor memory beside the cross-spectrum, as [i][slot pair w] (re_2w,
  // re_2w+1, im_2w, im_2w+1), or [i] (re, im) for a single slot (16 columns = BPL summed
  // blocks), with conj(c_hat) and bin 0's real pair applied at use.
  constexpr int XG = NT / HB;
  const int xk = threadIdx.x % HB, xo0 = threadIdx.x / HB;
  const int xkr = G::at(xk), xki = G::at(bin_im_slot<P>(xk));
  {
    float ch[CH];
#pragma unroll
    for (int u = 0; u < NS; ++u)
#pragma unroll
      for (int i = 0; i < Q; ++i) {
        const float* crow = chat + (int64_t)(i * Q + j0 + xo0 + u * XG) * P;
        const int c = NS == 1 ? CPI * i : CPI * i + 2 * (u & ~1) + (u & 1);
        ch[c] = __ldg(crow + xk);
        ch[c + (NS == 1 ? 1 : 2)] = __ldg(crow + bin_im_slot<P>(xk));
      }
#pragma unroll
    for (int c = 0; c < CH; c += 16) tc::tmem_st16(tch + c, ch + c);
  }
  tc::tmem_wait_st();

  bool failed = false;
  unsigned phase = 0;
  for (int64_t tok0 = tbeg; tok0 < tend; tok0 += TT) {
    const int ntok = (int)((tend - tok0) < TT ? (tend - tok0) : TT);
    if (tok0 != tbeg) __syncthreads();              // the previous tile is fully consumed
    if constexpr (SM::STG) {                        // this tile's rows have landed (bounded wait)
      const bool arrived = mbar_wait_bounded(mbar, phase);
      phase ^= 1u;
      if (!__syncthreads_and(arrived)) {
        if (threadIdx.x == 0) mbar_wait_bounded(mbar, phase ^ 1u, kWaitCycles / 8);   // copies in flight
        failed = true;
        break;
      }
    }
    // 1. rdFFT of g (rows t q + i) and of the group's x blocks (rows XR + t QJ + jl), read
    // from the staging buffer or from HBM
    auto src = [&](int r) -> const T* {
      if (r < XR) {
        const int t = r / q, b = r - t * q;
        if (t >= ntok) return nullptr;
        return SM::STG ? stage + (size_t)t * D + (size_t)b * P : g + (tok0 + t) * (int64_t)D + (int64_t)b * P;
      }
      const int t = (r - XR) / QJ, jl = r - XR - t * QJ;
      if (t >= ntok) return nullptr;
      return SM::STG ? stage + SM::STAGE_G + (size_t)(t * QJ + jl) * P
                     : x + (tok0 + t) * (int64_t)D + (int64_t)(j0 + jl) * P;
    };
    // only the rows of the tile's ntok tokens are transformed: the r-th is g row r for
    // r < ntok q, then x row XR + (r - ntok q), so a partial last tile takes fewer rounds
    // of rows (the rows of absent tokens keep stale values that nothing stores)
    const int ngr = ntok * q, nrows = ntok * (q + QJ);
    auto rowmap = [=](int r) { return r < ngr ? r : XR + (r - ngr); };
    {
      constexpr int TPR = G::TPR, RPR = NT / TPR;
      const int v = threadIdx.x % TPR;
      for (int rr = threadIdx.x / TPR; rr < nrows; rr += RPR) {
        const int r = rowmap(rr);
        fwd_pass0<G, T>(tile, r, v, src(r), true);
      }
    }
    if constexpr (SM::STG) {
      __syncthreads();                               // the staged rows are read: fetch the next tile's
      if (threadIdx.x == 0 && tok0 + TT < tend) fill(tok0 + TT);
    }
    fft_rows_rest_mapped<P, NT, T, 1>(tile, nrows, rowmap);
    __syncthreads();

    // 2. cross-spectrum: S_ij += G_i conj(X_j) over the tile's tokens, from and back to
    // tensor memory; input blocks b and b + 1 on packed fp32 pairs
#pragma unroll
    for (int c = 0; c < ACC; c += 16) tc::tmem_ld16_nowait(tacc + c, acc + c);
    tc::tmem_wait_ld();
    // G conj(X): re = gr xr + gi xi, im = gi xr - gr xi; bin 0 (real pair): (gr xr, gi xi),
    // written as re += gr xr + gi xa, im += gi xb + gr xc with the x terms chosen per
    // input-block pair; bin0 = false (warps with no bin-0 group) drops the selects
    auto accumulate = [&](bool bin0) {
      const bool gz = bin0 && (gk == 0);
      for (int t = 0; t < ntok; ++t) {
        float gr[RI], gi[RI];
#pragma unroll
        for (int a = 0; a < RI; ++a) {
          const int rb = G::row_base(t * q + gib * RI + a);
          gr[a] = tile[rb + gkr];
          gi[a] = tile[rb + gki];
        }
#pragma unroll
        for (int bp = 0; bp < RJP; ++bp) {
          float xr[2], xi[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int rb = G::row_base(XR + t * QJ + gjb * RJ + 2 * bp + h);
            xr[h] = tile[rb + gkr];
            xi[h] = tile[rb + gki];
          }
          const f2 vxr = f2_mk(xr[0], xr[1]);
          const f2 vxa = gz ? f2_bc(0.0f) : f2_mk(xi[0], xi[1]);
          const f2 vxb = gz ? f2_mk(xi[0], xi[1]) : vxr;
          const f2 vxc = gz ? f2_bc(0.0f) : f2_mk(-xi[0], -xi[1]);
#pragma unroll
          for (int a = 0; a < RI; ++a) {
            const int o = (a * RJP + bp) * 4;
            const f2 vgr = f2_bc(gr[a]), vgi = f2_bc(gi[a]);
            const f2 sr = f2_fma(vgr, vxr, f2_fma(vgi, vxa, f2_mk(acc[o], acc[o + 1])));
            const f2 si = f2_fma(vgi, vxb, f2_fma(vgr, vxc, f2_mk(acc[o + 2], acc[o + 3])));
            acc[o] = sr.x;
            acc[o + 1] = sr.y;
            acc[o + 2] = si.x;
            acc[o + 3] = si.y;
          }
        }
      }
    };
    if (gam < ng) {
      if (warp_bin0) accumulate(true);               // warp-uniform: each side is specialised
      else accumulate(false);
    }
#pragma unroll
    for (int c = 0; c < ACC; c += 16) tc::tmem_st16(tacc + c, acc + c);
    tc::tmem_wait_st();
    __syncthreads();                                 // X rows read: they become grad_x rows

    // 3. grad_x spectra over the X rows: Y_j = sum_i conj(C_ij) G_i, stored mirrored
    // (slot k = Re - Im, slot p - k = Re + Im; bin 0 keeps its real pair)
    // conj(c) G as yr += cr xa + ci xb, yi += cr xc + ci xd with the token's G terms
    //   complex bin: xa = gr, xb = gi, xc = gi, xd = -gr;  bin 0: xa = gr, xb = xc = 0, xd = gi
    if constexpr (NS % 2 == 0) {
      // all NS slots share the bin, so each G value is read once for all of them; slot
      // pairs (u, u + 1) accumulate on packed fp32 pairs
      f2 yr[NS / 2][TT], yi[NS / 2][TT];
#pragma unroll
      for (int w = 0; w < NS / 2; ++w)
#pragma unroll
        for (int t = 0; t < TT; ++t) yr[w][t] = yi[w][t] = f2_bc(0.0f);
      auto contract = [&](bool bin0) {
        const bool xz = bin0 && (xk == 0);
        float ch[16];
#pragma unroll
        for (int i = 0; i < Q; ++i) {
          if (i % BPL == 0) {
            tc::tmem_ld16_nowait(tch + CPI * i, ch);
            tc::tmem_wait_ld();
          }
          const int cb = CPI * (i % BPL);
          f2 cr[NS / 2], ci[NS / 2];
#pragma unroll
          for (int w = 0; w < NS / 2; ++w) {
            cr[w] = f2_mk(ch[cb + 4 * w], ch[cb + 4 * w + 1]);
            ci[w] = f2_mk(ch[cb + 4 * w + 2], ch[cb + 4 * w + 3]);
          }
#pragma unroll
          for (int t = 0; t < TT; ++t) {
            if (t < ntok) {
              const int rb = G::row_base(t * Q + i);
              const float vr = tile[rb + xkr], vi = tile[rb + xki];
              const f2 xa = f2_bc(vr);
              const f2 xb = f2_bc(xz ? 0.0f : vi);
              const f2 xc = xb;
              const f2 xd = f2_bc(xz ? vi : -vr);
#pragma unroll
              for (int w = 0; w < NS / 2; ++w) {
                yr[w][t] = f2_fma(cr[w], xa, f2_fma(ci[w], xb, yr[w][t]));
                yi[w][t] = f2_fma(cr[w], xc, f2_fma(ci[w], xd, yi[w][t]));
              }
            }
          }
        }
      };
      if (warp_bin0) contract(true);                 // warp-uniform: each side is specialised
      else contract(false);
#pragma unroll
      for (int u = 0; u < NS; ++u) {
        const int o = xo0 + u * XG;
#pragma unroll
        for (int t = 0; t < TT; ++t) {
          if (t < ntok) {
            const float ar = (u & 1) ? yr[u / 2][t].y : yr[u / 2][t].x;
            const float ai = (u & 1) ? yi[u / 2][t].y : yi[u / 2][t].x;
            const int rb = G::row_base(XR + t * QJ + o);
            tile[rb + xkr] = xk == 0 ? ar : ar - ai;
            tile[rb + xki] = xk == 0 ? ai : ar + ai;
          }
        }
      }
    } else {
      // one slot: token pairs (t, t + 1) accumulate on packed fp32 pairs, c_hat broadcast
      f2 yr[TT / 2], yi[TT / 2];
#pragma unroll
      for (int v = 0; v < TT / 2; ++v) yr[v] = yi[v] = f2_bc(0.0f);
      auto contract = [&](bool bin0) {
        const bool xz = bin0 && (xk == 0);
        float ch[16];
#pragma unroll
        for (int i = 0; i < Q; ++i) {
          if (i % BPL == 0) {
            tc::tmem_ld16_nowait(tch + CPI * i, ch);
            tc::tmem_wait_ld();
          }
          const int cb = CPI * (i % BPL);
          const f2 cr = f2_bc(ch[cb]), ci = f2_bc(ch[cb + 1]);
#pragma unroll
          for (int v = 0; v < TT / 2; ++v) {
            // a pair past the tile's tokens is skipped; in a pair whose second token is absent,
            // that lane works on a stale row and is never stored (the lanes are independent)
            if (2 * v >= ntok) break;
            const int rb0 = G::row_base(2 * v * Q + i), rb1 = G::row_base((2 * v + 1) * Q + i);
            const float vr0 = tile[rb0 + xkr], vi0 = tile[rb0 + xki];
            const float vr1 = tile[rb1 + xkr], vi1 = tile[rb1 + xki];
            const f2 xa = f2_mk(vr0, vr1);
            const f2 xb = xz ? f2_bc(0.0f) : f2_mk(vi0, vi1);
            const f2 xd = xz ? f2_mk(vi0, vi1) : f2_mk(-vr0, -vr1);
            yr[v] = f2_fma(cr, xa, f2_fma(ci, xb, yr[v]));
            yi[v] = f2_fma(cr, xb, f2_fma(ci, xd, yi[v]));
          }
        }
      };
      if (warp_bin0) contract(true);                 // warp-uniform: each side is specialised
      else contract(false);
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        if (t < ntok) {
          const float ar = (t & 1) ? yr[t / 2].y : yr[t / 2].x;
          const float ai = (t & 1) ? yi[t / 2].y : yi[t / 2].x;
          const int rb = G::row_base(XR + t * QJ + xo0);
          tile[rb + xkr] = xk == 0 ? ar : ar - ai;
          tile[rb + xki] = xk == 0 ? ai : ar + ai;
        }
      }
    }
    __syncthreads();
    // 4. rdIFFT (Hartley form) of the grad_x rows straight to HBM
    ifft_rows_mirrored<P, NT, T>(tile + G::row_base(XR), ntok * QJ, [&](int r) -> T* {
      const int t = r / QJ, jl = r - t * QJ;
      return grad_x + (tok0 + t) * (int64_t)D + (int64_t)(j0 + jl) * P;
    });
  }

  // 5. the CTA's cross-spectrum into grad_c (left unwritten after a wait gave up)
  griddep_launch_dependents();
#pragma unroll
  for (int c = 0; c < ACC; c += 16) tc::tmem_ld16_nowait(tacc + c, acc + c);
  tc::tmem_wait_ld();
  if (gam < ng && !failed) {
    const int kim = bin_im_slot<P>(gk);
#pragma unroll
    for (int a = 0; a < RI; ++a)
#pragma unroll
      for (int b = 0; b < RJ; ++b) {
        float* dst = gc_base + ((int64_t)(gib * RI + a) * q + (j0 + gjb * RJ + b)) * P;
        const int o = (a * RJP + b / 2) * 4 + (b & 1);
        const float vr = acc[o], vi = acc[o + 2];
        if (store) {
          dst[gk] = vr;
          dst[kim] = vi;
        } else {
          atomicAdd(dst + gk, vr);
          atomicAdd(dst + kim, vi);
        }
      }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem_holder, COLS);
}

template <int P, int Q, int QJ, typename T, int TT, int RI, int RJ>
cudaError_t run_fused(const void* g, const void* x, const float* chat, void* grad_x, float* grad_c, int64_t B,
                      cudaStream_t s, GcSink* sink) {
  constexpr int NT = 512;
  constexpr int q = Q;
  auto kern = k_circ_bwd_fused<P, Q, QJ, T, NT, TT, RI, RJ>;
  const size_t smem = FusedSmem<P, Q, QJ, T, TT>::BYTES;
  constexpr int NJG = Q / QJ;                      // input-block groups
  int64_t tiles_per = 1;
  const int slices = layer_gc_slices(NJG, (B + TT - 1) / TT, num_sms(), &tiles_per);
  float* partial = nullptr;
  cudaError_t e = sink_plan(sink, slices, (int64_t)q * q * P, &partial);
  if (e != cudaSuccess || (sink && sink->plan_only)) return e;
  e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  if (slices > 1 && !partial) {
    e = launch_zero_f32(grad_c, (int64_t)q * q * P, s);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(kern, dim3((unsigned)slices, (unsigned)NJG), dim3(NT), smem, s, static_cast<const T*>(g),
                    static_cast<const T*>(x), chat, static_cast<T*>(grad_x), grad_c, partial, B,
                    (int64_t)(tiles_per * TT));
}

// The same backward for layers of one or two blocks (q <= 2): the cross-spectrum
// S_ij = sum_b G_i conj(X_j) has q^2 p/2 complex bins, so each thread keeps its bins' sums
// (and its bins' c_hat) in registers, no tensor memory. A persistent CTA walks its token slice
// in tiles of TT tokens: rdFFT of g (tile rows t q + i) and x (rows TT q + t q + j), then per bin
// S_ij += G_i conj(X_j) and the grad_x spectra Y_j = sum_i conj(C_ij) G_i written mirrored over
// the x rows, then the Hartley-form rdIFFT of those rows to HBM: 3 row transforms per token and
// block against 2 + 2 for the two kernels. Bin 0 holds the real pair (y_0, y_{p/2}), whose
// products are component-wise.
template <int P, int Q, typename T, int NT, int TT>
__global__ void __launch_bounds__(NT, 1)
k_circ_bwd_small(const T* __restrict__ g, const T* __restrict__ x, const float* __restrict__ chat,
                 T* __restrict__ grad_x, float* __restrict__ grad_c, float* __restrict__ partial, int64_t B,
                 int64_t tok_per_cta) {
  using G = LayerGeo<P>;
  constexpr int HB = P / 2;
  constexpr int KB = (HB + NT - 1) / NT;            // bins per thread: k = tid + NT u
  constexpr int XR = TT * Q;                        // first x row of the tile
  constexpr int D = Q * P;
  static_assert(NT % G::TPR == 0 && (G::RW == 1 || XR % G::RW == 0), "whole rows; additive row bases");
  extern __shared__ float tile[];
  const int64_t tbeg = (int64_t)blockIdx.x * tok_per_cta;
  const int64_t tend = (tbeg + tok_per_cta < B) ? tbeg + tok_per_cta : B;
  const bool store = (gridDim.x == 1) || partial != nullptr;   // as in k_circ_bwd_fused
  float* const gc_base = partial != nullptr ? partial + (int64_t)blockIdx.x * Q * Q * P : grad_c;
  griddep_wait();

  float sr[KB][Q][Q], si[KB][Q][Q], cr[KB][Q][Q], ci[KB][Q][Q];
#pragma unroll
  for (int u = 0; u < KB; ++u) {
    const int k = threadIdx.x + NT * u;
#pragma unroll
    for (int i = 0; i < Q; ++i)
#pragma unroll
      for (int j = 0; j < Q; ++j) {
        const float* crow = chat + (int64_t)(i * Q + j) * P;
        sr[u][i][j] = si[u][i][j] = 0.0f;
        cr[u][i][j] = k < HB ? __ldg(crow + k) : 0.0f;
        ci[u][i][j] = k < HB ? __ldg(crow + bin_im_slot<P>(k)) : 0.0f;
      }
  }
  for (int64_t tok0 = tbeg; tok0 < tend; tok0 += TT) {
    const int ntok = (int)((tend - tok0) < TT ? (tend - tok0) : TT);
    if (tok0 != tbeg) __syncthreads();              // the previous tile is fully consumed
    // 1. rdFFT of g (rows t q + i) and x (rows XR + t q + j)
    fft_rows<P, NT, T>(tile, 2 * XR, [&](int r) -> const T* {
      const bool isx = r >= XR;
      const int rr = isx ? r - XR : r;
      const int t = rr / Q, b = rr - t * Q;
      if (t >= ntok) return nullptr;
      return (isx ? x : g) + (tok0 + t) * (int64_t)D + (int64_t)b * P;
    });
    __syncthreads();
    // 2. per bin: S_ij += G_i conj(X_j); Y_j = sum_i conj(C_ij) G_i over the x rows (mirrored:
    // slot k = Re - Im, slot p - k = Re + Im; bin 0 keeps its real pair). A thread reads and
    // writes only its own bins' slots.
#pragma unroll
    for (int u = 0; u < KB; ++u) {
      const int k = threadIdx.x + NT * u;
      if (k < HB) {
        const int kr = G::at(k), ki = G::at(bin_im_slot<P>(k));
        for (int t = 0; t < ntok; ++t) {
          float gr[Q], gi[Q], xr[Q], xi[Q];
#pragma unroll
          for (int b = 0; b < Q; ++b) {
            const int gb = G::row_base(t * Q + b), xb = G::row_base(XR + t * Q + b);
            gr[b] = tile[gb + kr];
            gi[b] = tile[gb + ki];
            xr[b] = tile[xb + kr];
            xi[b] = tile[xb + ki];
          }
#pragma unroll
          for (int j = 0; j < Q; ++j) {
            float yr = 0.0f, yi = 0.0f;
#pragma unroll
            for (int i = 0; i < Q; ++i) {
              if (k == 0) {
                sr[u][i][j] = fmaf(gr[i], xr[j], sr[u][i][j]);
                si[u][i][j] = fmaf(gi[i], xi[j], si[u][i][j]);
                yr = fmaf(cr[u][i][j], gr[i], yr);
                yi = fmaf(ci[u][i][j], gi[i], yi);
              } else {
                sr[u][i][j] = fmaf(gr[i], xr[j], fmaf(gi[i], xi[j], sr[u][i][j]));
                si[u][i][j] = fmaf(gi[i], xr[j], fmaf(-gr[i], xi[j], si[u][i][j]));
                yr = fmaf(cr[u][i][j], gr[i], fmaf(ci[u][i][j], gi[i], yr));
                yi = fmaf(cr[u][i][j], gi[i], fmaf(-ci[u][i][j], gr[i], yi));
              }
            }
            const int xb = G::row_base(XR + t * Q + j);
            tile[xb + kr] = k == 0 ? yr : yr - yi;
            tile[xb + ki] = k == 0 ? yi : yr + yi;
          }
        }
      }
    }
    __syncthreads();
    // 3. rdIFFT (Hartley form) of the grad_x rows straight to HBM
    ifft_rows_mirrored<P, NT, T>(tile + G::row_base(XR), XR, [&](int r) -> T* {
      const int t = r / Q, j = r - t * Q;
      return t < ntok ? grad_x + (tok0 + t) * (int64_t)D + (int64_t)j * P : nullptr;
    });
  }
  // 4. the CTA's cross-spectrum into grad_c (row i q + j)
  griddep_launch_dependents();
#pragma unroll
  for (int u = 0; u < KB; ++u) {
    const int k = threadIdx.x + NT * u;
    if (k < HB) {
#pragma unroll
      for (int i = 0; i < Q; ++i)
#pragma unroll
        for (int j = 0; j < Q; ++j) {
          float* dst = gc_base + (int64_t)(i * Q + j) * P;
          if (store) {
            dst[k] = sr[u][i][j];
            dst[bin_im_slot<P>(k)] = si[u][i][j];
          } else {
            atomicAdd(dst + k, sr[u][i][j]);
            atomicAdd(dst + bin_im_slot<P>(k), si[u][i][j]);
          }
        }
    }
  }
}

template <int P, int Q, typename T, int NT, int TT>
cudaError_t run_small(const void* g, const void* x, const float* chat, void* grad_x, float* grad_c, int64_t B,
                      cudaStream_t s, GcSink* sink) {
  auto kern = k_circ_bwd_small<P, Q, T, NT, TT>;
  const size_t smem = sizeof(float) * (size_t)LayerGeo<P>::words(2 * TT * Q);
  int64_t tiles_per = 1;
  const int slices = layer_gc_slices(1, (B + TT - 1) / TT, num_sms(), &tiles_per);
  float* partial = nullptr;
  cudaError_t e = sink_plan(sink, slices, (int64_t)Q * Q * P, &partial);
  if (e != cudaSuccess || (sink && sink->plan_only)) return e;
  e = set_smem(kern, smem);
  if (e != cudaSuccess) return e;
  if (slices > 1 && !partial) {
    e = launch_zero_f32(grad_c, (int64_t)Q * Q * P, s);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(kern, dim3((unsigned)slices), dim3(NT), smem, s, static_cast<const T*>(g),
                    static_cast<const T*>(x), chat, static_cast<T*>(grad_x), grad_c, partial, B,
                    (int64_t)(tiles_per * TT));
}

template <typename T>
cudaError_t fused_t(const void* g, const void* x, const float* chat, void* grad_x, float* grad_c, int64_t B, int q,
                    int p, cudaStream_t s, GcSink* sink) {
  if (q == 1) {
    // TT tokens per tile: 2 TT q rows of TPR = p/32 threads each fill the CTA in one round
    switch (p) {
      case 512: return run_small<512, 1, T, 128, 4>(g, x, chat, grad_x, grad_c, B, s, sink);
      case 1024: return run_small<1024, 1, T, 128, 2>(g, x, chat, grad_x, grad_c, B, s, sink);
      case 2048: return run_small<2048, 1, T, 256, 2>(g, x, chat, grad_x, grad_c, B, s, sink);
      case 4096: return run_small<4096, 1, T, 512, 2>(g, x, chat, grad_x, grad_c, B, s, sink);
      default: return cudaErrorInvalidValue;
    }
  }
  if (q == 2) {
    switch (p) {
      case 512: return run_small<512, 2, T, 128, 2>(g, x, chat, grad_x, grad_c, B, s, sink);
      case 1024: return run_small<1024, 2, T, 256, 2>(g, x, chat, grad_x, grad_c, B, s, sink);
      case 2048: return run_small<2048, 2, T, 512, 2>(g, x, chat, grad_x, grad_c, B, s, sink);
      case 4096: return run_small<4096, 2, T, 512, 1>(g, x, chat, grad_x, grad_c, B, s, sink);
      default: return cudaErrorInvalidValue;
    }
  }
  // tiles of 4 tokens (2 at p = 1024), or half that while all CTAs hold one tile in one wave
  const int nsm = num_sms();
  if (p == 128 && q == 32) {
    if (layer_fused_small_tiles(B, 2, 4, nsm)) return run_fused<128, 32, 8, T, 2, 4, 8>(g, x, chat, grad_x, grad_c, B, s, sink);
    return run_fused<128, 32, 8, T, 4, 4, 8>(g, x, chat, grad_x, grad_c, B, s, sink);
  }
  if (p == 512 && q == 8) {
    if (layer_fused_small_tiles(B, 2, 1, nsm)) return run_fused<512, 8, 8, T, 2, 4, 8>(g, x, chat, grad_x, grad_c, B, s, sink);
    return run_fused<512, 8, 8, T, 4, 4, 8>(g, x, chat, grad_x, grad_c, B, s, sink);
  }
  if (p == 1024 && q == 4) {
    if (layer_fused_small_tiles(B, 1, 1, nsm)) return run_fused<1024, 4, 4, T, 1, 4, 4>(g, x, chat, grad_x, grad_c, B, s, sink);
    return run_fused<1024, 4, 4, T, 2, 4, 4>(g, x, chat, grad_x, grad_c, B, s, sink);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t take_fused_device_error(unsigned int* flags) {
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  *flags = v;
  return e;
}

// p = 128 (q = 32) at every batch size (backward at D = 4096 with 2-token tiles: 13.8 against
// 14.7 us for the two kernels at B = 1, 16.7 against 19.7 at B = 4, 16.7 against 21.3 at
// B = 12; with 4-token tiles 24.0 against 31.8 at B = 128)
// One or two blocks (D = p or 2 p) from p = 512 on, at every batch size (backward at D = p =
// 4096: 15.0 against 17.3 us at B = 1, 15.4 against 21.7 at B = 256, 115.8 against 188.0 at
// B = 4096; at D = p = 1024, 11.1 / 14.1 against 15.6 / 18.5 us at B = 1 / 256, even at B = 4096;
// at D = 2 p = 2048, 9.2 / 12.5 / 70.3 against 13.0 / 18.8 / 121.8 us at B = 1 / 256 / 4096, and
// at D = 2 p = 8192, 13.4 / 25.8 / 229.5 against 18.1 / 33.5 / 321.1)
bool circ_bwd_fused_supported(int p, int D, int64_t B) {
  (void)B;
  return (p == 512 && D == 4096) || (p == 1024 && D == 4096) || (p == 128 && D == 4096) ||
         ((D == p || D == 2 * p) && p >= 512);
}

cudaError_t launch_circ_bwd_fused(const void* g, const void* x, const float* chat, void* grad_x, float* grad_c,
                                  int64_t B, int D, int p, int dtype, cudaStream_t s, GcSink* sink) {
  const int q = D / p;
  if (dtype == 0) return fused_t<float>(g, x, chat, grad_x, grad_c, B, q, p, s, sink);
  return fused_t<bf16_t>(g, x, chat, grad_x, grad_c, B, q, p, s, sink);
}

}  // namespace rdfft
