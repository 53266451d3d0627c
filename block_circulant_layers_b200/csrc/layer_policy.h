// Launch-shape rules of the block-circulant layer kernels. Plain host arithmetic,
// shared by the CUDA launchers (circ_kernels.cuh) and the host test library, so the
// rules are checked on the CPU.
#pragma once

#include <stdint.h>

namespace rdfft {

// Largest divisor of q that is at most cap (at least 1).
inline int largest_divisor_leq(int q, int cap) {
  for (int d = cap; d >= 1; --d)
    if (q % d == 0) return d;
  return 1;
}

// Output blocks per CTA of the forward / grad_x kernel: as many as the CTA's slots
// cover (qi_max, a divisor of q), and fewer while the grid of gx token groups times
// q / QI block groups would cover fewer than half of the n_sm SMs. The spare slots of
// a CTA then idle; every CTA waits on its own c_hat reads, so more CTAs finish sooner.
inline int layer_qi(int q, int qi_max, int64_t gx, int n_sm) {
  int qi = largest_divisor_leq(q, qi_max);
  while (qi > 1 && gx * (q / qi) < n_sm / 2) qi = largest_divisor_leq(q, qi - 1);
  return qi;
}

// Tokens per CTA of the forward / grad_x kernel for p <= 512: the largest of tt_max, 2, 1
// whose grid keeps all of a token's output blocks in one CTA, i.e. for which layer_qi does
// not split the output blocks over several CTAs (each of which would transform the same input
// rows again); 1 when every tile size would split them. More tokens per CTA let each c_hat
// value read serve more tokens, so the split is the only reason to take fewer (forward at
// D=4096 p=512: B=256 9.6 against 11.5 us, B=64 6.8 against 8.2; D=4096 p=256 B=32 6.5
// against 8.2; D=2048 p=512 B=128 5.8 against 6.6).
inline int layer_x_tokens(int64_t B, int q, int qi_max, int n_sm, int tt_max) {
  const int full = largest_divisor_leq(q, qi_max);
  for (int tt = tt_max; tt > 1; tt /= 2)
    if (layer_qi(q, qi_max, (B + tt - 1) / tt, n_sm) == full) return tt;
  return 1;
}

// Token tiles of the one-kernel backward (circ_bwd_fused.cu): the smaller of its two tile
// sizes (tt_small tokens) while every CTA of the njgroups block groups then holds one tile
// and they all fit in one wave (the kernel runs one CTA per SM); the larger one above. With
// few tokens a CTA's time is one tile's latency, and a smaller tile has less of it (D=4096,
// p=512: 17.4 against 23.1 us at B = 128; p=1024: 14.6 against 16.8 us at B = 128).
inline bool layer_fused_small_tiles(int64_t B, int tt_small, int njgroups, int n_sm) {
  return ((B + tt_small - 1) / tt_small) * njgroups <= n_sm;
}

// Input blocks per grad_c CTA group: a divisor of q, at most 8, with at most
// max_slots complex accumulators per CTA (hb bins x q output blocks x QJ), and fewer
// while ntiles token tiles times q / QJ groups would cover fewer than half the SMs
// (each group then transforms all of g again, which only pays with few tokens).
inline int layer_qj(int q, int hb, int64_t max_slots, int64_t ntiles, int n_sm) {
  int qj = largest_divisor_leq(q, 8);
  while (qj > 1 && (int64_t)hb * q * qj > max_slots) qj = largest_divisor_leq(q, qj - 1);
  while (qj > 1 && ntiles * (q / qj) < n_sm / 2) qj = largest_divisor_leq(q, qj - 1);
  return qj;
}

// Token tiles of the grad_c kernel: half of tt while the half-size tiles number at most half
// the SMs and their grid (tiles times the input-block groups layer_qj then sets) fits one
// wave; with that few tokens each CTA's time is one tile's latency, and a smaller tile has
// less of it. Above, the full tiles (more tokens per c_hat-free pass over g and x).
inline bool layer_gc_half_tiles(int64_t B, int tt, int q, int hb, int64_t max_slots, int n_sm) {
  const int th = tt / 2;
  if (th < 1) return false;
  const int64_t nt = (B + th - 1) / th;
  if (nt > n_sm / 2) return false;
  const int qj = layer_qj(q, hb, max_slots, nt, n_sm);
  return nt * (q / qj) <= n_sm;
}

// Token slices of the persistent grad_c grid: about n_sm CTAs over the njgroups
// input-block groups, each slice a whole number of token tiles (*tiles_per, at least
// 1). Returns the number of slices (at least 1).
inline int layer_gc_slices(int njgroups, int64_t ntiles, int n_sm, int64_t* tiles_per) {
  if (ntiles < 1) ntiles = 1;
  int64_t slices = (n_sm + njgroups - 1) / njgroups;
  if (slices < 1) slices = 1;
  if (slices > ntiles) slices = ntiles;
  *tiles_per = (ntiles + slices - 1) / slices;
  return (int)((ntiles + *tiles_per - 1) / *tiles_per);
}

}  // namespace rdfft
