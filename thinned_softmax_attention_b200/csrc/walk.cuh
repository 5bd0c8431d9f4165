// Device pieces of the Kernel Halving walk shared by the walk kernels (halving.cu) and the fused
// small-instance halving kernel (halving_fused.cu).
#pragma once

#include <cuda_runtime.h>

namespace thin {

// Approximate square root and reciprocal (MUFU): relative error ~1e-7, far below the 1e-4
// near-tie margin of the decisions; they sit on the walk's serial chain.
__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One step of the sigma recursion and the threshold of pair i.  With C = sqrt(2 ln(2/delta_i)) > 1:
//   b >= sigma C:  a = b^2,          sigma' = b
//   otherwise:     a = b sigma C,    sigma'^2 = sigma^2 + max(0, b^2 (1 + 1/C^2) - 2 b sigma / C)
// which is sigma'^2 = sigma^2 + b^2 max(0, 1 + (b^2 - 2a) sigma^2 / a^2) with the two cases of
// a = max(b sigma C, b^2) written out (in the first, sigma <= b/C < b gives sigma'^2 = b^2).
// Returns a; sigma is updated in place.  b^2 <= 0 (a repeated point) keeps sigma and returns 0.
// q = b^2 (1 + 1/C^2), r2 = 2 b / C.
__device__ __forceinline__ float sigma_step(float& sigma, float b2, float b, float C, float q, float r2) {
  const float sc = sigma * C;
  const bool first = b >= sc;
  const float s_else = sqrt_approx(fmaf(sigma, sigma, fmaxf(0.f, fmaf(-r2, sigma, q))));
  const bool live = b2 > 0.f;
  sigma = live ? (first ? b : s_else) : sigma;
  return first ? b2 : b * sc;
}

// The same threshold and recursion in a form with one square root on sigma's dependency chain:
//   a      = max(b^2, b sigma C)
//   sigma' = max(sigma, sqrt(max(sigma - b/C, 0)^2 + b^2))
// Equal to the above: when b >= sigma C the inner max is 0, sqrt(b^2) = b >= sigma, so sigma' = b;
// otherwise sigma'^2 = sigma^2 + max(0, b^2 + (sigma - b/C)^2 - sigma^2) = max(sigma^2,
// (sigma - b/C)^2 + b^2).  b^2 <= 0 (a repeated point) gives a = 0 and leaves sigma unchanged.
// Returns a; rC = 1/C.
__device__ __forceinline__ float sigma_thr(float& sigma, float b2, float C, float rC) {
  const float b2p = fmaxf(b2, 0.f), b = sqrt_approx(b2p);
  const float a = fmaxf(b2p, b * (sigma * C));
  const float d = fmaxf(fmaf(-b, rC, sigma), 0.f);
  sigma = fmaxf(sigma, sqrt_approx(fmaf(d, d, b2p)));
  return a;
}

// The walk of an instance of m <= SEG pairs held by one SEG-lane segment of a warp: lane l of the
// segment owns column l of Delta (d[s] = Delta[s][l]) and alpha of pair l; w_l = 1 - 2u of pair l.
// Pair s keeps its first point iff alpha_s < a_s w_s: every lane compares its own alpha with the
// segment's threshold of pair s and a ballot hands lane s's answer to all.  The thresholds do not
// depend on the decisions, so sigma's recursion runs one pair ahead of the alpha chain.  Returns
// the decision bits of the lane's segment (bit s set = first point kept).
template <int SEG>
__device__ __forceinline__ uint32_t walk_segment(const float (&d)[SEG], float w_l, float C, int lane) {
  const int sl = lane % SEG, shift = lane - sl;
  const float rC = 1.f / C;
  float sigma = 0.f, my = 0.f;
  uint32_t kb = 0;
  float b2n = __shfl_sync(0xffffffffu, d[0], 0, SEG);
  float thn = sigma_thr(sigma, b2n, C, rC) * __shfl_sync(0xffffffffu, w_l, 0, SEG);
#pragma unroll
  for (int s = 0; s < SEG; ++s) {
    const float b2 = b2n, th = thn;
    if (s + 1 < SEG) {
      b2n = __shfl_sync(0xffffffffu, d[s + 1], s + 1, SEG);
      thn = sigma_thr(sigma, b2n, C, rC) * __shfl_sync(0xffffffffu, w_l, s + 1, SEG);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, my < th);
    const bool keep = !(b2 > 0.f) || ((bal >> (shift + s)) & 1u);
    if (sl > s) my = fmaf(keep ? 1.f : -1.f, d[s], my);
    kb |= (uint32_t)keep << s;
  }
  if constexpr (SEG < 32) kb |= 0xFFFFFFFFu << (SEG & 31);   // pairs past the segment read as kept
  return kb;
}

// 32 decisions of the pairs base..base+31 by one warp (the same arithmetic as walk_segment<32>):
// lane l owns alpha of pair base+l in `my`, b2l = b^2 and wl = 1 - 2u of pair base+l, and col(s)
// returns Delta[base+s][base+l], the contribution of pair base+s to this lane's pair.  sigma carries
// over from block to block.  Lanes that hold no pair have b2l = 0 and wl = 0: their steps keep the
// first point and only change alpha of lanes that hold no pair either.
template <typename Col>
__device__ __forceinline__ uint32_t walk_block32(float& my, float& sigma, float b2l, float wl, float C, float rC, int lane,
                                                 Col col) {
  uint32_t kb = 0;
  float b2n = __shfl_sync(0xffffffffu, b2l, 0);
  float thn = sigma_thr(sigma, b2n, C, rC) * __shfl_sync(0xffffffffu, wl, 0);
#pragma unroll
  for (int s = 0; s < 32; ++s) {
    const float b2 = b2n, th = thn;
    if (s + 1 < 32) {
      b2n = __shfl_sync(0xffffffffu, b2l, s + 1);
      thn = sigma_thr(sigma, b2n, C, rC) * __shfl_sync(0xffffffffu, wl, s + 1);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, my < th);
    const bool keep = !(b2 > 0.f) || ((bal >> s) & 1u);
    if (lane > s) my = fmaf(keep ? 1.f : -1.f, col(s), my);
    kb |= (uint32_t)keep << s;
  }
  return kb;
}

// Thresholds of the pairs base..base+31, computed by one warp ahead of the warp that walks them:
// th = a (1 - 2u) for a pair with b^2 > 0 and +inf otherwise (such a pair keeps its first point).
// b2l and wl are b^2 and 1 - 2u of pair base + lane (0 for lanes that hold no pair); sigma carries
// over from block to block.  Lane l returns the threshold of pair base + l.  The sigma recursion,
// the threshold and their order are those of walk_block32, so the decisions are the same.
__device__ __forceinline__ float thresholds32(float& sigma, float b2l, float wl, float C, float rC, int lane) {
  float th_l = __int_as_float(0x7f800000);
#pragma unroll
  for (int s = 0; s < 32; ++s) {
    const float b2 = __shfl_sync(0xffffffffu, b2l, s);
    const float a = sigma_thr(sigma, b2, C, rC);
    if (lane == s && b2 > 0.f) th_l = a * wl;
  }
  return th_l;
}

// The decisions of pairs base..base+31 with thresholds from thresholds32 (th_l of pair base+lane):
// the warp's only serial chain is alpha -> ballot -> alpha.  Pairs s >= steps are padding and keep
// their first point; their alpha updates touch only lanes that hold no pair.
template <typename Col>
__device__ __forceinline__ uint32_t walk_block32_th(float& my, float th_l, int steps, int lane, Col col) {
  // the column is read into registers first so that no shared-memory load sits on the chain
  float d[32];
#pragma unroll
  for (int s = 0; s < 32; ++s) d[s] = col(s);
  uint32_t kb = 0;
#pragma unroll
  for (int s = 0; s < 32; ++s) {
    const float th = __shfl_sync(0xffffffffu, th_l, s);
    const uint32_t bal = __ballot_sync(0xffffffffu, my < th);
    const bool keep = s >= steps || ((bal >> s) & 1u);
    if (lane > s) my = fmaf(keep ? 1.f : -1.f, d[s], my);
    kb |= (uint32_t)keep << s;
  }
  return kb;
}

}  // namespace thin
