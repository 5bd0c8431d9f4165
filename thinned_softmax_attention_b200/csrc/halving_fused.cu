// Kernel Halving steps of up to 512 points per instance in one launch each.
//
// The three-launch step of halving.cu (c^2, pair-difference Gram, walk + gather) reads every
// point from HBM three times and round-trips the pair-difference matrix through HBM.  This file
// does a whole step in one pass over the points, in three kernels:
//   halve_fused_kernel<NP>  instances of <= 128 points (the bulk of the Express batch thinning),
//                           persistent, units of 128 rows -- described below;
//   halve256_kernel         129..256 points, one CTA per instance (further down);
//   halve512_kernel         257..512 points with D <= 128, one CTA per instance, the pair
//                           differences as a packed upper triangle (further down).
// The persistent kernel's steps per unit:
//
//   TMA      a unit of 128 point rows lands in one pipeline stage as (E+D)/64 chunks of
//            128 rows x 64 bf16 (128-byte swizzle); a unit is 4 instances of <= 32 points
//            (NP = 32), 2 of <= 64 (NP = 64) or 1 of <= 128 (NP = 128)
//   c^2      max |v| of each instance, read from the stage
//   tcgen05  kk = K K^T and vv = V V^T of each instance (A = the unit's 128 rows, B = the
//            instance's NP rows), fp32 accumulators in TMEM
//   epilogue kappa = 2^(kk s log2 e) (vv + c^2) and the pair differences
//            Delta[j][i] = kappa[2j][2i] - kappa[2j][2i+1] - kappa[2j+1][2i] + kappa[2j+1][2i+1]
//            into shared memory (thread = TMEM lane = point row; the row difference is a shuffle)
//   walk     the sequential decisions of each instance, with the same arithmetic as the walk
//            kernels of halving.cu, so the decisions are the same
//   gather   the kept rows, from the stage straight to the destination rows
//
// Warp roles (320 threads, one CTA per SM, persistent over units u = blockIdx.x + k gridDim.x):
//   warp 0     TMA producer (one thread)     warp 1     MMA issuer (one thread), TMEM owner
//   warps 2,3  walkers of even k             warps 4-7  epilogue (warp w reads TMEM lanes 32(w%4)..)
//   warps 8,9  walkers of odd k
// Pipeline: `nst` shared-memory stages, two TMEM accumulator buffers of 256 columns and two
// Delta buffers (one per walker set).  Every mbarrier wait is bounded; after a time-out the
// kernel stops, waits (bounded) for the copies and MMAs it started, frees TMEM and reports
// through the status word (code 3, status[1] = CTA).
#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "walk.cuh"

namespace thin {

namespace {

using namespace tc;

struct FusedMaps {
  CUtensorMap k, v;
};

constexpr uint32_t kChunk = 128 * 128;   // 128 rows x 64 bf16 (one feature chunk of a unit)
constexpr int kThreads = 320;
constexpr int kMaxChunks = 5;             // (E + D) / 64 <= 5 (the stages must fit in shared memory)

template <int NP>
struct FusedShape {
  static constexpr int PAIRS = NP / 2;                     // pairs per instance
  static constexpr int IPU = 128 / NP;                     // instances per unit
  static constexpr int LD = PAIRS + 1;                     // Delta row stride (floats): no bank conflicts
  static constexpr int DELTA_INST = PAIRS * LD;            // floats per instance
  static constexpr int DELTA_SET = IPU * DELTA_INST;       // floats per walker set
  static constexpr int SEG = PAIRS < 32 ? PAIRS : 32;      // walk lanes per instance (NP <= 64)
};

// Copy the kept point of pairs [i0, i1) of one instance from the stage (unit rows row0 + 2i or
// row0 + 2i + 1) to destination rows dst_row + i, with its token index.  One warp; lane = one
// 16-byte unit of a row (K units first), four rows in flight.
template <bool GAP = false, typename Bit>
__device__ __forceinline__ void gather_from_stage(const StepArgs& a, int64_t dst_row, int64_t src_row, uint32_t tok_base,
                                                  const uint8_t* st, int row0, int i0, int i1, Bit bit, int lane,
                                                  int EC, int NC, uint32_t chunk_bytes = kChunk, uint32_t gap_u = 0,
                                                  uint32_t gp0 = 0) {
  // token index of point p of the instance: tok_base + p k (k = subsample stride, 1 without
  // subsample); for a subsample of another ratio tok_base + floor(((gp0 + p) S + U) / S') with
  // gp0 = 2 pair0 and U = gap_u, the subsample's own formula
  const bool tokens = a.src_kind == SRC_TOKENS;
  constexpr bool gapped = GAP;   // (the caller's: tokens subsampled with a non-integer ratio)
  const uint32_t k = a.sub_stride > 1 ? (uint32_t)a.sub_stride : 1u;
  for (int i = i0 + lane; i < i1; i += 32) {
    const int p = 2 * i + (bit(i) ? 0 : 1);
    a.dstIdx[dst_row + i] =
        !tokens ? a.srcIdx[src_row + p]
                : gapped ? (int32_t)(tok_base + (uint32_t)(((uint64_t)(gp0 + p) * (uint64_t)a.S_full + gap_u) / (uint64_t)a.S_sub))
                         : (int32_t)(tok_base + (uint32_t)p * k);
  }
  const int units = NC * 8, kw = a.E / 8, vw = a.D / 8;
  uint4* dK = (uint4*)a.dstK;
  uint4* dV = (uint4*)a.dstV;
  for (int w = lane; w < units; w += 32) {
    const int c = w >> 3, x = w & 7;
    uint4* dst = c < EC ? dK + dst_row * kw + c * 8 + x : dV + dst_row * vw + (c - EC) * 8 + x;
    const int stride = c < EC ? kw : vw;
    const uint8_t* src = st + c * chunk_bytes;
    for (int i = i0; i < i1; i += 8) {
      uint4 buf[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (i + j < i1) {
          const int R = row0 + 2 * (i + j) + (bit(i + j) ? 0 : 1);
          buf[j] = *(const uint4*)(src + R * 128 + ((x ^ (R & 7)) << 4));
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (i + j < i1) dst[(int64_t)(i + j) * stride] = buf[j];
    }
  }
}

// GAP: token runs subsampled with a non-integer ratio (a separate instance of the kernel, so that
// the others carry none of its code).
template <int NP, bool GAP>
__global__ void __launch_bounds__(kThreads, 1) halve_fused_kernel(const __grid_constant__ FusedMaps maps,
                                                                  const StepArgs a, int n_units, int nst) {
  using Sh = FusedShape<NP>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, by an offset from the array itself so that the compiler keeps every pointer
  // derived from it in the shared address space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int EC = a.E / 64, NC = (a.E + a.D) / 64;
  const uint32_t stage_bytes = (uint32_t)NC * kChunk;
  float* delta = (float*)(smem + nst * stage_bytes);   // [2 sets][IPU][PAIRS][LD]
  __shared__ __align__(8) uint64_t bars[24];
  uint64_t* full = bars;            // [3] stage landed (TMA)
  uint64_t* empty = bars + 3;       // [3] stage gathered (64 walker lanes)
  uint64_t* tfull = bars + 6;       // [2] accumulators ready (MMA commit)
  uint64_t* tempty = bars + 8;      // [2] accumulators read (128 epilogue threads)
  uint64_t* dfull = bars + 10;      // [2] Delta written (128 epilogue threads)
  uint64_t* dempty = bars + 12;     // [2] Delta taken by the walkers (64 walker lanes)
  uint64_t* bitsf = bars + 14;      // [2] decisions of a 128-point instance published (32 lanes)
  uint64_t* cmax = bars + 16;       // partial max |v| exchanged among the epilogue threads
  uint64_t* mdone = bars + 17;      // every MMA of this CTA complete
  uint64_t* thf = bars + 18;        // [2] thresholds of one block of 32 pairs published (32 lanes)
  uint64_t* fixed = bars + 20;      // [3] stage compacted (subsample of a non-integer ratio; 128 threads)
  uint64_t* cfix = bars + 23;       // the compaction's loads of one chunk done / its stores done (128)
  __shared__ float red[2][4];
  __shared__ uint32_t bits_s[2][2];
  __shared__ float thr_s[2][64];
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_s = 0;
    for (int s = 0; s < nst; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 64);
      mbar_init(fixed + s, 128);
    }
    mbar_init(cfix, 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 128);
      mbar_init(dfull + b, 128);
      mbar_init(dempty + b, 64);
      mbar_init(bitsf + b, 32);
      mbar_init(thf + b, 32);
    }
    mbar_init(cmax, 128);
    mbar_init(mdone, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&tmem_base_s, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort = &abort_s;
  const int n_local = n_units > (int)blockIdx.x ? (n_units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  // token runs subsampled with a non-integer ratio: an instance's n points are n of the tokens
  // [t(2 pair0), t(2 pair0 + n - 1)] (t = the subsample's index formula), at most NP of them, so
  // the box of NP rows from the first holds them all; the epilogue warps move the selected rows
  // up to rows 0..n-1 before the MMAs read the stage
  constexpr bool gapped = GAP;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // lane ii < IPU handles instance ii of the unit: its record is read before the stage is free
    const bool tokens = a.src_kind == SRC_TOKENS;
    int issued = 0;
    for (int k = 0; k < n_local; ++k) {
      const int s = k % nst;
      const int u = blockIdx.x + k * gridDim.x;
      const int i0 = u * Sh::IPU, ni = min(Sh::IPU, a.n_inst - i0);
      int row = 0, h = 0;
      if (lane < ni) {
        const HalveInst in = a.inst[i0 + lane];
        // token runs: first row of the instance, in units of the subsample stride k for strided runs
        if (gapped) {
          const uint32_t U = sub_offset(a, in);
          row = (int)(in.src_row + (int64_t)(((uint64_t)(2 * in.pair0) * (uint64_t)a.S_full + U) / (uint64_t)a.S_sub));
        } else {
          row = (int)(tokens ? (a.sub_stride > 1 ? in.src_row / a.sub_stride : in.src_row) + 2 * (int64_t)in.pair0
                             : in.src_row);
        }
        h = (int)(in.bh % (uint32_t)a.H);
      }
      if (!warp_wait(empty + s, ((k / nst) & 1) ^ 1, abort)) break;
      if (lane == 0) mbar_expect_tx(full + s, (uint32_t)(ni * NC) * (NP * 128));
      __syncwarp();
      if (lane < ni) {
        uint8_t* st = smem + s * stage_bytes + lane * (NP * 128);
        for (int c = 0; c < NC; ++c) {
          const bool isk = c < EC;
          const CUtensorMap* m = isk ? &maps.k : &maps.v;
          const int x = (isk ? c : c - EC) * 64;
          if (!tokens) tma_load_2d(st + c * kChunk, m, full + s, x, row);
          else if (a.sub_stride > 1) tma_load_4d(st + c * kChunk, m, full + s, x, h, 0, row);
          else tma_load_3d(st + c * kChunk, m, full + s, x, h, row);
        }
      }
      issued = k + 1;
    }
    // leave no copy in flight: the last fill of every stage has landed
    if (lane == 0) {
      for (int k = max(0, issued - nst); k < issued; ++k) {
        const long long t0 = clock64();
        while (!mbar_try_wait(full + (k % nst), (k / nst) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, NP, false);
      const uint32_t base = smem_u32(smem);
      for (int k = 0; k < n_local; ++k) {
        const int s = k % nst, b = k & 1;
        if (!mbar_wait((gapped ? fixed : full) + s, (k / nst) & 1, abort)) break;
        if (!mbar_wait(tempty + b, ((k >> 1) & 1) ^ 1, abort)) break;
        tc_fence_after();
        const uint32_t st = base + s * stage_bytes;
        const uint32_t d = tmem + (uint32_t)b * 256u;
        for (int c = 0; c < NC; ++c) {
          const uint32_t ra = st + c * kChunk;
          const uint32_t dc = d + (c < EC ? 0u : 128u);
          const bool first = c == 0 || c == EC;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = sw128_desc(ra + kk * 32, 16, 1024);
#pragma unroll
            for (int ii = 0; ii < Sh::IPU; ++ii)
              umma_bf16(dc + ii * NP, adesc, sw128_desc(ra + ii * (NP * 128) + kk * 32, 16, 1024), IDESC,
                        (!first || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(tfull + b);
      }
      umma_commit(mdone);
      const long long t0 = clock64();
      while (!mbar_try_wait(mdone, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 4;                 // = warp % 4: TMEM lanes 32 ew .. 32 ew + 31
    const int r = ew * 32 + lane;            // unit row = TMEM lane
    const int ii = r / NP, lr = r % NP;      // instance within the unit, row within the instance
    const uint32_t lane_base = (uint32_t)(ew * 32) << 16;
    const int m = a.m;
    int cfix_uses = 0;   // completions of cfix so far (its parity)
    for (int k = 0; k < n_local; ++k) {
      const int s = k % nst, b = k & 1;
      const int u = blockIdx.x + k * gridDim.x;
      const bool live = u * Sh::IPU + ii < a.n_inst;
      if (!warp_wait(full + s, (k / nst) & 1, abort)) break;
      if (gapped) {
        // move the selected rows of each instance to rows 0..n-1 of its slot: thread item j is
        // unit row R = t/8 + 16 j (instance R / NP, point p = R % NP) and 16-byte unit x = t % 8;
        // all loads of a chunk, then all stores (a bounded wait on cfix between)
        const int t = ew * 32 + lane, x = t & 7;
        int srow[8];
        // the subsample offset U and first point of each instance of the unit, once per instance
        // (a thread's rows span at most a few instances; U costs a Philox evaluation)
        int cur_ii = -1;
        uint32_t cur_u = 0;
        uint64_t cur_g0 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int R = (t >> 3) + 16 * j, ii = R / NP, p = R % NP;
          srow[j] = R;
          const int inst = u * Sh::IPU + ii;
          if (p < a.n && inst < a.n_inst) {
            if (ii != cur_ii) {
              const HalveInst gi = a.inst[inst];
              cur_ii = ii;
              cur_u = sub_offset(a, gi);
              cur_g0 = 2ull * gi.pair0;
            }
            const int64_t t0 = (int64_t)((cur_g0 * (uint64_t)a.S_full + cur_u) / (uint64_t)a.S_sub);
            const int64_t tp = (int64_t)(((cur_g0 + p) * (uint64_t)a.S_full + cur_u) / (uint64_t)a.S_sub);
            srow[j] = ii * NP + (int)(tp - t0);
          }
        }
        uint8_t* stg = smem + s * stage_bytes;
        bool fok = true;
        for (int c = 0; c < NC && fok; ++c) {
          uint8_t* ch = stg + c * kChunk;
          uint4 buf[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) buf[j] = *(const uint4*)(ch + srow[j] * 128 + ((x ^ (srow[j] & 7)) << 4));
          mbar_arrive(cfix);
          fok = warp_wait(cfix, cfix_uses++ & 1, abort);
          if (!fok) break;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int R = (t >> 3) + 16 * j;
            if (srow[j] != R) *(uint4*)(ch + R * 128 + ((x ^ (R & 7)) << 4)) = buf[j];
          }
          mbar_arrive(cfix);
          fok = warp_wait(cfix, cfix_uses++ & 1, abort);
        }
        if (!fok) break;
        fence_proxy_async_smem();   // the MMAs read the stage through the async proxy
        mbar_arrive(fixed + s);
      }
      // c = max |v| over the instance: this row's part, then across the instance's threads
      float mx = 0.f;
      if (live && lr < a.n) {
        const uint8_t* rowp = smem + s * stage_bytes + r * 128;
        for (int c = EC; c < NC; ++c) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 w = *(const uint4*)(rowp + c * kChunk + ((q ^ (r & 7)) << 4));
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              mx = fmax3(mx, fabsf(__uint_as_float(ws[e] << 16)), fabsf(__uint_as_float(ws[e] & 0xFFFF0000u)));
          }
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) red[k & 1][ew] = mx;
      mbar_arrive(cmax);
      if (!warp_wait(cmax, k & 1, abort)) break;
      float cm;
      if (NP == 128) cm = fmaxf(fmaxf(red[k & 1][0], red[k & 1][1]), fmaxf(red[k & 1][2], red[k & 1][3]));
      else if (NP == 64) cm = fmaxf(red[k & 1][2 * ii], red[k & 1][2 * ii + 1]);
      else cm = red[k & 1][ii];
      const float c2 = cm * cm;
      if (!warp_wait(tfull + b, (k >> 1) & 1, abort)) break;
      if (!warp_wait(dempty + b, ((k >> 1) & 1) ^ 1, abort)) break;
      tc_fence_after();
      float* D = delta + b * Sh::DELTA_SET + ii * Sh::DELTA_INST;
      const int pj = lr >> 1;
      const bool writer = (lr & 1) == 0;
      const uint32_t kcol = tmem + lane_base + (uint32_t)b * 256u + (uint32_t)(ii * NP);
      // the walk reads Delta[j][i] for j <= i only: a chunk of columns left of this warp's 16 pair
      // rows (of its instance) holds none of those and is skipped
#pragma unroll 1
      for (int cc = ew % (NP / 32); cc < NP / 32; ++cc) {
        float kk[32], vv[32];
        tmem_ld32(kcol + cc * 32, kk);
        tmem_ld32(kcol + 128 + cc * 32, vv);
        tmem_ld_wait();
        float dd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float k0 = exp2f(kk[2 * i] * a.scale_log2e) * (vv[2 * i] + c2);
          const float k1 = exp2f(kk[2 * i + 1] * a.scale_log2e) * (vv[2 * i + 1] + c2);
          dd[i] = k0 - k1;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) dd[i] -= __shfl_xor_sync(0xffffffffu, dd[i], 1);
        if (writer) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int pi = cc * 16 + i;
            D[pj * Sh::LD + pi] = (live && pj < m && pi < m) ? dd[i] : 0.f;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty + b);
      mbar_arrive(dfull + b);
    }
  } else {
    // ------------------------------------------------------------------ walkers (warps 2, 3, 8, 9)
    const int set = warp >= 8 ? 1 : 0, wi = warp & 1;
    const int m = a.m, nb = a.m_pad >> 5;
    const float C = a.C;
    for (int k = set; k < n_local; k += 2) {
      const int s = k % nst;
      const int u = blockIdx.x + k * gridDim.x;
      const float* Dset = delta + set * Sh::DELTA_SET;
      const uint8_t* st = smem + s * stage_bytes;
      if constexpr (NP <= 64) {
        // one instance per SEG-lane segment: NP = 64 -> warp wi walks instance wi;
        // NP = 32 -> warp wi walks instances 2wi (lanes 0-15) and 2wi+1 (lanes 16-31)
        constexpr int SEG = Sh::SEG;
        const int seg = lane / SEG, sl = lane % SEG;
        const int ii = wi * (32 / SEG) + seg;
        const int inst = u * Sh::IPU + ii;
        const bool live = inst < a.n_inst;
        HalveInst in{};
        if (live) in = a.inst[inst];
        if (!warp_wait(dfull + set, (k >> 1) & 1, abort)) break;
        const float* D = Dset + ii * Sh::DELTA_INST;
        float d[SEG];
#pragma unroll
        for (int q = 0; q < SEG; ++q) d[q] = D[q * Sh::LD + sl];
        __syncwarp();
        mbar_arrive(dempty + set);
        const float w_l =
            (live && sl < m) ? 1.f - 2.f * philox_uniform(a.seed, in.ctr_bh, in.round_id, in.pair0 + (uint32_t)sl) : 0.f;
        const uint32_t kb = walk_segment<SEG>(d, w_l, C, lane);
        if (!warp_wait(full + s, (k / nst) & 1, abort)) break;   // (complete: orders the stage reads)
#pragma unroll
        for (int g = 0; g < 32 / SEG; ++g) {
          const int src = g * SEG;
          const int gi = u * Sh::IPU + wi * (32 / SEG) + g;
          const uint32_t kbg = __shfl_sync(0xffffffffu, kb, src);
          const int64_t dst_row = __shfl_sync(0xffffffffu, in.dst_row, src);
          const int64_t src_row = __shfl_sync(0xffffffffu, in.src_row, src);
          const uint32_t tok_base = __shfl_sync(
              0xffffffffu, gapped ? in.tok0 : in.tok0 + 2u * in.pair0 * (a.sub_stride > 1 ? (uint32_t)a.sub_stride : 1u), src);
          const uint32_t gap_u = __shfl_sync(0xffffffffu, gapped && live ? sub_offset(a, in) : 0u, src);
          const uint32_t gp0 = __shfl_sync(0xffffffffu, 2u * in.pair0, src);
          if (gi < a.n_inst) {
            if (a.trace && lane == 0) a.trace[a.trace_base + (size_t)gi * nb] = kbg;
            gather_from_stage<GAP>(a, dst_row, src_row, tok_base, st, (wi * (32 / SEG) + g) * NP, 0, m,
                              [kbg](int i) { return ((kbg >> i) & 1u) != 0; }, lane, EC, NC, kChunk, gap_u, gp0);
          }
        }
      } else {
        // one instance of <= 64 pairs as two blocks of 32: warp wi = 1 computes the thresholds
        // (sigma's recursion) of block 0 then block 1, warp wi = 0 walks each block as soon as its
        // thresholds are published (lane l owns pairs l and l + 32), then publishes the decisions;
        // both warps gather half of the kept rows
        const int inst = u;
        const bool live = inst < a.n_inst;
        const int half = (m + 1) / 2;
        HalveInst in{};
        if (live) in = a.inst[inst];
        if (!warp_wait(dfull + set, (k >> 1) & 1, abort)) break;
        const float* D = Dset;
        uint32_t kb0 = 0, kb1 = 0;
        if (wi == 1) {
          const float rC = 1.f / C;
          float sigma = 0.f;
#pragma unroll 1
          for (int blk = 0; blk < 2; ++blk) {
            const int p = 32 * blk + lane;
            const float b2l = D[p * Sh::LD + p];
            const float wl =
                (live && p < m) ? 1.f - 2.f * philox_uniform(a.seed, in.ctr_bh, in.round_id, in.pair0 + (uint32_t)p) : 0.f;
            thr_s[set][p] = thresholds32(sigma, b2l, wl, C, rC, lane);
            __syncwarp();
            mbar_arrive(thf + set);
          }
          __syncwarp();
          mbar_arrive(dempty + set);
          if (!warp_wait(bitsf + set, (k >> 1) & 1, abort)) break;
          kb0 = bits_s[set][0];
          kb1 = bits_s[set][1];
        } else {
          float my0 = 0.f, my1 = 0.f;
          if (!warp_wait(thf + set, 0, abort)) break;
          kb0 = walk_block32_th(my0, thr_s[set][lane], min(32, m), lane, [&](int q) { return D[q * Sh::LD + lane]; });
#pragma unroll
          for (int q = 0; q < 32; ++q) my1 = fmaf(((kb0 >> q) & 1u) ? 1.f : -1.f, D[q * Sh::LD + 32 + lane], my1);
          if (!warp_wait(thf + set, 1, abort)) break;
          kb1 = walk_block32_th(my1, thr_s[set][32 + lane], m - 32, lane,
                                [&](int q) { return D[(32 + q) * Sh::LD + 32 + lane]; });
          __syncwarp();
          mbar_arrive(dempty + set);
          if (lane == 0) {
            bits_s[set][0] = kb0;
            bits_s[set][1] = kb1;
          }
          __syncwarp();
          mbar_arrive(bitsf + set);
        }
        if (!warp_wait(full + s, (k / nst) & 1, abort)) break;   // (complete: orders the stage reads)
        if (live) {
          if (a.trace && wi == 0 && lane < nb) a.trace[a.trace_base + (size_t)inst * nb + lane] = lane ? kb1 : kb0;
          auto bit = [kb0, kb1](int i) { return (((i < 32 ? kb0 : kb1) >> (i & 31)) & 1u) != 0; };
          const uint32_t tok_base = gapped ? in.tok0 : in.tok0 + 2u * in.pair0 * (a.sub_stride > 1 ? (uint32_t)a.sub_stride : 1u);
          gather_from_stage<GAP>(a, in.dst_row, in.src_row, tok_base, st, 0, wi ? half : 0, wi ? m : half, bit, lane, EC, NC,
                            kChunk, gapped ? sub_offset(a, in) : 0u, 2u * in.pair0);
        }
      }
      __syncwarp();
      mbar_arrive(empty + s);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_s && threadIdx.x == 0 && a.status) {
    if (atomicCAS(a.status, 0, 3) == 0) a.status[1] = (int)blockIdx.x;
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int NP>
cudaError_t launch_np(const StepArgs& a, cudaStream_t st) {
  FusedMaps maps;
  bool ok;
  if (a.src_kind == SRC_TOKENS && a.sub_stride > 1) {
    ok = make_map_4d_strided(&maps.k, a.srcK, a.src_rows, a.H, a.E, a.sub_stride, NP) &&
         make_map_4d_strided(&maps.v, a.srcV, a.src_rows, a.H, a.D, a.sub_stride, NP);
  } else if (a.src_kind == SRC_TOKENS) {
    ok = make_map_3d(&maps.k, a.srcK, a.src_rows, a.H, a.E, NP) && make_map_3d(&maps.v, a.srcV, a.src_rows, a.H, a.D, NP);
  } else {
    ok = make_map_2d(&maps.k, a.srcK, a.src_rows, a.E, a.E, NP) && make_map_2d(&maps.v, a.srcV, a.src_rows, a.D, a.D, NP);
  }
  if (!ok) return cudaErrorInvalidValue;
  const int NC = (a.E + a.D) / 64;
  const size_t delta_bytes = 2 * (size_t)FusedShape<NP>::DELTA_SET * 4;
  const size_t static_bytes = 1024;   // barriers and small arrays declared in the kernel
  int nst = 3;
  while (nst > 2 && 1024 + (size_t)nst * NC * kChunk + delta_bytes + static_bytes > 227 * 1024) --nst;
  size_t sm = 1024 + (size_t)nst * NC * kChunk + delta_bytes;
  if (sm < 120 * 1024) sm = 120 * 1024;   // one CTA per SM: each holds all 512 TMEM columns
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const bool gap = a.src_kind == SRC_TOKENS && a.S_sub < a.S_full && a.sub_stride < 2;
  auto kern = gap ? halve_fused_kernel<NP, true> : halve_fused_kernel<NP, false>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const int n_units = (a.n_inst + FusedShape<NP>::IPU - 1) / FusedShape<NP>::IPU;
  const int grid = n_units < sms ? n_units : sms;
  kern<<<grid, kThreads, sm, st>>>(maps, a, n_units, nst);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Instances of 129..256 points: one CTA per instance (its 256 rows, 32 KB per feature chunk, and the
// 128 x 128 pair differences take the shared memory of an SM).  Warps: 0 TMA, 1 MMA (TMEM owner),
// 2-5 epilogue (warp w reads TMEM lanes 32 (w % 4)..), 6 sigma's recursion, 7 the walk; all eight
// gather.  The Gram takes two passes through the 512 TMEM columns: rows 0..127 against all 256 rows
// (kk in columns 0..255, vv in 256..511), then rows 128..255 against themselves (columns 0..127 and
// 256..383), so Delta rows 0..63 are written while the second pass runs.  Every barrier is used
// once (phase 0) and every wait is bounded.
// One instance (`inst` of step `a`) with the CTA's 256 threads; `smem` is the 1024-byte aligned
// dynamic shared memory, `tmem` 512 allocated TMEM columns.  The barriers are initialised here and
// invalidated before returning, so a persistent caller can run one instance after another.
// Returns false when a bounded wait gave up (reported in a.status).
__device__ __forceinline__ bool halve256_body(const FusedMaps& maps, const StepArgs& a, const int inst, uint8_t* smem,
                                              const uint32_t tmem) {
  constexpr int LD = 129;                       // Delta row stride (floats)
  constexpr uint32_t CB = 2 * kChunk;           // one feature chunk: 256 rows x 64 bf16
  const int EC = a.E / 64, NC = (a.E + a.D) / 64;
  float* D = (float*)(smem + NC * CB);          // [128][LD]
  __shared__ __align__(8) uint64_t bars[20];
  uint64_t* full = bars;          // rows landed
  uint64_t* tfull0 = bars + 1;    // first-pass accumulators ready
  uint64_t* tempty0 = bars + 2;   // first-pass accumulators read (128)
  uint64_t* tfull1 = bars + 3;    // second-pass accumulators ready
  uint64_t* cmax = bars + 4;      // c exchanged among the epilogue threads (128)
  uint64_t* dhalf = bars + 5;     // Delta rows 0..63 written (128)
  uint64_t* dfull = bars + 6;     // Delta rows 64..127 written (128)
  uint64_t* mdone = bars + 8;     // every MMA complete
  uint64_t* thf = bars + 9;       // [4] thresholds of pair block b published (32)
  uint64_t* bitsb = bars + 13;    // [4] decisions of pair block b published (32; blocks in order)
  __shared__ float red[4];
  __shared__ float thr_s[128];
  __shared__ uint32_t bits_s[4];
  __shared__ volatile int abort_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = a.m, n = a.n;
  if (threadIdx.x == 0) {
    abort_s = 0;
    mbar_init(full, 1);
    mbar_init(tfull0, 1);
    mbar_init(tempty0, 128);
    mbar_init(tfull1, 1);
    mbar_init(cmax, 128);
    mbar_init(dhalf, 128);
    mbar_init(dfull, 128);
    mbar_init(mdone, 1);
    for (int b = 0; b < 4; ++b) {
      mbar_init(thf + b, 32);
      mbar_init(bitsb + b, 32);
    }
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  volatile int* abort = &abort_s;
  const HalveInst in = a.inst[inst];
  const bool tokens = a.src_kind == SRC_TOKENS;
  const int ks = a.sub_stride > 1 ? a.sub_stride : 1;

  if (warp == 0) {
    if (lane == 0) {
      const int row = (int)(tokens ? in.src_row / ks + 2 * (int64_t)in.pair0 : in.src_row);
      const int h = (int)(in.bh % (uint32_t)a.H);
      mbar_expect_tx(full, (uint32_t)NC * CB);
      for (int c = 0; c < NC; ++c) {
        const bool isk = c < EC;
        const CUtensorMap* mp = isk ? &maps.k : &maps.v;
        const int x = (isk ? c : c - EC) * 64;
        for (int blk = 0; blk < 2; ++blk) {
          uint8_t* dst = smem + c * CB + blk * kChunk;
          if (!tokens) tma_load_2d(dst, mp, full, x, row + 128 * blk);
          else if (ks > 1) tma_load_4d(dst, mp, full, x, h, 0, row + 128 * blk);
          else tma_load_3d(dst, mp, full, x, h, row + 128 * blk);
        }
      }
      const long long t0 = clock64();
      while (!mbar_try_wait(full, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t base = smem_u32(smem);
      bool ok = mbar_wait(full, 0, abort);
      if (ok) {
        tc_fence_after();
        constexpr uint32_t I256 = idesc_bf16(128, 256, false), I128 = idesc_bf16(128, 128, false);
        for (int c = 0; c < NC; ++c) {
          const uint32_t ra = base + c * CB;
          const uint32_t dc = tmem + (c < EC ? 0u : 256u);
          const bool first = c == 0 || c == EC;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(dc, sw128_desc(ra + kk * 32, 16, 1024), sw128_desc(ra + kk * 32, 16, 1024), I256,
                      (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit(tfull0);
        ok = mbar_wait(tempty0, 0, abort);
        if (ok) {
          tc_fence_after();
          for (int c = 0; c < NC; ++c) {
            const uint32_t rb = base + c * CB + kChunk;
            const uint32_t dc = tmem + (c < EC ? 0u : 256u);
            const bool first = c == 0 || c == EC;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(dc, sw128_desc(rb + kk * 32, 16, 1024), sw128_desc(rb + kk * 32, 16, 1024), I128,
                        (!first || kk > 0) ? 1u : 0u);
          }
          umma_commit(tfull1);
        }
      }
      umma_commit(mdone);
      const long long t0 = clock64();
      while (!mbar_try_wait(mdone, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------------ epilogue
    const int q4 = warp & 3;                    // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;               // row r of the first pass (row 128 + r of the second)
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    bool ok = warp_wait(full, 0, abort);
    float c2 = 0.f;
    if (ok) {
      // four independent max chains (one per 32-bit word of a 16-byte unit)
      float m4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        const int R = r + 128 * blk;
        if (R < n) {
          const uint8_t* rowp = smem + blk * kChunk + r * 128;
          for (int c = EC; c < NC; ++c) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint4 w = *(const uint4*)(rowp + c * CB + ((q ^ (r & 7)) << 4));
              const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                m4[e] = fmax3(m4[e], fabsf(__uint_as_float(ws[e] << 16)), fabsf(__uint_as_float(ws[e] & 0xFFFF0000u)));
            }
          }
        }
      }
      float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) red[q4] = mx;
      mbar_arrive(cmax);
      ok = warp_wait(cmax, 0, abort);
      const float cm = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
      c2 = cm * cm;
    }
    // first pass: pair rows 0..63 against pair columns 0..127
    if (ok) ok = warp_wait(tfull0, 0, abort);
    if (ok) {
      tc_fence_after();
      const int pj = r >> 1;
      const bool writer = (r & 1) == 0;
      // chunks of columns left of this warp's 16 pair rows hold no entry the walk reads (j <= i)
#pragma unroll 1
      for (int cc = q4; cc < 8; ++cc) {
        float kk[32], vv[32];
        tmem_ld32(tmem + lane_base + cc * 32, kk);
        tmem_ld32(tmem + lane_base + 256 + cc * 32, vv);
        tmem_ld_wait();
        float dd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float k0 = exp2f(kk[2 * i] * a.scale_log2e) * (vv[2 * i] + c2);
          const float k1 = exp2f(kk[2 * i + 1] * a.scale_log2e) * (vv[2 * i + 1] + c2);
          dd[i] = k0 - k1;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) dd[i] -= __shfl_xor_sync(0xffffffffu, dd[i], 1);
        if (writer) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int pi = cc * 16 + i;
            D[pj * LD + pi] = (pj < m && pi < m) ? dd[i] : 0.f;
          }
        }
      }
      tc_fence_before();
    }
    mbar_arrive(tempty0);
    mbar_arrive(dhalf);
    // second pass: pair rows 64..127 against pair columns 64..127
    if (ok) ok = warp_wait(tfull1, 0, abort);
    if (ok) {
      tc_fence_after();
      const int pj = 64 + (r >> 1);
      const bool writer = (r & 1) == 0;
#pragma unroll 1
      for (int cc = q4; cc < 4; ++cc) {
        float kk[32], vv[32];
        tmem_ld32(tmem + lane_base + cc * 32, kk);
        tmem_ld32(tmem + lane_base + 256 + cc * 32, vv);
        tmem_ld_wait();
        float dd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float k0 = exp2f(kk[2 * i] * a.scale_log2e) * (vv[2 * i] + c2);
          const float k1 = exp2f(kk[2 * i + 1] * a.scale_log2e) * (vv[2 * i + 1] + c2);
          dd[i] = k0 - k1;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) dd[i] -= __shfl_xor_sync(0xffffffffu, dd[i], 1);
        if (writer) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int pi = 64 + cc * 16 + i;
            D[pj * LD + pi] = (pj < m && pi < m) ? dd[i] : 0.f;
          }
        }
      }
      tc_fence_before();
    }
    mbar_arrive(dfull);
  } else if (warp == 6) {
    // ------------------------------------------------------------------ sigma's recursion
    const float C = a.C, rC = 1.f / C;
    float sigma = 0.f;
    // the random numbers of all four blocks first, while Delta is still being formed
    float wls[4];
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      const int p = 32 * blk + lane;
      wls[blk] = p < m ? 1.f - 2.f * philox_uniform(a.seed, in.ctr_bh, in.round_id, in.pair0 + (uint32_t)p) : 0.f;
    }
#pragma unroll 1
    for (int blk = 0; blk < 4; ++blk) {
      if (!warp_wait(blk < 2 ? dhalf : dfull, 0, abort)) break;
      const int p = 32 * blk + lane;
      const float wl = blk == 0 ? wls[0] : blk == 1 ? wls[1] : blk == 2 ? wls[2] : wls[3];
      thr_s[p] = thresholds32(sigma, D[p * LD + p], wl, C, rC, lane);
      __syncwarp();
      mbar_arrive(thf + blk);
    }
  } else {
    // ------------------------------------------------------------------ the walk (warp 7)
    float my[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t kb[4] = {0u, 0u, 0u, 0u};
    bool ok = true;
#pragma unroll 1
    for (int blk = 0; blk < 4 && ok; ++blk) {
      ok = warp_wait(thf + blk, 0, abort);
      if (!ok) break;
      const int base = 32 * blk;
      float cur = blk == 0 ? my[0] : blk == 1 ? my[1] : blk == 2 ? my[2] : my[3];
      const uint32_t bb = walk_block32_th(cur, thr_s[base + lane], m - base, lane,
                                          [&](int q) { return D[(base + q) * LD + base + lane]; });
      kb[blk] = bb;
      if (lane == 0) bits_s[blk] = bb;
      __syncwarp();
      mbar_arrive(bitsb + blk);   // the gatherers of this block may start
      // this block's contribution to the alpha of every later pair, in pair order
#pragma unroll 1
      for (int b2 = blk + 1; b2 < 4; ++b2) {
        float acc = b2 == 1 ? my[1] : b2 == 2 ? my[2] : my[3];
#pragma unroll 8
        for (int q = 0; q < 32; ++q) acc = fmaf(((bb >> q) & 1u) ? 1.f : -1.f, D[(base + q) * LD + 32 * b2 + lane], acc);
        if (b2 == 1) my[1] = acc;
        else if (b2 == 2) my[2] = acc;
        else my[3] = acc;
      }
    }
  }
  // ------------------------------------------------------------------ gather
  // pair block t's kept rows from the stage as soon as its decisions are out: blocks 0..2 by warp
  // pairs (0,1), (2,3), (4,5) -- idle by then -- while the walk goes on, block 3 by all eight warps
  __syncwarp();
  {
    auto bit = [&](int i) { return ((bits_s[i >> 5] >> (i & 31)) & 1u) != 0; };
    const uint32_t tok_base = in.tok0 + 2u * in.pair0 * (uint32_t)ks;
    if (warp < 6 && warp_wait(bitsb + (warp >> 1), 0, abort)) {
      const int i0 = 32 * (warp >> 1) + 16 * (warp & 1);
      gather_from_stage(a, in.dst_row, in.src_row, tok_base, smem, 0, min(m, i0), min(m, i0 + 16), bit, lane, EC, NC, CB);
    }
  }
  if (warp_wait(bitsb + 3, 0, abort)) {
    const uint32_t b0 = bits_s[0], b1 = bits_s[1], b2 = bits_s[2], b3 = bits_s[3];
    auto bit = [b0, b1, b2, b3](int i) {
      const uint32_t w = i < 64 ? (i < 32 ? b0 : b1) : (i < 96 ? b2 : b3);
      return ((w >> (i & 31)) & 1u) != 0;
    };
    const uint32_t tok_base = in.tok0 + 2u * in.pair0 * (uint32_t)ks;
    gather_from_stage(a, in.dst_row, in.src_row, tok_base, smem, 0, min(m, 96 + 4 * warp), min(m, 100 + 4 * warp),
                      bit, lane, EC, NC, CB);
    if (a.trace && warp == 0 && lane < 4) {
      const int nb = a.m_pad >> 5;
      if (lane < nb) a.trace[a.trace_base + (size_t)inst * nb + lane] = lane == 0 ? b0 : lane == 1 ? b1 : lane == 2 ? b2 : b3;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (abort_s && threadIdx.x == 0 && a.status) {
    if (atomicCAS(a.status, 0, 5) == 0) a.status[1] = inst;
  }
  const bool ok = !abort_s;
  __syncthreads();
  if (threadIdx.x == 0 && ok) {   // after a time-out the CTA stops; nothing re-initialises them
    for (int i = 0; i < 17; ++i)
      if (i != 7) mbar_inval(bars + i);
  }
  return ok;
}

__global__ void __launch_bounds__(256, 1) halve256_kernel(const __grid_constant__ FusedMaps maps, const StepArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint32_t tmem_base_s;
  if (threadIdx.x >> 5 == 1) tmem_alloc(&tmem_base_s, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  halve256_body(maps, a, blockIdx.x, smem, tmem_base_s);
  if (threadIdx.x >> 5 == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base_s, 512);
  }
}

// ------------------------------------------------------------------------------------------------
// Instances of 257..512 points (the first step of a HALVE merge of four 128-point nodes): one CTA per
// instance.  The 256 x 256 pair differences are kept as the packed upper triangle (row j holds
// columns j..255, 131.6 KB) in shared memory (before the first Delta is written, that area holds the
// instance's V rows, loaded by TMA for c = max |v| in one pass for D <= 128, two for D <= 256); the
// 512 point rows do not fit beside it, so the Gram
// runs over the 10 upper-triangle pairs (bi <= bj) of 128-row blocks in row-block order, each a
// (128 x 128) kk and vv product streamed through a two-stage ring of 64-column chunks (A = rows of
// block bi, B = rows of block bj), accumulators double-buffered in TMEM.  The kept rows are gathered
// from global memory
// (still in L2: the ring read them moments before).  Warps: 0 TMA, 1 MMA (TMEM owner), 2-5 epilogue
// (warp w reads TMEM lanes 32 (w % 4)..), 6 sigma's recursion, 7 the walk; all eight gather.  The
// walk of pair block t starts once Delta rows 32t..32t+31 (row block t/2) are complete.  Every wait
// is bounded.
constexpr int kH512Pairs = 256;

// Blocks of 128 V rows staged per pass in the 131.6 KB Delta area: all four for D <= 128 (at most
// 8 chunks of 16 KB), two for D <= 256.
__host__ __device__ __forceinline__ int v_blocks_per_pass(int DCn) { return DCn <= 2 ? 4 : 2; }

__device__ __forceinline__ int tri_offset(int j) { return j * kH512Pairs - (j * (j - 1)) / 2; }

// Copy the kept point of pairs [i0, i1) of one instance from its source rows in global memory to
// destination rows dst_row + i, with its token index.  One warp; lane = one 16-byte unit of a row
// (K units first), ROWS rows in flight.  Token runs: point p is token tok0 + (2 pair0 + p) k of
// the (b,h) run (k = subsample stride, 1 without subsample).
template <int ROWS, typename Bit>
__device__ __forceinline__ void gather_global(const StepArgs& a, const HalveInst& in, int i0, int i1, Bit bit, int lane) {
  const bool tokens = a.src_kind == SRC_TOKENS;
  const int64_t k = a.sub_stride > 1 ? a.sub_stride : 1;
  const int h = (int)(in.bh % (uint32_t)a.H);
  const int kw = a.E / 8, vw = a.D / 8, units = kw + vw;
  const uint4* K = (const uint4*)a.srcK;
  const uint4* V = (const uint4*)a.srcV;
  uint4* dK = (uint4*)a.dstK;
  uint4* dV = (uint4*)a.dstV;
  for (int g = i0; g < i1; g += 32) {
    const int i = g + lane;
    int64_t row = 0;
    if (i < i1) {
      const int p = 2 * i + (bit(i) ? 0 : 1);
      if (tokens) {
        const int64_t t = (2 * (int64_t)in.pair0 + p) * k;
        row = (in.src_row + t) * a.H + h;
        a.dstIdx[in.dst_row + i] = (int32_t)(in.tok0 + t);
      } else {
        row = in.src_row + p;
        a.dstIdx[in.dst_row + i] = a.srcIdx[row];
      }
    }
    const int nrows = min(32, i1 - g);
    for (int w0 = 0; w0 < units; w0 += 32) {
      const int w = w0 + lane;
      const bool act = w < units, isk = w < kw;
      for (int j = 0; j < nrows; j += ROWS) {
        uint4 buf[ROWS];
#pragma unroll
        for (int jj = 0; jj < ROWS; ++jj) {
          const int64_t r = __shfl_sync(0xffffffffu, row, (j + jj) & 31);
          if (act && j + jj < nrows) buf[jj] = isk ? K[r * kw + w] : V[r * vw + (w - kw)];
        }
#pragma unroll
        for (int jj = 0; jj < ROWS; ++jj) {
          const int64_t d = in.dst_row + g + j + jj;
          if (act && j + jj < nrows) {
            if (isk) dK[d * kw + w] = buf[jj];
            else dV[d * vw + (w - kw)] = buf[jj];
          }
        }
      }
    }
  }
}

// One instance with the CTA's 256 threads, as halve256_body (barriers initialised here and
// invalidated before returning; false when a bounded wait gave up).
__device__ __forceinline__ bool halve512_body(const FusedMaps& maps, const StepArgs& a, const int inst, uint8_t* smem,
                                              const uint32_t tmem) {
  constexpr int NBP = 10;                       // block pairs (bi <= bj) of four 128-row blocks
  const int EC = a.E / 64, NC = (a.E + a.D) / 64;
  float* D = (float*)(smem + 4 * kChunk);       // packed upper triangle, row j at tri_offset(j)
  __shared__ __align__(8) uint64_t bars[24];
  uint64_t* full = bars;          // [2] ring stage landed
  uint64_t* empty = bars + 2;     // [2] ring stage read by its MMAs (commit)
  uint64_t* tfull = bars + 4;     // [2] accumulators ready (commit)
  uint64_t* tempty = bars + 6;    // [2] accumulators read (128)
  uint64_t* cmax = bars + 8;      // c exchanged among the epilogue threads (128)
  uint64_t* drow = bars + 9;      // [4] Delta rows of row block b complete (128)
  uint64_t* mdone = bars + 14;    // every MMA complete
  uint64_t* vfull = bars + 15;    // a pass of the instance's V rows landed in the Delta area
  uint64_t* vread = bars + 16;    // a pass of V rows read by every epilogue thread (128)
  __shared__ __align__(8) uint64_t thf[8];   // thresholds of pair block t published (32)
  __shared__ __align__(8) uint64_t bitsb[8]; // decisions of pair block t published (32; blocks in order)
  __shared__ float red[4];
  __shared__ float thr_s[kH512Pairs];
  __shared__ float alpha_s[kH512Pairs];
  __shared__ uint32_t bits_s[8];
  __shared__ volatile int abort_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = a.m, n = a.n;
  if (threadIdx.x == 0) {
    abort_s = 0;
    for (int b = 0; b < 2; ++b) {
      mbar_init(full + b, 1);
      mbar_init(empty + b, 1);
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, 128);
    }
    mbar_init(cmax, 128);
    for (int b = 0; b < 4; ++b) mbar_init(drow + b, 128);
    mbar_init(mdone, 1);
    mbar_init(vfull, 1);
    mbar_init(vread, 128);
    for (int t = 0; t < 8; ++t) {
      mbar_init(thf + t, 32);
      mbar_init(bitsb + t, 32);
    }
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  volatile int* abort = &abort_s;
  const HalveInst in = a.inst[inst];
  const bool tokens = a.src_kind == SRC_TOKENS;
  const int ks = a.sub_stride > 1 ? a.sub_stride : 1;
  // block pair q -> (bi, bj), row-block order: (0,0) (0,1) (0,2) (0,3) (1,1) (1,2) (1,3) (2,2) (2,3) (3,3)
  auto pair_of = [](int q, int& bi, int& bj) {
    bi = q < 4 ? 0 : q < 7 ? 1 : q < 9 ? 2 : 3;
    const int first = bi == 0 ? 0 : bi == 1 ? 4 : bi == 2 ? 7 : 9;
    bj = bi + (q - first);
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    const int row = (int)(tokens ? in.src_row / ks + 2 * (int64_t)in.pair0 : in.src_row);
    const int h = (int)(in.bh % (uint32_t)a.H);
    if (lane == 1) {
      // V rows into the Delta area for c, in passes of bpr blocks (DC chunks of 128 rows x 64
      // columns per block); a pass overwrites the area once every epilogue thread read the last
      const int DCn = NC - EC, bpr = v_blocks_per_pass(DCn);
      for (int r0 = 0; r0 < 4; r0 += bpr) {
        if (r0 > 0 && !mbar_wait(vread, (r0 / bpr - 1) & 1, abort)) break;
        mbar_expect_tx(vfull, (uint32_t)(bpr * DCn) * kChunk);
        for (int blk = r0; blk < r0 + bpr; ++blk)
          for (int c = 0; c < DCn; ++c) {
            uint8_t* dst = (uint8_t*)D + ((blk - r0) * DCn + c) * kChunk;
            if (!tokens) tma_load_2d(dst, &maps.v, vfull, c * 64, row + 128 * blk);
            else if (ks > 1) tma_load_4d(dst, &maps.v, vfull, c * 64, h, 0, row + 128 * blk);
            else tma_load_3d(dst, &maps.v, vfull, c * 64, h, row + 128 * blk);
          }
        // leave no copy in flight
        const long long t0 = clock64();
        while (!mbar_try_wait(vfull, (r0 / bpr) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int q = 0; q < NBP && ok; ++q) {
        int bi, bj;
        pair_of(q, bi, bj);
        for (int c = 0; c < NC; ++c, ++g) {
          const int s = g & 1;
          if (g >= 2 && !mbar_wait(empty + s, ((g >> 1) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          const bool isk = c < EC;
          const CUtensorMap* mp = isk ? &maps.k : &maps.v;
          const int x = (isk ? c : c - EC) * 64;
          mbar_expect_tx(full + s, (bi == bj ? 1u : 2u) * kChunk);
          for (int side = 0; side < (bi == bj ? 1 : 2); ++side) {
            uint8_t* dst = smem + s * 2 * kChunk + side * kChunk;
            const int r0 = row + 128 * (side ? bj : bi);
            if (!tokens) tma_load_2d(dst, mp, full + s, x, r0);
            else if (ks > 1) tma_load_4d(dst, mp, full + s, x, h, 0, r0);
            else tma_load_3d(dst, mp, full + s, x, h, r0);
          }
        }
      }
      // leave no copy in flight: the last fill of each stage has landed
      for (int gg = max(0, g - 2); gg < g; ++gg) {
        const long long t0 = clock64();
        while (!mbar_try_wait(full + (gg & 1), (gg >> 1) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t I128 = idesc_bf16(128, 128, false);
      const uint32_t base = smem_u32(smem);
      int g = 0;
      bool ok = true;
      for (int q = 0; q < NBP && ok; ++q) {
        int bi, bj;
        pair_of(q, bi, bj);
        const int tb = q & 1;
        if (q >= 2 && !mbar_wait(tempty + tb, ((q >> 1) & 1) ^ 1, abort)) break;
        for (int c = 0; c < NC; ++c, ++g) {
          const int s = g & 1;
          if (!mbar_wait(full + s, (g >> 1) & 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ra = base + s * 2 * kChunk;
          const uint32_t rb = bi == bj ? ra : ra + kChunk;
          const uint32_t dc = tmem + tb * 256u + (c < EC ? 0u : 128u);
          const bool first = c == 0 || c == EC;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(dc, sw128_desc(ra + kk * 32, 16, 1024), sw128_desc(rb + kk * 32, 16, 1024), I128,
                      (!first || kk > 0) ? 1u : 0u);
          umma_commit(empty + s);
        }
        if (ok) umma_commit(tfull + tb);
      }
      umma_commit(mdone);
      const long long t0 = clock64();
      while (!mbar_try_wait(mdone, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------------ epilogue
    const int q4 = warp & 3;                    // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;               // row within a 128-row block = TMEM lane
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    // c = max |v| over the instance's rows, from the V rows staged in the Delta area pass by
    // pass (row R of a block: 128 bytes per chunk, 16-byte units swizzled by R & 7)
    bool ok = true;
    float mx = 0.f;
    {
      const int DCn = NC - EC, bpr = v_blocks_per_pass(DCn);
      for (int r0 = 0; r0 < 4 && ok; r0 += bpr) {
        ok = warp_wait(vfull, (r0 / bpr) & 1, abort);
        if (!ok) break;
        for (int blk = r0; blk < r0 + bpr; ++blk) {
          if (128 * blk + r >= n) break;
          for (int c = 0; c < DCn; ++c) {
            const uint8_t* rowp = (const uint8_t*)D + ((blk - r0) * DCn + c) * kChunk + r * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint4 w = *(const uint4*)(rowp + ((q ^ (r & 7)) << 4));
              const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                mx = fmax3(mx, fabsf(__uint_as_float(ws[e] << 16)), fabsf(__uint_as_float(ws[e] & 0xFFFF0000u)));
            }
          }
        }
        mbar_arrive(vread);   // this thread's reads of the pass are done
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[q4] = mx;
    mbar_arrive(cmax);   // every epilogue thread has read its V rows: the area may take Delta now
    if (ok) ok = warp_wait(cmax, 0, abort);
    const float cm = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float c2 = cm * cm;
    for (int q = 0; q < NBP; ++q) {
      int bi, bj;
      pair_of(q, bi, bj);
      const int tb = q & 1;
      if (ok) ok = warp_wait(tfull + tb, (q >> 1) & 1, abort);
      if (ok) {
        tc_fence_after();
        const int pj = bi * 64 + (r >> 1);
        const bool writer = (r & 1) == 0;
        // on a diagonal block the chunks left of this warp's 16 pair rows hold no upper-triangle entry
#pragma unroll 1
        for (int cc = (bi == bj ? q4 : 0); cc < 4; ++cc) {
          float kk[32], vv[32];
          tmem_ld32(tmem + lane_base + tb * 256u + cc * 32, kk);
          tmem_ld32(tmem + lane_base + tb * 256u + 128 + cc * 32, vv);
          tmem_ld_wait();
          float dd[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float k0 = exp2f(kk[2 * i] * a.scale_log2e) * (vv[2 * i] + c2);
            const float k1 = exp2f(kk[2 * i + 1] * a.scale_log2e) * (vv[2 * i + 1] + c2);
            dd[i] = k0 - k1;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) dd[i] -= __shfl_xor_sync(0xffffffffu, dd[i], 1);
          if (writer) {
            float* Drow = D + tri_offset(pj) - pj;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int pi = bj * 64 + cc * 16 + i;
              if (pi >= pj) Drow[pi] = (pj < m && pi < m) ? dd[i] : 0.f;
            }
          }
        }
        tc_fence_before();
      }
      mbar_arrive(tempty + tb);
      if (bj == 3) mbar_arrive(drow + bi);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------------ sigma's recursion
    const float C = a.C, rC = 1.f / C;
    float sigma = 0.f;
#pragma unroll 1
    for (int t = 0; t < 8; ++t) {
      if (!warp_wait(drow + (t >> 1), 0, abort)) break;
      const int p = 32 * t + lane;
      const float wl = p < m ? 1.f - 2.f * philox_uniform(a.seed, in.ctr_bh, in.round_id, in.pair0 + (uint32_t)p) : 0.f;
      thr_s[p] = thresholds32(sigma, D[tri_offset(p)], wl, C, rC, lane);
      __syncwarp();
      mbar_arrive(thf + t);
    }
  } else {
    // ------------------------------------------------------------------ the walk (warp 7)
    // alpha of pair 32 t2 + lane lives in alpha_s (no register array indexed by block); each block's
    // terms are added to every later pair's alpha in row order, as the walk kernels do
    for (int i = lane; i < kH512Pairs; i += 32) alpha_s[i] = 0.f;
    __syncwarp();
    bool ok = true;
#pragma unroll 1
    for (int t = 0; t < 8; ++t) {
      uint32_t bb = 0u;
      if (ok) ok = warp_wait(thf + t, 0, abort);
      if (ok) {
        const int base = 32 * t;
        float my = alpha_s[base + lane];
        bb = walk_block32_th(my, thr_s[base + lane], m - base, lane,
                             [&](int q) { return D[tri_offset(base + q) - (base + q) + base + lane]; });
        // the later blocks' sums run side by side (seven independent chains, each in row order)
        float acc[7];
#pragma unroll
        for (int j = 0; j < 7; ++j) acc[j] = t + 1 + j < 8 ? alpha_s[32 * (t + 1 + j) + lane] : 0.f;
#pragma unroll 4
        for (int q = 0; q < 32; ++q) {
          const float* Dq = D + tri_offset(base + q) - (base + q) + lane;
          const float sg = ((bb >> q) & 1u) ? 1.f : -1.f;
#pragma unroll
          for (int j = 0; j < 7; ++j)
            if (t + 1 + j < 8) acc[j] = fmaf(sg, Dq[32 * (t + 1 + j)], acc[j]);
        }
#pragma unroll
        for (int j = 0; j < 7; ++j)
          if (t + 1 + j < 8) alpha_s[32 * (t + 1 + j) + lane] = acc[j];
      }
      if (lane == 0) bits_s[t] = bb;
      __syncwarp();
      mbar_arrive(bitsb + t);
    }
  }
  // ------------------------------------------------------------------ gather (all warps)
  __syncwarp();
  if (warp_wait(bitsb + 7, 0, abort)) {
    auto bit = [&](int i) { return ((bits_s[i >> 5] >> (i & 31)) & 1u) != 0; };
    const int per = (m + 7) / 8;
    gather_global<8>(a, in, min(m, warp * per), min(m, (warp + 1) * per), bit, lane);
    if (a.trace && warp == 0) {
      const int nb = a.m_pad >> 5;
      if (lane < nb) a.trace[a.trace_base + (size_t)inst * nb + lane] = bits_s[lane];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (abort_s && threadIdx.x == 0 && a.status) {
    if (atomicCAS(a.status, 0, 6) == 0) a.status[1] = inst;
  }
  const bool ok = !abort_s;
  __syncthreads();
  if (threadIdx.x == 0 && ok) {   // after a time-out the CTA stops; nothing re-initialises them
    for (int i = 0; i < 17; ++i)
      if (i != 13) mbar_inval(bars + i);
    for (int t = 0; t < 8; ++t) {
      mbar_inval(thf + t);
      mbar_inval(bitsb + t);
    }
  }
  return ok;
}

__global__ void __launch_bounds__(256, 1) halve512_kernel(const __grid_constant__ FusedMaps maps, const StepArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint32_t tmem_base_s;
  if (threadIdx.x >> 5 == 1) tmem_alloc(&tmem_base_s, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  halve512_body(maps, a, blockIdx.x, smem, tmem_base_s);
  if (threadIdx.x >> 5 == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base_s, 512);
  }
}

// TMA maps of a step's source rows (128-row boxes): tokens, every k-th token, or compact rows.
bool make_step_maps(const StepArgs& a, FusedMaps* maps) {
  if (a.src_kind == SRC_TOKENS && a.sub_stride > 1)
    return make_map_4d_strided(&maps->k, a.srcK, a.src_rows, a.H, a.E, a.sub_stride, 128) &&
           make_map_4d_strided(&maps->v, a.srcV, a.src_rows, a.H, a.D, a.sub_stride, 128);
  if (a.src_kind == SRC_TOKENS)
    return make_map_3d(&maps->k, a.srcK, a.src_rows, a.H, a.E, 128) && make_map_3d(&maps->v, a.srcV, a.src_rows, a.H, a.D, 128);
  return make_map_2d(&maps->k, a.srcK, a.src_rows, a.E, a.E, 128) && make_map_2d(&maps->v, a.srcV, a.src_rows, a.D, a.D, 128);
}

constexpr size_t kDelta512Bytes = (size_t)(kH512Pairs * (kH512Pairs + 1) / 2) * 4;
size_t smem_512() { return 1024 + 4 * (size_t)kChunk + kDelta512Bytes; }
size_t smem_256(const StepArgs& a) { return 1024 + (size_t)((a.E + a.D) / 64) * 2 * kChunk + (size_t)128 * 129 * 4; }

cudaError_t launch_512(const StepArgs& a, cudaStream_t st) {
  FusedMaps maps;
  if (!make_step_maps(a, &maps)) return cudaErrorInvalidValue;
  if ((size_t)v_blocks_per_pass(a.D / 64) * (a.D / 64) * kChunk > kDelta512Bytes) return cudaErrorInvalidValue;
  const size_t sm = smem_512();
  cudaError_t e = cudaFuncSetAttribute(halve512_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  halve512_kernel<<<a.n_inst, 256, sm, st>>>(maps, a);
  return cudaGetLastError();
}

cudaError_t launch_256(const StepArgs& a, cudaStream_t st) {
  FusedMaps maps;
  if (!make_step_maps(a, &maps)) return cudaErrorInvalidValue;
  const size_t sm = smem_256(a);
  cudaError_t e = cudaFuncSetAttribute(halve256_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  halve256_kernel<<<a.n_inst, 256, sm, st>>>(maps, a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------------
// Several steps of 129..512-point instances in one persistent launch (the last thinning level of the
// Express batches and both steps of every HALVE merge): one CTA per SM takes work items (step,
// instance) from a counter in the host-built queue order, waits until the items that write its
// source rows -- or read or write its destination rows -- have finished, runs the instance with the
// body of halve256_kernel or halve512_kernel, and publishes its completion.  A merge thus starts as
// soon as its four child coresets exist, and the SMs that one level leaves idle at its tail take the
// next level's ready instances.  The queue order is a topological order of those dependencies (the
// host simulates a list schedule of the items on the SMs), so an item only ever waits for items that
// CTAs already hold, and every wait is bounded: a wait that gives up (or any failure reported in the
// status word) stops every CTA at its next item.
constexpr int kSchedMaxSteps = 12;

struct SchedParams {
  FusedMaps maps[kSchedMaxSteps];
  StepArgs steps[kSchedMaxSteps];
  const int2* items;      // (step, instance) in queue order
  const int* pred_off;    // predecessors of item i: preds[pred_off[i] .. pred_off[i + 1])
  const int* preds;
  int n_items;
  int* done;              // per item: `epoch` once its outputs are written
  int epoch;
  int* sched;             // [0] next item, [1] CTAs that have left (the last one resets both)
  int* status;
  int inject_item;        // test hook: this item's wait never succeeds (-1: none)
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__global__ void __launch_bounds__(256, 1) halve_sched_kernel(const __grid_constant__ SchedParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint32_t tmem_base_s;
  __shared__ int item_s;
  if (threadIdx.x >> 5 == 1) tmem_alloc(&tmem_base_s, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  volatile int* status = P.status;
  for (;;) {
    if (threadIdx.x == 0) {
      int it = status[0] == 0 ? atomicAdd(P.sched, 1) : P.n_items;
      if (it >= P.n_items) it = -1;
      if (it >= 0) {
        bool ok = true;
        const long long t0 = clock64();
        for (int q = P.pred_off[it]; q < P.pred_off[it + 1] && ok; ++q) {
          const int* flag = P.done + P.preds[q];
          while (ld_acquire(flag) != P.epoch) {
            if (status[0] != 0 || clock64() - t0 > kWaitCycles) {
              ok = false;
              break;
            }
          }
        }
        if (ok && it == P.inject_item) {   // a flag that nothing sets: the wait runs out
          while (status[0] == 0 && clock64() - t0 <= kWaitCycles) {
          }
          ok = false;
        }
        if (!ok) {
          if (atomicCAS(P.status, 0, 7) == 0) P.status[1] = it;
          it = -1;
        }
      }
      item_s = it;
    }
    __syncthreads();
    const int it = item_s;
    if (it < 0) break;
    // the predecessors' outputs were written by other CTAs' ordinary stores: make them visible to
    // this CTA's tensor-memory-access loads
    asm volatile("fence.proxy.async.global;" ::: "memory");
    const int2 w = P.items[it];
    const bool ok = P.steps[w.x].n > 256 ? halve512_body(P.maps[w.x], P.steps[w.x], w.y, smem, tmem)
                                         : halve256_body(P.maps[w.x], P.steps[w.x], w.y, smem, tmem);
    __threadfence();
    __syncthreads();
    if (!ok) break;
    if (threadIdx.x == 0) st_release(P.done + it, P.epoch);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(P.sched + 1, 1) == (int)gridDim.x - 1) {
      atomicExch(P.sched, 0);
      atomicExch(P.sched + 1, 0);
    }
  }
  if (threadIdx.x >> 5 == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// The shapes the one-launch kernels take (independent of the driver and the environment).
bool halving_fused_shape_ok(const StepArgs& a) {
  if (a.E % 64 || a.D % 64 || (a.E + a.D) / 64 > kMaxChunks || a.n < 2 || a.n > 512 || a.n % 2) return false;
  if (a.src_rows <= 0) return false;
  // subsampled rows: an integer ratio is a strided view (runs on multiples of it); another ratio
  // needs the tokens spanned by an instance's n points, at most ceil((n-1) S / S') + 1, to fit the
  // box of NP rows of the persistent kernel
  if (a.src_kind == SRC_TOKENS && a.S_sub < a.S_full && a.sub_stride < 2) {
    if (a.n > 128) return false;
    const int NP = a.n <= 32 ? 32 : a.n <= 64 ? 64 : 128;
    const int64_t span = ((int64_t)(a.n - 1) * a.S_full + a.S_sub - 1) / a.S_sub + 1;
    if (span > NP) return false;
  }
  return true;
}

bool halving_fused_supported(const StepArgs& a) {
  return std::getenv("THIN_ATTN_UNFUSED_HALVING") == nullptr && halving_fused_shape_ok(a) && tensor_maps_available();
}

// Dynamic shared memory the scheduler can give an instance: 227 KB per CTA less the static arrays of
// both instance bodies (about 3.1 KB), with room to spare.
constexpr size_t kSchedDynSmemMax = 232448 - 4096;

bool halving_sched_shape_ok(const StepArgs& a) {
  if (!halving_fused_shape_ok(a) || a.n <= 128) return false;
  if (a.n <= 256) return smem_256(a) <= kSchedDynSmemMax;
  return smem_512() <= kSchedDynSmemMax && (size_t)v_blocks_per_pass(a.D / 64) * (a.D / 64) * kChunk <= kDelta512Bytes;
}

bool halving_sched_step_supported(const StepArgs& a) { return halving_fused_supported(a) && halving_sched_shape_ok(a); }

int halving_sched_max_steps() { return kSchedMaxSteps; }

cudaError_t launch_halving_sched(const StepArgs* steps, int n_steps, const SchedTables& t, cudaStream_t st) {
  if (n_steps < 1 || n_steps > kSchedMaxSteps || t.n_items == 0) return cudaErrorInvalidValue;
  SchedParams P{};
  size_t sm = 0;
  for (int i = 0; i < n_steps; ++i) {
    if (!halving_sched_step_supported(steps[i]) || !make_step_maps(steps[i], &P.maps[i])) return cudaErrorInvalidValue;
    P.steps[i] = steps[i];
    sm = std::max(sm, steps[i].n > 256 ? smem_512() : smem_256(steps[i]));
  }
  P.items = t.items;
  P.pred_off = t.pred_off;
  P.preds = t.preds;
  P.n_items = t.n_items;
  P.done = t.done;
  P.epoch = t.epoch;
  P.sched = t.sched;
  P.status = t.status;
  P.inject_item = t.inject_item;
  int dev = 0, sms = 0, optin = 0;
  cudaFuncAttributes fa{};
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, halve_sched_kernel);
  if (e != cudaSuccess) return e;
  if (sm + fa.sharedSizeBytes > (size_t)optin) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(halve_sched_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  halve_sched_kernel<<<std::min(t.n_items, sms), 256, sm, st>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_halving_fused(const StepArgs& a, cudaStream_t st) {
  if (a.n_inst == 0) return cudaSuccess;
  if (a.n <= 32) return launch_np<32>(a, st);
  if (a.n <= 64) return launch_np<64>(a, st);
  if (a.n <= 128) return launch_np<128>(a, st);
  if (a.n <= 256) return launch_256(a, st);
  return launch_512(a, st);
}

}  // namespace thin
