// Weighted softmax attention over key segments on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
//   o_t = sum_j w_j e^{s q_t.k_j} v_j / sum_j w_j e^{s q_t.k_j},  lse_t = ln sum_j w_j e^{s q_t.k_j}
// for a tile of up to 128 queries of one (b,h) against its key segments (exact prefix, Express
// nodes with weight 4^l b/c, the causal in-batch keys, or a Thinformer coreset with weight S/|C|),
// in key tiles of 128 rows.
//
// CTA = 6 warps:
//   warps 0-3  softmax: thread i owns query row i (TMEM lane i); reads S from TMEM, writes
//              P = exp2(z - m) as bf16 into shared memory (128-byte swizzled, K-major),
//              rescales O in TMEM when its running max grows by more than 2^8, epilogue
//   warp 4     TMA producer: Q once, then K and V tiles into a 2-stage ring
//   warp 5     MMA issuer (one thread): S = Q K^T into a double-buffered TMEM tile (cols 0/128),
//              O += P V into TMEM cols 256..256+D; also owns the TMEM allocation
// Every wait on an mbarrier is bounded; a CTA that gives up records the failure in the status
// word and leaves through the normal exit path (TMEM freed, its TMA copies landed).
#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "thin_attn.h"

namespace thin {

namespace {

using namespace tc;

constexpr int BM = 128;   // queries per tile
constexpr int BN = 128;   // keys per tile
constexpr int NSTAGE = 2;

template <int E, int D>
struct TcLayout {
  static constexpr int EC = E / 64, DC = D / 64;
  static constexpr uint32_t Q_BYTES = BM * E * 2;
  static constexpr uint32_t K_BYTES = BN * E * 2;
  static constexpr uint32_t V_BYTES = BN * D * 2;
  static constexpr uint32_t P_BYTES = BM * BN * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NSTAGE * K_BYTES;
  static constexpr uint32_t OFF_P = OFF_V + NSTAGE * V_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_P + P_BYTES;
  static constexpr uint32_t BYTES = OFF_BAR + 256 + 1024;   // barriers + alignment slack
};

struct TcMaps {
  CUtensorMap q, k, v, ck, cv;
};

// 128-key tiles of a query tile (counted by the host, so that a kernel learns an item's length from
// the tile record alone instead of walking its segments in global memory)
__device__ __forceinline__ int count_key_tiles(const AttnArgs&, const AttnTile& t) { return t.nkt; }

template <int E, int D>
__global__ void __launch_bounds__(192, 1) attn_tc_kernel(const __grid_constant__ TcMaps maps, const AttnArgs a,
                                                         int* status) {
  using Lay = TcLayout<E, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem + Lay::OFF_Q;
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  uint8_t* sP = smem + Lay::OFF_P;
  uint64_t* bars = (uint64_t*)(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;     // [NSTAGE]
  uint64_t* kv_empty = bars + 3;    // [NSTAGE]
  uint64_t* s_full = bars + 5;      // [2]
  uint64_t* s_free = bars + 7;      // [2]
  uint64_t* p_full = bars + 9;
  uint64_t* pv_done = bars + 10;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ volatile int where_s;   // first wait that gave up: code * 1000 + iteration

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile_id = a.tile0 + a.n_tiles - 1 - (int)blockIdx.x;   // heaviest (latest) query tiles first
  const AttnTile tile = a.tiles[tile_id];
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int n_kt = count_key_tiles(a, tile);

  if (threadIdx.x == 0) {
    abort_s = 0;
    where_s = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, 128);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(&tmem_base_s, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort = &abort_s;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_kt > 0) {
      mbar_expect_tx(q_full, Lay::Q_BYTES);
#pragma unroll
      for (int c = 0; c < Lay::EC; ++c) tma_load_3d(sQ + c * 16384, &maps.q, q_full, c * 64, h, b * a.T + tile.q0);
      int it = 0;
      int last_fill[NSTAGE] = {-1, -1};
      bool ok = true;
      for (int si = 0; si < tile.nseg && ok; ++si) {
        const AttnSeg sg = a.segs[tile.seg0 + si];
        for (int j0 = 0; j0 < sg.len && ok; j0 += BN, ++it) {
          const int st = it % NSTAGE;
          if (it >= NSTAGE && !mbar_wait(kv_empty + st, ((it / NSTAGE) - 1) & 1, abort)) {
            ok = false;
            atomicCAS((int*)&where_s, 0, 1000 + min(it, 999));
            break;
          }
          mbar_expect_tx(kv_full + st, Lay::K_BYTES + Lay::V_BYTES);
          uint8_t* dK = sK + st * Lay::K_BYTES;
          uint8_t* dV = sV + st * Lay::V_BYTES;
          if (sg.kind == SEG_TOKENS) {
            const int row = b * a.L + sg.first + j0;
#pragma unroll
            for (int c = 0; c < Lay::EC; ++c) tma_load_3d(dK + c * 16384, &maps.k, kv_full + st, c * 64, h, row);
#pragma unroll
            for (int c = 0; c < Lay::DC; ++c) tma_load_3d(dV + c * 16384, &maps.v, kv_full + st, c * 64, h, row);
          } else {
            const int row = (bh * a.n_slots + sg.first) * a.slot_rows + j0;
#pragma unroll
            for (int c = 0; c < Lay::EC; ++c) tma_load_2d(dK + c * 16384, &maps.ck, kv_full + st, c * 64, row);
#pragma unroll
            for (int c = 0; c < Lay::DC; ++c) tma_load_2d(dV + c * 16384, &maps.cv, kv_full + st, c * 64, row);
          }
          last_fill[st] = it;
        }
      }
      // never leave with a copy in flight into this CTA's shared memory
      for (int st = 0; st < NSTAGE; ++st)
        if (last_fill[st] >= 0) {
          const long long t0 = clock64();
          while (!mbar_try_wait(kv_full + st, (last_fill[st] / NSTAGE) & 1) && clock64() - t0 < kWaitCycles) {
          }
        }
      {
        const long long t0 = clock64();
        while (!mbar_try_wait(q_full, 0) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_kt > 0) {
      constexpr uint32_t IQK = idesc_bf16(BM, BN, false);
      constexpr uint32_t IPV = idesc_bf16(BM, D, true);
      const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK), va = smem_u32(sV), pa = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, abort);
      auto issue_s = [&](int it) -> bool {
        const int st = it % NSTAGE, sb = it & 1;
        if (!mbar_wait(kv_full + st, (it / NSTAGE) & 1, abort)) {
          atomicCAS((int*)&where_s, 0, 3000 + min(it, 999));
          return false;
        }
        if (it >= 2 && !mbar_wait(s_free + sb, ((it >> 1) - 1) & 1, abort)) {
          atomicCAS((int*)&where_s, 0, 4000 + min(it, 999));
          return false;
        }
        tc_fence_after();
        const uint32_t kb = ka + st * Lay::K_BYTES;
#pragma unroll
        for (int k = 0; k < E / 16; ++k) {
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
          umma_bf16(tmem + sb * BN, sw128_desc(qa + off, 16, 1024), sw128_desc(kb + off, 16, 1024), IQK, k > 0);
        }
        umma_commit(s_full + sb);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int it = 0; it < n_kt && ok; ++it) {
        if (it + 1 < n_kt && !issue_s(it + 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait(p_full, it & 1, abort)) {
          atomicCAS((int*)&where_s, 0, 5000 + min(it, 999));
          ok = false;
          break;
        }
        tc_fence_after();
        const int st = it % NSTAGE;
        const uint32_t vb = va + st * Lay::V_BYTES;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          const uint32_t aoff = (k >> 2) * 16384 + (k & 3) * 32;
          umma_bf16(tmem + 256, sw128_desc(pa + aoff, 16, 1024), sw128_desc(vb + k * 2048, 16384, 1024), IPV,
                    (it > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(kv_empty + st);
        umma_commit(pv_done);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroup
    const int row = warp * 32 + lane;
    const int tq = tile.q0 + row;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    int it = 0, where = 0;
    bool ok = true;
    for (int si = 0; si < tile.nseg && ok; ++si) {
      const AttnSeg sg = a.segs[tile.seg0 + si];
      const float lw2 = sg.logw * 1.4426950408889634f;
      for (int j0 = 0; j0 < sg.len; j0 += BN, ++it) {
        const int sb = it & 1;
        if (!warp_wait(s_full + sb, (it >> 1) & 1, abort)) {
          ok = false;
          where = 6;
          break;
        }
        tc_fence_after();
        float z[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32(tmem + lane_base + sb * BN + c * 32, z + c * 32);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(s_free + sb);
        // Masked keys -> -inf.  A tile every query of the CTA sees in full (the usual case) skips
        // the mask; otherwise key c is visible to this row iff c <= lim.
        const int nvalid = min(BN, sg.len - j0);
        const int kt0 = sg.first + j0;
        const bool causal = sg.kind == SEG_TOKENS && sg.causal;
        if (nvalid < BN || (causal && kt0 + BN - 1 > tile.q0)) {
          const int lim = min(nvalid - 1, causal ? tq - kt0 : BN - 1);
#pragma unroll
          for (int c = 0; c < BN; ++c) z[c] = c <= lim ? z[c] : -INFINITY;
        }
        // row max of the raw scores (scale > 0 keeps the order), 8 independent chains
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = z[i];
#pragma unroll
        for (int c = 8; c < BN; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], z[c]);
        const float smax = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                 fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float mx = smax == -INFINITY ? -INFINITY : fmaf(smax, a.scale_log2e, lw2);
        // P of the previous tile must be consumed (PV done) before P and O are touched
        if (it > 0 && !warp_wait(pv_done, (it - 1) & 1, abort)) {
          ok = false;
          where = 7;
          break;
        }
        tc_fence_after();
        // New running max: rescale the accumulated O and l, lazily (only when the max grows by
        // more than 2^8).  The TMEM round trip is warp-wide (.sync.aligned): a lane that needs
        // no rescale multiplies by 1.
        const bool grow = mx > m_used + 8.f;
        float corr = 1.f;
        if (grow) {
          corr = ex2_approx(m_used - mx);
          l *= corr;
          m_used = mx;
        }
        if (it > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(tmem + lane_base + 256 + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= corr;
            tmem_st32(tmem + lane_base + 256 + c * 32, o);
          }
          tmem_st_wait();
        }
        // p = 2^(s * scale * log2e + log2 w - m) in one FMA + EX2; a row that has seen no key yet
        // (m = -inf) has only -inf scores and gets p = 0.
        const float off = m_used == -INFINITY ? 0.f : lw2 - m_used;
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int g = 0; g < BN / 8; ++g) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = ex2_approx(fmaf(z[g * 8 + 2 * e], a.scale_log2e, off));
            const float p1 = ex2_approx(fmaf(z[g * 8 + 2 * e + 1], a.scale_log2e, off));
            ls[e] += p0 + p1;
            const __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
            pk[e] = *reinterpret_cast<const uint32_t*>(&pp);
          }
          // K-major 128B-swizzled layout: chunk g/8 (64 keys), 16-byte granule g%8 of row `row`
          const int chunk = g >> 3, gran = g & 7;
          uint8_t* dst = sP + chunk * 16384 + row * 128 + ((gran ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
      }
    }
    // epilogue: O / l to global, lse
    if (ok && n_kt > 0 && !warp_wait(pv_done, (n_kt - 1) & 1, abort)) where = 8;
    if (ok && n_kt > 0 && where == 0) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* out = (__nv_bfloat16*)a.out;
      const bool live = row < tile.qlen;
      __nv_bfloat16* orow = out + ((int64_t)(b * a.T + tq) * a.H + h) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_base + 256 + c * 32, o);
        tmem_ld_wait();
        if (live) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 u;
            __nv_bfloat162 t0 = __floats2bfloat162_rn(o[i] * inv, o[i + 1] * inv);
            __nv_bfloat162 t1 = __floats2bfloat162_rn(o[i + 2] * inv, o[i + 3] * inv);
            __nv_bfloat162 t2 = __floats2bfloat162_rn(o[i + 4] * inv, o[i + 5] * inv);
            __nv_bfloat162 t3 = __floats2bfloat162_rn(o[i + 6] * inv, o[i + 7] * inv);
            u.x = *reinterpret_cast<uint32_t*>(&t0);
            u.y = *reinterpret_cast<uint32_t*>(&t1);
            u.z = *reinterpret_cast<uint32_t*>(&t2);
            u.w = *reinterpret_cast<uint32_t*>(&t3);
            *reinterpret_cast<uint4*>(orow + c * 32 + i) = u;
          }
        }
      }
      if (live && a.lse) a.lse[(int64_t)bh * a.T + tq] = (m_used + log2f(l)) * 0.6931471805599453f;
    }
    if (where && lane == 0) atomicCAS((int*)&where_s, 0, where * 1000 + min(it, 999));
  }
  tc_fence_before();
  __syncthreads();
  if (abort_s && threadIdx.x == 0 && status) {
    if (atomicCAS(status, 0, 1) == 0) {
      status[1] = tile_id * 65536 + bh;
      status[2] = where_s;
    }
  }
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// Two CTAs per SM variant (D <= 128): 96 KB of shared memory and 256 TMEM columns per CTA, so
// one CTA's MMAs overlap the other's softmax.  S lives in TMEM columns 0..127; the softmax writes
// P (bf16, two per column) back into columns 0..63 and the PV MMA reads it from there as its A
// operand; O accumulates in columns 128..128+D.  K and V have one stage each with separate
// barriers: K(j+1) loads as soon as S(j) is done, V(j+1) as soon as PV(j) is done.  The MMA
// thread issues S(j+1) right after PV(j): the tensor-core pipeline runs one thread's MMAs in
// issue order, so PV(j) reads P(j) before S(j+1) overwrites it.
// The softmax reads S twice (max pass, then exponent pass) to stay within 170 registers.
template <int E, int D, bool FP8 = false>
struct Tc2Layout {
  // Q and K in 128-byte rows of chunks: 64 bf16 or 128 e4m3 elements each
  static constexpr int CW = FP8 ? 128 : 64;
  static constexpr int EC = E / CW, DC = D / 64;
  static constexpr uint32_t Q_BYTES = BM * E * (FP8 ? 1 : 2);
  static constexpr uint32_t K_BYTES = BN * E * (FP8 ? 1 : 2);
  static constexpr uint32_t V_BYTES = BN * D * 2;
  static constexpr uint32_t OFF_K = Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + K_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + V_BYTES;
  static constexpr uint32_t BYTES = OFF_BAR + 128 + 1024;
};


// Softmax of one key tile for the thread's row (TMEM address ts of its 128 S columns, to of its O
// columns): reads S twice -- row max, then P = 2^(s scale log2e + log2 w - m) as bf16 written over
// the S columns already read (16 columns per 32 read) -- and rescales O lazily (warp-wide TMEM
// round trip when some row's max grew by more than 2^8).  MASKED: keys c > lim are invisible.
template <bool MASKED, int D>
__device__ __forceinline__ void softmax_tile(uint32_t ts, uint32_t to, int lim, float sl2e, float lw2, int it,
                                             float& m_used, float& l, uint64_t* p_half) {
  float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  // row max: two 32-column loads in flight per wait
#pragma unroll
  for (int c2 = 0; c2 < BN / 64; ++c2) {
    float z[2][32];
    tmem_ld32(ts + c2 * 64, z[0]);
    tmem_ld32(ts + c2 * 64 + 32, z[1]);
    tmem_ld_wait();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = 2 * c2 + h;
      if (MASKED) {
#pragma unroll
        for (int i = 0; i < 32; ++i) z[h][i] = c * 32 + i <= lim ? z[h][i] : -INFINITY;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        mx4[0] = fmax3(mx4[0], z[h][i], z[h][i + 1]);
        mx4[1] = fmax3(mx4[1], z[h][i + 2], z[h][i + 3]);
        mx4[2] = fmax3(mx4[2], z[h][i + 4], z[h][i + 5]);
        mx4[3] = fmax3(mx4[3], z[h][i + 6], z[h][i + 7]);
      }
    }
  }
  const float smax = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
  const float mx = smax == -INFINITY ? -INFINITY : fmaf(smax, sl2e, lw2);
  const bool grow = mx > m_used + 8.f;
  float corr = 1.f;
  if (grow) {
    corr = ex2_approx(m_used - mx);
    l *= corr;
    m_used = mx;
  }
  if (it > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      tmem_ld32(to + c * 32, o);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] *= corr;
      tmem_st32(to + c * 32, o);
    }
  }
  const float off = m_used == -INFINITY ? 0.f : lw2 - m_used;
  // two scores per instruction: the scale-and-offset FMA and the row-sum add run on packed fp32
  // pairs (sm_100 FFMA2 / FADD2), which leaves one EX2 per score and one bf16x2 pack per pair
  const float2 sl2e2 = make_float2(sl2e, sl2e), off2 = make_float2(off, off);
  float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  // 32 columns at a time, the next 32 loading while these are exponentiated
  float zb[2][32];
  tmem_ld32(ts, zb[0]);
  tmem_ld_wait();
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    if (c + 1 < BN / 32) tmem_ld32(ts + (c + 1) * 32, zb[(c + 1) & 1]);
    const float* z = zb[c & 1];
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float z0 = z[2 * e], z1 = z[2 * e + 1];
      if (MASKED) {
        z0 = c * 32 + 2 * e <= lim ? z0 : -INFINITY;
        z1 = c * 32 + 2 * e + 1 <= lim ? z1 : -INFINITY;
      }
      const float2 t = __ffma2_rn(make_float2(z0, z1), sl2e2, off2);
      const float p0 = ex2_approx(t.x);
      const float p1 = ex2_approx(t.y);
      ls2[e & 1] = __fadd2_rn(ls2[e & 1], make_float2(p0, p1));
      const __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
      pk[e] = *reinterpret_cast<const uint32_t*>(&pp);
    }
    tmem_st16(ts + c * 16, pk);
    if (c == BN / 64 - 1) {
      // P of the first half of the keys is in place: the MMA warp starts its half of PV
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_half);
    }
    if (c + 1 < BN / 32) tmem_ld_wait();
  }
  l += (ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y);
}

template <int E, int D>
__global__ void __launch_bounds__(192, 2) attn_tc2_kernel(const __grid_constant__ TcMaps maps, const AttnArgs a,
                                                          int* status) {
  using Lay = Tc2Layout<E, D>;
  constexpr uint32_t O_COL = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  uint64_t* bars = (uint64_t*)(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 2;
  uint64_t* v_full = bars + 3;
  uint64_t* v_empty = bars + 4;
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;      // P of all keys of the tile written (128 threads)
  uint64_t* pv_done = bars + 7;
  uint64_t* p_half = bars + 8;      // P of keys 0..BN/2-1 written (128 threads)
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ volatile int where_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile_id = a.tile0 + a.n_tiles - 1 - (int)blockIdx.x;
  const AttnTile tile = a.tiles[tile_id];
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int n_kt = count_key_tiles(a, tile);

  if (threadIdx.x == 0) {
    abort_s = 0;
    where_s = 0;
    mbar_init(q_full, 1);
    mbar_init(k_full, 1);
    mbar_init(k_empty, 1);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(p_half, 128);
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(&tmem_base_s, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort = &abort_s;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_kt > 0) {
      mbar_expect_tx(q_full, Lay::Q_BYTES);
#pragma unroll
      for (int c = 0; c < Lay::EC; ++c) tma_load_3d(sQ + c * 16384, &maps.q, q_full, c * 64, h, b * a.T + tile.q0);
      int it = 0;
      bool ok = true;
      for (int si = 0; si < tile.nseg && ok; ++si) {
        const AttnSeg sg = a.segs[tile.seg0 + si];
        const bool tok = sg.kind == SEG_TOKENS;
        for (int j0 = 0; j0 < sg.len; j0 += BN, ++it) {
          const int row = tok ? b * a.L + sg.first + j0 : (bh * a.n_slots + sg.first) * a.slot_rows + j0;
          if (it > 0 && !mbar_wait(k_empty, (it - 1) & 1, abort)) {
            ok = false;
            atomicCAS((int*)&where_s, 0, 1000 + min(it, 999));
            break;
          }
          const bool withhold = a.inject_timeout && a.tile0 == 0 && it == 0 && blockIdx.x == 0 && blockIdx.y == 0;
          if (!withhold) {
            mbar_expect_tx(k_full, Lay::K_BYTES);
#pragma unroll
            for (int c = 0; c < Lay::EC; ++c) {
              if (tok) tma_load_3d(sK + c * 16384, &maps.k, k_full, c * 64, h, row);
              else tma_load_2d(sK + c * 16384, &maps.ck, k_full, c * 64, row);
            }
          }
          if (it > 0 && !mbar_wait(v_empty, (it - 1) & 1, abort)) {
            ok = false;
            atomicCAS((int*)&where_s, 0, 2000 + min(it, 999));
            break;
          }
          mbar_expect_tx(v_full, Lay::V_BYTES);
#pragma unroll
          for (int c = 0; c < Lay::DC; ++c) {
            if (tok) tma_load_3d(sV + c * 16384, &maps.v, v_full, c * 64, h, row);
            else tma_load_2d(sV + c * 16384, &maps.cv, v_full, c * 64, row);
          }
        }
      }
      // never leave with a copy in flight into this CTA's shared memory
      if (it > 0) {
        long long t0 = clock64();
        while (!mbar_try_wait(k_full, (it - 1) & 1) && clock64() - t0 < kWaitCycles) {
        }
        t0 = clock64();
        while (!mbar_try_wait(v_full, (it - 1) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
      const long long t0 = clock64();
      while (!mbar_try_wait(q_full, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_kt > 0) {
      constexpr uint32_t IQK = idesc_bf16(BM, BN, false);
      constexpr uint32_t IPV = idesc_bf16(BM, D, true);
      const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK), va = smem_u32(sV);
      bool ok = mbar_wait(q_full, 0, abort);
      for (int it = 0; it < n_kt && ok; ++it) {
        // No wait for PV(it-1) before S(it) overwrites the P columns it reads: tcgen05.mma ops
        // issued by one thread execute in issue order, and the commit after S(it) tracks PV(it-1)
        // too, so s_full(it) also tells the softmax that O is complete up to tile it-1.
        if (!mbar_wait(k_full, it & 1, abort)) {
          atomicCAS((int*)&where_s, 0, 3000 + min(it, 999));
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < E / 16; ++k) {
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
          umma_bf16(tmem, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), IQK, k > 0);
        }
        umma_commit(s_full);
        umma_commit(k_empty);
        // PV in two halves over the keys: the first as soon as P of keys 0..BN/2-1 is written
        if (!mbar_wait(p_half, it & 1, abort) || !mbar_wait(v_full, it & 1, abort)) {
          atomicCAS((int*)&where_s, 0, 5000 + min(it, 999));
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < BN / 32; ++k)
          umma_bf16_tmem_a(tmem + O_COL, tmem + k * 8, sw128_desc(va + k * 2048, 16384, 1024), IPV,
                           (it > 0 || k > 0) ? 1u : 0u);
        if (!mbar_wait(p_full, it & 1, abort)) {
          atomicCAS((int*)&where_s, 0, 7000 + min(it, 999));
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = BN / 32; k < BN / 16; ++k)
          umma_bf16_tmem_a(tmem + O_COL, tmem + k * 8, sw128_desc(va + k * 2048, 16384, 1024), IPV, 1u);
        umma_commit(pv_done);
        umma_commit(v_empty);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroup
    const int row = warp * 32 + lane;
    const int tq = tile.q0 + row;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    int it = 0, where = 0;
    bool ok = true;
    for (int si = 0; si < tile.nseg && ok; ++si) {
      const AttnSeg sg = a.segs[tile.seg0 + si];
      const float lw2 = sg.logw * 1.4426950408889634f;
      for (int j0 = 0; j0 < sg.len; j0 += BN, ++it) {
        if (!warp_wait(s_full, it & 1, abort)) {
          ok = false;
          where = 6;
          break;
        }
        tc_fence_after();
        const int nvalid = min(BN, sg.len - j0);
        const int kt0 = sg.first + j0;
        const bool causal = sg.kind == SEG_TOKENS && sg.causal;
        const bool masked = nvalid < BN || (causal && kt0 + BN - 1 > tile.q0);
        const int lim = min(nvalid - 1, causal ? tq - kt0 : BN - 1);
        if (masked) softmax_tile<true, D>(tmem + lane_base, tmem + lane_base + 128, lim, a.scale_log2e, lw2, it, m_used, l, p_half);
        else softmax_tile<false, D>(tmem + lane_base, tmem + lane_base + 128, lim, a.scale_log2e, lw2, it, m_used, l, p_half);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
      }
    }
    if (ok && n_kt > 0 && !warp_wait(pv_done, (n_kt - 1) & 1, abort)) where = 8;
    if (ok && n_kt > 0 && where == 0) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* out = (__nv_bfloat16*)a.out;
      const bool live = row < tile.qlen;
      __nv_bfloat16* orow = out + ((int64_t)(b * a.T + tq) * a.H + h) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_base + O_COL + c * 32, o);
        tmem_ld_wait();
        if (live) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 u;
            __nv_bfloat162 t0 = __floats2bfloat162_rn(o[i] * inv, o[i + 1] * inv);
            __nv_bfloat162 t1 = __floats2bfloat162_rn(o[i + 2] * inv, o[i + 3] * inv);
            __nv_bfloat162 t2 = __floats2bfloat162_rn(o[i + 4] * inv, o[i + 5] * inv);
            __nv_bfloat162 t3 = __floats2bfloat162_rn(o[i + 6] * inv, o[i + 7] * inv);
            u.x = *reinterpret_cast<uint32_t*>(&t0);
            u.y = *reinterpret_cast<uint32_t*>(&t1);
            u.z = *reinterpret_cast<uint32_t*>(&t2);
            u.w = *reinterpret_cast<uint32_t*>(&t3);
            *reinterpret_cast<uint4*>(orow + c * 32 + i) = u;
          }
        }
      }
      if (live && a.lse) a.lse[(int64_t)bh * a.T + tq] = (m_used + log2f(l)) * 0.6931471805599453f;
    }
    if (where && lane == 0) atomicCAS((int*)&where_s, 0, where * 1000 + min(it, 999));
  }
  tc_fence_before();
  __syncthreads();
  if (abort_s && threadIdx.x == 0 && status) {
    if (atomicCAS(status, 0, 1) == 0) {
      status[1] = tile_id * 65536 + bh;
      status[2] = where_s;
    }
  }
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}


// Persistent form of attn_tc2_kernel: two CTAs per SM, each looping over work items (query tile,
// (b,h)).  Items are handed out dynamically in the order the per-tile grid runs -- (b,h) by
// (b,h), the last (heaviest) tiles first: item j = tile n_tiles-1 - j % n_tiles of (b,h)
// j / n_tiles -- so the CTAs running at one time read the keys of one or two heads (they stay in
// L2) and the load balances like the hardware's own block scheduling.  The producer takes the next
// item from a counter in global memory (sched[0]) and passes it to the MMA and softmax roles
// through a two-slot ring in shared memory; the last CTA to leave resets the counter (sched[1]
// counts the CTAs that left).  Per item the roles run the same key-tile pipeline as attn_tc2_kernel; what persistence
// adds is the overlap between items: the producer loads the next item's Q as soon as the last S
// MMA of the current item has read Q (q_empty), and the next item's first S MMA runs while the
// softmax warps write the current item's O (the first PV of an item waits for that: o_empty).
// Barrier parities follow a key-tile count and an item count that run across items.
template <int E, int D, bool FP8 = false>
__global__ void __launch_bounds__(192, 2) attn_tc2p_kernel(const __grid_constant__ TcMaps maps, const AttnArgs a,
                                                           int* status) {
  using Lay = Tc2Layout<E, D, FP8>;
  constexpr uint32_t O_COL = 128;
  // S/P and O: 256 TMEM columns for D <= 128 (two CTAs per SM), 512 for D = 256 (one CTA per SM)
  constexpr uint32_t TCOLS = D <= 128 ? 256 : 512;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  uint64_t* bars = (uint64_t*)(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 2;
  uint64_t* v_full = bars + 3;
  uint64_t* v_empty = bars + 4;
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;      // P of all keys of the tile written (128 threads)
  uint64_t* pv_done = bars + 7;
  uint64_t* p_half = bars + 8;      // P of keys 0..BN/2-1 written (128 threads)
  uint64_t* q_empty = bars + 9;     // the item's last S MMA has read Q (commit)
  uint64_t* o_empty = bars + 10;    // the item's O has been read out of TMEM (128 threads)
  uint64_t* item_full = bars + 11;  // [2] next item index published (producer)
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ volatile int where_s;
  __shared__ int item_s;
  __shared__ int item_ring[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.n_tiles * a.B * a.H;
  int* sched = status + 4;

  if (threadIdx.x == 0) {
    abort_s = 0;
    where_s = 0;
    item_s = -1;
    mbar_init(q_full, 1);
    mbar_init(k_full, 1);
    mbar_init(k_empty, 1);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(p_half, 128);
    mbar_init(q_empty, 1);
    mbar_init(o_empty, 128);
    mbar_init(item_full, 1);
    mbar_init(item_full + 1, 1);
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(&tmem_base_s, TCOLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort = &abort_s;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int git = 0, r = 0;
      bool ok = true;
      for (;; ++r) {
        // the ring slot of item r was last read at the start of item r-2, before q_empty(r-1)
        if (r > 0 && !mbar_wait(q_empty, (r - 1) & 1, abort)) {
          atomicCAS((int*)&where_s, 0, 9000 + min(r, 999));
          ok = false;
        }
        const int j = ok ? atomicAdd(sched, 1) : n_items;
        item_ring[r & 1] = j < n_items ? j : -1;
        mbar_arrive(item_full + (r & 1));
        if (j >= n_items) break;
        const AttnTile tile = a.tiles[a.tile0 + a.n_tiles - 1 - j % a.n_tiles];
        const int bh = j / a.n_tiles, b = bh / a.H, h = bh % a.H;
        mbar_expect_tx(q_full, Lay::Q_BYTES);
#pragma unroll
        for (int c = 0; c < Lay::EC; ++c) tma_load_3d(sQ + c * 16384, &maps.q, q_full, c * Lay::CW, h, b * a.T + tile.q0);
        for (int si = 0; si < tile.nseg && ok; ++si) {
          const AttnSeg sg = a.segs[tile.seg0 + si];
          const bool tok = sg.kind == SEG_TOKENS;
          for (int j0 = 0; j0 < sg.len; j0 += BN, ++git) {
            const int row = tok ? b * a.L + sg.first + j0 : (bh * a.n_slots + sg.first) * a.slot_rows + j0;
            if (git > 0 && !mbar_wait(k_empty, (git - 1) & 1, abort)) {
              ok = false;
              atomicCAS((int*)&where_s, 0, 1000 + min(git, 999));
              break;
            }
            const bool withhold = a.inject_timeout && a.tile0 == 0 && git == 0 && blockIdx.x == 0;
            if (!withhold) {
              mbar_expect_tx(k_full, Lay::K_BYTES);
#pragma unroll
              for (int c = 0; c < Lay::EC; ++c) {
                if (tok) tma_load_3d(sK + c * 16384, &maps.k, k_full, c * Lay::CW, h, row);
                else tma_load_2d(sK + c * 16384, &maps.ck, k_full, c * Lay::CW, row);
              }
            }
            if (git > 0 && !mbar_wait(v_empty, (git - 1) & 1, abort)) {
              ok = false;
              atomicCAS((int*)&where_s, 0, 2000 + min(git, 999));
              break;
            }
            mbar_expect_tx(v_full, Lay::V_BYTES);
#pragma unroll
            for (int c = 0; c < Lay::DC; ++c) {
              if (tok) tma_load_3d(sV + c * 16384, &maps.v, v_full, c * 64, h, row);
              else tma_load_2d(sV + c * 16384, &maps.cv, v_full, c * 64, row);
            }
          }
        }
        if (!ok) break;   // abort is set: every other role's next wait returns at once
      }
      // never leave with a copy in flight into this CTA's shared memory
      if (git > 0) {
        long long t0 = clock64();
        while (!mbar_try_wait(k_full, (git - 1) & 1) && clock64() - t0 < kWaitCycles) {
        }
        t0 = clock64();
        while (!mbar_try_wait(v_full, (git - 1) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
      if (r > 0) {
        const long long t0 = clock64();
        while (!mbar_try_wait(q_full, (r - 1) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IQK = FP8 ? idesc_e4m3(BM, BN) : idesc_bf16(BM, BN, false);
      constexpr uint32_t IPV = idesc_bf16(BM, D, true);
      const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK), va = smem_u32(sV);
      int git = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        if (!mbar_wait(item_full + (r & 1), (r >> 1) & 1, abort)) break;
        const int j = item_ring[r & 1];
        if (j < 0) break;
        const AttnTile tile = a.tiles[a.tile0 + a.n_tiles - 1 - j % a.n_tiles];
        const int n_kt = count_key_tiles(a, tile);
        if (!mbar_wait(q_full, r & 1, abort)) {
          atomicCAS((int*)&where_s, 0, 4000 + min(r, 999));
          break;
        }
        for (int it = 0; it < n_kt; ++it, ++git) {
          // S(it) may overwrite the P columns PV(it-1) reads: tcgen05.mma ops issued by one thread
          // execute in issue order, and the commit after S(it) tracks PV(it-1) too
          if (!mbar_wait(k_full, git & 1, abort)) {
            ok = false;
            atomicCAS((int*)&where_s, 0, 3000 + min(git, 999));
            break;
          }
          tc_fence_after();
#pragma unroll
          // 32 bytes of K per instruction: 16 bf16 or 32 e4m3 elements
          for (int k = 0; k < E / (FP8 ? 32 : 16); ++k) {
            const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
            if (FP8) umma_e4m3(tmem, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), IQK, k > 0);
            else umma_bf16(tmem, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), IQK, k > 0);
          }
          umma_commit(s_full);
          umma_commit(k_empty);
          if (it == n_kt - 1) umma_commit(q_empty);
          if (!mbar_wait(p_half, git & 1, abort) || !mbar_wait(v_full, git & 1, abort) ||
              (it == 0 && r > 0 && !mbar_wait(o_empty, (r - 1) & 1, abort))) {
            ok = false;
            atomicCAS((int*)&where_s, 0, 5000 + min(git, 999));
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < BN / 32; ++k)
            umma_bf16_tmem_a(tmem + O_COL, tmem + k * 8, sw128_desc(va + k * 2048, 16384, 1024), IPV,
                             (it > 0 || k > 0) ? 1u : 0u);
          if (!mbar_wait(p_full, git & 1, abort)) {
            ok = false;
            atomicCAS((int*)&where_s, 0, 7000 + min(git, 999));
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = BN / 32; k < BN / 16; ++k)
            umma_bf16_tmem_a(tmem + O_COL, tmem + k * 8, sw128_desc(va + k * 2048, 16384, 1024), IPV, 1u);
          umma_commit(pv_done);
          umma_commit(v_empty);
        }
        if (n_kt == 0) umma_commit(q_empty);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroup
    const int row = warp * 32 + lane;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    int git = 0, where = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      if (!warp_wait(item_full + (r & 1), (r >> 1) & 1, abort)) {
        where = 10;
        break;
      }
      const int j = item_ring[r & 1];
      if (j < 0) break;
      const int tile_id = a.tile0 + a.n_tiles - 1 - j % a.n_tiles;
      const AttnTile tile = a.tiles[tile_id];
      const int bh = j / a.n_tiles, b = bh / a.H, h = bh % a.H;
      if (tile.nkt == 0) {
        mbar_arrive(o_empty);
        continue;
      }
      // the tile's segment records into L1: the loads at the segment boundaries below then hit there
      if (lane == 0) prefetch_l1(a.segs + tile.seg0, tile.nseg * (int)sizeof(AttnSeg));
      if (threadIdx.x == 0) item_s = tile_id * 65536 + bh;
      const int tq = tile.q0 + row;
      // e4m3 scores are q k^T times scale_q scale_k: the (b,h) factor that undoes it joins s log2 e
      const float sl2e = FP8 ? a.scale_log2e * a.qk_inv[bh] : a.scale_log2e;
      float m_used = -INFINITY, l = 0.f;
      int it = 0;
      for (int si = 0; si < tile.nseg && ok; ++si) {
        const AttnSeg sg = a.segs[tile.seg0 + si];
        const float lw2 = sg.logw * 1.4426950408889634f;
        for (int j0 = 0; j0 < sg.len; j0 += BN, ++it, ++git) {
          if (!warp_wait(s_full, git & 1, abort)) {
            ok = false;
            where = 6;
            break;
          }
          tc_fence_after();
          const int nvalid = min(BN, sg.len - j0);
          const int kt0 = sg.first + j0;
          const bool causal = sg.kind == SEG_TOKENS && sg.causal;
          const bool masked = nvalid < BN || (causal && kt0 + BN - 1 > tile.q0);
          const int lim = min(nvalid - 1, causal ? tq - kt0 : BN - 1);
          if (masked) softmax_tile<true, D>(tmem + lane_base, tmem + lane_base + 128, lim, sl2e, lw2, it, m_used, l, p_half);
          else softmax_tile<false, D>(tmem + lane_base, tmem + lane_base + 128, lim, sl2e, lw2, it, m_used, l, p_half);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(p_full);
        }
      }
      if (!ok) break;
      if (!warp_wait(pv_done, (git - 1) & 1, abort)) {
        where = 8;
        break;
      }
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* out = (__nv_bfloat16*)a.out;
      const bool live = row < tile.qlen;
      __nv_bfloat16* orow = out + ((int64_t)(b * a.T + tq) * a.H + h) * D;
      if constexpr (D <= 128) {
        // the row of O, normalised and packed to bf16 pairs in registers (64 columns per TMEM wait),
        // then O is released to the next item's first PV before the stores go out
        uint32_t pk[D / 2];
#pragma unroll
        for (int c2 = 0; c2 < D / 64; ++c2) {
          float o[2][32];
          tmem_ld32(tmem + lane_base + O_COL + c2 * 64, o[0]);
          tmem_ld32(tmem + lane_base + O_COL + c2 * 64 + 32, o[1]);
          tmem_ld_wait();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const __nv_bfloat162 t = __floats2bfloat162_rn(o[hh][i] * inv, o[hh][i + 1] * inv);
              pk[(c2 * 64 + hh * 32 + i) / 2] = *reinterpret_cast<const uint32_t*>(&t);
            }
        }
        tc_fence_before();
        mbar_arrive(o_empty);
        if (live) {
#pragma unroll
          for (int i = 0; i < D / 8; ++i)
            *reinterpret_cast<uint4*>(orow + 8 * i) = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      } else {
        // D = 256: a packed row would not fit in registers; every 64 columns go out as they are
        // packed, and O is released after the last of them
#pragma unroll 1
        for (int c2 = 0; c2 < D / 64; ++c2) {
          float o[2][32];
          tmem_ld32(tmem + lane_base + O_COL + c2 * 64, o[0]);
          tmem_ld32(tmem + lane_base + O_COL + c2 * 64 + 32, o[1]);
          tmem_ld_wait();
          uint32_t pk[32];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const __nv_bfloat162 t = __floats2bfloat162_rn(o[hh][i] * inv, o[hh][i + 1] * inv);
              pk[(hh * 32 + i) / 2] = *reinterpret_cast<const uint32_t*>(&t);
            }
          if (live) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *reinterpret_cast<uint4*>(orow + c2 * 64 + 8 * i) =
                  make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
        tc_fence_before();
        mbar_arrive(o_empty);
      }
      if (live && a.lse) a.lse[(int64_t)bh * a.T + tq] = (m_used + log2f(l)) * 0.6931471805599453f;
    }
    if (where && lane == 0) atomicCAS((int*)&where_s, 0, where * 1000 + min(git, 999));
  }
  tc_fence_before();
  __syncthreads();
  if (abort_s && threadIdx.x == 0) {
    if (atomicCAS(status, 0, 1) == 0) {
      status[1] = item_s;
      status[2] = where_s;
    }
  }
  if (threadIdx.x == 0) {
    // every CTA has taken its last item before it counts itself out: the last one resets
    __threadfence();
    if (atomicAdd(sched + 1, 1) == (int)gridDim.x - 1) {
      atomicExch(sched, 0);
      atomicExch(sched + 1, 0);
    }
  }
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TCOLS);
  }
}

// ---------------------------------------------------------------------------------------------
// Ping-pong form (E, D <= 128): one persistent CTA per SM runs two query tiles of one (b,h) at a
// time, tile A and tile B, against a single stream of K/V tiles.  The host pairs tiles whose key
// lists nest: A's key tiles are the first n_A key tiles of B's (two neighbouring tiles of one
// Express batch, the exact phase, or any two tiles of a Thinformer head), so every K/V tile is
// loaded once for both; the K and V rings fill the shared memory beside the Q buffers.
//   TMEM (512 columns): S_A / P_A 0..127, S_B / P_B 128..255, O_A 256..383, O_B 384..511.
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B (thread = query row = TMEM lane)
//   warp 8     TMA producer: work items (published one item ahead), K per key tile into the K ring
//   warp 10    TMA producer: V per key tile into the V ring
//   warp 11    TMA producer: Q_A and Q_B of every item into a ring of NQ Q buffers (item r takes
//              fills 2r and 2r + 1), each refilled once the last S MMA reading it has completed, so
//              that the next item's Q_A loads while the current item's B tile still runs
// After set-up the softmax warpgroups take 192 registers per thread and warps 8-11 keep 120, so a
// softmax thread holds its row of S and reads it from TMEM once per key tile.
//   warp 9     MMA issuer: per key tile j, PV_A(j), S_A(j+1), PV_B(j), S_B(j+1) -- while one
//              softmax warpgroup turns its S into P, the tensor pipe runs the other tile's PV and S.
//              A's key list ends no later than B's, so in an item's last step the A slot is free:
//              the next item's S_A(0) is issued there, ahead of the last PV_B, and the A softmax
//              starts the next item while B finishes this one.
// The per-row arithmetic is softmax_tile's, as in the two-CTA kernels, so outputs equal theirs bit
// for bit.
// Items (tile pair, (b,h)) come from the work counter in the handle's status buffer, heaviest
// pairs first, through a two-slot ring whose slots are released by every reader (item_empty).
template <int E, int D, int NQ>
struct PpLayout {
  static constexpr int EC = E / 64, DC = D / 64;
  static constexpr uint32_t Q_BYTES = BM * E * 2;
  static constexpr uint32_t K_BYTES = BN * E * 2;
  static constexpr uint32_t V_BYTES = BN * D * 2;
  // K and V rings as deep as the shared memory beside the Q buffers allows (227 KB per CTA, less
  // barriers and alignment slack), at most 4 stages each: E = D = 128 gives 3 K and 2 V stages
  // beside two Q buffers, 2 and 2 beside three
  static constexpr uint32_t AVAIL = 232448 - 2048 - NQ * Q_BYTES;
  static constexpr int NK = (AVAIL - 2 * V_BYTES) / K_BYTES < 4 ? (int)((AVAIL - 2 * V_BYTES) / K_BYTES) : 4;
  static constexpr int NV = (AVAIL - NK * K_BYTES) / V_BYTES < 4 ? (int)((AVAIL - NK * K_BYTES) / V_BYTES) : 4;
  static_assert(NQ >= 2 && NK >= 2 && NV >= 2, "two Q buffers and two stages of K and V at least");
  static constexpr uint32_t OFF_K = NQ * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + NK * K_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + NV * V_BYTES;
  static constexpr int N_BARS = 2 * NQ + 2 * NK + 2 * NV + 14;
  static constexpr uint32_t BYTES = OFF_BAR + ((N_BARS * 8 + 127) / 128) * 128 + 1024;
  static_assert(BYTES <= 232448, "shared memory per CTA");
};

// softmax_tile with the thread's whole row of S in registers (one TMEM read per tile; the
// ping-pong kernel's softmax threads hold 192 registers): the same arithmetic in the same order,
// so the same P, row sum and rescale decisions.
template <bool MASKED, int D>
__device__ __forceinline__ void softmax_tile_reg(uint32_t ts, uint32_t to, int lim, float sl2e, float lw2, int it,
                                                 float& m_used, float& l, uint64_t* p_half) {
  float z[BN];
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) tmem_ld32(ts + c * 32, z + c * 32);
  tmem_ld_wait();
  if (MASKED) {
#pragma unroll
    for (int i = 0; i < BN; ++i) z[i] = i <= lim ? z[i] : -INFINITY;
  }
  float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int i = 0; i < BN; i += 8) {
    mx4[0] = fmax3(mx4[0], z[i], z[i + 1]);
    mx4[1] = fmax3(mx4[1], z[i + 2], z[i + 3]);
    mx4[2] = fmax3(mx4[2], z[i + 4], z[i + 5]);
    mx4[3] = fmax3(mx4[3], z[i + 6], z[i + 7]);
  }
  const float smax = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
  const float mx = smax == -INFINITY ? -INFINITY : fmaf(smax, sl2e, lw2);
  const bool grow = mx > m_used + 8.f;
  float corr = 1.f;
  if (grow) {
    corr = ex2_approx(m_used - mx);
    l *= corr;
    m_used = mx;
  }
  if (it > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      tmem_ld32(to + c * 32, o);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] *= corr;
      tmem_st32(to + c * 32, o);
    }
  }
  const float off = m_used == -INFINITY ? 0.f : lw2 - m_used;
  const float2 sl2e2 = make_float2(sl2e, sl2e), off2 = make_float2(off, off);
  float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float2 t = __ffma2_rn(make_float2(z[c * 32 + 2 * e], z[c * 32 + 2 * e + 1]), sl2e2, off2);
      const float p0 = ex2_approx(t.x);
      const float p1 = ex2_approx(t.y);
      ls2[e & 1] = __fadd2_rn(ls2[e & 1], make_float2(p0, p1));
      const __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
      pk[e] = *reinterpret_cast<const uint32_t*>(&pp);
    }
    tmem_st16(ts + c * 16, pk);
    if (c == BN / 64 - 1) {
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_half);
    }
  }
  l += (ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y);
}

// Registers per thread of the ping-pong kernel after its reallocation: the two softmax warpgroups
// take kPpSoftmaxRegs, the producer / MMA warpgroup keeps kPpOtherRegs; the sum fits the launch's
// 384 x kPpLaunchRegs (checked on the host before every launch).
constexpr int kPpLaunchRegs = 168, kPpSoftmaxRegs = 192, kPpOtherRegs = 120;
static_assert(256 * kPpSoftmaxRegs + 128 * kPpOtherRegs <= 384 * kPpLaunchRegs, "register split");

template <int E, int D, int NQ>
__global__ void __launch_bounds__(384, 1) attn_pp_kernel(const __grid_constant__ TcMaps maps, const AttnArgs a,
                                                         int* status) {
  using Lay = PpLayout<E, D, NQ>;
  constexpr int NK = Lay::NK, NV = Lay::NV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  uint64_t* bars = (uint64_t*)(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars;                // [NQ] the Q buffer's fill landed (or, for an absent A tile, was skipped)
  uint64_t* q_empty = q_full + NQ;        // [NQ] the last S MMA reading the buffer has completed (commit)
  uint64_t* k_full = q_empty + NQ;        // [NK]
  uint64_t* k_empty = k_full + NK;        // [NK] S_A and S_B of the tile have read K (commit)
  uint64_t* v_full = k_empty + NK;        // [NV]
  uint64_t* v_empty = v_full + NV;        // [NV] PV_A and PV_B of the tile have read V (commit)
  uint64_t* s_full = v_empty + NV;        // [2] S_x ready (commit after S_x)
  uint64_t* p_half = s_full + 2;          // [2] P_x of keys 0..63 written (128 threads)
  uint64_t* p_full = p_half + 2;          // [2] P_x of all keys written (128 threads)
  uint64_t* pv_done = p_full + 2;         // [2] the item's last PV_x done (commit)
  uint64_t* o_empty = pv_done + 2;        // [2] O_x read out of TMEM (128 threads)
  uint64_t* item_full = o_empty + 2;      // [2] ring slot written (K producer)
  uint64_t* item_empty = item_full + 2;   // [2] ring slot read by the V and Q producers, the MMA thread
                                          //     and all 256 softmax threads
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;
  __shared__ volatile int where_s;
  __shared__ int item_s;
  __shared__ int item_ring[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.n_pairs * a.B * a.H;
  int* sched = status + 4;

  if (threadIdx.x == 0) {
    abort_s = 0;
    where_s = 0;
    item_s = -1;
    for (int s = 0; s < NQ; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    for (int s = 0; s < NK; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full + x, 1);
      mbar_init(p_half + x, 128);
      mbar_init(p_full + x, 128);
      mbar_init(pv_done + x, 1);
      mbar_init(o_empty + x, 128);
      mbar_init(item_full + x, 1);
      mbar_init(item_empty + x, 259);
    }
    fence_barrier_init();
  }
  if (warp == 9) tmem_alloc(&tmem_base_s, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort = &abort_s;
  // item j: pair n_pairs - 1 - j % n_pairs (the heaviest first) of (b,h) j / n_pairs
  auto pair_of = [&](int j) { return a.pairs[a.pair0 + a.n_pairs - 1 - j % a.n_pairs]; };
  auto tiles_of = [&](int t) { return t < 0 ? 0 : count_key_tiles(a, a.tiles[t]); };

  if (warp >= 8) {
  regs_dec<kPpOtherRegs>();   // the whole warpgroup 8-11
  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer: work items and K
    if (lane == 0) {
      int g = 0, r = 0;
      bool ok = true;
      // item r + 1 is taken and published when item r's K loads start, so that the Q producer loads
      // its Q tiles a whole item ahead; its first key tile is prefetched into L2 meanwhile
      auto prefetch = [&](int jn) {
        const int2 pn = pair_of(jn);
        const int bhn = jn / a.n_pairs, bn = bhn / a.H, hn = bhn % a.H;
        const AttnTile tn = a.tiles[pn.y];
        if (tn.nseg > 0) {
          const AttnSeg sg = a.segs[tn.seg0];
          if (sg.kind == SEG_TOKENS) {
            for (int c = 0; c < Lay::EC; ++c) tma_prefetch_3d(&maps.k, c * 64, hn, bn * a.L + sg.first);
            for (int c = 0; c < Lay::DC; ++c) tma_prefetch_3d(&maps.v, c * 64, hn, bn * a.L + sg.first);
          } else {
            const int row = (bhn * a.n_slots + sg.first) * a.slot_rows;
            for (int c = 0; c < Lay::EC; ++c) tma_prefetch_2d(&maps.ck, c * 64, row);
            for (int c = 0; c < Lay::DC; ++c) tma_prefetch_2d(&maps.cv, c * 64, row);
          }
        }
      };
      // ring slot rr & 1 holds item rr; it is rewritten once all readers have taken item rr - 2
      auto publish = [&](int rr, int jv) -> bool {
        if (rr >= 2 && !mbar_wait(item_empty + (rr & 1), ((rr >> 1) - 1) & 1, abort)) {
          atomicCAS((int*)&where_s, 0, 11000 + min(rr, 999));
          return false;
        }
        item_ring[rr & 1] = jv < n_items ? jv : -1;
        mbar_arrive(item_full + (rr & 1));
        return true;
      };
      int j = atomicAdd(sched, 1);
      ok = publish(0, j);
      for (; ok && j < n_items; ++r) {
        const int j_next = atomicAdd(sched, 1);
        if (!publish(r + 1, j_next)) {
          ok = false;
          break;
        }
        if (j_next < n_items) prefetch(j_next);
        const int2 pr = pair_of(j);
        const int bh = j / a.n_pairs, b = bh / a.H, h = bh % a.H;
        const AttnTile tB = a.tiles[pr.y];
        for (int si = 0; si < tB.nseg && ok; ++si) {
          const AttnSeg sg = a.segs[tB.seg0 + si];
          const bool tok = sg.kind == SEG_TOKENS;
          for (int j0 = 0; j0 < sg.len; j0 += BN, ++g) {
            const int row = tok ? b * a.L + sg.first + j0 : (bh * a.n_slots + sg.first) * a.slot_rows + j0;
            const int st = g % NK;
            if (g >= NK && !mbar_wait(k_empty + st, ((g / NK) - 1) & 1, abort)) {
              ok = false;
              atomicCAS((int*)&where_s, 0, 1000 + min(g, 999));
              break;
            }
            if (a.inject_timeout && g == 0 && blockIdx.x == 0) continue;   // test hook: K(0) withheld
            mbar_expect_tx(k_full + st, Lay::K_BYTES);
#pragma unroll
            for (int c = 0; c < Lay::EC; ++c) {
              if (tok) tma_load_3d(sK + st * Lay::K_BYTES + c * 16384, &maps.k, k_full + st, c * 64, h, row);
              else tma_load_2d(sK + st * Lay::K_BYTES + c * 16384, &maps.ck, k_full + st, c * 64, row);
            }
          }
        }
        j = j_next;
      }
      // never leave with a copy in flight into this CTA's shared memory: wait (bounded) for the
      // last fill of every K stage
      for (int st = 0; st < NK; ++st) {
        const int last = g - 1 - ((g - 1 - st) % NK + NK) % NK;   // largest g' < g with g' % NK == st
        if (last < 0) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(k_full + st, (last / NK) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp == 11) {
    // ------------------------------------------------------------ TMA producer: Q
    if (lane == 0) {
      int nq = 0;   // fills issued
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int slot = r & 1;
        if (!mbar_wait(item_full + slot, (r >> 1) & 1, abort)) break;
        const int j = item_ring[slot];
        mbar_arrive(item_empty + slot);
        if (j < 0) break;
        const int2 pr = pair_of(j);
        const int bh = j / a.n_pairs, b = bh / a.H, h = bh % a.H;
        for (int x = 0; x < 2; ++x) {
          const int n = 2 * r + x, buf = n % NQ;
          if (n >= NQ && !mbar_wait(q_empty + buf, ((n / NQ) - 1) & 1, abort)) {
            atomicCAS((int*)&where_s, 0, 9000 + min(n, 999));
            ok = false;
            break;
          }
          ++nq;
          const int t = x ? pr.y : pr.x;
          if (x == 0 && tiles_of(t) == 0) {
            mbar_arrive(q_full + buf);   // no A tile: the fill is empty
            continue;
          }
          mbar_expect_tx(q_full + buf, Lay::Q_BYTES);
          const int q0 = a.tiles[t].q0;
#pragma unroll
          for (int c = 0; c < Lay::EC; ++c)
            tma_load_3d(sQ + buf * Lay::Q_BYTES + c * 16384, &maps.q, q_full + buf, c * 64, h, b * a.T + q0);
        }
      }
      for (int buf = 0; buf < NQ; ++buf) {
        const int last = nq - 1 - ((nq - 1 - buf) % NQ + NQ) % NQ;
        if (last < 0) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(q_full + buf, (last / NQ) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ TMA producer: V, on its own so that
    // a K load never waits for a V stage to drain
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int slot = r & 1;
        if (!mbar_wait(item_full + slot, (r >> 1) & 1, abort)) break;
        const int j = item_ring[slot];
        mbar_arrive(item_empty + slot);
        if (j < 0) break;
        const int2 pr = pair_of(j);
        const int bh = j / a.n_pairs, b = bh / a.H, h = bh % a.H;
        const AttnTile tB = a.tiles[pr.y];
        for (int si = 0; si < tB.nseg && ok; ++si) {
          const AttnSeg sg = a.segs[tB.seg0 + si];
          const bool tok = sg.kind == SEG_TOKENS;
          for (int j0 = 0; j0 < sg.len; j0 += BN, ++g) {
            const int row = tok ? b * a.L + sg.first + j0 : (bh * a.n_slots + sg.first) * a.slot_rows + j0;
            const int st = g % NV;
            if (g >= NV && !mbar_wait(v_empty + st, ((g / NV) - 1) & 1, abort)) {
              ok = false;
              atomicCAS((int*)&where_s, 0, 2000 + min(g, 999));
              break;
            }
            mbar_expect_tx(v_full + st, Lay::V_BYTES);
#pragma unroll
            for (int c = 0; c < Lay::DC; ++c) {
              if (tok) tma_load_3d(sV + st * Lay::V_BYTES + c * 16384, &maps.v, v_full + st, c * 64, h, row);
              else tma_load_2d(sV + st * Lay::V_BYTES + c * 16384, &maps.cv, v_full + st, c * 64, row);
            }
          }
        }
      }
      for (int st = 0; st < NV; ++st) {
        const int last = g - 1 - ((g - 1 - st) % NV + NV) % NV;
        if (last < 0) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(v_full + st, (last / NV) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IQK = idesc_bf16(BM, BN, false);
      constexpr uint32_t IPV = idesc_bf16(BM, D, true);
      const uint32_t q0 = smem_u32(sQ), ka = smem_u32(sK), va = smem_u32(sV);
      int g = 0, gx[2] = {0, 0}, ix[2] = {0, 0};
      bool ok = true;
      auto fail = [&](int code, int at) {
        ok = false;
        atomicCAS((int*)&where_s, 0, code + min(at, 999));
      };
      // S_x = Q (fill n) K^T of ring position gg into TMEM columns 128 x
      auto issue_s = [&](int x, int gg, int n) {
        const uint32_t q = q0 + (n % NQ) * Lay::Q_BYTES;
        const uint32_t kb = ka + (gg % NK) * Lay::K_BYTES;
#pragma unroll
        for (int k = 0; k < E / 16; ++k) {
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
          umma_bf16(tmem + 128 * x, sw128_desc(q + off, 16, 1024), sw128_desc(kb + off, 16, 1024), IQK, k > 0);
        }
        umma_commit(s_full + x);
      };
      // the Q buffer of fill n is free again once every MMA issued so far has completed
      auto q_release = [&](int n) { umma_commit(q_empty + n % NQ); };
      auto q_wait = [&](int n) -> bool {
        if (!mbar_wait(q_full + n % NQ, (n / NQ) & 1, abort)) {
          fail(4000, n);
          return false;
        }
        tc_fence_after();
        return true;
      };
      // O_x += P_x V of ring position gg, in two halves over the keys (the first once P of keys 0..63
      // is written); the first of an item waits for the previous item's O_x to be read out
      auto issue_pv = [&](int x, int gg, bool first) -> bool {
        const int st = gg % NV;
        if (!mbar_wait(p_half + x, gx[x] & 1, abort) || !mbar_wait(v_full + st, (gg / NV) & 1, abort) ||
            (first && ix[x] > 0 && !mbar_wait(o_empty + x, (ix[x] - 1) & 1, abort))) {
          fail(5000, gg);
          return false;
        }
        tc_fence_after();
        const uint32_t vb = va + st * Lay::V_BYTES;
#pragma unroll
        for (int k = 0; k < BN / 32; ++k)
          umma_bf16_tmem_a(tmem + 256 + 128 * x, tmem + 128 * x + k * 8, sw128_desc(vb + k * 2048, 16384, 1024), IPV,
                           (!first || k > 0) ? 1u : 0u);
        if (!mbar_wait(p_full + x, gx[x] & 1, abort)) {
          fail(7000, gg);
          return false;
        }
        tc_fence_after();
#pragma unroll
        for (int k = BN / 32; k < BN / 16; ++k)
          umma_bf16_tmem_a(tmem + 256 + 128 * x, tmem + 128 * x + k * 8, sw128_desc(vb + k * 2048, 16384, 1024), IPV,
                           1u);
        ++gx[x];
        return true;
      };
      auto wait_k = [&](int gg) -> bool {
        if (!mbar_wait(k_full + gg % NK, (gg / NK) & 1, abort)) {
          fail(3000, gg);
          return false;
        }
        tc_fence_after();
        return true;
      };
      auto fetch = [&](int rr) -> int {
        if (!mbar_wait(item_full + (rr & 1), (rr >> 1) & 1, abort)) {
          fail(12000, rr);
          return -1;
        }
        const int jv = item_ring[rr & 1];
        mbar_arrive(item_empty + (rr & 1));
        return jv;
      };
      // an item's key-tile counts, read from its tile records
      auto lengths = [&](int jv, int& na, int& nb) {
        na = nb = 0;
        if (jv >= 0) {
          const int2 pv = pair_of(jv);
          na = tiles_of(pv.x);
          nb = tiles_of(pv.y);
        }
      };
      int j = fetch(0), n_a = 0, n_b = 0;
      lengths(j, n_a, n_b);
      bool pre = false;   // S_A(0) of item r was issued in item r - 1's last step
      for (int r = 0; ok && j >= 0; ++r) {
        const int fa = 2 * r, fb = 2 * r + 1;   // the item's Q fills
        if ((!pre && !q_wait(fa)) || !q_wait(fb)) break;
        if (n_b == 0) {
          q_release(fa);
          q_release(fb);
          j = fetch(r + 1);
          lengths(j, n_a, n_b);
          continue;
        }
        if (!pre) {
          if (!wait_k(g)) break;
          if (n_a > 0) issue_s(0, g, fa);
          if (n_a <= 1) q_release(fa);
        }
        issue_s(1, g, fb);
        umma_commit(k_empty + g % NK);
        if (n_b == 1) q_release(fb);
        // the next item is taken now (it is published an item ahead), so that reading its tile
        // records overlaps this item instead of stalling the tensor pipe at the boundary
        const int jn = fetch(r + 1);
        if (!ok) break;
        int n_a_next = 0, n_b_next = 0;
        lengths(jn, n_a_next, n_b_next);
        bool pre_next = false;
        for (int jj = 0; jj < n_b && ok; ++jj) {
          const int gg = g + jj;
          // S_x(jj + 1) overwrites the columns PV_x(jj) reads P_x from: tcgen05.mma ops issued by one
          // thread execute in issue order, and the commit after S_x(jj + 1) tracks PV_x(jj) too
          if (jj < n_a) {
            if (!issue_pv(0, gg, jj == 0)) break;
            if (jj == n_a - 1) {
              umma_commit(pv_done + 0);
              ++ix[0];
            }
            if (jj + 1 < n_a) {
              if (!wait_k(gg + 1)) break;
              issue_s(0, gg + 1, fa);
              if (jj + 1 == n_a - 1) q_release(fa);
            }
          }
          if (jj == n_b - 1) {
            // the A slot is done with this item: the next item's S_A(0) goes ahead of the last PV_B
            // if its Q fill and first key tile land before B's last P is half written (neither
            // depends on anything issued from here on); otherwise it waits for the next item's start
            if (jn >= 0) {
              const int fn = fa + 2, kn = g + n_b;
              const long long t0 = clock64();
              while (n_a_next > 0) {
                if (mbar_test(q_full + fn % NQ, (fn / NQ) & 1) && mbar_test(k_full + kn % NK, (kn / NK) & 1)) {
                  pre_next = true;
                  break;
                }
                if (mbar_test(p_half + 1, gx[1] & 1) || *abort || clock64() - t0 > kWaitCycles) break;
              }
              if (pre_next) {
                tc_fence_after();
                issue_s(0, kn, fn);
                if (n_a_next == 1) q_release(fn);
              }
            }
          }
          if (!issue_pv(1, gg, jj == 0)) break;
          umma_commit(v_empty + gg % NV);
          if (jj == n_b - 1) {
            umma_commit(pv_done + 1);
            ++ix[1];
          } else {
            if (!wait_k(gg + 1)) break;
            issue_s(1, gg + 1, fb);
            umma_commit(k_empty + (gg + 1) % NK);
            if (jj + 1 == n_b - 1) q_release(fb);
          }
        }
        if (!ok) break;
        g += n_b;
        j = jn;
        n_a = n_a_next;
        n_b = n_b_next;
        pre = pre_next;
      }
    }
  }
  } else {
    regs_inc<kPpSoftmaxRegs>();
    // ------------------------------------------------------------ softmax warpgroups A (warps 0-3), B (4-7)
    const int x = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t ts = tmem + lane_base + 128 * x, to = tmem + lane_base + 256 + 128 * x;
    int gx = 0, ix = 0, where = 0;
    bool ok = true;
    // item rr of the ring: its index and this warpgroup's tile, read ahead of the previous item's
    // epilogue, and the tile's segment records pulled into L1, so that none of these loads sits on
    // the slot's critical path
    struct Next {
      int j, tile_id;
      AttnTile tile;
    };
    auto take = [&](int rr, Next& nx) -> bool {
      if (!warp_wait(item_full + (rr & 1), (rr >> 1) & 1, abort)) {
        where = 10;
        return false;
      }
      nx.j = item_ring[rr & 1];
      mbar_arrive(item_empty + (rr & 1));
      nx.tile_id = -1;
      nx.tile = AttnTile{0, 0, 0, 0};
      if (nx.j < 0) return true;
      const int2 pr = pair_of(nx.j);
      nx.tile_id = x ? pr.y : pr.x;
      if (nx.tile_id >= 0) nx.tile = a.tiles[nx.tile_id];
      if (nx.tile.nkt > 0 && lane == 0) prefetch_l1(a.segs + nx.tile.seg0, nx.tile.nseg * (int)sizeof(AttnSeg));
      return true;
    };
    Next cur;
    if (!take(0, cur)) ok = false;
    for (int r = 0; ok && cur.j >= 0; ++r) {
      if (cur.tile.nkt == 0) {
        if (!take(r + 1, cur)) break;
        continue;
      }
      const int tile_id = cur.tile_id;
      const AttnTile tile = cur.tile;
      const int bh = cur.j / a.n_pairs, b = bh / a.H, h = bh % a.H;
      if (row == 0) item_s = tile_id * 65536 + bh;
      const int tq = tile.q0 + row;
      float m_used = -INFINITY, l = 0.f;
      int it = 0;
      for (int si = 0; si < tile.nseg && ok; ++si) {
        const AttnSeg sg = a.segs[tile.seg0 + si];
        const float lw2 = sg.logw * 1.4426950408889634f;
        for (int j0 = 0; j0 < sg.len; j0 += BN, ++it, ++gx) {
          if (!warp_wait(s_full + x, gx & 1, abort)) {
            ok = false;
            where = 6;
            break;
          }
          tc_fence_after();
          const int nvalid = min(BN, sg.len - j0);
          const int kt0 = sg.first + j0;
          const bool causal = sg.kind == SEG_TOKENS && sg.causal;
          const bool masked = nvalid < BN || (causal && kt0 + BN - 1 > tile.q0);
          const int lim = min(nvalid - 1, causal ? tq - kt0 : BN - 1);
          if (masked) softmax_tile_reg<true, D>(ts, to, lim, a.scale_log2e, lw2, it, m_used, l, p_half + x);
          else softmax_tile_reg<false, D>(ts, to, lim, a.scale_log2e, lw2, it, m_used, l, p_half + x);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(p_full + x);
        }
      }
      if (!ok) break;
      if (!take(r + 1, cur)) break;
      if (!warp_wait(pv_done + x, ix & 1, abort)) {
        where = 8;
        break;
      }
      ++ix;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* out = (__nv_bfloat16*)a.out;
      const bool live = row < tile.qlen;
      __nv_bfloat16* orow = out + ((int64_t)(b * a.T + tq) * a.H + h) * D;
      uint32_t pk[D / 2];
#pragma unroll
      for (int c2 = 0; c2 < D / 64; ++c2) {
        float o[2][32];
        tmem_ld32(to + c2 * 64, o[0]);
        tmem_ld32(to + c2 * 64 + 32, o[1]);
        tmem_ld_wait();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const __nv_bfloat162 t = __floats2bfloat162_rn(o[hh][i] * inv, o[hh][i + 1] * inv);
            pk[(c2 * 64 + hh * 32 + i) / 2] = *reinterpret_cast<const uint32_t*>(&t);
          }
      }
      tc_fence_before();
      mbar_arrive(o_empty + x);
      if (live) {
#pragma unroll
        for (int i = 0; i < D / 8; ++i)
          *reinterpret_cast<uint4*>(orow + 8 * i) = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
      if (live && a.lse) a.lse[(int64_t)bh * a.T + tq] = (m_used + log2f(l)) * 0.6931471805599453f;
    }
    if (where && lane == 0) atomicCAS((int*)&where_s, 0, where * 1000 + min(gx, 999));
  }
  tc_fence_before();
  __syncthreads();
  if (abort_s && threadIdx.x == 0) {
    if (atomicCAS(status, 0, 1) == 0) {
      status[1] = item_s;
      status[2] = where_s;
    }
  }
  if (threadIdx.x == 0) {
    // every CTA has taken its last item before it counts itself out: the last one resets
    __threadfence();
    if (atomicAdd(sched + 1, 1) == (int)gridDim.x - 1) {
      atomicExch(sched, 0);
      atomicExch(sched + 1, 0);
    }
  }
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int E, int D>
cudaError_t launch_tc_t(const AttnArgs& a, int* status, cudaStream_t st) {
  TcMaps maps;
  const int64_t compact_rows = (int64_t)a.B * a.H * a.n_slots * a.slot_rows;
  bool ok = make_map_3d(&maps.q, a.q, (int64_t)a.B * a.T, a.H, E, 128) &&
            make_map_3d(&maps.k, a.k, (int64_t)a.B * a.L, a.H, E, 128) &&
            make_map_3d(&maps.v, a.v, (int64_t)a.B * a.L, a.H, D, 128);
  if (ok && a.ck && compact_rows > 0) {
    ok = make_map_2d(&maps.ck, a.ck, compact_rows, E, E, 128) && make_map_2d(&maps.cv, a.cv, compact_rows, D, D, 128);
  } else if (ok) {
    maps.ck = maps.k;
    maps.cv = maps.v;
  }
  if (!ok) return cudaErrorInvalidValue;
  if constexpr (E == 128 && D <= 128) {
    if (a.q8) {
      // e4m3 QK^T: the persistent two-CTA kernel with its S MMAs on e4m3 copies of q and the keys
      TcMaps m8 = maps;
      bool ok8 = status && make_map_3d_u8(&m8.q, a.q8, (int64_t)a.B * a.T, a.H, E, 128) &&
                 make_map_3d_u8(&m8.k, a.k8, (int64_t)a.B * a.L, a.H, E, 128);
      if (ok8 && a.ck8 && compact_rows > 0) ok8 = make_map_2d_u8(&m8.ck, a.ck8, compact_rows, E, E, 128);
      else m8.ck = m8.k;
      if (!ok8) return cudaErrorInvalidValue;
      int dev = 0, sms = 0;
      cudaError_t e = cudaGetDevice(&dev);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      const size_t sm = Tc2Layout<E, D, true>::BYTES;
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(attn_tc2p_kernel<E, D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e != cudaSuccess) return e;
      const int64_t items = (int64_t)a.n_tiles * a.B * a.H;
      attn_tc2p_kernel<E, D, true><<<(int)std::min<int64_t>(items, 2 * (int64_t)sms), 192, sm, st>>>(m8, a, status);
      return cudaGetLastError();
    }
  }
  if constexpr (D <= 128 && E <= 128) {
    if (a.pairs && a.n_pairs > 0 && status && std::getenv("THIN_ATTN_TC1") == nullptr &&
        std::getenv("THIN_ATTN_TC2_PER_TILE") == nullptr) {
      int dev = 0, sms = 0;
      cudaError_t e = cudaGetDevice(&dev);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      // two Q buffers: a third costs a K stage (E = D = 128) and measured no faster
      const size_t sm = PpLayout<E, D, 2>::BYTES;
      auto kern = attn_pp_kernel<E, D, 2>;
      if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      int per_sm = 0;
      if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 384, sm);
      cudaFuncAttributes fa{};
      if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kern);
      if (e != cudaSuccess) return e;
      // the register reallocation inside the kernel is sized for a launch of exactly kPpLaunchRegs per
      // thread: with any other count the two-CTA kernel below runs instead
      if (per_sm >= 1 && fa.numRegs == kPpLaunchRegs) {
        const int64_t items = (int64_t)a.n_pairs * a.B * a.H;
        const int grid = (int)std::min<int64_t>(items, (int64_t)sms);
        kern<<<grid, 384, sm, st>>>(maps, a, status);
        return cudaGetLastError();
      }
    }
  }
  if constexpr (D == 256 && E == 64) {
    // D = 256 (BigGAN): the persistent kernel, one CTA per SM (S and O take 384 TMEM columns)
    if (std::getenv("THIN_ATTN_TC1") == nullptr && status != nullptr) {
      int dev = 0, sms = 0;
      cudaError_t e = cudaGetDevice(&dev);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      // more shared memory than half an SM's, so that no second CTA lands on an SM and waits for TMEM
      const size_t sm = std::max<size_t>(Tc2Layout<E, D>::BYTES, 120 * 1024);
      if (e == cudaSuccess) e = cudaFuncSetAttribute(attn_tc2p_kernel<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e != cudaSuccess) return e;
      const int64_t items = (int64_t)a.n_tiles * a.B * a.H;
      attn_tc2p_kernel<E, D><<<(int)std::min<int64_t>(items, sms), 192, sm, st>>>(maps, a, status);
      return cudaGetLastError();
    }
  }
  if constexpr (D <= 128) {
    if (std::getenv("THIN_ATTN_TC1") == nullptr) {
      const size_t sm = Tc2Layout<E, D>::BYTES;
      if (std::getenv("THIN_ATTN_TC2_PER_TILE") != nullptr || status == nullptr) {
        cudaError_t e = cudaFuncSetAttribute(attn_tc2_kernel<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        attn_tc2_kernel<E, D><<<dim3(a.n_tiles, a.B * a.H), 192, sm, st>>>(maps, a, status);
        return cudaGetLastError();
      }
      int dev = 0, sms = 0;
      cudaError_t e = cudaGetDevice(&dev);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      if (e == cudaSuccess) e = cudaFuncSetAttribute(attn_tc2p_kernel<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e != cudaSuccess) return e;
      const int64_t items = (int64_t)a.n_tiles * a.B * a.H;
      const int grid = (int)std::min<int64_t>(items, 2 * (int64_t)sms);
      attn_tc2p_kernel<E, D><<<grid, 192, sm, st>>>(maps, a, status);
      return cudaGetLastError();
    }
  }
  const size_t sm = TcLayout<E, D>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<E, D><<<dim3(a.n_tiles, a.B * a.H), 192, sm, st>>>(maps, a, status);
  return cudaGetLastError();
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// rows x width bf16 matrix whose rows are `row_stride` elements apart, in (64 x 128) boxes.
bool make_map_2d(CUtensorMap* m, const void* base, int64_t rows, int width, int64_t row_stride, int box_rows) {
  cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)base, dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (B*L, H, width) view of a (B, L, H, width) bf16 tensor, boxes of (64, 1 head, 128 rows).
bool make_map_3d(CUtensorMap* m, const void* base, int64_t BL, int H, int width, int box_rows) {
  cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)H, (cuuint64_t)BL};
  cuuint64_t strides[2] = {(cuuint64_t)width * 2, (cuuint64_t)width * H * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)base, dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (B*L/k, k, H, width) view of a (B, L, H, width) bf16 tensor, boxes of (64, 1 head, 1, box_rows):
// a box starting at (x, h, 0, R) holds rows R k, (R+1) k, ... -- every k-th row.
bool make_map_4d_strided(CUtensorMap* m, const void* base, int64_t BL, int H, int width, int k, int box_rows) {
  if (k < 1 || BL / k < 1) return false;
  cuuint64_t dims[4] = {(cuuint64_t)width, (cuuint64_t)H, (cuuint64_t)k, (cuuint64_t)(BL / k)};
  cuuint64_t strides[3] = {(cuuint64_t)width * 2, (cuuint64_t)width * H * 2, (cuuint64_t)width * H * k * 2};
  cuuint32_t box[4] = {64, 1, 1, (cuuint32_t)box_rows};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, (void*)base, dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// e4m3 (one byte per element) forms of make_map_2d / make_map_3d: boxes of 128 elements (128 bytes).
bool make_map_2d_u8(CUtensorMap* m, const void* base, int64_t rows, int width, int64_t row_stride, int box_rows) {
  cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride};
  cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void*)base, dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool make_map_3d_u8(CUtensorMap* m, const void* base, int64_t BL, int H, int width, int box_rows) {
  cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)H, (cuuint64_t)BL};
  cuuint64_t strides[2] = {(cuuint64_t)width, (cuuint64_t)width * H};
  cuuint32_t box[3] = {128, 1, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, (void*)base, dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tensor_maps_available() { return encode_fn() != nullptr; }

bool attention_tc_supported(int dtype, int E, int D) {
  if (dtype != 1) return false;
  return (E == 64 && (D == 64 || D == 128 || D == 256)) || (E == 128 && (D == 64 || D == 128));
}

int attention_tc_tile_rows() { return BM; }

cudaError_t launch_attention_tc(const AttnArgs& a, int* status, cudaStream_t st, bool* done) {
  *done = false;
  if (!tensor_maps_available() || a.n_tiles == 0 || a.B * a.H == 0) return cudaSuccess;
  cudaError_t e = cudaErrorInvalidValue;
  if (a.E == 64 && a.D == 64) e = launch_tc_t<64, 64>(a, status, st);
  else if (a.E == 64 && a.D == 128) e = launch_tc_t<64, 128>(a, status, st);
  else if (a.E == 64 && a.D == 256) e = launch_tc_t<64, 256>(a, status, st);
  else if (a.E == 128 && a.D == 64) e = launch_tc_t<128, 64>(a, status, st);
  else if (a.E == 128 && a.D == 128) e = launch_tc_t<128, 128>(a, status, st);
  else return cudaSuccess;
  if (e == cudaSuccess) *done = true;
  return e;
}

}  // namespace thin
