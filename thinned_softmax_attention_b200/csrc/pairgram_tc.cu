// Pair-difference Gram of the key-value attention kernel on the sm_100a tensor cores.
//
// For an instance of n points p_0..p_{n-1} (pairs (p_2i, p_2i+1)) and one tile of P x P points
// (row block tj <= column block ti):
//   kk = K_rows K_cols^T and vv = V_rows V_cols^T   (tcgen05, bf16 in, fp32 accumulators in TMEM)
//   kappa = 2^(kk s log2 e) (vv + c^2)               (epilogue, one row of the tile per thread)
//   Delta[j][i] = kappa[2j][2i] - kappa[2j][2i+1] - (kappa[2j+1][2i] - kappa[2j+1][2i+1])
// Rows 2j and 2j+1 sit in adjacent TMEM lanes, i.e. adjacent threads of one warp, so the
// second difference is one shuffle.  The (E + D) feature dimension is streamed through a
// 2-stage ring of 64-wide TMA boxes; the first E/64 chunks accumulate kk, the rest vv.
//
// CTA = 4 warps: thread 0 issues the TMA loads and the MMAs; all four warps run the epilogue
// (thread = tile row = TMEM lane).  Every mbarrier wait is bounded.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace thin {

namespace {

using namespace tc;

struct GramMaps {
  CUtensorMap k, v;
};

template <int P>
struct GramLayout {
  static constexpr uint32_t CHUNK = P * 64 * 2;        // one (P x 64) bf16 box
  static constexpr uint32_t STAGE = 2 * CHUNK;         // row box + column box
  static constexpr uint32_t SLACK = 16384;             // an M=128 operand reads 128 rows
  static constexpr uint32_t OFF_BAR = 2 * STAGE + SLACK;
  static constexpr uint32_t BYTES = OFF_BAR + 64 + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * P < 32 ? 32 : 2 * P;
};

template <int P>
__global__ void __launch_bounds__(128) pairgram_tc_kernel(const __grid_constant__ GramMaps maps, const StepArgs a,
                                                          int* status) {
  using Lay = GramLayout<P>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + Lay::OFF_BAR);
  uint64_t* full = bars;        // [2]
  uint64_t* empty = bars + 2;   // [2]
  uint64_t* done = bars + 4;
  __shared__ uint32_t tmem_base_s;
  __shared__ volatile int abort_s;

  const int inst = blockIdx.x;
  const int nt = (a.n + P - 1) / P;
  int t = blockIdx.y, tj = 0;
  while (t >= nt - tj) {
    t -= nt - tj;
    ++tj;
  }
  const int ti = tj + t;
  const bool diag = tj == ti;
  const HalveInst in = a.inst[inst];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int EC = a.E / 64, NC = (a.E + a.D) / 64;

  if (threadIdx.x == 0) {
    abort_s = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base_s, Lay::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort = &abort_s;

  if (threadIdx.x == 0) {
    const bool tokens = a.src_kind == SRC_TOKENS;
    const int h = (int)(in.bh % (uint32_t)a.H);
    // first source row of the instance: a token run starts 2*pair0 points into its (b,h) run
    const int64_t base_row = tokens ? (a.sub_stride > 1 ? in.src_row / a.sub_stride : in.src_row) + 2 * (int64_t)in.pair0
                                    : in.src_row;
    const int row_r = (int)(base_row + (int64_t)tj * P), row_c = (int)(base_row + (int64_t)ti * P);
    auto load = [&](int c) {
      const int st = c & 1;
      uint8_t* dst = smem + st * Lay::STAGE;
      mbar_expect_tx(full + st, diag ? Lay::CHUNK : 2 * Lay::CHUNK);
      const bool isk = c < EC;
      const CUtensorMap* m = isk ? &maps.k : &maps.v;
      const int x = (isk ? c : c - EC) * 64;
      if (tokens && a.sub_stride > 1) {
        tma_load_4d(dst, m, full + st, x, h, 0, row_r);
        if (!diag) tma_load_4d(dst + Lay::CHUNK, m, full + st, x, h, 0, row_c);
      } else if (tokens) {
        tma_load_3d(dst, m, full + st, x, h, row_r);
        if (!diag) tma_load_3d(dst + Lay::CHUNK, m, full + st, x, h, row_c);
      } else {
        tma_load_2d(dst, m, full + st, x, row_r);
        if (!diag) tma_load_2d(dst + Lay::CHUNK, m, full + st, x, row_c);
      }
    };
    constexpr uint32_t IDESC = idesc_bf16(128, P, false);
    const uint32_t base = smem_u32(smem);
    bool ok = true;
    load(0);
    if (NC > 1) load(1);
    int last = -1;
    for (int c = 0; c < NC && ok; ++c) {
      const int st = c & 1;
      if (!mbar_wait(full + st, (c >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t ra = base + st * Lay::STAGE;
      const uint32_t cb = diag ? ra : ra + Lay::CHUNK;
      const uint32_t d = tmem + (c < EC ? 0u : (uint32_t)P);
      const bool first = c == 0 || c == EC;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_bf16(d, sw128_desc(ra + k * 32, 16, 1024), sw128_desc(cb + k * 32, 16, 1024), IDESC,
                  (!first || k > 0) ? 1u : 0u);
      umma_commit(empty + st);
      last = c;
      if (c + 2 < NC) {
        if (!mbar_wait(empty + st, (c >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        load(c + 2);
      }
    }
    umma_commit(done);
    // leave no copy in flight: the last fill of each stage has landed
    for (int c = (last >= 0 ? last + 1 : 0); c < NC && c <= last + 2; ++c) {
      const long long t0 = clock64();
      while (!mbar_try_wait(full + (c & 1), (c >> 1) & 1) && clock64() - t0 < kWaitCycles) {
      }
    }
  }
  // ------------------------------------------------------------------ epilogue
  const int r = warp * 32 + lane;              // tile row = TMEM lane
  const bool ok = warp_wait(done, 0, abort);
  tc_fence_after();
  if (ok && warp * 32 < P) {
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float c2 = a.c2[inst];
    const int pj = (tj * P + r) >> 1;
    float* Drow = a.delta + (size_t)inst * a.m_pad * a.m_pad + (size_t)pj * a.m_pad;
    const bool writer = (r & 1) == 0 && pj < a.m;
#pragma unroll 1
    for (int cc = 0; cc < P / 32; ++cc) {
      float kk[32], vv[32];
      tmem_ld32(tmem + lane_base + cc * 32, kk);
      tmem_ld32(tmem + lane_base + P + cc * 32, vv);
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
      const int pi0 = (ti * P + cc * 32) >> 1;
      if (writer) {
        if (pi0 + 16 <= a.m) {
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(Drow + pi0 + i) = make_float4(dd[i], dd[i + 1], dd[i + 2], dd[i + 3]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (pi0 + i < a.m) Drow[pi0 + i] = dd[i];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (abort_s && threadIdx.x == 0 && status) {
    if (atomicCAS(status, 0, 2) == 0) status[1] = inst;
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

template <int P>
cudaError_t launch_p(const StepArgs& a, int* status, cudaStream_t st) {
  GramMaps maps;
  bool ok;
  if (a.src_kind == SRC_TOKENS && a.sub_stride > 1) {
    ok = make_map_4d_strided(&maps.k, a.srcK, a.src_rows, a.H, a.E, a.sub_stride, P) &&
         make_map_4d_strided(&maps.v, a.srcV, a.src_rows, a.H, a.D, a.sub_stride, P);
  } else if (a.src_kind == SRC_TOKENS) {
    ok = make_map_3d(&maps.k, a.srcK, a.src_rows, a.H, a.E, P) && make_map_3d(&maps.v, a.srcV, a.src_rows, a.H, a.D, P);
  } else {
    ok = make_map_2d(&maps.k, a.srcK, a.src_rows, a.E, a.E, P) && make_map_2d(&maps.v, a.srcV, a.src_rows, a.D, a.D, P);
  }
  if (!ok) return cudaErrorInvalidValue;
  const int nt = (a.n + P - 1) / P;
  const size_t sm = GramLayout<P>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(pairgram_tc_kernel<P>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  pairgram_tc_kernel<P><<<dim3(a.n_inst, nt * (nt + 1) / 2), 128, sm, st>>>(maps, a, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pairgram_tc(const StepArgs& a, cudaStream_t st, bool* done) {
  *done = false;
  if (a.E % 64 || a.D % 64 || a.src_rows <= 0 || !tensor_maps_available()) return cudaSuccess;
  // subsampled rows are a box only as a strided view (integer ratio, runs on multiples of it)
  if (a.src_kind == SRC_TOKENS && a.S_sub < a.S_full && a.sub_stride < 2) return cudaSuccess;
  cudaError_t e;
  if (a.n <= 32) e = launch_p<32>(a, a.status, st);
  else if (a.n <= 64) e = launch_p<64>(a, a.status, st);
  else e = launch_p<128>(a, a.status, st);
  if (e == cudaSuccess) *done = true;
  return e;
}

}  // namespace thin
