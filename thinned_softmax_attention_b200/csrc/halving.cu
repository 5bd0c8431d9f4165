// Kernel Halving on the GPU: one "step" halves n_inst independent instances of n points.
//
// The walk is the self-balancing walk of Kernel Halving (Dwivedi & Mackey,
// "Kernel Thinning"), run on the key-value attention kernel kappa_att that the
// "Express Language Modeling" summary names for Thinformer Express:
//   kappa((k,v),(k',v')) = exp(s <k,k'>) (<v,v'> + c^2),  c = max |v| of the instance.
//
// A step is three launches (instances of <= 128 bf16 points whose rows form TMA boxes take the
// one-launch kernel of halving_fused.cu instead):
//   1. c2_kernel        c^2 of every instance
//   2. pairgram kernel   pair-difference matrix Delta[j][i] = k(x_j,x_i) - k(y_j,x_i)
//                        - k(x_j,y_i) + k(y_j,y_i) for j <= i (upper triangle, 32x32 pair
//                        tiles; Delta[i][i] = b_i^2)
//   3. walk_kernel       the sequential decisions, then the gather of the survivors
//
// The decision for pair i keeps its first point iff alpha_i < a_i (1 - 2 u_i), which
// is u_i < clip((1 - alpha_i/a_i)/2, 0, 1) rearranged (a_i > 0).
#include "common.cuh"
#include "kernels.h"
#include "walk.cuh"

namespace thin {

// ---------------------------------------------------------------------------
// 1. c^2 = (max |v|)^2 over the instance's points
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) c2_kernel(StepArgs a) {
  const int inst = blockIdx.x;
  const HalveInst in = a.inst[inst];
  __shared__ uint32_t U_s;
  __shared__ float red[8];
  if (threadIdx.x == 0) U_s = sub_offset(a, in);
  __syncthreads();
  const int epc = 16 / (int)sizeof(T);            // elements per 16-byte chunk
  const int cpp = a.D / epc;                       // chunks per point
  const uint4* V = (const uint4*)a.srcV;
  float mx = 0.f;
  const int total = a.n * cpp;
  // 8 independent 16-byte loads in flight per thread
  for (int e0 = threadIdx.x; e0 < total; e0 += 8 * blockDim.x) {
    uint4 w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + u * blockDim.x;
      if (e < total) {
        const int p = e / cpp, c = e - p * cpp;
        int64_t kr, vr;
        point_rows(a, in, p, U_s, &kr, &vr);
        w[u] = V[vr / epc + c];
      } else {
        w[u] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (sizeof(T) == 2) {
        const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = __uint_as_float(ws[i] << 16), hi = __uint_as_float(ws[i] & 0xFFFF0000u);
          mx = fmaxf(mx, fmaxf(fabsf(lo), fabsf(hi)));
        }
      } else {
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(__uint_as_float(w[u].x)), fabsf(__uint_as_float(w[u].y))),
                             fmaxf(fabsf(__uint_as_float(w[u].z)), fabsf(__uint_as_float(w[u].w)))));
      }
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) v = fmaxf(v, red[w]);
    a.c2[inst] = v * v;
  }
}

// ---------------------------------------------------------------------------
// 2. pair-difference Gram, CUDA-core version (fp32 inputs, and any bf16 shape)
//    CTA = one 32x32 tile of Delta = one 64x64 tile of the point Gram.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) pairgram_simt_kernel(StepArgs a) {
  const int inst = blockIdx.x;
  const int nb = a.m_pad >> 5;
  int t = blockIdx.y, tj = 0;
  while (t >= nb - tj) {
    t -= nb - tj;
    ++tj;
  }
  const int ti = tj + t;
  const HalveInst in = a.inst[inst];

  __shared__ float As[64][33];
  __shared__ float Bs[64][33];
  __shared__ int64_t rK[64], rV[64], cK[64], cV[64];
  __shared__ uint32_t U_s;
  if (threadIdx.x == 0) U_s = sub_offset(a, in);
  __syncthreads();
  if (threadIdx.x < 128) {
    const int which = threadIdx.x >> 6, r = threadIdx.x & 63;
    const int p = (which ? ti : tj) * 64 + r;
    int64_t ko = -1, vo = -1;
    if (p < a.n) {
      const PointRef pr = point_ref(a, in, p, U_s);
      ko = pr.krow;
      vo = pr.vrow;
    }
    if (which) { cK[r] = ko; cV[r] = vo; } else { rK[r] = ko; rV[r] = vo; }
  }
  __syncthreads();

  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  float kk[4][4], vv[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) kk[i][j] = vv[i][j] = 0.f;

  for (int part = 0; part < 2; ++part) {
    const T* X = (const T*)(part ? a.srcV : a.srcK);
    const int W = part ? a.D : a.E;
    const int64_t* ro = part ? rV : rK;
    const int64_t* co = part ? cV : cK;
    for (int d0 = 0; d0 < W; d0 += 32) {
      for (int e = threadIdx.x; e < 64 * 32; e += 256) {
        const int r = e >> 5, c = e & 31;
        const bool okc = d0 + c < W;
        As[r][c] = (ro[r] >= 0 && okc) ? to_f(X[ro[r] + d0 + c]) : 0.f;
        Bs[r][c] = (co[r] >= 0 && okc) ? to_f(X[co[r] + d0 + c]) : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int c = 0; c < 32; ++c) {
        float av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = As[ty * 4 + i][c];
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = Bs[tx * 4 + j][c];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (part) vv[i][j] = fmaf(av[i], bv[j], vv[i][j]);
            else kk[i][j] = fmaf(av[i], bv[j], kk[i][j]);
          }
      }
      __syncthreads();
    }
  }
  const float c2 = a.c2[inst];
  float kap[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) kap[i][j] = exp2f(kk[i][j] * a.scale_log2e) * (vv[i][j] + c2);
  float* Dl = a.delta + (size_t)inst * a.m_pad * a.m_pad;
#pragma unroll
  for (int pa = 0; pa < 2; ++pa)
#pragma unroll
    for (int pb = 0; pb < 2; ++pb) {
      const int pj = tj * 32 + ty * 2 + pa, pi = ti * 32 + tx * 2 + pb;
      const float d = kap[2 * pa][2 * pb] - kap[2 * pa + 1][2 * pb] - kap[2 * pa][2 * pb + 1] +
                      kap[2 * pa + 1][2 * pb + 1];
      if (pj < a.m && pi < a.m) Dl[(size_t)pj * a.m_pad + pi] = d;
    }
}

// ---------------------------------------------------------------------------
// 3. the walk and the gather.  CTA = one instance, 128 threads.
//    Pairs are taken in blocks of 32: warp 0 runs the 32 dependent decisions
//    of a block from its diagonal Delta tile (lane l holds alpha of pair 32t+l),
//    then all threads add the block's contribution eta_s Delta[32t+s][k] to the
//    alpha of every later pair k.  alpha_i therefore accumulates its terms in
//    pair order j = 0, 1, ..., i-1.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128, 8) walk_kernel(StepArgs a) {
  extern __shared__ float sm[];
  const int inst = blockIdx.x;
  const HalveInst in = a.inst[inst];
  const int m = a.m, mp = a.m_pad, nb = mp >> 5;
  float* alpha = sm;                              // mp
  float* ubuf = alpha + mp;                       // mp
  float* tile = ubuf + mp;                        // 32 x 33
  uint32_t* bits = (uint32_t*)(tile + 32 * 33);   // nb
  __shared__ uint32_t U_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* Dl = a.delta + (size_t)inst * mp * mp;

  for (int i = tid; i < mp; i += 128) {
    alpha[i] = 0.f;
    ubuf[i] = i < m ? philox_uniform(a.seed, in.ctr_bh, in.round_id, in.pair0 + (uint32_t)i) : 0.5f;
  }
  if (tid == 0) U_s = sub_offset(a, in);
  float sigma = 0.f;
  for (int t = 0; t < nb; ++t) {
    const int base = t * 32;
    __syncthreads();
    for (int e = tid; e < 1024; e += 128) {
      const int r = e >> 5, c = e & 31;
      tile[r * 33 + c] = (base + r < m && base + c < m) ? Dl[(size_t)(base + r) * mp + base + c] : 0.f;
    }
    __syncthreads();
    const int steps = min(32, m - base);
    if (warp == 0) {
      // lane l holds pair base + l; the tile is zero past m, so padded pairs are no-ops
      float my = alpha[base + lane];
      const uint32_t kb = walk_block32(my, sigma, tile[lane * 33 + lane], 1.f - 2.f * ubuf[base + lane], a.C,
                                       1.f / a.C, lane, [&](int s) { return tile[s * 33 + lane]; });
      if (lane == 0) bits[t] = kb;
    }
    __syncthreads();
    const uint32_t kb = bits[t];
    for (int k = base + 32 + tid; k < m; k += 128) {
      float acc = alpha[k];
#pragma unroll
      for (int s0 = 0; s0 < 32; s0 += 8) {
        float d[8];
#pragma unroll
        for (int s = 0; s < 8; ++s) d[s] = s0 + s < steps ? Dl[(size_t)(base + s0 + s) * mp + k] : 0.f;
#pragma unroll
        for (int s = 0; s < 8; ++s) acc = fmaf(((kb >> (s0 + s)) & 1u) ? 1.f : -1.f, d[s], acc);
      }
      alpha[k] = acc;
    }
  }
  __syncthreads();
  if (a.trace)
    for (int w = tid; w < nb; w += 128) a.trace[a.trace_base + (size_t)inst * nb + w] = bits[w];

  // gather the kept point of every pair into row i of the destination
  const int kw = a.E * (int)sizeof(T) / 16, vw = a.D * (int)sizeof(T) / 16;
  const uint4* K = (const uint4*)a.srcK;
  const uint4* V = (const uint4*)a.srcV;
  uint4* dK = (uint4*)a.dstK;
  uint4* dV = (uint4*)a.dstV;
  const int epw = 16 / (int)sizeof(T);
  for (int i = warp; i < m; i += 4) {
    const bool keep = (bits[i >> 5] >> (i & 31)) & 1u;
    const PointRef r = point_ref(a, in, 2 * i + (keep ? 0 : 1), U_s);
    const int64_t drow = in.dst_row + i;
    for (int w = lane; w < kw; w += 32) dK[drow * kw + w] = K[r.krow / epw + w];
    for (int w = lane; w < vw; w += 32) dV[drow * vw + w] = V[r.vrow / epw + w];
    if (lane == 0) a.dstIdx[drow] = r.idx;
  }
}


// Gather the kept point of pairs [i0, i1) (bit i of `bits(i)` set = first point kept) into
// destination rows dst_row + i, by one warp.  Lane l resolves pair i0 + 32q + l; the warp then
// copies the rows four at a time with all their 16-byte loads in flight before the stores.
template <typename T, bool WIDE, typename Bits>
__device__ __forceinline__ void gather_pairs(const StepArgs& a, const HalveInst& in, uint32_t U, int i0, int i1,
                                             Bits bits, int lane) {
  const int kw = a.E * (int)sizeof(T) / 16, vw = a.D * (int)sizeof(T) / 16, rw = kw + vw;
  const int epw = 16 / (int)sizeof(T);
  const uint4* K = (const uint4*)a.srcK;
  const uint4* V = (const uint4*)a.srcV;
  uint4* dK = (uint4*)a.dstK;
  uint4* dV = (uint4*)a.dstV;
  for (int g = i0; g < i1; g += 32) {
    const int i = g + lane;
    int64_t kr = 0, vr = 0;
    if (i < i1) {
      const bool keep = bits(i);
      const int pnt = 2 * i + (keep ? 0 : 1);
      point_rows(a, in, pnt, U, &kr, &vr);
      a.dstIdx[in.dst_row + i] =
          a.src_kind == SRC_TOKENS ? (int32_t)(in.tok0 + (int)(kr / a.E / a.H - in.src_row)) : a.srcIdx[in.src_row + pnt];
    }
    kr /= epw;
    vr /= epw;
    const int nrows = min(32, i1 - g);
    if (WIDE && rw <= 32) {
      // one 16-byte chunk per lane per row: 8 rows in flight
      for (int j = 0; j < nrows; j += 8) {
        uint4 buf[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int64_t krj = __shfl_sync(0xffffffffu, kr, (j + jj) & 31);
          const int64_t vrj = __shfl_sync(0xffffffffu, vr, (j + jj) & 31);
          if (j + jj < nrows && lane < rw) buf[jj] = lane < kw ? K[krj + lane] : V[vrj + (lane - kw)];
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int64_t drow = in.dst_row + g + j + jj;
          if (j + jj < nrows && lane < rw) {
            if (lane < kw) dK[drow * kw + lane] = buf[jj];
            else dV[drow * vw + (lane - kw)] = buf[jj];
          }
        }
      }
      continue;
    }
    for (int j = 0; j < nrows; j += 4) {
      uint4 buf[4][4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int64_t krj = __shfl_sync(0xffffffffu, kr, (j + jj) & 31);
        const int64_t vrj = __shfl_sync(0xffffffffu, vr, (j + jj) & 31);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int w = lane + 32 * q;
          if (j + jj < nrows && w < rw) buf[jj][q] = w < kw ? K[krj + w] : V[vrj + (w - kw)];
        }
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int64_t drow = in.dst_row + g + j + jj;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int w = lane + 32 * q;
          if (j + jj < nrows && w < rw) {
            if (w < kw) dK[drow * kw + w] = buf[jj][q];
            else dV[drow * vw + (w - kw)] = buf[jj][q];
          }
        }
      }
    }
  }
}

// Walk of instances with m <= 32 pairs: one warp per instance.  Lane l holds column l of the
// pair-difference matrix (Delta[s][l] for every s) and alpha of pair l.
template <typename T>
__global__ void __launch_bounds__(128) walk_small_kernel(StepArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int inst = blockIdx.x * 4 + warp;
  if (inst >= a.n_inst) return;
  const HalveInst in = a.inst[inst];
  const int m = a.m;
  const float* Dl = a.delta + (size_t)inst * a.m_pad * a.m_pad;
  float d[32];
#pragma unroll
  for (int s = 0; s < 32; ++s) d[s] = (s < m && lane < m) ? Dl[(size_t)s * a.m_pad + lane] : 0.f;
  const float w_l = lane < m ? 1.f - 2.f * philox_uniform(a.seed, in.ctr_bh, in.round_id, in.pair0 + (uint32_t)lane) : 0.f;
  const uint32_t U = sub_offset(a, in);
  // Pairs s >= m are no-ops: their Delta entries are 0, so b^2 = 0 keeps sigma and alpha as they
  // are, and their bits are never read.
  const uint32_t kb = walk_segment<32>(d, w_l, a.C, lane);
  if (a.trace && lane == 0) a.trace[a.trace_base + inst] = kb;
  gather_pairs<T, false>(a, in, U, 0, m, [kb](int i) { return ((kb >> i) & 1u) != 0; }, lane);
}

// Walk of instances with 32 < m <= 256 pairs: one CTA of 128 threads per instance.  The 32 rows
// of Delta of pair block t (columns >= 32t) are staged in shared memory with cp.async while
// block t-1 is walked; warp 0 runs the 32 dependent decisions of a block, then all threads add
// the block's contribution to the alpha of the later pairs.
constexpr int kWalkMidMaxPad = 256;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename T>
__global__ void __launch_bounds__(128) walk_mid_kernel(StepArgs a) {
  extern __shared__ __align__(16) float smf[];
  const int inst = blockIdx.x;
  const HalveInst in = a.inst[inst];
  const int m = a.m, mp = a.m_pad, nb = mp >> 5;
  float* alpha = smf;                          // mp
  float* wbuf = alpha + mp;                    // mp: 1 - 2u
  float* rb = wbuf + mp;                       // 2 x 32 x mp
  uint32_t* bits = (uint32_t*)(rb + 64 * mp);  // nb
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* Dl = a.delta + (size_t)inst * mp * mp;
  auto stage = [&](int t) {   // rows [32t, 32t+32), columns [32t, mp) -> rb[t & 1]
    float* dst = rb + (t & 1) * 32 * mp;
    const int c0 = 32 * t, nq = (mp - c0) / 4;
    for (int e = tid; e < 32 * nq; e += 128) {
      const int r = e / nq, q = e - r * nq;
      cp_async16(dst + r * mp + c0 + 4 * q, Dl + (size_t)(c0 + r) * mp + c0 + 4 * q);
    }
    cp_async_commit();
  };
  stage(0);
  for (int i = tid; i < mp; i += 128) {
    alpha[i] = 0.f;
    wbuf[i] = i < m ? 1.f - 2.f * philox_uniform(a.seed, in.ctr_bh, in.round_id, in.pair0 + (uint32_t)i) : 0.f;
  }
  const float C = a.C, rC = 1.f / C;
  float sigma = 0.f;
  for (int t = 0; t < nb; ++t) {
    const int base = 32 * t;
    __syncthreads();                 // rb[(t+1)&1] is no longer read (update of block t-1)
    if (t + 1 < nb) {
      stage(t + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const float* R = rb + (t & 1) * 32 * mp;
    const int steps = min(32, m - base);
    if (warp == 0) {
      const float dl = lane < steps ? R[lane * mp + base + lane] : 0.f;   // b^2 of pair base+lane
      float my = alpha[base + lane];
      // Pairs s >= steps are no-ops (b^2 = 0 keeps sigma; they only touch alpha of lanes that are
      // no pair), so the 32 steps run without a guard.
      const uint32_t kb = walk_block32(my, sigma, dl, wbuf[base + lane], C, rC, lane,
                                       [&](int s) { return R[s * mp + base + lane]; });
      if (lane == 0) bits[t] = kb;
    }
    __syncthreads();
    const uint32_t kb = bits[t];
    for (int k = base + 32 + tid; k < m; k += 128) {
      float acc = alpha[k];
#pragma unroll 8
      for (int s = 0; s < steps; ++s) acc = fmaf(((kb >> s) & 1u) ? 1.f : -1.f, R[s * mp + k], acc);
      alpha[k] = acc;
    }
  }
  __syncthreads();
  if (a.trace)
    for (int w = tid; w < nb; w += 128) a.trace[a.trace_base + (size_t)inst * nb + w] = bits[w];
  const uint32_t U = sub_offset(a, in);
  const int per = (m + 3) / 4;
  gather_pairs<T, true>(a, in, U, warp * per, min(m, (warp + 1) * per),
                  [bits](int i) { return ((bits[i >> 5] >> (i & 31)) & 1u) != 0; }, lane);
}

// Copy runs of tokens unchanged into compact rows (Express batches that need no thinning).
template <typename T>
__global__ void copy_tokens_kernel(StepArgs a) {
  const int inst = blockIdx.x;
  const HalveInst in = a.inst[inst];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kw = a.E * (int)sizeof(T) / 16, vw = a.D * (int)sizeof(T) / 16;
  const int epw = 16 / (int)sizeof(T);
  const uint4* K = (const uint4*)a.srcK;
  const uint4* V = (const uint4*)a.srcV;
  uint4* dK = (uint4*)a.dstK;
  uint4* dV = (uint4*)a.dstV;
  for (int p = warp; p < a.n; p += blockDim.x / 32) {
    const PointRef r = point_ref(a, in, p, 0u);
    const int64_t drow = in.dst_row + p;
    for (int w = lane; w < kw; w += 32) dK[drow * kw + w] = K[r.krow / epw + w];
    for (int w = lane; w < vw; w += 32) dV[drow * vw + w] = V[r.vrow / epw + w];
    if (lane == 0) a.dstIdx[drow] = r.idx;
  }
}

__global__ void iota_kernel(int32_t* idx, int64_t rows, int period) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i < rows) idx[i] = (int32_t)(i % period);
}

size_t walk_smem_bytes(int m_pad) { return (size_t)(2 * m_pad + 32 * 33 + m_pad / 32) * 4; }

template <typename T>
static cudaError_t launch_step_t(const StepArgs& a, bool use_tc, cudaStream_t st) {
  if (a.n_inst == 0) return cudaSuccess;
  if (sizeof(T) == 2 && use_tc && halving_fused_supported(a)) return launch_halving_fused(a, st);
  c2_kernel<T><<<a.n_inst, 256, 0, st>>>(a);
  const int nb = a.m_pad / 32;
  const int ntri = nb * (nb + 1) / 2;
  bool done = false;
  if (use_tc) {
    cudaError_t e = launch_pairgram_tc(a, st, &done);
    if (e != cudaSuccess) return e;
  }
  if (!done) pairgram_simt_kernel<T><<<dim3(a.n_inst, ntri), 256, 0, st>>>(a);
  if (a.m <= 32) {
    walk_small_kernel<T><<<(a.n_inst + 3) / 4, 128, 0, st>>>(a);
    return cudaGetLastError();
  }
  if (a.m_pad <= kWalkMidMaxPad) {
    const size_t sm = (size_t)(2 * a.m_pad + 64 * a.m_pad + a.m_pad / 32) * 4;
    cudaError_t e = cudaFuncSetAttribute(walk_mid_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    walk_mid_kernel<T><<<a.n_inst, 128, sm, st>>>(a);
    return cudaGetLastError();
  }
  const size_t sm = walk_smem_bytes(a.m_pad);
  if (sm > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(walk_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
  }
  walk_kernel<T><<<a.n_inst, 128, sm, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_halving_step(const StepArgs& a, int dtype, bool use_tc, cudaStream_t st) {
  return dtype == 0 ? launch_step_t<float>(a, false, st) : launch_step_t<__nv_bfloat16>(a, use_tc, st);
}

cudaError_t launch_copy_step(const StepArgs& a, int dtype, cudaStream_t st) {
  if (a.n_inst == 0) return cudaSuccess;
  if (dtype == 0) copy_tokens_kernel<float><<<a.n_inst, 128, 0, st>>>(a);
  else copy_tokens_kernel<__nv_bfloat16><<<a.n_inst, 128, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_iota(int32_t* idx, int64_t rows, int period, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  iota_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(idx, rows, period);
  return cudaGetLastError();
}

}  // namespace thin
