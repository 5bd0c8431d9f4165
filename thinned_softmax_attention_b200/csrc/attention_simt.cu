// Weighted softmax attention of a query tile against a list of key segments, on CUDA cores.
//
//   o_t   = sum_j w_j e^{s q_t.k_j} v_j / sum_j w_j e^{s q_t.k_j}
//   lse_t = ln sum_j w_j e^{s q_t.k_j}
// over the keys j of every segment visible to t (w_j = e^{logw} of the segment).
// This is the fp32 path (IEEE fp32 throughout) and the reference-shape fallback;
// bf16 workloads on E = D = 128 use the tensor-core kernel.
//
// CTA = up to 64 queries of one (b,h): 16 warps x 4 queries; key chunks of 64 rows are
// staged in shared memory (fp32) and shared by all 64 queries.  Online softmax in base 2.
#include "common.cuh"
#include "kernels.h"

namespace thin {

constexpr int SQ = 64;      // queries per CTA
constexpr int SK = 64;      // keys per chunk
constexpr int QPW = 4;      // queries per warp

template <typename T, int DV>
__global__ void __launch_bounds__(512) attn_simt_kernel(AttnArgs a) {
  extern __shared__ float sm[];
  const int E = a.E, D = a.D;
  float* Ks = sm;                       // SK x (E+1)
  float* Vs = Ks + SK * (E + 1);        // SK x D
  float* Qs = Vs + SK * D;              // SQ x E
  const AttnTile tile = a.tiles[a.tile0 + blockIdx.x];
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* q = (const T*)a.q;
  for (int e = threadIdx.x; e < SQ * E; e += blockDim.x) {
    const int r = e / E, c = e % E;
    Qs[e] = r < tile.qlen ? to_f(q[((int64_t)(b * a.T + tile.q0 + r) * a.H + h) * E + c]) : 0.f;
  }
  float mrow[QPW], lrow[QPW], o[QPW][DV];
#pragma unroll
  for (int i = 0; i < QPW; ++i) {
    mrow[i] = -INFINITY;
    lrow[i] = 0.f;
#pragma unroll
    for (int d = 0; d < DV; ++d) o[i][d] = 0.f;
  }
  for (int si = 0; si < tile.nseg; ++si) {
    const AttnSeg sg = a.segs[tile.seg0 + si];
    const float lw2 = sg.logw * 1.4426950408889634f;
    for (int j0 = 0; j0 < sg.len; j0 += SK) {
      const int nk = min(SK, sg.len - j0);
      __syncthreads();
      for (int e = threadIdx.x; e < SK * (E + D); e += blockDim.x) {
        const int r = e / (E + D), c = e % (E + D);
        float val = 0.f;
        if (r < nk) {
          const bool isk = c < E;
          const int cc = isk ? c : c - E;
          const int W = isk ? E : D;
          int64_t row;
          const T* base;
          if (sg.kind == SEG_TOKENS) {
            row = (int64_t)(b * a.L + sg.first + j0 + r) * a.H + h;
            base = (const T*)(isk ? a.k : a.v);
          } else {
            row = ((int64_t)bh * a.n_slots + sg.first) * a.slot_rows + j0 + r;
            base = (const T*)(isk ? a.ck : a.cv);
          }
          val = to_f(base[row * W + cc]);
        }
        if (c < E) Ks[r * (E + 1) + c] = val;
        else Vs[r * D + (c - E)] = val;
      }
      __syncthreads();
#pragma unroll
      for (int qi = 0; qi < QPW; ++qi) {
        const int ql = warp * QPW + qi;
        if (ql >= tile.qlen) continue;
        const int tq = tile.q0 + ql;
        float z[2];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int j = lane + 32 * kk;
          float acc = 0.f;
          for (int c = 0; c < E; ++c) acc = fmaf(Qs[ql * E + c], Ks[j * (E + 1) + c], acc);
          bool vis = j < nk;
          if (sg.kind == SEG_TOKENS && sg.causal) vis = vis && (sg.first + j0 + j <= tq);
          z[kk] = vis ? fmaf(acc, a.scale_log2e, lw2) : -INFINITY;
        }
        float cm = fmaxf(z[0], z[1]);
#pragma unroll
        for (int off = 16; off; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
        if (cm == -INFINITY) continue;
        const float mnew = fmaxf(mrow[qi], cm);
        const float corr = exp2f(mrow[qi] - mnew);
        const float p0 = exp2f(z[0] - mnew), p1 = exp2f(z[1] - mnew);
        float ps = p0 + p1;
#pragma unroll
        for (int off = 16; off; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        lrow[qi] = lrow[qi] * corr + ps;
        mrow[qi] = mnew;
#pragma unroll
        for (int d = 0; d < DV; ++d) o[qi][d] *= corr;
        for (int j = 0; j < nk; ++j) {
          const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
#pragma unroll
          for (int d = 0; d < DV; ++d) {
            const int dd = lane + 32 * d;
            if (dd < D) o[qi][d] = fmaf(pj, Vs[j * D + dd], o[qi][d]);
          }
        }
      }
    }
  }
  T* out = (T*)a.out;
#pragma unroll
  for (int qi = 0; qi < QPW; ++qi) {
    const int ql = warp * QPW + qi;
    if (ql >= tile.qlen) continue;
    const int tq = tile.q0 + ql;
    const float inv = 1.f / lrow[qi];
#pragma unroll
    for (int d = 0; d < DV; ++d) {
      const int dd = lane + 32 * d;
      if (dd < D) out[((int64_t)(b * a.T + tq) * a.H + h) * D + dd] = from_f<T>(o[qi][d] * inv);
    }
    if (a.lse && lane == 0)
      a.lse[((int64_t)bh) * a.T + tq] = (mrow[qi] + log2f(lrow[qi])) * 0.6931471805599453f;
  }
}

template <typename T, int DV>
static cudaError_t launch_simt_t(const AttnArgs& a, cudaStream_t st) {
  const size_t sm = (size_t)(SK * (a.E + 1) + SK * a.D + SQ * a.E) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<T, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  attn_simt_kernel<T, DV><<<dim3(a.n_tiles, a.B * a.H), 512, sm, st>>>(a);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_simt_d(const AttnArgs& a, cudaStream_t st) {
  if (a.D <= 64) return launch_simt_t<T, 2>(a, st);
  if (a.D <= 128) return launch_simt_t<T, 4>(a, st);
  return launch_simt_t<T, 8>(a, st);
}

cudaError_t launch_attention_simt(const AttnArgs& a, int dtype, cudaStream_t st) {
  if (a.n_tiles == 0 || a.B * a.H == 0) return cudaSuccess;
  return dtype == 0 ? launch_simt_d<float>(a, st) : launch_simt_d<__nv_bfloat16>(a, st);
}

int attention_simt_tile_rows() { return SQ; }

}  // namespace thin
