// Attention of one query per (b,h) against its key segments, split over the keys (decode).
//
// A decoded position attends to a few thousand keys (exact prefix, snapshot nodes, the batch in
// progress) with a single query.  Split kernel: CTA (chunk, b*h) takes 128 consecutive keys of the
// concatenated segments, one warp per 32 keys, one key per lane:
//   scores   lane i reads its key's row whole (all 16-byte pieces in flight) and forms
//            z = s q.k log2e + log2 w (w = the segment's weight) against q held in shared memory
//   softmax  m = the chunk's max z, p = 2^(z - m), l = sum p (CTA-wide through shared memory)
//   PV       lane-parallel over D: o += p_i v_i, the p_i broadcast from lane i
// and writes the partial (m, l, o) of its chunk.  The last CTA of a (b,h) to finish (an arrival
// counter per (b,h)) merges the partials
//   M = max m,  L = sum l 2^(m - M),  out = sum o 2^(m - M) / L,  lse = (M + log2 L) ln 2,
// appends the decoded token's key and value to the cache and clears the counter: one launch per
// token.  Base 2 throughout, fp32 accumulation, one pass over every key and value row.
#include "common.cuh"
#include "kernels.h"

namespace thin {

namespace {

constexpr int kDecodeChunk = 128;     // keys per CTA
constexpr int kDecodeThreads = 128;   // 4 warps x 32 keys

// A lane's DPL elements of a value row, kept as loaded (bf16 pairs or fp32 words) until used, so that
// a round of rows in flight costs half the registers in bf16.
template <typename T, int DPL>
struct RawSlice {
  static constexpr int W = DPL * (int)sizeof(T) / 4;
  uint32_t w[W];
};
template <typename T, int DPL>
__device__ __forceinline__ void load_raw(const T* row, int lane, RawSlice<T, DPL>& r) {
  const uint32_t* src = (const uint32_t*)(row + lane * DPL);
  if constexpr (RawSlice<T, DPL>::W == 1) {
    r.w[0] = src[0];
  } else if constexpr (RawSlice<T, DPL>::W == 2) {
    const uint2 u = *(const uint2*)src;
    r.w[0] = u.x;
    r.w[1] = u.y;
  } else {
#pragma unroll
    for (int c = 0; c < RawSlice<T, DPL>::W / 4; ++c) {
      const uint4 u = ((const uint4*)src)[c];
      r.w[4 * c] = u.x;
      r.w[4 * c + 1] = u.y;
      r.w[4 * c + 2] = u.z;
      r.w[4 * c + 3] = u.w;
    }
  }
}
template <typename T, int DPL>
__device__ __forceinline__ void fma_raw(float p, const RawSlice<T, DPL>& r, float (&o)[DPL]) {
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < DPL / 2; ++i) {
      o[2 * i] = fmaf(p, __uint_as_float(r.w[i] << 16), o[2 * i]);
      o[2 * i + 1] = fmaf(p, __uint_as_float(r.w[i] & 0xFFFF0000u), o[2 * i + 1]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[i] = fmaf(p, __uint_as_float(r.w[i]), o[i]);
  }
}

// partials merged by the last CTA of a (b,h): at most this many chunks per position
constexpr int kDecodeMaxSplits = 512;   // 64K visible keys

template <typename T, int E, int D>
__device__ __forceinline__ void decode_combine(const AttnArgs& a, const float* part, int n_splits,
                                               const DecodeAppend& ap, int bh);

template <typename T, int EPL, int DPL>
__global__ void __launch_bounds__(kDecodeThreads) decode_split_kernel(AttnArgs a, float* part, int n_splits,
                                                                       DecodeAppend ap) {
  const int split = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int E = EPL * 32, D = DPL * 32;
  constexpr int KV = E * (int)sizeof(T) / 16;     // 16-byte pieces of a key row
  __shared__ AttnSeg segs[32];
  __shared__ int seg_start[33];
  __shared__ __align__(16) float q_s[E];
  __shared__ float red_m[4], red_l[4];
  __shared__ float o_s[4][D];
  // launched with programmatic stream serialisation: the next token's launch may start now; it
  // sets up and loads its query, then waits (griddepcontrol.wait) for this grid to complete before
  // it touches the cache, the partials or any output
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const bool own = ap.nseg >= 0;   // segments passed in the launch
  const AttnTile tile = own ? AttnTile{0, 1, 0, ap.nseg} : a.tiles[a.tile0];
  const int nseg = min(tile.nseg, 32);
  if (warp == 0) {
    // one segment per lane (all in flight at once), start offsets by a warp prefix sum
    int len = 0;
    if (lane < nseg) {
      segs[lane] = own ? ap.segs[lane] : a.segs[tile.seg0 + lane];
      len = segs[lane].len;
    }
    int incl = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < nseg) seg_start[lane] = incl - len;
    if (lane == nseg - 1) seg_start[nseg] = incl;
    if (nseg == 0 && lane == 0) seg_start[0] = 0;
  }
  // every load the chunk needs goes out before any of them is used (a token is a chain of
  // dependent memory latencies, so the fewer rounds the better): q, this lane's key row and the
  // first RV value rows of the warp, then the rest of the value rows once the key row is consumed
  const T* q = (const T*)a.q + ((int64_t)b * a.T * a.H + h) * E;   // the tile's single query row
  float q_mine = 0.f;
  if (threadIdx.x < E) q_mine = to_f(q[threadIdx.x]);
  static_assert(E <= kDecodeThreads, "one q element per thread");
  __syncthreads();   // seg_start
  // this lane's key: j = chunk start + 32 warp + lane -> K and V rows, log2 weight
  const int j = split * kDecodeChunk + warp * 32 + lane;
  const bool valid = j < seg_start[nseg];
  const T *kr = nullptr, *vr = nullptr;
  float lw2 = 0.f;
  if (valid) {
    int s = 0;
    while (s + 1 < nseg && seg_start[s + 1] <= j) ++s;
    const AttnSeg sg = segs[s];
    const int off = j - seg_start[s];
    if (sg.kind == SEG_TOKENS) {
      const int64_t row = ((int64_t)b * a.L + sg.first + off) * a.H + h;
      kr = (const T*)a.k + row * E;
      vr = (const T*)a.v + row * D;
    } else {
      const int64_t row = ((int64_t)bh * a.n_slots + sg.first) * a.slot_rows + off;
      kr = (const T*)a.ck + row * E;
      vr = (const T*)a.cv + row * D;
    }
    lw2 = sg.logw * 1.4426950408889634f;
    if (ap.new_k && j == seg_start[nseg] - 1) {
      // the last key is the token being decoded: read it from the caller's rows (it is appended to
      // the cache by the merging CTA, after every chunk has been read)
      kr = (const T*)ap.new_k + ((int64_t)b * a.T * a.H + h) * E;
      vr = (const T*)ap.new_v + ((int64_t)b * a.T * a.H + h) * D;
    }
  }
  const int nvalid = __popc(__ballot_sync(0xffffffffu, valid));   // the valid keys are the first ones
  // everything below reads what the previous launch on this stream wrote (the cache rows, the
  // node buffers) or writes what it reads (the partials, the arrival counters)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  uint4 kv[KV];
  if (valid) {
#pragma unroll
    for (int c = 0; c < KV; ++c) kv[c] = ((const uint4*)kr)[c];
  }
  // o = sum p_i v_i over the warp's keys, lane-parallel over D: rows 0..RV-1 now, RV..31 later
  constexpr int RV = 16;
  RawSlice<T, DPL> v0[RV], v1[RV];
#pragma unroll
  for (int u = 0; u < RV; ++u) {
    const T* r = (const T*)__shfl_sync(0xffffffffu, (unsigned long long)vr, u);
    if (u < nvalid) load_raw<T, DPL>(r, lane, v0[u]);
  }
  if (threadIdx.x < E) q_s[threadIdx.x] = q_mine * a.scale_log2e;
  __syncthreads();
  // score of this lane's key against q (pre-scaled by s log2 e, broadcast from shared memory)
  float z_mine = -INFINITY;
  if (valid) {
    // four independent partial sums (one per 16-byte piece position mod 4), added at the end
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < KV; ++c) {
      const uint32_t w[4] = {kv[c].x, kv[c].y, kv[c].z, kv[c].w};
      float& ac = acc[c & 3];
      if constexpr (sizeof(T) == 2) {
        const float4 qa = *(const float4*)(q_s + c * 8), qb = *(const float4*)(q_s + c * 8 + 4);
        const float qq[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ac = fmaf(qq[2 * i], __uint_as_float(w[i] << 16), ac);
          ac = fmaf(qq[2 * i + 1], __uint_as_float(w[i] & 0xFFFF0000u), ac);
        }
      } else {
        const float4 qa = *(const float4*)(q_s + c * 4);
        const float qq[4] = {qa.x, qa.y, qa.z, qa.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) ac = fmaf(qq[i], __uint_as_float(w[i]), ac);
      }
    }
    z_mine = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + lw2;
  }
#pragma unroll
  for (int u = 0; u < RV; ++u) {
    const T* r = (const T*)__shfl_sync(0xffffffffu, (unsigned long long)vr, RV + u);
    if (RV + u < nvalid) load_raw<T, DPL>(r, lane, v1[u]);
  }
  // chunk max and 2^(z - m)
  float wm = z_mine;
#pragma unroll
  for (int o = 16; o; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
  if (lane == 0) red_m[warp] = wm;
  __syncthreads();
  const float m = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));
  const float p_mine = (z_mine == -INFINITY || m == -INFINITY) ? 0.f : exp2f(z_mine - m);
  float wl = p_mine;
#pragma unroll
  for (int o = 16; o; o >>= 1) wl += __shfl_xor_sync(0xffffffffu, wl, o);
  if (lane == 0) red_l[warp] = wl;
  float ov[DPL];
#pragma unroll
  for (int d = 0; d < DPL; ++d) ov[d] = 0.f;
#pragma unroll
  for (int u = 0; u < RV; ++u) {
    const float pu = __shfl_sync(0xffffffffu, p_mine, u);
    if (u < nvalid) fma_raw<T, DPL>(pu, v0[u], ov);
  }
#pragma unroll
  for (int u = 0; u < RV; ++u) {
    const float pu = __shfl_sync(0xffffffffu, p_mine, RV + u);
    if (RV + u < nvalid) fma_raw<T, DPL>(pu, v1[u], ov);
  }
#pragma unroll
  for (int d = 0; d < DPL; ++d) o_s[warp][lane * DPL + d] = ov[d];
  __syncthreads();
  float* out = part + ((size_t)bh * n_splits + split) * (D + 2);
  for (int d = threadIdx.x; d < D; d += kDecodeThreads) out[d] = o_s[0][d] + o_s[1][d] + o_s[2][d] + o_s[3][d];
  if (threadIdx.x == 0) {
    out[D] = m;
    out[D + 1] = red_l[0] + red_l[1] + red_l[2] + red_l[3];
  }
  // the last chunk of this (b,h) to finish merges them all
  __shared__ int last_s;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last_s = atomicAdd(ap.arrive + bh, 1) == n_splits - 1;
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  decode_combine<T, E, D>(a, part, n_splits, ap, bh);
  if (threadIdx.x == 0) ap.arrive[bh] = 0;   // ready for the next token (a later launch)
}

// Merge of the chunks' partials of (b,h) `bh` by one CTA (partials written by other CTAs of this
// launch: read through L2), append of the decoded token.
template <typename T, int E, int D>
__device__ __forceinline__ void decode_combine(const AttnArgs& a, const float* part, int n_splits,
                                               const DecodeAppend& ap, int bh) {
  const int b = bh / a.H, h = bh % a.H;
  if (ap.new_k) {
    // append the decoded token's key and value to the cache row of this position
    const int64_t src = (int64_t)b * a.T * a.H + h, dst = ((int64_t)b * a.L + ap.row) * a.H + h;
    for (int e = threadIdx.x; e < E; e += blockDim.x) ((T*)a.k)[dst * E + e] = ((const T*)ap.new_k)[src * E + e];
    for (int d = threadIdx.x; d < D; d += blockDim.x) ((T*)a.v)[dst * D + d] = ((const T*)ap.new_v)[src * D + d];
  }
  // the chunks' (m, l) in one round of loads, one chunk per thread, then M, the chunks' factors
  // 2^(m - M) and L through shared memory; o in rounds of sixteen chunks' loads, the first of
  // them issued with (m, l)
  __shared__ float m_s[kDecodeMaxSplits], f_s[kDecodeMaxSplits], l_s[kDecodeMaxSplits];
  __shared__ float red[4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* p = part + (size_t)bh * n_splits * (D + 2);
  // this thread's first column of o for the first sixteen chunks, loaded in the same round as (m, l)
  constexpr int RO = 16;
  float x0[RO];
#pragma unroll
  for (int u = 0; u < RO; ++u)
    x0[u] = (u < n_splits && (int)threadIdx.x < D) ? __ldcg(p + (size_t)u * (D + 2) + threadIdx.x) : 0.f;
  float mloc = -INFINITY;
  for (int s = threadIdx.x; s < n_splits; s += blockDim.x) {
    const float ms = __ldcg(p + (size_t)s * (D + 2) + D), ls = __ldcg(p + (size_t)s * (D + 2) + D + 1);
    m_s[s] = ms;
    l_s[s] = ls;
    mloc = fmaxf(mloc, ms);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
  if (lane == 0) red[warp] = mloc;
  __syncthreads();
  const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float lloc = 0.f;
  for (int s = threadIdx.x; s < n_splits; s += blockDim.x) {
    const float f = m_s[s] == -INFINITY ? 0.f : exp2f(m_s[s] - M);
    f_s[s] = f;
    lloc += l_s[s] * f;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) lloc += __shfl_xor_sync(0xffffffffu, lloc, o);
  if (lane == 0) red[warp] = lloc;
  __syncthreads();
  const float L = (red[0] + red[1]) + (red[2] + red[3]);
  const float inv = L > 0.f ? 1.f / L : 0.f;
  T* out = (T*)a.out + ((int64_t)b * a.T * a.H + h) * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float o = 0.f;
    for (int s0 = 0; s0 < n_splits; s0 += RO) {
      float x[RO];
      if (s0 == 0 && d == (int)threadIdx.x) {
#pragma unroll
        for (int u = 0; u < RO; ++u) x[u] = x0[u];
      } else {
#pragma unroll
        for (int u = 0; u < RO; ++u) x[u] = s0 + u < n_splits ? __ldcg(p + (size_t)(s0 + u) * (D + 2) + d) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < RO; ++u)
        if (s0 + u < n_splits) o = fmaf(x[u], f_s[s0 + u], o);
    }
    out[d] = from_f<T>(o * inv);
  }
  if (threadIdx.x == 0 && a.lse) a.lse[(int64_t)bh * a.T] = (M + log2f(L)) * 0.6931471805599453f;
}

template <typename T, int EPL, int DPL>
cudaError_t launch_t(const AttnArgs& a, int n_splits, float* part, const DecodeAppend& ap, cudaStream_t st) {
  // programmatic stream serialisation: consecutive tokens' launches overlap their set-up with the
  // previous token's tail (the kernel waits on griddepcontrol before its first dependent access)
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(n_splits, a.B * a.H);
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_split_kernel<T, EPL, DPL>, a, part, n_splits, ap);
}

template <typename T>
cudaError_t launch_dt(const AttnArgs& a, int n_splits, float* part, const DecodeAppend& ap, cudaStream_t st) {
  const int epl = a.E / 32, dpl = a.D / 32;
#define THIN_DECODE_CASE(X, Y) \
  if (epl == X && dpl == Y) return launch_t<T, X, Y>(a, n_splits, part, ap, st);
  THIN_DECODE_CASE(2, 2)
  THIN_DECODE_CASE(2, 4)
  THIN_DECODE_CASE(2, 8)
  THIN_DECODE_CASE(4, 2)
  THIN_DECODE_CASE(4, 4)
  THIN_DECODE_CASE(4, 8)
#undef THIN_DECODE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

bool decode_attention_supported(int E, int D, int max_segments, int max_splits) {
  const bool ok_e = E == 64 || E == 128, ok_d = D == 64 || D == 128 || D == 256;
  return ok_e && ok_d && max_segments <= 32 && max_splits <= kDecodeMaxSplits;
}

int decode_chunk_keys() { return kDecodeChunk; }

cudaError_t launch_decode_attention(const AttnArgs& a, int dtype, int n_splits, float* part, const DecodeAppend& ap,
                                    cudaStream_t st) {
  if (a.B * a.H == 0 || n_splits <= 0) return cudaSuccess;
  return dtype == 0 ? launch_dt<float>(a, n_splits, part, ap, st) : launch_dt<__nv_bfloat16>(a, n_splits, part, ap, st);
}

}  // namespace thin
