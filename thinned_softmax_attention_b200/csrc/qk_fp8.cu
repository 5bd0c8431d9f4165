// e4m3 copies of q, k and the compact key rows for the FP8 QK^T of the attention kernel.
//
// One scale per (b,h) slice and tensor: the slice's largest |x| maps to 448, the largest e4m3
// value, so every element rounds (to nearest even, saturating) into range.  Three passes, each a
// streaming read of bf16 rows in 16-byte vectors (8 elements, one head's consecutive columns):
// the per-(b,h) maxima of q and of k, the scales, then the conversions.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace thin {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerBlock = 32;
constexpr int kMaxVecPerThread = 8;   // H E / 8 <= 8 * 256

__device__ __forceinline__ float absmax8(uint4 w) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(__uint_as_float(ws[e] << 16)), fabsf(__uint_as_float(ws[e] & 0xFFFF0000u))));
  return m;
}

// grid (ceil(Lr / kRowsPerBlock), B, 2): z = 0 q (Lr = T), z = 1 k (Lr = L).  Thread t owns the
// 16-byte vectors t, t + 256, ... of every row of its block (fixed heads); groups of E / 8
// neighbouring threads share a head and combine their maxima before one atomic per group.
__global__ void __launch_bounds__(kThreads) qk_amax_kernel(QkFp8Args a) {
  const int z = blockIdx.z, b = blockIdx.y;
  const int Lr = z ? a.L : a.T;
  const uint4* src = (const uint4*)(z ? a.k : a.q);
  const int vpr = a.H * a.E / 8;                 // vectors per row
  const int r0 = blockIdx.x * kRowsPerBlock, r1 = min(Lr, r0 + kRowsPerBlock);
  float m[kMaxVecPerThread];
#pragma unroll
  for (int j = 0; j < kMaxVecPerThread; ++j) m[j] = 0.f;
  for (int r = r0; r < r1; ++r) {
    const uint4* row = src + ((int64_t)b * Lr + r) * vpr;
#pragma unroll
    for (int j = 0; j < kMaxVecPerThread; ++j) {
      const int v = threadIdx.x + j * kThreads;
      if (v < vpr) m[j] = fmaxf(m[j], absmax8(row[v]));
    }
  }
  const int g = a.E / 8;                         // threads per head (8 or 16 or 32): power of two
#pragma unroll
  for (int j = 0; j < kMaxVecPerThread; ++j) {
    const int v = threadIdx.x + j * kThreads;
    float x = m[j];
    for (int o = g >> 1; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    if (v < vpr && (threadIdx.x & (g - 1)) == 0)
      atomicMax(a.amax + z * a.B * a.H + b * a.H + v * 8 / a.E, __float_as_uint(x));
  }
}

__global__ void qk_scales_kernel(QkFp8Args a) {
  const int BH = a.B * a.H;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < BH; i += gridDim.x * blockDim.x) {
    const float mq = __uint_as_float(a.amax[i]), mk = __uint_as_float(a.amax[BH + i]);
    const float sq = mq > 0.f ? 448.f / mq : 1.f, sk = mk > 0.f ? 448.f / mk : 1.f;
    a.scales[i] = sq;
    a.scales[BH + i] = sk;
    a.qk_inv[i] = 1.f / (sq * sk);
  }
}

__device__ __forceinline__ uint2 to_e4m3x8(uint4 w, float s) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t r = 0;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const uint32_t x = ws[2 * h + e];
      const float2 f = make_float2(__uint_as_float(x << 16) * s, __uint_as_float(x & 0xFFFF0000u) * s);
      const __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
      r |= (uint32_t)p << (16 * e);
    }
    out[h] = r;
  }
  return make_uint2(out[0], out[1]);
}

// Token rows: grid-stride over the 16-byte vectors of q (z = 0) or k (z = 1).
__global__ void __launch_bounds__(kThreads) qk_quant_kernel(QkFp8Args a) {
  const int z = blockIdx.y;
  const int Lr = z ? a.L : a.T;
  const uint4* src = (const uint4*)(z ? a.k : a.q);
  uint2* dst = (uint2*)(z ? a.k8 : a.q8);
  const float* sc = a.scales + z * a.B * a.H;
  const int vph = a.E / 8, vpr = a.H * vph;
  const int64_t n = (int64_t)a.B * Lr * vpr;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kThreads) {
    const int64_t row = i / vpr;
    const int h = (int)(i % vpr) / vph;
    const int b = (int)(row / Lr);
    dst[i] = to_e4m3x8(src[i], sc[b * a.H + h]);
  }
}

// Compact key rows: (b,h) = row / rows_per_bh.
__global__ void __launch_bounds__(kThreads) ck_quant_kernel(QkFp8Args a) {
  const uint4* src = (const uint4*)a.ck;
  uint2* dst = (uint2*)a.ck8;
  const float* sc = a.scales + a.B * a.H;
  const int vpr = a.E / 8;
  const int64_t n = a.ck_rows * vpr;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kThreads)
    dst[i] = to_e4m3x8(src[i], sc[(i / vpr) / a.rows_per_bh]);
}

}  // namespace

bool qk_fp8_supported(int H, int E) {
  return E % 8 == 0 && E / 8 <= 32 && ((E / 8) & (E / 8 - 1)) == 0 && H * E / 8 <= kMaxVecPerThread * kThreads;
}

cudaError_t launch_qk_fp8(const QkFp8Args& a, cudaStream_t st) {
  if (!qk_fp8_supported(a.H, a.E)) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(a.amax, 0, sizeof(unsigned) * 2 * a.B * a.H, st);
  if (e != cudaSuccess) return e;
  const int Lmax = std::max(a.T, a.L);
  qk_amax_kernel<<<dim3((Lmax + kRowsPerBlock - 1) / kRowsPerBlock, a.B, 2), kThreads, 0, st>>>(a);
  qk_scales_kernel<<<(a.B * a.H + 255) / 256, 256, 0, st>>>(a);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  qk_quant_kernel<<<dim3(sms * 8, 2), kThreads, 0, st>>>(a);
  if (a.ck && a.ck_rows > 0) ck_quant_kernel<<<sms * 4, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace thin
