// Kernel Halving without device allocation.
//
// thin_attn_halve_noalloc halves caller-provided point sets with the same three kernels as a
// halving step of thin_attn_forward (c^2 pass, pair-difference Gram, walk + gather).  The
// scratch those kernels need -- the instance table, the point-index table, c^2 per instance
// and the pair-difference matrices -- lives in one file-scope __device__ array of
// kHalveScratchBytes, which every device that loads this library keeps until the process
// exits.  Nothing here calls cudaMalloc, cudaFree or an allocating library routine.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "thin_attn.h"

namespace thin {
int record_error(int s, const char* msg);
}

namespace {

using namespace thin;

constexpr size_t kHalveScratchBytes = (size_t)16 << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_halve_scratch[kHalveScratchBytes];

// Device address of g_halve_scratch per device ordinal (host code must not use the symbol
// itself: on the host it is only a stand-in, not a device address).
constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

thin_attn_status err(thin_attn_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  return (thin_attn_status)record_error((int)s, buf);
}

// Set-up, once per device, with that device current.
thin_attn_status scratch_address(int dev, unsigned char** out) {
  if (dev < 0 || dev >= kMaxDevices) return err(THIN_ATTN_EUNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_halve_scratch);
    if (e != cudaSuccess || !p)
      return err(THIN_ATTN_ECUDA, "cudaGetSymbolAddress of the halving scratch: %s", cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = (unsigned char*)g_scratch_addr[dev];
  return THIN_ATTN_OK;
}

// Instance i: points rows [i n, (i+1) n) of K/V, survivors rows [i m, (i+1) m); Philox counter
// (pair, round_id, i, 0); the point index table holds the position of a row within its set.
__global__ void fill_noalloc_tables(HalveInst* inst, int32_t* pidx, int n_inst, int n, int m, uint32_t round_id) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t i = t0; i < n_inst; i += stride) {
    HalveInst h{};
    h.src_row = i * n;
    h.dst_row = i * m;
    h.bh = (uint32_t)i;
    h.ctr_bh = (uint32_t)i;
    h.round_id = round_id;
    inst[i] = h;
  }
  for (int64_t r = t0; r < (int64_t)n_inst * n; r += stride) pidx[r] = (int32_t)(r % n);
}

}  // namespace

extern "C" THIN_ATTN_API thin_attn_status thin_attn_halve_noalloc(int dtype, const void* K, const void* V,
                                                                 int n_inst, int n, int E, int D, float scale,
                                                                 uint64_t seed, uint32_t round_id, void* K_out,
                                                                 void* V_out, int32_t* idx_out,
                                                                 uint32_t* keep_bits_opt, void* stream) {
  if (dtype != THIN_ATTN_FP32 && dtype != THIN_ATTN_BF16) return err(THIN_ATTN_EINVAL, "dtype %d", dtype);
  if (!K || !V || !K_out || !V_out || !idx_out) return err(THIN_ATTN_EINVAL, "null tensor pointer");
  if (n_inst < 1 || n < 2 || n % 2 || n > 4096)
    return err(THIN_ATTN_EINVAL, "n_inst=%d n=%d: need n_inst >= 1 and an even n in [2, 4096]", n_inst, n);
  if (E < 8 || E > 256 || E % 8 || D < 8 || D > 256 || D % 8)
    return err(THIN_ATTN_EINVAL, "E=%d D=%d: widths must be multiples of 8 in [8, 256]", E, D);
  for (const void* p : {K, V, (const void*)K_out, (const void*)V_out})
    if ((uintptr_t)p % 16) return err(THIN_ATTN_EINVAL, "tensor pointers must be 16-byte aligned");
  const int m = n / 2, m_pad = (m + 31) / 32 * 32;
  const size_t off_idx = al256((size_t)n_inst * sizeof(HalveInst));
  const size_t off_c2 = off_idx + al256((size_t)n_inst * n * 4);
  const size_t off_delta = off_c2 + al256((size_t)n_inst * 4);
  const size_t need = off_delta + (size_t)n_inst * m_pad * m_pad * 4;
  if (need > kHalveScratchBytes)
    return err(THIN_ATTN_EINVAL, "%d sets of %d points need %zu bytes of scratch; the maximum is %zu", n_inst, n,
               need, kHalveScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return err(THIN_ATTN_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  unsigned char* scratch = nullptr;
  thin_attn_status s = scratch_address(dev, &scratch);
  if (s != THIN_ATTN_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  HalveInst* inst = (HalveInst*)scratch;
  int32_t* pidx = (int32_t*)(scratch + off_idx);
  const int64_t work = std::max<int64_t>(n_inst, (int64_t)n_inst * n);
  fill_noalloc_tables<<<(unsigned)std::min<int64_t>((work + 255) / 256, 4096), 256, 0, st>>>(inst, pidx, n_inst, n, m,
                                                                                            round_id);
  StepArgs a{};
  a.src_kind = SRC_COMPACT;
  a.srcK = K;
  a.srcV = V;
  a.srcIdx = pidx;
  a.H = 1;
  a.src_rows = (int64_t)n_inst * n;
  a.S_full = a.S_sub = n;
  a.dstK = K_out;
  a.dstV = V_out;
  a.dstIdx = idx_out;
  a.inst = inst;
  a.n_inst = n_inst;
  a.n = n;
  a.m = m;
  a.m_pad = m_pad;
  a.E = E;
  a.D = D;
  const float sc = scale > 0.f ? scale : (float)(1.0 / std::sqrt((double)E));
  a.scale_log2e = (float)((double)sc * 1.4426950408889634);
  a.C = (float)std::sqrt(2.0 * std::log(4.0 * m));
  a.seed = seed;
  a.c2 = (float*)(scratch + off_c2);
  a.delta = (float*)(scratch + off_delta);
  a.trace = keep_bits_opt;
  a.trace_base = 0;
  e = launch_halving_step(a, dtype, true, st);
  if (e != cudaSuccess) return err(THIN_ATTN_ECUDA, "halving: %s", cudaGetErrorString(e));
  return THIN_ATTN_OK;
}
