// Shared definitions of the thin_attn CUDA library (device structs, Philox, element access).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace thin {

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC'11).  Counter (pair, round id, b*H+h, 0), key = seed.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ uint32_t mulhi32(uint32_t a, uint32_t b) {
#ifdef __CUDA_ARCH__
  return __umulhi(a, b);
#else
  return (uint32_t)(((uint64_t)a * b) >> 32);
#endif
}

__host__ __device__ __forceinline__ uint32_t philox_x0(uint64_t seed, uint32_t bh, uint32_t round_id,
                                                        uint32_t pair) {
  uint32_t c0 = pair, c1 = round_id, c2 = bh, c3 = 0;
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c0, hi0 = mulhi32(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = mulhi32(0xCD9E8D57u, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return c0;
}

// u = ((x0 >> 9) + 1/2) 2^-23: an odd multiple of 2^-24 in (0,1), exact in fp32.
__host__ __device__ __forceinline__ float philox_uniform(uint64_t seed, uint32_t bh, uint32_t round_id,
                                                         uint32_t pair) {
  return ((float)(philox_x0(seed, bh, round_id, pair) >> 9) + 0.5f) * (1.0f / 8388608.0f);
}

// ---------------------------------------------------------------------------
// Element access
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------------------
// Halving steps.  One step = one launch group (max|v| pass, pair-difference
// Gram, walk + gather) over n_inst independent instances of n points each.
// ---------------------------------------------------------------------------
enum SrcKind : int { SRC_TOKENS = 0, SRC_COMPACT = 1 };

struct HalveInst {
  int64_t src_row;     // SRC_TOKENS: b*L_seq + tok0 ; SRC_COMPACT: first source row
  int64_t dst_row;     // first destination row (compact buffer)
  uint32_t bh;         // b*H + h
  uint32_t round_id;   // Philox round id
  uint32_t pair0;      // Philox pair index of pair 0
  uint32_t sub_round;  // Philox round of the subsample word (SRC_TOKENS with S_sub < S_full)
  uint32_t tok0;       // SRC_TOKENS: token index of the run start (stored in idx)
  uint32_t ctr_bh;     // (b,h) word of the Philox counter: (b0 + b) * H_total + h0 + h of the whole problem
};

struct StepArgs {
  // source
  int src_kind;
  const void* srcK;        // SRC_TOKENS: k (B,L,H,E); SRC_COMPACT: (rows, E)
  const void* srcV;
  const int32_t* srcIdx;   // SRC_COMPACT only
  int H;                   // heads (SRC_TOKENS row addressing)
  int64_t src_rows;        // rows of the source: B*L (SRC_TOKENS) or compact rows; 0 = unknown
  int S_full, S_sub;       // SRC_TOKENS subsample: token = floor((p*S_full + U)/S_sub)
  int sub_stride;          // k = S_full / S_sub when that is an integer and every run starts on a multiple
                           // of k: the subsample is then tokens 0, k, 2k, ... (U < S_sub drops out), a
                           // strided box for TMA; 0 otherwise
  // destination
  void* dstK;
  void* dstV;
  int32_t* dstIdx;
  // instances
  const HalveInst* inst;
  int n_inst;
  int n;                   // points per instance
  int m;                   // pairs per instance
  int m_pad;               // m rounded up to 32 (row stride of the pair-difference matrix)
  int E, D;
  float scale_log2e;       // s * log2(e)
  float C;                 // sqrt(2 ln(2/delta_i)), delta_i = 1/(2m)
  uint64_t seed;
  // scratch
  float* c2;               // (n_inst) squared max |v|
  float* delta;            // (n_inst, m_pad, m_pad)
  int* status;             // device status word for bounded waits (may be null)
  // trace (may be null)
  uint32_t* trace;
  uint64_t trace_base;     // first word of this step
};

// Subsample word U of an instance (0 when no subsample).
__device__ __forceinline__ uint32_t sub_offset(const StepArgs& a, const HalveInst& in) {
  if (a.src_kind != SRC_TOKENS || a.S_sub >= a.S_full) return 0u;
  return philox_x0(a.seed, in.ctr_bh, in.sub_round, 0u) % (uint32_t)a.S_sub;
}

// Row of point p (0..n-1) of an instance: element offset of its K row, V row, and its token index.
struct PointRef {
  int64_t krow;    // element offset into srcK
  int64_t vrow;    // element offset into srcV
  int32_t idx;     // token index
};

__device__ __forceinline__ PointRef point_ref(const StepArgs& a, const HalveInst& in, int p, uint32_t U) {
  PointRef r;
  if (a.src_kind == SRC_TOKENS) {
    const int64_t gp = 2 * (int64_t)in.pair0 + p;  // point index within the (sub)sampled run
    const int64_t t = (a.S_sub < a.S_full) ? (gp * a.S_full + U) / a.S_sub : gp;
    const int h = (int)(in.bh % (uint32_t)a.H);
    const int64_t row = (in.src_row + t) * a.H + h;
    r.krow = row * a.E;
    r.vrow = row * a.D;
    r.idx = (int32_t)(in.tok0 + t);
  } else {
    const int64_t row = in.src_row + p;
    r.krow = row * a.E;
    r.vrow = row * a.D;
    r.idx = a.srcIdx[row];
  }
  return r;
}

// Element offsets of the K and V rows of point p (no token-index lookup).
__device__ __forceinline__ void point_rows(const StepArgs& a, const HalveInst& in, int p, uint32_t U, int64_t* krow,
                                           int64_t* vrow) {
  int64_t row;
  if (a.src_kind == SRC_TOKENS) {
    const int64_t gp = 2 * (int64_t)in.pair0 + p;
    const int64_t t = (a.S_sub < a.S_full) ? (gp * a.S_full + U) / a.S_sub : gp;
    row = (in.src_row + t) * a.H + (int)(in.bh % (uint32_t)a.H);
  } else {
    row = in.src_row + p;
  }
  *krow = row * a.E;
  *vrow = row * a.D;
}

// ---------------------------------------------------------------------------
// Attention over key segments.
// ---------------------------------------------------------------------------
enum SegKind : int { SEG_TOKENS = 0, SEG_COMPACT = 1 };

struct AttnSeg {
  int kind;      // SEG_TOKENS: tokens [first, first+len) of this (b,h) in k/v
                 // SEG_COMPACT: rows (bh*n_slots + first)*slot_rows + [0, len) of the compact buffers
  int first;
  int len;
  int causal;    // SEG_TOKENS only: key token j visible to query t iff j <= t
  float logw;    // ln of the weight of every key of the segment
  int pad;
};

struct AttnTile {
  int q0;        // first query token
  int qlen;      // queries in the tile
  int seg0;      // first segment in the segment table
  int nseg;
  int nkt = 0;   // 128-key tiles over its segments (sum of ceil(len / 128)), filled by the host before upload
};

struct AttnArgs {
  const void* q;        // (B,T,H,E)
  const void* k;        // (B,L,H,E) original keys (L = S non-causal, T causal)
  const void* v;        // (B,L,H,D)
  const void* ck;       // compact keys (rows, E)
  const void* cv;       // compact values (rows, D)
  void* out;            // (B,T,H,D)
  float* lse;           // (B,H,T) or null
  const AttnTile* tiles;
  const AttnSeg* segs;
  int tile0;            // first tile of this launch
  int n_tiles;          // tiles of this launch
  int B, T, L, H, E, D;
  int n_slots, slot_rows;
  float scale_log2e;
  int inject_timeout;   // test hook: CTA (0,0) withholds its first key tile so a bounded wait runs out
  // tile pairs of the ping-pong kernel: (x, y) = tiles A and B, A's key tiles the first ones of B's
  // (x = -1: B alone); pairs [pair0, pair0 + n_pairs) of the table.  Null: no pairs.
  const int2* pairs;
  int pair0, n_pairs;
  // e4m3 QK^T (null: bf16): q8, k8 and ck8 hold q, k and the compact keys times the (b,h) scales,
  // rounded to e4m3 (same layouts, one byte per element); qk_inv[bh] = 1 / (scale_q * scale_k)
  const void* q8;
  const void* k8;
  const void* ck8;
  const float* qk_inv;
};

}  // namespace thin
