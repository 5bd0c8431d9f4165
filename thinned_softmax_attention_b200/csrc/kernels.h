// Kernel launchers of the thin_attn library (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace thin {

// Halving step (c^2, pair-difference Gram, walk + gather).  dtype 0 = fp32, 1 = bf16.
cudaError_t launch_halving_step(const StepArgs& a, int dtype, bool use_tc, cudaStream_t st);
// Tensor-core pair-difference Gram (bf16, E and D multiples of 64); *done = false when the
// shape is not covered and the CUDA-core kernel must run instead.
cudaError_t launch_pairgram_tc(const StepArgs& a, cudaStream_t st, bool* done);
// One-launch halving of instances of <= 128 points (bf16, E and D multiples of 64, E + D <= 320,
// rows that form TMA boxes): c^2, Gram, walk and gather fused, the points read once.
bool halving_fused_supported(const StepArgs& a);
cudaError_t launch_halving_fused(const StepArgs& a, cudaStream_t st);
// Several halving steps of 129..512-point instances in one persistent launch, each work item (step,
// instance) waiting for the items it depends on.  Tables in device memory, built by the host:
struct SchedTables {
  const int2* items;      // (step, instance) in queue order (a topological order of the dependencies)
  const int* pred_off;    // predecessors of item i: preds[pred_off[i] .. pred_off[i + 1]) (item indices)
  const int* preds;
  int n_items;
  int* done;              // per item: completion epoch (zeroed once; never equal to a live epoch before)
  int epoch;              // this launch's epoch (>= 1, different from every earlier launch's)
  int* sched;             // two ints: work counter and exit count, zero between launches
  int* status;            // the handle's status word (code 7: a dependency wait gave up, [1] = item)
  int inject_item;        // test hook: item whose wait runs out (-1: none)
};
bool halving_sched_shape_ok(const StepArgs& a);         // the plan's choice (shapes only)
bool halving_sched_step_supported(const StepArgs& a);   // the launch's (and the driver's TMA, the environment)
int halving_sched_max_steps();
cudaError_t launch_halving_sched(const StepArgs* steps, int n_steps, const SchedTables& t, cudaStream_t st);
// Copy of token runs into compact rows (batches that are not thinned).
cudaError_t launch_copy_step(const StepArgs& a, int dtype, cudaStream_t st);
cudaError_t launch_iota(int32_t* idx, int64_t rows, int period, cudaStream_t st);
size_t walk_smem_bytes(int m_pad);

// Attention over key segments.
cudaError_t launch_attention_simt(const AttnArgs& a, int dtype, cudaStream_t st);
int attention_simt_tile_rows();
// Tensor-core attention (bf16, E = D = 128); *done = false when the shape is not covered.
// Device status buffer of a handle (zeroed at creation): ints [0..3] the status word (code and
// detail of a bounded wait that gave up), [4..5] the work counter of the persistent attention
// kernels, [6..7] that of the halving scheduler (each left at zero by every launch).
constexpr size_t kStatusBytes = 32;

cudaError_t launch_attention_tc(const AttnArgs& a, int* status_word, cudaStream_t st, bool* done);
int attention_tc_tile_rows();
bool attention_tc_supported(int dtype, int E, int D);

// Split-key attention of one query per (b,h) (decode): n_splits chunks of decode_chunk_keys() keys
// of the tile a.tile0, partials (m, l, o) in `part` (n_splits x B*H x (D + 2) floats), merged into
// out and lse by the last chunk of each (b,h) to finish (one launch).
// With new_k set, the last key of the tile is the token being decoded: it is read from new_k / new_v
// (batch entry b a.T token rows after entry 0, like q and out; lse of (b,h) i at a.lse[i a.T]) and
// then written to row `row` of every (b,h) of a.k / a.v.
struct DecodeAppend {
  const void* new_k = nullptr;
  const void* new_v = nullptr;
  int row = 0;
  int* arrive = nullptr;   // B*H arrival counters of the chunks, zero between launches (required)
  // the tile's segments, copied from the host's tables into the launch (saves two dependent loads at
  // the head of a token's latency chain); nseg = -1: read a.tiles / a.segs instead
  int nseg = -1;
  AttnSeg segs[32];
};
bool decode_attention_supported(int E, int D, int max_segments, int max_splits);
int decode_chunk_keys();
cudaError_t launch_decode_attention(const AttnArgs& a, int dtype, int n_splits, float* part, const DecodeAppend& ap,
                                    cudaStream_t st);

// bf16 TMA tensor maps with 128-byte swizzle and (64 elements x box_rows) boxes:
// 2D over `rows` rows of `width` elements, rows `row_stride` elements apart;
// 3D over a (B*L, H, width) view of a (B, L, H, width) tensor, one head per box.
bool tensor_maps_available();
bool make_map_2d(CUtensorMap* m, const void* base, int64_t rows, int width, int64_t row_stride, int box_rows);
bool make_map_3d(CUtensorMap* m, const void* base, int64_t BL, int H, int width, int box_rows);
// 4D view over every k-th row (a systematic subsample with integer ratio k): box (64, 1, 1, box_rows)
// at (x, h, 0, R) holds rows R k, (R+1) k, ...
bool make_map_4d_strided(CUtensorMap* m, const void* base, int64_t BL, int H, int width, int k, int box_rows);
// The same 2D / 3D maps over one-byte (e4m3) elements, boxes of 128 elements.
bool make_map_2d_u8(CUtensorMap* m, const void* base, int64_t rows, int width, int64_t row_stride, int box_rows);
bool make_map_3d_u8(CUtensorMap* m, const void* base, int64_t BL, int H, int width, int box_rows);

// e4m3 copies for QK^T (thin_attn_config::qk_fp8).  Per (b,h): scale_q = 448 / max|q| over its T
// rows, scale_k = 448 / max|k| over its L token rows (1 when the maximum is 0); q8 = e4m3(q scale_q),
// k8 = e4m3(k scale_k), ck8 = e4m3(ck scale_k) for the compact key rows (rows_per_bh rows per (b,h));
// qk_inv[bh] = 1 / (scale_q scale_k).  `amax` (2 B H words) is cleared here.  bf16 inputs, E a
// multiple of 8 and H E / 8 <= 2048.
struct QkFp8Args {
  const void* q;
  const void* k;
  const void* ck;          // may be null (no compact rows)
  int B, T, L, H, E;
  int64_t ck_rows, rows_per_bh;
  uint8_t* q8;
  uint8_t* k8;
  uint8_t* ck8;
  unsigned* amax;          // [2][B H] scratch
  float* scales;           // [2][B H]: scale_q, scale_k
  float* qk_inv;           // [B H]
};
bool qk_fp8_supported(int H, int E);
cudaError_t launch_qk_fp8(const QkFp8Args& a, cudaStream_t st);

}  // namespace thin
