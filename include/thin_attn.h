/*
 * thin_attn -- Thinformer and Thinformer Express attention on NVIDIA B200 (sm_100a).
 *
 * C ABI of the library.  Every entry point takes plain pointers and sizes; no
 * framework types cross this boundary.
 *
 * The operation (Thinformer README, "Getting Started"; "Express Language
 * Modeling" summary, Methodology):
 *   non-causal  out = attention of every query against a kernel-halving coreset
 *               C of the S key/value pairs of its (b,h), each coreset point
 *               weighted S/|C|  ("Thinformer" for unmasked attention);
 *   causal      Thinformer Express prefill: an exact phase of n_exact tokens,
 *               then batches of `batch` tokens thinned to coresets as they
 *               complete, then HALVE merges of four equal-level coresets into
 *               one of four times the weight.
 *
 * Tensor layouts (README, "Getting Started"), all row-major and contiguous:
 *   q   (B, T, H, E)        k (B, S, H, E)        v (B, S, H, D)
 *   out (B, T, H, D)        lse (B, H, T) fp32    (causal: S = T)
 * q, k, v and out share the handle's element type (fp32 or bf16).
 *
 * Ownership: the caller owns every tensor it passes; the library never frees
 * caller memory.  A handle owns its device workspace (allocated on first use
 * of a (causal, g) plan, or by thin_attn_reserve) and releases it in
 * thin_attn_destroy.
 *
 * Execution: device entry points enqueue kernels on the caller's stream and
 * return without synchronising.  The host-buffer entry point synchronises.
 * A handle's forwards share its workspace (and the work counter of its
 * attention kernel), so they must not overlap on the GPU: issue them on one
 * stream, or order the streams; use one handle per concurrent stream.
 *
 * Errors: every entry point returns a thin_attn_status; on failure the
 * calling thread's message is available from thin_attn_last_error().  Invalid
 * arguments are rejected on the host before anything is enqueued.
 */
#ifndef THIN_ATTN_H_
#define THIN_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define THIN_ATTN_API __attribute__((visibility("default")))
#else
#define THIN_ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct thin_attn_s* thin_attn_t;

typedef enum {
  THIN_ATTN_OK = 0,
  THIN_ATTN_EINVAL = 1,        /* bad argument: null pointer, shape, g out of range */
  THIN_ATTN_ENOMEM = 2,        /* device or host allocation failed */
  THIN_ATTN_ECUDA = 3,         /* a CUDA call failed (message holds the CUDA error) */
  THIN_ATTN_ETIMEOUT = 4,      /* a bounded device-side wait gave up */
  THIN_ATTN_EUNSUPPORTED = 5   /* valid request outside what this library implements */
} thin_attn_status;

typedef enum { THIN_ATTN_FP32 = 0, THIN_ATTN_BF16 = 1 } thin_attn_dtype;

typedef struct {
  int dtype;       /* thin_attn_dtype of q, k, v, out */
  int B, T, S, H;  /* batch, queries, keys (ignored when causal: S = T), heads */
  int E, D;        /* key/query width, value width: multiples of 8, E <= 256, D <= 256 */
  float scale;     /* softmax scale s; <= 0 selects 1/sqrt(E) */
  int n_exact;     /* Express exact phase length (causal only) */
  int batch;       /* Express thin batch length (causal only; > 0) */
  int device;      /* CUDA device ordinal the handle's memory lives on */
  /* Shard of a larger problem (batch- or head-parallel runs, one handle per GPU).  The Philox
   * counter of (b,h) is keyed on the whole problem's (b0 + b) * H_total + h0 + h, so the decisions,
   * coresets and outputs of a shard equal those of the whole problem's run for its (b,h).  Zero
   * gives the unsharded problem.  EINVAL when b0 < 0, h0 < 0, h0 + H > H_total or
   * (b0 + B) * H_total >= 2^32. */
  int b0;          /* whole-problem index of this handle's batch row 0 */
  int h0;          /* whole-problem index of this handle's head 0 */
  int H_total;     /* heads of the whole problem; <= 0 selects H */
  /* QK^T in e4m3 (FP8; "Express Language Modeling", Limitations, lists FP8 as unexploited): 0 keeps
   * bf16.  1: after the thinning, q, k and the coreset keys are copied to e4m3 with one scale per
   * (b,h) and tensor (its largest |x| maps to 448), S = q8 k8^T on the tensor cores' e4m3 path and
   * the scales undone in the softmax; P V stays bf16.  The thinning always uses the bf16 keys.  bf16
   * handles with E = 128, D <= 128, H <= 128; EUNSUPPORTED otherwise.  The decode cache ignores it. */
  int qk_fp8;
  /* Query-row shard: attend only the query rows [q_begin, q_end) of every (b,h).  The thinning still
   * runs over all keys, so these rows come out bit-identical to the whole run's, and the rows of out
   * and lse outside the range are not written: ranks holding disjoint ranges of one sequence need
   * no communication (sequence parallelism when B*H is below the GPU count).  Both zero: every row.
   * EINVAL unless 0 <= q_begin < q_end <= T, q_begin a multiple of 128 and q_end a multiple of 128
   * or T.  thin_attn_forward_host and the decode cache take no range (EUNSUPPORTED / EINVAL). */
  int q_begin;
  int q_end;
  /* Express sequence shards with the thinning split too (causal = 1 only): with thin_split = 1 the
   * handle thins only the batches it owns -- batch k is owned by the range [q_begin, q_end) that
   * holds its last token ("Express Language Modeling", The EXPRESS Meta-Procedure: batches are
   * thinned independently) -- and the other batches' coresets come from the ranks that own them.
   * A forward then runs in two calls of thin_attn_forward_phase: phase 1 thins the owned batches;
   * the caller exchanges the batch coresets (thin_attn_nodes_export on every rank, an all-gather,
   * thin_attn_nodes_import of the others' batches); phase 2 runs every HALVE merge and the
   * attention of the range.  Outputs equal the whole run's bit for bit.  0: thin every batch. */
  int thin_split;
} thin_attn_config;

/* Sizes of one (causal, g) plan. */
typedef struct {
  int levels;                  /* halving levels r of KH-Compress (per sequence or per batch) */
  int leaf;                    /* leaf size L (points per leaf run) */
  int subsampled;              /* S' = L 4^r points kept by the systematic subsample */
  int coreset_rows;            /* non-causal: |C| per (b,h); causal: c per node */
  int n_batches;               /* causal: completed thin batches n_b */
  int n_nodes;                 /* causal: node slots (level-0 nodes, then level 1, ...) */
  int n_halvings;              /* halving instances (entries of the trace layout) */
  int kernel_launches;         /* kernels one forward launches (without the optional outputs) */
  uint64_t trace_words;        /* uint32 words of the decision trace */
  uint64_t coreset_idx_elems;  /* int32 elements of coreset_idx_opt */
  uint64_t workspace_bytes;    /* device workspace the plan needs */
  int attn_rows;               /* query rows of each (b,h) the attention writes (T, or q_end - q_begin) */
} thin_attn_plan_info;

/* Where the decisions of one halving instance sit in the trace. */
typedef struct {
  uint32_t bh;           /* b * H + h */
  uint32_t round_id;     /* Philox round identifier of the halving */
  uint32_t pair0;        /* Philox pair index of the instance's first pair */
  uint32_t n_pairs;      /* pairs m of the instance */
  uint64_t word_offset;  /* first uint32 word; bit i%32 of word i/32 = 1 iff pair i kept its first point */
} thin_attn_trace_entry;

/* Library version string. */
THIN_ATTN_API const char* thin_attn_version(void);

/* Message of the last failure on the calling thread ("" when none). */
THIN_ATTN_API const char* thin_attn_last_error(void);

/* Create a handle for one problem shape.  *out receives the handle. */
THIN_ATTN_API thin_attn_status thin_attn_create(thin_attn_t* out, const thin_attn_config* cfg);

/* Release the handle and its workspace.  Null is accepted. */
THIN_ATTN_API thin_attn_status thin_attn_destroy(thin_attn_t h);

/* Sizes of the (causal, g) plan; 0 <= g <= 6. */
THIN_ATTN_API thin_attn_status thin_attn_plan(thin_attn_t h, int causal, int g, thin_attn_plan_info* info);

/* One phase of a forward of a thin_split handle (see thin_attn_config::thin_split): phase 1 thins
 * the owned batches into their level-0 nodes; phase 2 runs the merges and the attention of the
 * query-row range and writes out, lse_opt, coreset_idx_opt (every node; valid once the other
 * ranks' batches have been imported) and trace_opt (this handle's halvings).  Arguments as for
 * thin_attn_forward.  EINVAL unless the handle has thin_split = 1, causal = 1 and phase is 1 or 2;
 * thin_attn_forward on such a handle is EINVAL. */
THIN_ATTN_API thin_attn_status thin_attn_forward_phase(thin_attn_t h, const void* q, const void* k, const void* v,
                                                       void* out, int causal, int g, uint64_t seed, float* lse_opt,
                                                       int32_t* coreset_idx_opt, uint32_t* trace_opt, int phase,
                                                       void* stream);

/* The batch coresets of a causal (Express, causal = 1) plan, for the exchange between thin_split
 * ranks.  *own_begin, *own_end: the batches this handle thins; *n_batches: all completed batches;
 * *bytes_per_batch: bytes of one batch's exchange block -- its level-0 node of every (b,h): keys
 * (B*H*c*E elements), values (B*H*c*D elements), then token indices (B*H*c int32), each (b,h)-major. */
THIN_ATTN_API thin_attn_status thin_attn_nodes_layout(thin_attn_t h, int causal, int g, int* own_begin, int* own_end,
                                                      int* n_batches, uint64_t* bytes_per_batch);
/* Copy the owned batches' blocks, in batch order, into dst (device memory, (own_end - own_begin) *
 * bytes_per_batch bytes, 16-byte aligned), on stream after the phase-1 work queued there. */
THIN_ATTN_API thin_attn_status thin_attn_nodes_export(thin_attn_t h, int causal, int g, void* dst, void* stream);
/* Write the blocks of batches [batch_begin, batch_end) from src (device memory, in batch order) into
 * this handle's level-0 nodes, on stream, before phase 2.  EINVAL for batches outside [0, n_batches). */
THIN_ATTN_API thin_attn_status thin_attn_nodes_import(thin_attn_t h, int causal, int g, const void* src,
                                                      int batch_begin, int batch_end, void* stream);

/* Allocate the workspace of the (causal, g) plan now (so the first forward allocates nothing). */
THIN_ATTN_API thin_attn_status thin_attn_reserve(thin_attn_t h, int causal, int g);

/* Copy the trace layout of the (causal, g) plan into entries[0 .. min(capacity, n)-1];
 * *count receives n (the number of halving instances). */
THIN_ATTN_API thin_attn_status thin_attn_trace_layout(thin_attn_t h, int causal, int g,
                                        thin_attn_trace_entry* entries, size_t capacity,
                                        size_t* count);

/*
 * Forward pass on device memory.
 *   q, k, v, out      device pointers in the layouts above
 *   causal            0: Thinformer; 1: Thinformer Express prefill (exact prefix of n_exact tokens,
 *                     batches of `batch` tokens, 4-ary counter of HALVE merges); 2: Thinformer
 *                     Express with the cache of "The EXPRESS Meta-Procedure" read literally: an exact
 *                     phase of n_out = n_exact tokens, batches of m n_out tokens thinned to n_out points
 *                     of weight m, the whole cache halved twice at 4 n_out with m <- 4m (`batch` unused)
 *   g                 oversampling parameter of KH-Compress, 0..6 (coreset ~ 2^g sqrt(S))
 *   seed              Philox key of the thinning decisions
 *   lse_opt           device (B,H,T) fp32 log-sum-exp ln sum_j w_j e^{s q.k_j}, or NULL
 *   coreset_idx_opt   device int32: non-causal (B,H,|C|) token indices of the coreset;
 *                     causal (B,H,n_nodes,c) token indices of every node; or NULL
 *   trace_opt         device uint32[trace_words] decision bits (thin_attn_trace_layout), or NULL
 *   stream            cudaStream_t to enqueue on (NULL = legacy default stream)
 * Allocates the plan's workspace on first use (not inside stream capture).
 * THIN_ATTN_EUNSUPPORTED when a halving instance would hold more than 4096 points: the last
 * KH-Compress level halves 2|C| points (2c per Express batch) and a HALVE merge 4c points.
 */
THIN_ATTN_API thin_attn_status thin_attn_forward(thin_attn_t h, const void* q, const void* k, const void* v,
                                   void* out, int causal, int g, uint64_t seed, float* lse_opt,
                                   int32_t* coreset_idx_opt, uint32_t* trace_opt, void* stream);

/*
 * Forward pass on host memory: copies q, k, v to device staging owned by the
 * handle, runs the forward, copies out (and lse when lse_opt is not NULL) back,
 * and synchronises `stream`.  Page-locked host buffers give asynchronous
 * copies; pageable ones work too.  When q, k and v hold 64 MB or more and H (or
 * else B) is a multiple of 4, the problem runs as eight (H or B a multiple of 8) or
 * four shards of its heads (or batch rows), each a handle with this one's random
 * stream (config b0/h0/H_total),
 * in a pipeline on internal streams ordered after `stream`: the copy-in of one
 * shard and the copy-out of another overlap the compute of a third.  Results
 * are those of one thin_attn_forward of the whole problem, bit for bit.
 * The staging belongs to the handle: run one host-buffer forward per handle at
 * a time (one handle per host thread).  Errors: THIN_ATTN_ENOMEM when the
 * staging cannot be allocated, the creation error of a shard handle, or
 * THIN_ATTN_ECUDA when a stream or event cannot be made; none of the pieces is
 * kept then, so a later call starts over.
 */
THIN_ATTN_API thin_attn_status thin_attn_forward_host(thin_attn_t h, const void* q, const void* k,
                                        const void* v, void* out, int causal, int g,
                                        uint64_t seed, float* lse_opt, void* stream);

/* Per-phase device timing: when enabled, every forward records CUDA events on its
 * stream between its phases (thinning of sequences or batches, HALVE merges,
 * attention).  No effect on results. */
THIN_ATTN_API thin_attn_status thin_attn_profile(thin_attn_t h, int enable);

/* Wait for the recorded forwards and return their summed times in milliseconds:
 * ms[0] thinning of sequences or batches, ms[1] HALVE merges, ms[2] attention (the
 * summed durations of its launches, which may overlap the halving steps), ms[3] the
 * whole forward; *calls = forwards recorded.  Resets the sums. */
THIN_ATTN_API thin_attn_status thin_attn_profile_read(thin_attn_t h, double* ms, int* calls);

/* The same recordings per halving step, in launch order: ms[i] the summed device time of step i
 * (from the end of the previous step, or the start of the forward, to its end), n_inst[i] its
 * instances and n_points[i] the points of each.  Up to max_steps entries are written;
 * *n_steps = steps of the most recently profiled plan (the sums restart when a forward of another
 * plan is recorded), *calls = forwards summed.  Steps that ran together in the persistent halving
 * launch (thin_attn_sched_layout) report its time on the first of them and 0 on the others.
 * Resets the step sums.  Both readers wait for the
 * recorded forwards; each returns and resets only its own sums, so each sees every forward. */
THIN_ATTN_API thin_attn_status thin_attn_profile_steps(thin_attn_t h, int max_steps, double* ms, int* n_inst,
                                                       int* n_points, int* n_steps, int* calls);

/* The halving steps of a plan that run as one persistent launch (the last thinning level of the
 * Express batches and the HALVE merges, or the last levels of a Thinformer compress): work item i
 * runs the halving of trace entry entry[i] (thin_attn_trace_layout's order) once the items
 * preds[pred_off[i] .. pred_off[i+1]) have finished (items are numbered in queue order; every
 * predecessor comes earlier).  Call with max_items = max_preds = 0 for the sizes (*n_items,
 * *n_preds); the arrays then need n_items, n_items + 1 and n_preds elements.  n_items = 0: the
 * plan runs every step as its own launch.  Host arrays; nothing is enqueued. */
THIN_ATTN_API thin_attn_status thin_attn_sched_layout(thin_attn_t h, int causal, int g, int32_t* entry,
                                                     int32_t* pred_off, int32_t* preds, size_t max_items,
                                                     size_t max_preds, size_t* n_items, size_t* n_preds);

/* Synchronise `stream` and report a device-side failure recorded by the
 * handle's kernels since the last call (THIN_ATTN_ETIMEOUT, ...). */
THIN_ATTN_API thin_attn_status thin_attn_check(thin_attn_t h, void* stream);

/*
 * Express decode cache -- the updatable weighted cache object of "The EXPRESS Meta-Procedure"
 * (Express Language Modeling).  One token of every (b,h) per call:
 *   thin_attn_cache_decode appends k_t, v_t, writes out_t = the attention of q_t against the
 *   cache (exact prefix, the coresets present after the completed batches, the tokens of the
 *   batch in progress), then -- when the token completes a batch -- KH-Compresses the batch into a
 *   level-0 coreset and runs the HALVE merges of the 4-ary counter.  Decisions use the same
 *   Philox rounds and pairs as thin_attn_forward(causal=1), so the coresets and out_t equal the
 *   prefill's row t (up to the attention kernel's rounding).
 * cfg: as for thin_attn_create with T = capacity in tokens (S ignored), n_exact, batch >= 1.
 * q, k, v, out: device (B,1,H,E), (B,1,H,E), (B,1,H,D), (B,1,H,D); lse_opt device (B,H) or NULL.
 * Raw keys/values are kept only for the exact prefix and the batch in progress; every coreset slot
 * of the capacity is allocated at creation (no allocation while decoding).
 */
typedef struct thin_attn_cache_s* thin_attn_cache_t;
THIN_ATTN_API thin_attn_status thin_attn_cache_create(thin_attn_cache_t* out, const thin_attn_config* cfg, int g,
                                                      uint64_t seed);
THIN_ATTN_API thin_attn_status thin_attn_cache_destroy(thin_attn_cache_t c);
/* Tokens decoded so far. */
THIN_ATTN_API thin_attn_status thin_attn_cache_length(thin_attn_cache_t c, int64_t* t);
THIN_ATTN_API thin_attn_status thin_attn_cache_decode(thin_attn_cache_t c, const void* q, const void* k,
                                                      const void* v, void* out, float* lse_opt, void* stream);
/* n consecutive tokens of every (b,h) in one call: q, k (B,n,H,E), v, out (B,n,H,D) device, lse_opt
 * (B,H,n) or NULL.  Token i attends to the cache after tokens 0..i-1 of the call, exactly as n calls
 * of thin_attn_cache_decode would (same kernels, bit-identical results), without a host round trip
 * per token.  EINVAL if the capacity would be exceeded; EUNSUPPORTED for n > 1 when B*H > 64 (the
 * query-tile decode path). */
THIN_ATTN_API thin_attn_status thin_attn_cache_decode_n(thin_attn_cache_t c, const void* q, const void* k,
                                                       const void* v, void* out, float* lse_opt, int n,
                                                       void* stream);
/* Device int32 (B,H,n_nodes,c) token indices of every coreset slot (-1 while empty), in the
 * node order of thin_attn_forward's coreset output. */
THIN_ATTN_API thin_attn_status thin_attn_cache_nodes(thin_attn_cache_t c, int32_t* idx_out, void* stream);

/* Synchronise `stream` and report a device-side failure of the cache's kernels. */
THIN_ATTN_API thin_attn_status thin_attn_cache_check(thin_attn_cache_t c, void* stream);

/*
 * Kernel Halving of caller-provided point sets, allocating no device memory.
 * The pages have no counterpart of this entry point: it exists for callers that
 * cannot allocate -- an application whose device memory is owned by its own pool
 * or budgeted up front, or one that cannot accept the device-wide synchronisation
 * and failure modes that cudaMalloc/cudaFree bring in the middle of a run.
 *
 *   K (n_inst, n, E), V (n_inst, n, D)   device, contiguous, fp32 or bf16 (dtype)
 *   K_out, V_out (n_inst, n/2, E|D)      device: the kept point of every pair, pair order
 *   idx_out (n_inst, n/2) int32          device: position (0..n-1) of each kept point in its set
 *   keep_bits_opt                        device uint32[n_inst * ceil(n/64)] or NULL: bit i%32 of
 *                                        word i/32 of set s (words ceil(n/64) apart) = 1 iff pair i
 *                                        kept its first point
 * Set s is halved with the Philox counter (pair, round_id, s, 0) keyed by seed, with the same
 * kernel-halving walk and kernel as thin_attn_forward; scale <= 0 selects 1/sqrt(E).
 * n is even, 2 <= n <= 4096; E, D multiples of 8 in [8, 256].
 *
 * Scratch is a 16 MiB array in the library's device memory, held by every device that loads
 * the library until the process exits.  It needs
 *   n_inst*40 + n_inst*n*4 + n_inst*4 (each rounded up to 256) + n_inst*ceil(n/64)^2*4096
 * bytes; larger requests fail with THIN_ATTN_EINVAL before anything is enqueued.  All calls
 * share the array: calls whose work overlaps on the GPU (other streams, other threads) race
 * on it and must be serialised by the caller.  Every scratch element a call reads is written
 * earlier in the same call, so nothing needs clearing between calls.
 * Runs on the current device; the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and should come before any stream capture.
 */
THIN_ATTN_API thin_attn_status thin_attn_halve_noalloc(int dtype, const void* K, const void* V, int n_inst,
                                                      int n, int E, int D, float scale, uint64_t seed,
                                                      uint32_t round_id, void* K_out, void* V_out,
                                                      int32_t* idx_out, uint32_t* keep_bits_opt,
                                                      void* stream);

#ifdef __cplusplus
}
#endif

#endif /* THIN_ATTN_H_ */
