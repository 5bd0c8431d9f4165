// C ABI of thin_attn: argument checks, the (causal, g) plans, workspace, launch sequence.
//
// Plan of the non-causal path (Thinformer; README "Getting Started" layouts):
//   per (b,h): systematic subsample of the S keys to S' = L 4^r, then r halving
//   levels over groups of 4 L 2^(l-1) consecutive points (KH-Compress), then
//   attention of every query against the |C| = L 2^r survivors, weight S/|C|.
// Plan of the causal path (Thinformer Express; "Express Language Modeling",
// "The EXPRESS Meta-Procedure"):
//   exact phase [0, n_e); batch k = [n_e + k b, n_e + (k+1) b) compressed to c
//   points (weight b/c); a 4-ary counter merges four level-l nodes by two
//   halvings (4c -> 2c -> c, weight x4); a query of batch k attends to the exact
//   prefix, the nodes present after k completed batches, and its batch causally.
// Plan of the causal path with the page-literal cache (causal = 2, "The EXPRESS Meta-Procedure"
// read literally): exact phase [0, n_out); batches of m n_out tokens thinned to n_out points of
// weight m; the whole cache halved twice when it holds 4 n_out points, m <- 4m.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <queue>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "thin_attn.h"

using namespace thin;

namespace {

thread_local std::string g_err;

thin_attn_status fail(thin_attn_status s, const char* fmt, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

#define CK(call)                                                                               \
  do {                                                                                         \
    cudaError_t e_ = (call);                                                                   \
    if (e_ != cudaSuccess) return fail(THIN_ATTN_ECUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

struct Sizes {
  int r, L, S_sub, C;
};

// Least r with 4^(g+r) >= S, lowered (g = 0 only) until 4^r <= S; L = floor(S/4^r).
Sizes compress_sizes(int64_t S, int g) {
  if (S <= 0) return {0, 0, 0, 0};
  int r = 0;
  auto p4 = [](int e) { return (int64_t)1 << (2 * e); };
  while (p4(g + r) < S) ++r;
  while (r > 0 && p4(r) > S) --r;
  const int64_t L = S / p4(r);
  return {r, (int)L, (int)(L * p4(r)), (int)(L << r)};
}

// Reading A of Express: thinning a batch of N points to n_out: S' = L 4^r = n_out 2^r (a systematic
// uniform subsample when S' < N) through r KH-Compress levels over leaves of L = n_out / 2^r; 2^r is
// the largest power of two with 2^r <= N / n_out and 2^r <= n_out / 4^g (S' <= n_out^2 / 4^g).
Sizes express_a_sizes(int64_t N, int n_out, int g) {
  int r = 0;
  while (((int64_t)n_out << (r + 1)) <= N && ((int64_t)1 << (r + 1 + 2 * g)) <= n_out && n_out % (1 << (r + 1)) == 0)
    ++r;
  const int L = n_out >> r;
  return {r, L, L << (2 * r), n_out};
}

// Batches of reading A after the exact phase [0, n_out): level i holds three batches of 4^i n_out
// tokens (the last batch may be partial).
struct ABatch {
  int level, s;
  int64_t start, len;
};
std::vector<ABatch> express_a_layout(int64_t T, int n_out) {
  std::vector<ABatch> out;
  int64_t start = n_out;
  for (int i = 0; start < T; ++i)
    for (int s = 1; s <= 3 && start < T; ++s) {
      const int64_t size = ((int64_t)n_out) << (2 * i);
      out.push_back({i, s, start, std::min(size, T - start)});
      start += size;
    }
  return out;
}

uint32_t round_noncausal(int level) { return (uint32_t)level; }
uint32_t round_batch(int k, int level) { return 0x40000000u | ((uint32_t)k << 4) | (uint32_t)level; }
uint32_t round_merge(int level, int node, int step) {
  return 0x80000000u | ((uint32_t)level << 24) | ((uint32_t)node << 1) | (uint32_t)step;
}
uint32_t round_subsample(int k) { return 0xC0000000u | (uint32_t)k; }

enum : int { BUF_TOKENS = -1, BUF_NODES = -2, BUF_MTEMP = -3 };

struct BufSpec {
  int64_t rows = 0;
  size_t k_off = 0, v_off = 0, idx_off = 0;
};

struct StepPlan {
  bool copy_only = false;
  int phase = 0;   // 0: thinning of sequences / batches, 1: HALVE merges
  int merge_level = 0;   // phase 1: target level of the merge
  int src_buf = BUF_TOKENS, dst_buf = 0;
  int n = 0, m = 0, m_pad = 0;
  int S_full = 0, S_sub = 0;
  int sub_stride = 0;    // see StepArgs::sub_stride
  std::vector<HalveInst> inst;
  size_t inst_off = 0;
  uint64_t trace_base = 0;
};

// Subsample stride of a token-source step (StepArgs::sub_stride).
int sub_stride_of(const StepPlan& sp) {
  if (sp.src_buf != BUF_TOKENS || sp.S_sub <= 0 || sp.S_sub >= sp.S_full || sp.S_full % sp.S_sub) return 0;
  const int k = sp.S_full / sp.S_sub;
  for (const HalveInst& in : sp.inst)
    if (in.src_row % k) return 0;
  return k;
}

// A wave: consecutive attention tiles that can run as soon as halving step `after` (and all
// earlier steps) has run; after = -1: as soon as the forward starts.
struct AttnWave {
  int tile0, count, after;
};

struct AttnTables {
  int rows_per_tile = 0;
  std::vector<AttnTile> tiles;
  std::vector<AttnSeg> segs;
  std::vector<AttnWave> waves;
  std::vector<int2> pairs;   // tile pairs of the ping-pong attention kernel (AttnArgs::pairs)
  double key_tiles_per_tile = 0;   // mean 128-key tiles a query tile attends to
  size_t tiles_off = 0, segs_off = 0, pairs_off = 0;
};

struct Plan {
  int causal = 0, g = 0;
  Sizes sz{};
  int n_b = 0, n_slots = 0, c = 0;
  int own_k0 = 0, own_k1 = 0;    // causal: the batches this handle thins (all unless thin_split)
  std::vector<int> level_base;   // causal: first slot of each node level
  // causal == 2 (Express, page-literal cache): batches, slot of H_i, slot of thinned batch (i, s)
  std::vector<ABatch> a_batches;
  std::map<int, int> a_slot_h;
  std::map<std::pair<int, int>, int> a_slot_b;
  std::vector<StepPlan> steps;
  std::vector<BufSpec> levels;   // intermediate halving outputs
  BufSpec nodes, mtemp;
  std::vector<thin_attn_trace_entry> trace;
  uint64_t trace_words = 0;
  uint64_t coreset_idx_elems = 0;
  int final_buf = BUF_TOKENS;    // compact buffer holding the coreset / nodes
  int att_slots = 1, att_slot_rows = 0;
  AttnTables simt, tc;
  // steps [sched_s0, sched_s1) run as one persistent launch (launch_halving_sched); s0 == s1: none
  int sched_s0 = 0, sched_s1 = 0;
  std::vector<int2> sched_items;            // (step - sched_s0, instance) in queue order
  std::vector<int> sched_pred_off, sched_preds;
  size_t sched_items_off = 0, sched_pred_off_off = 0, sched_preds_off = 0, sched_done_off = 0;
  int sched_epoch = 0;
  size_t delta_off = 0, c2_off = 0, delta_floats = 0, c2_floats = 0;
  // e4m3 QK^T (thin_attn_config::qk_fp8): q8, k8, ck8 copies, the amax words, scales and 1/(sq sk)
  size_t fp8_q_off = 0, fp8_k_off = 0, fp8_ck_off = 0, fp8_amax_off = 0, fp8_scales_off = 0, fp8_inv_off = 0;
  int64_t fp8_ck_rows = 0;
  size_t bytes = 0;
  void* d_mem = nullptr;
};

}  // namespace

namespace thin {
// Record `msg` as the calling thread's last error (read by thin_attn_last_error) and return s.
int record_error(int s, const char* msg) {
  g_err = msg;
  return s;
}
}  // namespace thin

struct thin_attn_s {
  thin_attn_config cfg{};
  float scale = 0.f;
  std::mutex mu;
  std::map<std::pair<int, int>, Plan*> plans;
  int* d_status = nullptr;
  // host-buffer staging
  void* st_mem = nullptr;
  size_t st_bytes = 0;
  // pipelined host path: one handle per group of heads (or batch rows), copy-in / compute / copy-out
  // streams and their events (one set per group)
  std::vector<thin_attn_s*> hp_sub;
  bool hp_by_heads = true;
  int hp_groups = 0;
  cudaStream_t hp_in = nullptr, hp_comp = nullptr, hp_out = nullptr;
  std::vector<cudaEvent_t> hp_ev;   // [3 * groups + 1]: in_done, comp_done, out_done per group; start
  // side stream of the attention waves and its fork/join events
  cudaStream_t side = nullptr, main = nullptr;
  cudaEvent_t ev_join = nullptr, ev_join2 = nullptr, ev_fork = nullptr;
  std::vector<cudaEvent_t> ev_dep;
  // per-phase device timing (thin_attn_profile): event sets and their wave counts
  bool prof_on = false;
  struct ProfPending {
    std::vector<cudaEvent_t> ev;
    size_t waves;
    int group0, group1;   // steps [group0, group1) ran as one launch (none when equal)
  };
  std::vector<ProfPending> prof_pending;
  std::vector<std::vector<cudaEvent_t>> prof_free;
  double prof_ms[3] = {0, 0, 0};
  double prof_total = 0;
  int prof_calls = 0;
  // per halving step: summed ms and the step's shape (instances, points per instance)
  std::vector<double> prof_step_ms;
  std::vector<int> prof_step_inst, prof_step_n;
  int prof_step_calls = 0;
};

namespace {

size_t elt(const thin_attn_config& c) { return c.dtype == THIN_ATTN_FP32 ? 4 : 2; }
// Philox (b,h) word of the handle's local b * H + h: its index in the whole problem.
uint32_t ctr_bh_of(const thin_attn_config& c, uint32_t bh) {
  const uint32_t Ht = (uint32_t)(c.H_total > 0 ? c.H_total : c.H);
  return ((uint32_t)c.b0 + bh / (uint32_t)c.H) * Ht + (uint32_t)c.h0 + bh % (uint32_t)c.H;
}
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (dev < 0) return;   // nothing on a device to touch
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

// Wave structure of the tiles: a tile of Express batch k reads the nodes present after k
// completed batches, whose highest level is floor(log4 k); it can run once the batch thinning
// (k >= 1) and the merges up to that level are done.  Exact-phase tiles and batch 0 read no node.
void build_waves(const thin_attn_config& cf, const Plan& p, AttnTables& t) {
  t.waves.clear();
  const int n_steps = (int)p.steps.size();
  int last_thin = -1;
  std::vector<int> last_merge;
  for (int i = 0; i < n_steps; ++i) {
    if (p.steps[i].phase == 0) last_thin = i;
    else {
      const int lv = p.steps[i].merge_level;
      if ((int)last_merge.size() <= lv) last_merge.resize(lv + 1, -1);
      last_merge[lv] = i;
    }
  }
  const int ne = std::min(cf.n_exact, cf.T);
  for (int i = 0; i < (int)t.tiles.size(); ++i) {
    int after = n_steps - 1;
    if (p.causal == 2) {
      if (t.tiles[i].q0 < 4 * p.c) after = -1;   // the exact tiles need no halving step
    } else if (p.causal) {
      const int q0 = t.tiles[i].q0;
      const int64_t k = q0 < ne ? -1 : (q0 - ne) / cf.batch;
      if (k <= 0) after = -1;
      else {
        int lv = 0;
        while (((int64_t)1 << (2 * (lv + 1))) <= k) ++lv;
        after = lv == 0 ? last_thin : (lv < (int)last_merge.size() ? last_merge[lv] : n_steps - 1);
      }
    }
    if (!t.waves.empty() && t.waves.back().after == after) t.waves.back().count++;
    else t.waves.push_back({i, 1, after});
  }
}

void build_attn_tables(const thin_attn_config& cf, const Plan& p, int QT, AttnTables& t) {
  t.rows_per_tile = QT;
  t.tiles.clear();
  t.segs.clear();
  if (!p.causal) {
    AttnSeg s{};
    if (p.sz.r == 0) {
      s.kind = SEG_TOKENS;
      s.first = 0;
      s.len = cf.S;
      s.logw = 0.f;
    } else {
      s.kind = SEG_COMPACT;
      s.first = 0;
      s.len = p.sz.C;
      s.logw = (float)std::log((double)cf.S / (double)p.sz.C);
    }
    t.segs.push_back(s);
    for (int q0 = 0; q0 < cf.T; q0 += QT) t.tiles.push_back({q0, std::min(QT, cf.T - q0), 0, 1});
    return;
  }
  if (p.causal == 2) {
    // tokens [0, 4 n_out) exactly; a query of batch (i, s), i >= 1: H_i and the thinned batches
    // (i, 1..s-1), all of weight 4^i, and its batch causally
    const int T = cf.T, n_out = p.c;
    const int ex = (int)std::min<int64_t>((int64_t)4 * n_out, T);
    for (int q0 = 0; q0 < ex; q0 += QT) {
      const int ql = std::min(QT, ex - q0);
      t.tiles.push_back({q0, ql, (int)t.segs.size(), 1});
      t.segs.push_back({SEG_TOKENS, 0, q0 + ql, 1, 0.f, 0});
    }
    for (const ABatch& b : p.a_batches) {
      if (b.level < 1) continue;
      const float lw = (float)std::log(std::ldexp(1.0, 2 * b.level));
      for (int64_t q0 = b.start; q0 < b.start + b.len; q0 += QT) {
        const int ql = (int)std::min<int64_t>(QT, b.start + b.len - q0);
        const int seg0 = (int)t.segs.size();
        t.segs.push_back({SEG_COMPACT, p.a_slot_h.at(b.level), n_out, 0, lw, 0});
        for (int s2 = 1; s2 < b.s; ++s2) t.segs.push_back({SEG_COMPACT, p.a_slot_b.at({b.level, s2}), n_out, 0, lw, 0});
        t.segs.push_back({SEG_TOKENS, (int)b.start, (int)(q0 + ql - b.start), 1, 0.f, 0});
        t.tiles.push_back({(int)q0, ql, seg0, (int)t.segs.size() - seg0});
      }
    }
    return;
  }
  const int T = cf.T, ne = std::min(cf.n_exact, T), bsz = cf.batch;
  for (int q0 = 0; q0 < ne; q0 += QT) {
    const int ql = std::min(QT, ne - q0);
    t.tiles.push_back({q0, ql, (int)t.segs.size(), 1});
    t.segs.push_back({SEG_TOKENS, 0, q0 + ql, 1, 0.f, 0});
  }
  for (int k = 0;; ++k) {
    const int64_t start = (int64_t)ne + (int64_t)k * bsz;
    if (start >= T) break;
    const int end = (int)std::min<int64_t>(start + bsz, T);
    // nodes after k completed batches: base-4 digit d_l of k -> d_l nodes of level l
    std::vector<std::pair<int, int>> snap;
    for (int lv = 0; ((int64_t)1 << (2 * lv)) <= k; ++lv) {
      const int64_t p4 = (int64_t)1 << (2 * lv);
      const int d = (int)((k / p4) % 4);
      const int base = (int)((k / (p4 * 4)) * 4);
      for (int j = 0; j < d; ++j) snap.push_back({lv, base + j});
    }
    for (int q0 = (int)start; q0 < end; q0 += QT) {
      const int ql = std::min(QT, end - q0);
      const int seg0 = (int)t.segs.size();
      if (ne > 0) t.segs.push_back({SEG_TOKENS, 0, ne, 0, 0.f, 0});
      for (auto& nd : snap) {
        const double w = std::ldexp((double)bsz / p.c, 2 * nd.first);
        t.segs.push_back({SEG_COMPACT, p.level_base[nd.first] + nd.second, p.c, 0, (float)std::log(w), 0});
      }
      t.segs.push_back({SEG_TOKENS, (int)start, q0 + ql - (int)start, 1, 0.f, 0});
      t.tiles.push_back({q0, ql, seg0, (int)t.segs.size() - seg0});
    }
  }
}

// A query-row shard (config q_begin, q_end): keep the tiles that hold rows of the range, each clipped
// to it.  A clipped tile keeps its key segments; a row's arithmetic depends on its own position only
// (the causal mask is per row), so its output is the whole run's.
void restrict_rows(const thin_attn_config& cf, AttnTables& t) {
  if (cf.q_begin == 0 && cf.q_end == 0) return;
  std::vector<AttnTile> kept;
  for (AttnTile tl : t.tiles) {
    const int a = std::max(tl.q0, cf.q_begin), b = std::min(tl.q0 + tl.qlen, cf.q_end);
    if (a >= b) continue;
    tl.q0 = a;
    tl.qlen = b - a;
    kept.push_back(tl);
  }
  t.tiles.swap(kept);
}

// Each tile's count of 128-key tiles (AttnTile::nkt), which the attention kernels read.
void set_key_tile_counts(AttnTables& t) {
  for (AttnTile& tl : t.tiles) {
    tl.nkt = 0;
    for (int s = 0; s < tl.nseg; ++s) tl.nkt += (t.segs[tl.seg0 + s].len + 127) / 128;
  }
}

// Whether tile A's key tiles are the first key tiles of tile B's: the same segments, except that
// A's last one may stop earlier in B's segment of the same place (the causal in-batch keys of two
// neighbouring query tiles).  Such a pair shares one stream of K/V tiles.
bool key_tiles_nest(const AttnTables& t, const AttnTile& A, const AttnTile& B) {
  if (A.nseg < 1 || A.nseg > B.nseg) return false;
  for (int i = 0; i < A.nseg; ++i) {
    const AttnSeg& x = t.segs[A.seg0 + i];
    const AttnSeg& y = t.segs[B.seg0 + i];
    if (x.kind != y.kind || x.first != y.first || x.causal != y.causal || x.logw != y.logw) return false;
    if (i + 1 < A.nseg ? x.len != y.len : x.len > y.len) return false;
  }
  return true;
}

// Pair neighbouring tiles (i, i+1) whose key lists nest, in either order; a tile left over runs alone.
void build_pairs(AttnTables& t) {
  t.pairs.clear();
  const int n = (int)t.tiles.size();
  int64_t kt = 0;
  for (const AttnTile& tl : t.tiles)
    for (int s = 0; s < tl.nseg; ++s) kt += (t.segs[tl.seg0 + s].len + 127) / 128;
  t.key_tiles_per_tile = n ? (double)kt / n : 0.0;
  for (int i = 0; i < n;) {
    if (i + 1 < n && key_tiles_nest(t, t.tiles[i], t.tiles[i + 1])) {
      t.pairs.push_back(make_int2(i, i + 1));
      i += 2;
    } else if (i + 1 < n && key_tiles_nest(t, t.tiles[i + 1], t.tiles[i])) {
      t.pairs.push_back(make_int2(i + 1, i));
      i += 2;
    } else {
      t.pairs.push_back(make_int2(-1, i));
      i += 1;
    }
  }
}

// Append the halving steps of KH-Compress of `runs` token runs of length S_run each.
// run r: (bh, b*L_seq + tok0, tok0, batch id k for round ids, dst rows of the final level).
struct RunDesc {
  uint32_t bh;
  int64_t src_row;
  uint32_t tok0;
  int k;                 // -1: non-causal (round = level), else Express batch index
  int64_t final_dst;     // first destination row of the level-r output (buffer final_buf)
};

void add_compress_steps(Plan& p, const std::vector<RunDesc>& runs, int S_run, int final_buf,
                        std::vector<int64_t>& level_rows_per_run, const Sizes* sizes = nullptr) {
  const Sizes sz = sizes ? *sizes : compress_sizes(S_run, p.g);
  level_rows_per_run.clear();
  const int nr = (int)runs.size();
  for (int lv = 1; lv <= sz.r; ++lv) {
    StepPlan st;
    st.n = 4 * sz.L * (1 << (lv - 1));
    st.m = st.n / 2;
    st.m_pad = (st.m + 31) / 32 * 32;
    const int in_rows = sz.S_sub >> (lv - 1);   // points per run entering this level
    const int G = in_rows / st.n;
    const int out_rows = in_rows / 2;
    st.src_buf = lv == 1 ? BUF_TOKENS : (int)p.levels.size() - 1;
    if (lv == sz.r) {
      st.dst_buf = final_buf;
    } else {
      BufSpec b;
      b.rows = (int64_t)nr * out_rows;
      p.levels.push_back(b);
      st.dst_buf = (int)p.levels.size() - 1;
    }
    st.S_full = S_run;
    st.S_sub = sz.S_sub;
    for (int r = 0; r < nr; ++r) {
      const RunDesc& rd = runs[r];
      for (int gi = 0; gi < G; ++gi) {
        HalveInst in{};
        in.src_row = lv == 1 ? rd.src_row : (int64_t)r * in_rows + (int64_t)gi * st.n;
        in.dst_row = (lv == sz.r ? rd.final_dst : (int64_t)r * out_rows) + (int64_t)gi * st.m;
        in.bh = rd.bh;
        in.round_id = rd.k < 0 ? round_noncausal(lv) : round_batch(rd.k, lv);
        in.pair0 = (uint32_t)(gi * st.m);
        in.sub_round = round_subsample(rd.k < 0 ? 0 : rd.k);
        in.tok0 = rd.tok0;
        st.inst.push_back(in);
      }
    }
    p.steps.push_back(std::move(st));
  }
}

int64_t src_rows_of(const thin_attn_config& cf, const Plan* p, const StepPlan& sp);

// Whether the persistent halving scheduler can run this step (instances of 129..512 points that the
// one-launch kernels take).
bool sched_step_ok(const thin_attn_config& cf, const Plan* p, const StepPlan& sp) {
  if (sp.copy_only || sp.inst.empty() || sp.n <= 128 || sp.n > 512 || cf.dtype != THIN_ATTN_BF16) return false;
  StepArgs a{};
  a.src_kind = sp.src_buf == BUF_TOKENS ? SRC_TOKENS : SRC_COMPACT;
  a.src_rows = src_rows_of(cf, p, sp);
  a.S_full = sp.S_full;
  a.S_sub = sp.S_sub;
  a.sub_stride = sp.sub_stride;
  a.n = sp.n;
  a.E = cf.E;
  a.D = cf.D;
  return halving_sched_shape_ok(a);
}

// The scheduled group -- the longest run of two or more consecutive steps the scheduler can run, when
// it holds HALVE merges --
// its work items, their dependencies and the queue order.  Item X of a later step depends on item Y
// of an earlier one when X reads rows Y writes, writes rows Y reads, or writes rows Y writes (same
// buffer, overlapping row ranges).  The queue order comes from a list schedule of the items on the
// SMs with durations proportional to the measured instance times (a 512-point instance ~2.4 times a
// 256-point one), taking among the ready items the one with the longest chain of work after it; so
// the order is topological and puts the instances that feed the deepest merges first.
void build_sched(const thin_attn_config& cf, Plan* p, int n_sms) {
  p->sched_s0 = p->sched_s1 = 0;
  p->sched_items.clear();
  p->sched_pred_off.clear();
  p->sched_preds.clear();
  if (cf.thin_split) return;   // the batch steps and the merges run in different phases
  const int ns = (int)p->steps.size(), cap = halving_sched_max_steps();
  int best0 = 0, best1 = 0;
  for (int i = 0; i < ns;) {
    if (!sched_step_ok(cf, p, p->steps[i])) {
      ++i;
      continue;
    }
    int j = i;
    while (j < ns && j - i < cap && sched_step_ok(cf, p, p->steps[j])) ++j;
    if (j - i > best1 - best0) best0 = i, best1 = j;
    i = j;
  }
  // only where HALVE merges follow the last thinning level: a Thinformer compress's last two levels
  // (ViT) ran slower as one launch than as two (15 us of 240)
  bool merges = false;
  for (int si = best0; si < best1; ++si) merges = merges || p->steps[si].phase == 1;
  if (best1 - best0 < 2 || !merges) return;
  struct It {
    int step, inst;
  };
  std::vector<It> items;
  std::vector<int> first(best1 - best0 + 1, 0);
  for (int si = best0; si < best1; ++si) {
    first[si - best0] = (int)items.size();
    for (int i = 0; i < (int)p->steps[si].inst.size(); ++i) items.push_back({si, i});
  }
  first[best1 - best0] = (int)items.size();
  const int n = (int)items.size();
  auto src_range = [&](const It& x, int64_t* lo, int64_t* hi) {
    const StepPlan& sp = p->steps[x.step];
    *lo = sp.inst[x.inst].src_row;
    *hi = *lo + sp.n;
  };
  auto dst_range = [&](const It& x, int64_t* lo, int64_t* hi) {
    const StepPlan& sp = p->steps[x.step];
    *lo = sp.inst[x.inst].dst_row;
    *hi = *lo + sp.m;
  };
  // per earlier step: its items' source and destination ranges, each sorted by start
  struct Rg {
    int64_t lo, hi;
    int item;
  };
  std::vector<std::vector<Rg>> by_src(best1 - best0), by_dst(best1 - best0);
  for (int x = 0; x < n; ++x) {
    Rg r{0, 0, x};
    const int k = items[x].step - best0;
    src_range(items[x], &r.lo, &r.hi);
    by_src[k].push_back(r);
    dst_range(items[x], &r.lo, &r.hi);
    by_dst[k].push_back(r);
  }
  for (auto* v : {&by_src, &by_dst})
    for (auto& l : *v) std::sort(l.begin(), l.end(), [](const Rg& a, const Rg& b) { return a.lo < b.lo; });
  auto overlapping = [](const std::vector<Rg>& l, int64_t lo, int64_t hi, std::vector<int>& out) {
    // ranges of one step do not overlap each other, so their ends are sorted too
    auto it = std::lower_bound(l.begin(), l.end(), lo, [](const Rg& r, int64_t v) { return r.hi <= v; });
    for (; it != l.end() && it->lo < hi; ++it) out.push_back(it->item);
  };
  std::vector<std::vector<int>> preds(n), succs(n);
  for (int x = 0; x < n; ++x) {
    const StepPlan& sx = p->steps[items[x].step];
    int64_t slo, shi, dlo, dhi;
    src_range(items[x], &slo, &shi);
    dst_range(items[x], &dlo, &dhi);
    std::vector<int> c;
    for (int sy = best0; sy < items[x].step; ++sy) {
      const StepPlan& so = p->steps[sy];
      if (sx.src_buf != BUF_TOKENS && sx.src_buf == so.dst_buf) overlapping(by_dst[sy - best0], slo, shi, c);
      if (sx.dst_buf == so.src_buf) overlapping(by_src[sy - best0], dlo, dhi, c);
      if (sx.dst_buf == so.dst_buf) overlapping(by_dst[sy - best0], dlo, dhi, c);
    }
    std::sort(c.begin(), c.end());
    c.erase(std::unique(c.begin(), c.end()), c.end());
    preds[x] = c;
    for (int y : c) succs[y].push_back(x);
  }
  // list schedule: longest chain of (estimated) work after each item first
  std::vector<double> dur(n), chain(n, 0.0);
  for (int x = 0; x < n; ++x) dur[x] = p->steps[items[x].step].n > 256 ? 2.4 : 1.0;
  for (int x = n - 1; x >= 0; --x) {   // successors always come later in step order
    double mx = 0.0;
    for (int y : succs[x]) mx = std::max(mx, chain[y]);
    chain[x] = dur[x] + mx;
  }
  auto worse = [&](int a, int b) { return chain[a] < chain[b] || (chain[a] == chain[b] && a > b); };
  std::priority_queue<int, std::vector<int>, decltype(worse)> ready(worse);
  std::vector<int> left(n);
  for (int x = 0; x < n; ++x)
    if ((left[x] = (int)preds[x].size()) == 0) ready.push(x);
  using Ev = std::pair<double, int>;
  std::priority_queue<Ev, std::vector<Ev>, std::greater<Ev>> running;
  std::vector<int> order;
  order.reserve(n);
  int free_sms = std::max(1, n_sms);
  while ((int)order.size() < n) {
    while (free_sms > 0 && !ready.empty()) {
      const int x = ready.top();
      ready.pop();
      order.push_back(x);
      running.push({dur[x], x});   // times of running items are relative to the current time
      --free_sms;
    }
    if (running.empty()) break;   // cannot happen: the dependencies point forward in step order
    const double t = running.top().first;
    while (!running.empty() && running.top().first <= t) {
      const int x = running.top().second;
      running.pop();
      ++free_sms;
      for (int y : succs[x])
        if (--left[y] == 0) ready.push(y);
    }
    // items started later start at t: shift the clock of what is still running
    std::vector<Ev> keep;
    while (!running.empty()) {
      keep.push_back({running.top().first - t, running.top().second});
      running.pop();
    }
    for (auto& e : keep) running.push(e);
  }
  std::vector<int> pos(n);
  for (int i = 0; i < n; ++i) pos[order[i]] = i;
  p->sched_s0 = best0;
  p->sched_s1 = best1;
  p->sched_pred_off.push_back(0);
  for (int i = 0; i < n; ++i) {
    const int x = order[i];
    p->sched_items.push_back(make_int2(items[x].step - best0, items[x].inst));
    for (int y : preds[x]) p->sched_preds.push_back(pos[y]);
    p->sched_pred_off.push_back((int)p->sched_preds.size());
  }
}

thin_attn_status build_plan(thin_attn_s* h, int causal, int g, Plan** out) {
  const thin_attn_config& cf = h->cfg;
  Plan* p = new Plan();
  p->causal = causal;
  p->g = g;
  const int BH = cf.B * cf.H;
  if (!causal) {
    p->sz = compress_sizes(cf.S, g);
    p->final_buf = BUF_TOKENS;
    if (p->sz.r > 0) {
      p->levels.reserve(p->sz.r + 1);
      std::vector<RunDesc> runs;
      for (int bh = 0; bh < BH; ++bh) {
        const int b = bh / cf.H;
        runs.push_back({(uint32_t)bh, (int64_t)b * cf.S, 0u, -1, (int64_t)bh * p->sz.C});
      }
      // the final level writes into its own buffer appended after the intermediates
      std::vector<int64_t> lr;
      const int final_index = p->sz.r - 1;   // levels 1..r-1 are intermediates -> indices 0..r-2
      add_compress_steps(*p, runs, cf.S, final_index, lr);
      BufSpec fb;
      fb.rows = (int64_t)BH * p->sz.C;
      p->levels.push_back(fb);
      p->final_buf = final_index;
      p->att_slots = 1;
      p->att_slot_rows = p->sz.C;
    }
    p->coreset_idx_elems = (uint64_t)BH * (p->sz.r > 0 ? p->sz.C : cf.S);
  } else if (causal == 2) {
    // Express with the page-literal cache: thinned batches (independent of the cache), then the
    // HALVEs H_1, H_2, ... in order (H_i consumes H_{i-1} and the three thinned batches of level
    // i-1, or the raw tokens [0, 4 n_out) for H_1)
    const int T = cf.T, n_out = std::min(cf.n_exact, T);
    p->c = n_out;
    p->a_batches = express_a_layout(T, n_out);
    const auto& L = p->a_batches;
    std::map<std::pair<int, int>, size_t> have;
    for (size_t j = 0; j < L.size(); ++j) have[{L[j].level, L[j].s}] = j;
    std::vector<int> need_h;
    for (const auto& b : L)
      if (b.level >= 1 && (need_h.empty() || need_h.back() != b.level)) need_h.push_back(b.level);
    auto needs_h = [&](int i) { return std::find(need_h.begin(), need_h.end(), i) != need_h.end(); };
    std::vector<std::pair<int, int>> need_b;
    for (const auto& b : L)
      if (b.level >= 1 && (have.count({b.level, b.s + 1}) || needs_h(b.level + 1))) need_b.push_back({b.level, b.s});
    for (int i : need_h) {
      p->a_slot_h[i] = p->n_slots++;
      for (int s2 = 1; s2 <= 3; ++s2)
        if (std::find(need_b.begin(), need_b.end(), std::make_pair(i, s2)) != need_b.end()) p->a_slot_b[{i, s2}] = p->n_slots++;
    }
    p->n_b = (int)need_b.size();
    p->nodes.rows = (int64_t)BH * p->n_slots * n_out;
    p->final_buf = BUF_NODES;
    p->att_slots = std::max(1, p->n_slots);
    p->att_slot_rows = n_out;
    // thinned batches, level by level (one set of steps per batch size)
    for (int i : need_h) {
      std::vector<RunDesc> runs;
      int64_t len = 0;
      for (int bh = 0; bh < BH; ++bh)
        for (int s2 = 1; s2 <= 3; ++s2) {
          auto it = p->a_slot_b.find({i, s2});
          if (it == p->a_slot_b.end()) continue;
          const ABatch& b = L[have[{i, s2}]];
          len = b.len;
          const int kb = (int)have[{i, s2}];
          runs.push_back({(uint32_t)bh, (int64_t)(bh / cf.H) * T + b.start, (uint32_t)b.start, kb,
                          ((int64_t)bh * p->n_slots + it->second) * n_out});
        }
      if (runs.empty()) continue;
      const Sizes sz = express_a_sizes(len, n_out, g);
      std::vector<int64_t> lr;
      if (sz.r > 0) add_compress_steps(*p, runs, (int)len, BUF_NODES, lr, &sz);
    }
    // HALVEs: 4 n_out points -> 2 n_out (MTEMP) -> n_out (slot H_i)
    p->mtemp.rows = (int64_t)BH * 2 * n_out;
    for (int i : need_h) {
      for (int step = 0; step < 2; ++step) {
        StepPlan st;
        st.phase = 1;
        st.merge_level = i;
        st.n = (step == 0 ? 4 : 2) * n_out;
        st.m = st.n / 2;
        st.m_pad = (st.m + 31) / 32 * 32;
        st.src_buf = step == 0 ? (i == 1 ? BUF_TOKENS : BUF_NODES) : BUF_MTEMP;
        st.dst_buf = step == 0 ? BUF_MTEMP : BUF_NODES;
        st.S_full = st.S_sub = st.n;
        for (int bh = 0; bh < BH; ++bh) {
          HalveInst in{};
          const int64_t mt = (int64_t)bh * 2 * n_out;
          if (step == 0) {
            in.src_row = i == 1 ? (int64_t)(bh / cf.H) * T : ((int64_t)bh * p->n_slots + p->a_slot_h[i - 1]) * n_out;
            in.dst_row = mt;
          } else {
            in.src_row = mt;
            in.dst_row = ((int64_t)bh * p->n_slots + p->a_slot_h[i]) * n_out;
          }
          in.bh = (uint32_t)bh;
          in.round_id = round_merge(i, 0, step);
          in.pair0 = 0;
          in.tok0 = 0;
          st.inst.push_back(in);
        }
        p->steps.push_back(std::move(st));
      }
    }
    p->coreset_idx_elems = (uint64_t)p->nodes.rows;
  } else {
    const int T = cf.T, ne = std::min(cf.n_exact, T), bsz = cf.batch;
    p->n_b = T > ne ? (T - ne) / bsz : 0;
    p->own_k0 = 0;
    p->own_k1 = p->n_b;
    if (cf.thin_split) {
      // batch k belongs to the query-row range holding its last token ne + (k + 1) b - 1
      // (the batches whose last token lies before q_begin, and before q_end: a range owning no batch
      // gets an empty range in place)
      const int qb = cf.q_begin, qe = (cf.q_begin == 0 && cf.q_end == 0) ? T : cf.q_end;
      auto before = [&](int64_t t) {
        int n = 0;
        while (n < p->n_b && (int64_t)ne + (int64_t)(n + 1) * bsz - 1 < t) ++n;
        return n;
      };
      p->own_k0 = before(qb);
      p->own_k1 = before(qe);
    }
    p->sz = compress_sizes(bsz, g);
    p->c = p->sz.C;
    for (int lv = 0; (p->n_b >> (2 * lv)) > 0; ++lv) {
      p->level_base.push_back(p->n_slots);
      p->n_slots += p->n_b >> (2 * lv);
    }
    p->nodes.rows = (int64_t)BH * p->n_slots * p->c;
    p->final_buf = BUF_NODES;
    p->att_slots = p->n_slots;
    p->att_slot_rows = p->c;
    if (p->n_b > 0) {
      std::vector<RunDesc> runs;
      for (int bh = 0; bh < BH; ++bh)
        for (int k = p->own_k0; k < p->own_k1; ++k) {
          const int b = bh / cf.H;
          const uint32_t tok0 = (uint32_t)(ne + k * bsz);
          runs.push_back({(uint32_t)bh, (int64_t)b * T + tok0, tok0, k,
                          ((int64_t)bh * p->n_slots + k) * p->c});
        }
      if (p->sz.r == 0) {
        StepPlan st;
        st.copy_only = true;
        st.n = bsz;
        st.src_buf = BUF_TOKENS;
        st.dst_buf = BUF_NODES;
        st.S_full = st.S_sub = bsz;
        for (auto& rd : runs) {
          HalveInst in{};
          in.src_row = rd.src_row;
          in.dst_row = rd.final_dst;
          in.bh = rd.bh;
          in.tok0 = rd.tok0;
          st.inst.push_back(in);
        }
        p->steps.push_back(std::move(st));
      } else {
        std::vector<int64_t> lr;
        add_compress_steps(*p, runs, bsz, BUF_NODES, lr);
      }
      // HALVE merges: target level L' takes level L'-1 slots 4j'..4j'+3.  The first step's output
      // goes to rows of the merge buffer of its own (level, b, h, node), so merges of different
      // levels never share rows (the halving scheduler runs them concurrently)
      int64_t merges = 0;
      for (int lv = 1; (p->n_b >> (2 * lv)) > 0; ++lv) merges += (int64_t)BH * (p->n_b >> (2 * lv));
      p->mtemp.rows = merges * 2 * p->c;
      int64_t level_first = 0;
      for (int lv = 1; (p->n_b >> (2 * lv)) > 0; level_first += (int64_t)BH * (p->n_b >> (2 * lv)), ++lv) {
        const int nj = p->n_b >> (2 * lv);
        for (int step = 0; step < 2; ++step) {
          StepPlan st;
          st.phase = 1;
          st.merge_level = lv;
          st.n = (step == 0 ? 4 : 2) * p->c;
          st.m = st.n / 2;
          st.m_pad = (st.m + 31) / 32 * 32;
          st.src_buf = step == 0 ? BUF_NODES : BUF_MTEMP;
          st.dst_buf = step == 0 ? BUF_MTEMP : BUF_NODES;
          st.S_full = st.S_sub = st.n;
          for (int bh = 0; bh < BH; ++bh)
            for (int j = 0; j < nj; ++j) {
              HalveInst in{};
              const int64_t mt = (level_first + (int64_t)bh * nj + j) * 2 * p->c;
              if (step == 0) {
                in.src_row = ((int64_t)bh * p->n_slots + p->level_base[lv - 1] + 4 * j) * p->c;
                in.dst_row = mt;
              } else {
                in.src_row = mt;
                in.dst_row = ((int64_t)bh * p->n_slots + p->level_base[lv] + j) * p->c;
              }
              in.bh = (uint32_t)bh;
              in.round_id = round_merge(lv, j, step);
              in.pair0 = 0;
              st.inst.push_back(in);
            }
          p->steps.push_back(std::move(st));
        }
      }
    }
    p->coreset_idx_elems = (uint64_t)p->nodes.rows;
  }
  // trace layout and scratch sizes
  for (auto& st : p->steps) {
    st.sub_stride = sub_stride_of(st);
    for (auto& in : st.inst) in.ctr_bh = ctr_bh_of(cf, in.bh);
    if (st.copy_only) continue;
    st.trace_base = p->trace_words;
    const int nw = st.m_pad / 32;
    for (size_t i = 0; i < st.inst.size(); ++i) {
      const HalveInst& in = st.inst[i];
      p->trace.push_back({in.bh, in.round_id, in.pair0, (uint32_t)st.m, st.trace_base + i * nw});
    }
    p->trace_words += (uint64_t)st.inst.size() * nw;
    p->delta_floats = std::max(p->delta_floats, st.inst.size() * (size_t)st.m_pad * st.m_pad);
    p->c2_floats = std::max(p->c2_floats, st.inst.size());
  }
  build_attn_tables(cf, *p, attention_simt_tile_rows(), p->simt);
  restrict_rows(cf, p->simt);
  build_waves(cf, *p, p->simt);
  if (attention_tc_supported(cf.dtype, cf.E, cf.D)) {
    build_attn_tables(cf, *p, attention_tc_tile_rows(), p->tc);
    restrict_rows(cf, p->tc);
    build_waves(cf, *p, p->tc);
    build_pairs(p->tc);
  }
  {
    int sms = 148;
    if (cf.device >= 0) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, cf.device);
    cudaGetLastError();
    build_sched(cf, p, sms);
  }
  // memory layout: tables first, then buffers
  size_t off = 0;
  for (auto& st : p->steps) {
    st.inst_off = off;
    off = align256(off + st.inst.size() * sizeof(HalveInst));
  }
  p->sched_items_off = off;
  off = align256(off + p->sched_items.size() * sizeof(int2));
  p->sched_pred_off_off = off;
  off = align256(off + p->sched_pred_off.size() * sizeof(int));
  p->sched_preds_off = off;
  off = align256(off + p->sched_preds.size() * sizeof(int));
  p->sched_done_off = off;   // zeros, uploaded with the tables
  off = align256(off + p->sched_items.size() * sizeof(int));
  for (AttnTables* t : {&p->simt, &p->tc}) {
    t->tiles_off = off;
    off = align256(off + t->tiles.size() * sizeof(AttnTile));
    t->segs_off = off;
    off = align256(off + t->segs.size() * sizeof(AttnSeg));
    t->pairs_off = off;
    off = align256(off + t->pairs.size() * sizeof(int2));
  }
  const size_t es = elt(cf);
  auto place = [&](BufSpec& b) {
    b.k_off = off;
    off = align256(off + (size_t)b.rows * cf.E * es);
    b.v_off = off;
    off = align256(off + (size_t)b.rows * cf.D * es);
    b.idx_off = off;
    off = align256(off + (size_t)b.rows * 4);
  };
  for (auto& b : p->levels) place(b);
  place(p->nodes);
  place(p->mtemp);
  p->delta_off = off;
  off = align256(off + p->delta_floats * 4);
  p->c2_off = off;
  off = align256(off + p->c2_floats * 4);
  if (cf.qk_fp8) {
    const int64_t BH = (int64_t)cf.B * cf.H, L = causal ? cf.T : cf.S;
    p->fp8_ck_rows = p->final_buf != BUF_TOKENS ? BH * p->att_slots * p->att_slot_rows : 0;
    p->fp8_q_off = off;
    off = align256(off + (size_t)cf.B * cf.T * cf.H * cf.E);
    p->fp8_k_off = off;
    off = align256(off + (size_t)cf.B * L * cf.H * cf.E);
    p->fp8_ck_off = off;
    off = align256(off + (size_t)p->fp8_ck_rows * cf.E);
    p->fp8_amax_off = off;
    off = align256(off + (size_t)2 * BH * 4);
    p->fp8_scales_off = off;
    off = align256(off + (size_t)2 * BH * 4);
    p->fp8_inv_off = off;
    off = align256(off + (size_t)BH * 4);
  }
  p->bytes = off;
  *out = p;
  return THIN_ATTN_OK;
}

thin_attn_status materialise(thin_attn_s* h, Plan* p) {
  if (!h->d_status) {
    cudaError_t e = cudaMalloc(&h->d_status, kStatusBytes);
    if (e != cudaSuccess) {
      cudaGetLastError();
      h->d_status = nullptr;
      return fail(THIN_ATTN_ENOMEM, "status word: %s", cudaGetErrorString(e));
    }
    e = cudaMemset(h->d_status, 0, kStatusBytes);
    if (e != cudaSuccess) {  // a status word that is not zero is never kept
      cudaFree(h->d_status);
      h->d_status = nullptr;
      return fail(THIN_ATTN_ECUDA, "status word: %s", cudaGetErrorString(e));
    }
  }
  if (p->d_mem) return THIN_ATTN_OK;
  void* mem = nullptr;
  cudaError_t e = cudaMalloc(&mem, std::max<size_t>(p->bytes, 256));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(THIN_ATTN_ENOMEM, "workspace of %zu bytes: %s", p->bytes, cudaGetErrorString(e));
  }
  // upload tables
  std::vector<char> host(p->steps.empty() && p->simt.tiles.empty() ? 0 : p->delta_off);
  size_t tbl_end = 0;
  for (auto& st : p->steps) {
    if (!st.inst.empty()) std::memcpy(host.data() + st.inst_off, st.inst.data(), st.inst.size() * sizeof(HalveInst));
    tbl_end = std::max(tbl_end, st.inst_off + st.inst.size() * sizeof(HalveInst));
  }
  if (!p->sched_items.empty()) {
    std::memcpy(host.data() + p->sched_items_off, p->sched_items.data(), p->sched_items.size() * sizeof(int2));
    std::memcpy(host.data() + p->sched_pred_off_off, p->sched_pred_off.data(), p->sched_pred_off.size() * sizeof(int));
    if (!p->sched_preds.empty())
      std::memcpy(host.data() + p->sched_preds_off, p->sched_preds.data(), p->sched_preds.size() * sizeof(int));
    tbl_end = std::max(tbl_end, p->sched_done_off + p->sched_items.size() * sizeof(int));
  }
  for (AttnTables* t : {&p->simt, &p->tc}) {
    set_key_tile_counts(*t);
    if (!t->tiles.empty()) std::memcpy(host.data() + t->tiles_off, t->tiles.data(), t->tiles.size() * sizeof(AttnTile));
    if (!t->segs.empty()) std::memcpy(host.data() + t->segs_off, t->segs.data(), t->segs.size() * sizeof(AttnSeg));
    if (!t->pairs.empty()) std::memcpy(host.data() + t->pairs_off, t->pairs.data(), t->pairs.size() * sizeof(int2));
    tbl_end = std::max(tbl_end, t->pairs_off + t->pairs.size() * sizeof(int2));
  }
  if (tbl_end) {
    e = cudaMemcpy(mem, host.data(), tbl_end, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      cudaFree(mem);
      return fail(THIN_ATTN_ECUDA, "table upload: %s", cudaGetErrorString(e));
    }
  }
  p->d_mem = mem;
  return THIN_ATTN_OK;
}

thin_attn_status check_cfg(const thin_attn_config* c) {
  if (!c) return fail(THIN_ATTN_EINVAL, "config is null");
  if (c->dtype != THIN_ATTN_FP32 && c->dtype != THIN_ATTN_BF16) return fail(THIN_ATTN_EINVAL, "dtype %d", c->dtype);
  if (c->B < 1 || c->T < 1 || c->H < 1) return fail(THIN_ATTN_EINVAL, "B, T, H must be >= 1");
  if (c->E < 8 || c->E > 256 || c->E % 8 || c->D < 8 || c->D > 256 || c->D % 8)
    return fail(THIN_ATTN_EINVAL, "E=%d D=%d: widths must be multiples of 8 in [8, 256]", c->E, c->D);
  if ((int64_t)c->B * c->T * c->H > ((int64_t)1 << 31) / 4) return fail(THIN_ATTN_EINVAL, "B*T*H too large");
  const int64_t Ht = c->H_total > 0 ? c->H_total : c->H;
  if (c->b0 < 0 || c->h0 < 0 || c->h0 + (int64_t)c->H > Ht)
    return fail(THIN_ATTN_EINVAL, "shard b0=%d h0=%d H=%d outside the whole problem's H_total=%lld", c->b0, c->h0, c->H,
                (long long)Ht);
  if (((int64_t)c->b0 + c->B) * Ht > (int64_t)UINT32_MAX)
    return fail(THIN_ATTN_EINVAL, "(b0 + B) * H_total exceeds the 32-bit Philox (b,h) word");
  if (c->q_begin != 0 || c->q_end != 0) {
    if (c->q_begin < 0 || c->q_end <= c->q_begin || c->q_end > c->T)
      return fail(THIN_ATTN_EINVAL, "query rows [%d, %d) are not a range inside [0, T=%d)", c->q_begin, c->q_end, c->T);
    if (c->q_begin % 128 || (c->q_end % 128 && c->q_end != c->T))
      return fail(THIN_ATTN_EINVAL, "query rows [%d, %d): both ends must be multiples of 128 (the end may be T)",
                  c->q_begin, c->q_end);
  }
  if (c->thin_split != 0 && c->thin_split != 1) return fail(THIN_ATTN_EINVAL, "thin_split must be 0 or 1");
  if (c->thin_split && c->qk_fp8) return fail(THIN_ATTN_EUNSUPPORTED, "thin_split takes no qk_fp8");
  if (c->qk_fp8 != 0 && c->qk_fp8 != 1) return fail(THIN_ATTN_EINVAL, "qk_fp8 must be 0 or 1");
  if (c->qk_fp8 && (c->dtype != THIN_ATTN_BF16 || c->E != 128 || c->D > 128 || c->D % 64 || !qk_fp8_supported(c->H, c->E)))
    return fail(THIN_ATTN_EUNSUPPORTED, "qk_fp8 needs bf16 with E = 128, D = 64 or 128 and H <= 128 (E=%d D=%d H=%d)", c->E,
                c->D, c->H);
  return THIN_ATTN_OK;
}


thin_attn_status get_plan(thin_attn_s* h, int causal, int g, Plan** out) {
  if (causal < 0 || causal > 2) return fail(THIN_ATTN_EINVAL, "causal must be 0, 1 or 2");
  if (g < 0 || g > 6) return fail(THIN_ATTN_EINVAL, "g=%d outside 0..6", g);
  const thin_attn_config& c = h->cfg;
  if (!causal && (c.S < 1)) return fail(THIN_ATTN_EINVAL, "non-causal attention needs S >= 1");
  if (causal == 1 && (c.batch < 1 || c.n_exact < 0))
    return fail(THIN_ATTN_EINVAL, "causal attention needs batch >= 1 and n_exact >= 0");
  if (causal == 2 && c.n_exact < 2)
    return fail(THIN_ATTN_EINVAL, "Express with the page-literal cache needs n_exact (the cache size n_out) >= 2");
  if (c.thin_split && causal != 1)
    return fail(THIN_ATTN_EUNSUPPORTED, "thin_split runs Express (causal = 1) with its batch cache only");
  auto key = std::make_pair(causal, g);
  auto it = h->plans.find(key);
  if (it != h->plans.end()) {
    *out = it->second;
    return THIN_ATTN_OK;
  }
  Plan* p = nullptr;
  thin_attn_status s = build_plan(h, causal, g, &p);
  if (s != THIN_ATTN_OK) return s;
  for (auto& st : p->steps)
    if (!st.copy_only && st.m_pad > 2048) {
      delete p;
      return fail(THIN_ATTN_EUNSUPPORTED, "halving instance of %d points exceeds 4096", st.n);
    }
  h->plans[key] = p;
  *out = p;
  return THIN_ATTN_OK;
}

char* base_of(Plan* p) { return (char*)p->d_mem; }

void buf_ptrs(Plan* p, int id, const void* k, const void* v, const void** K, const void** V,
              int32_t** idx) {
  if (id == BUF_TOKENS) {
    *K = k;
    *V = v;
    *idx = nullptr;
    return;
  }
  const BufSpec& b = id == BUF_NODES ? p->nodes : id == BUF_MTEMP ? p->mtemp : p->levels[id];
  *K = base_of(p) + b.k_off;
  *V = base_of(p) + b.v_off;
  *idx = (int32_t*)(base_of(p) + b.idx_off);
}

// Rows of a step's source: the (B*L) token rows, or the rows of its compact buffer.
int64_t src_rows_of(const thin_attn_config& cf, const Plan* p, const StepPlan& sp) {
  return sp.src_buf == BUF_TOKENS ? (int64_t)cf.B * (p->causal ? cf.T : cf.S)
         : (sp.src_buf == BUF_NODES ? p->nodes : sp.src_buf == BUF_MTEMP ? p->mtemp : p->levels[sp.src_buf]).rows;
}

// Kernels a step launches: 1 (copy, or the fused small-instance kernel) or 3 (c^2, Gram, walk).
int step_launches(const thin_attn_config& cf, const Plan* p, const StepPlan& sp) {
  if (sp.inst.empty()) return 0;
  if (sp.copy_only) return 1;
  StepArgs a{};
  a.src_kind = sp.src_buf == BUF_TOKENS ? SRC_TOKENS : SRC_COMPACT;
  a.src_rows = src_rows_of(cf, p, sp);
  a.S_full = sp.S_full;
  a.S_sub = sp.S_sub;
  a.sub_stride = sp.sub_stride;
  a.n = sp.n;
  a.E = cf.E;
  a.D = cf.D;
  const bool tc = cf.dtype == 1 && std::getenv("THIN_ATTN_SIMT_GRAM") == nullptr;
  return tc && halving_fused_supported(a) ? 1 : 3;
}

// phase 0: the whole forward.  Sequence shards with split thinning (thin_split) run it in two calls:
// phase 1 the batch-thinning steps only, phase 2 the merge steps, the attention and the coreset
// output (the other ranks' batch coresets imported in between).
thin_attn_status run_forward(thin_attn_s* h, Plan* p, const void* q, const void* k, const void* v, void* out,
                             uint64_t seed, float* lse, int32_t* cidx, uint32_t* trace, cudaStream_t st,
                             int phase = 0) {
  const thin_attn_config& cf = h->cfg;
  const bool use_tc_gram = std::getenv("THIN_ATTN_SIMT_GRAM") == nullptr;
  const bool use_tc_attn = !p->tc.tiles.empty() && tensor_maps_available() && std::getenv("THIN_ATTN_SIMT_ATTN") == nullptr;
  const AttnTables& tab = use_tc_attn ? p->tc : p->simt;
  // With THIN_ATTN_OVERLAP set, attention runs as waves on a side stream, each after the halving
  // step it depends on, so the tensor cores work while later (latency-bound) halving steps run.
  // By default one attention launch follows all halving steps on the caller's stream: the waves
  // save ~3 % of an Express step but share SMs with the halving kernels.
  const bool fp8 = cf.qk_fp8 && use_tc_attn;
  const bool side = phase == 0 && tab.waves.size() > 1 && std::getenv("THIN_ATTN_OVERLAP") != nullptr && !fp8;
  const std::vector<AttnWave> one_wave = {{0, (int)tab.tiles.size(), (int)p->steps.size() - 1}};
  const std::vector<AttnWave>& waves = side ? tab.waves : one_wave;
  cudaStream_t sa = st;
  cudaStream_t caller = st;
  if (side) {
    // halving steps on a high-priority stream (their CTAs are dispatched ahead of pending
    // attention CTAs), attention waves on a low-priority one; both fork from and join back
    // into the caller's stream
    if (!h->side) {
      int lo = 0, hi = 0;
      CK(cudaDeviceGetStreamPriorityRange(&lo, &hi));
      CK(cudaStreamCreateWithPriority(&h->side, cudaStreamNonBlocking, lo));
      CK(cudaStreamCreateWithPriority(&h->main, cudaStreamNonBlocking, hi));
      CK(cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming));
      CK(cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming));
      CK(cudaEventCreateWithFlags(&h->ev_join2, cudaEventDisableTiming));
    }
    while (h->ev_dep.size() < waves.size() + 1) {
      cudaEvent_t e;
      CK(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
      h->ev_dep.push_back(e);
    }
    CK(cudaEventRecord(h->ev_fork, caller));
    CK(cudaStreamWaitEvent(h->main, h->ev_fork, 0));
    CK(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
    st = h->main;
    sa = h->side;
  }
  // profiling events: [0] start, [1] first merge step, [2] all halving steps, [3] end (joined),
  // then a (start, stop) pair per attention wave on the attention stream, then the end of every
  // halving step on the halving stream
  std::vector<cudaEvent_t> ev;
  const size_t ev_steps = 4 + 2 * waves.size();
  if (h->prof_on && phase == 0) {
    const size_t need = ev_steps + p->steps.size();
    if (!h->prof_free.empty() && h->prof_free.back().size() >= need) {
      ev = h->prof_free.back();
      h->prof_free.pop_back();
    } else {
      ev.resize(need);
      for (auto& e : ev) CK(cudaEventCreate(&e));
    }
    CK(cudaEventRecord(ev[0], st));
  }
  AttnArgs aa{};
  aa.q = q;
  aa.k = k;
  aa.v = v;
  if (p->final_buf != BUF_TOKENS) {
    int32_t* didx;
    buf_ptrs(p, p->final_buf, k, v, &aa.ck, &aa.cv, &didx);
  }
  aa.out = out;
  aa.lse = lse;
  aa.B = cf.B;
  aa.T = cf.T;
  aa.L = p->causal ? cf.T : cf.S;
  aa.H = cf.H;
  aa.E = cf.E;
  aa.D = cf.D;
  aa.n_slots = p->att_slots;
  aa.slot_rows = p->att_slot_rows;
  aa.scale_log2e = (float)((double)h->scale * 1.4426950408889634);
  // Test hook for failure detection: one CTA's bounded wait runs out (no fault, no hang).
  aa.inject_timeout = std::getenv("THIN_ATTN_INJECT_WAIT_TIMEOUT") != nullptr;
  aa.tiles = (const AttnTile*)(base_of(p) + tab.tiles_off);
  aa.segs = (const AttnSeg*)(base_of(p) + tab.segs_off);
  // The ping-pong kernel (tile pairs sharing one K/V stream) pays a Q reload and a pipeline refill
  // at every pair it starts and gains in every key tile after that, so it runs where a query tile
  // attends to kPpMinKeyTiles key tiles or more on average (Express 128K: 28; Express 32K: 15, ViT
  // 2 stay on the two-CTA kernel, measured faster there).  THIN_ATTN_PP / THIN_ATTN_TC2P force
  // one form or the other.
  constexpr double kPpMinKeyTiles = 24.0;
  const bool want_pp = std::getenv("THIN_ATTN_TC2P") == nullptr &&
                       (std::getenv("THIN_ATTN_PP") != nullptr || tab.key_tiles_per_tile >= kPpMinKeyTiles);
  if (!side && use_tc_attn && want_pp && !tab.pairs.empty()) {
    aa.pairs = (const int2*)(base_of(p) + tab.pairs_off);
    aa.pair0 = 0;
    aa.n_pairs = (int)tab.pairs.size();
  }
  size_t next_wave = 0, dep_i = 0;
  auto launch_waves_after = [&](int step) -> thin_attn_status {
    if (phase == 1) return THIN_ATTN_OK;   // no attention in the thinning phase
    while (next_wave < waves.size() && waves[next_wave].after <= step) {
      const AttnWave& w = waves[next_wave];
      if (side) {
        CK(cudaEventRecord(h->ev_dep[dep_i], st));
        CK(cudaStreamWaitEvent(sa, h->ev_dep[dep_i], 0));
        ++dep_i;
      }
      aa.tile0 = w.tile0;
      aa.n_tiles = w.count;
      // (with e4m3 QK^T the attention phase starts before the copies of q and k, recorded there)
      if (!ev.empty() && !(fp8 && next_wave == 0)) CK(cudaEventRecord(ev[4 + 2 * next_wave], sa));
      bool done = false;
      cudaError_t e = cudaSuccess;
      if (use_tc_attn) e = launch_attention_tc(aa, h->d_status, sa, &done);
      if (e == cudaSuccess && !done) e = launch_attention_simt(aa, cf.dtype, sa);
      if (e != cudaSuccess) return fail(THIN_ATTN_ECUDA, "attention: %s", cudaGetErrorString(e));
      if (!ev.empty()) CK(cudaEventRecord(ev[5 + 2 * next_wave], sa));
      ++next_wave;
    }
    return THIN_ATTN_OK;
  };
  thin_attn_status ls = launch_waves_after(-1);
  if (ls != THIN_ATTN_OK) return ls;
  bool merged_mark = false;
  // the scheduled group runs as one launch unless THIN_ATTN_LEVELWISE asks for a launch per step
  const bool sched = p->sched_s1 > p->sched_s0 && use_tc_gram && std::getenv("THIN_ATTN_LEVELWISE") == nullptr;
  std::vector<StepArgs> group;
  for (size_t si = 0; si < p->steps.size(); ++si) {
    const StepPlan& sp = p->steps[si];
    if ((phase == 1 && sp.phase != 0) || (phase == 2 && sp.phase == 0)) continue;
    const bool in_group = sched && (int)si >= p->sched_s0 && (int)si < p->sched_s1;
    if (!ev.empty() && !merged_mark) {
      // the first merge step; a scheduled group that holds merges counts as merging from its start
      bool merges = sp.phase == 1;
      if (in_group && (int)si == p->sched_s0)
        for (int sj = p->sched_s0; sj < p->sched_s1; ++sj) merges = merges || p->steps[sj].phase == 1;
      if (merges && (!in_group || (int)si == p->sched_s0)) {
        CK(cudaEventRecord(ev[1], st));
        merged_mark = true;
      }
    }
    StepArgs a{};
    const void *sk, *sv;
    int32_t* sidx;
    buf_ptrs(p, sp.src_buf, k, v, &sk, &sv, &sidx);
    const void *dk, *dv;
    int32_t* didx;
    buf_ptrs(p, sp.dst_buf, k, v, &dk, &dv, &didx);
    a.src_kind = sp.src_buf == BUF_TOKENS ? SRC_TOKENS : SRC_COMPACT;
    a.src_rows = src_rows_of(cf, p, sp);
    a.status = h->d_status;
    a.srcK = sk;
    a.srcV = sv;
    a.srcIdx = sidx;
    a.H = cf.H;
    a.S_full = sp.S_full;
    a.S_sub = sp.S_sub;
    a.sub_stride = sp.sub_stride;
    a.dstK = (void*)dk;
    a.dstV = (void*)dv;
    a.dstIdx = didx;
    a.inst = (const HalveInst*)(base_of(p) + sp.inst_off);
    a.n_inst = (int)sp.inst.size();
    a.n = sp.n;
    a.m = sp.m;
    a.m_pad = sp.m_pad;
    a.E = cf.E;
    a.D = cf.D;
    a.scale_log2e = (float)((double)h->scale * 1.4426950408889634);
    a.C = sp.m > 0 ? (float)std::sqrt(2.0 * std::log(4.0 * sp.m)) : 0.f;
    a.seed = seed;
    a.c2 = (float*)(base_of(p) + p->c2_off);
    a.delta = (float*)(base_of(p) + p->delta_off);
    a.trace = trace;
    a.trace_base = sp.trace_base;
    if (in_group) {
      group.push_back(a);
      if ((int)si + 1 < p->sched_s1) continue;
      bool ok = true;
      for (const StepArgs& ga : group) ok = ok && halving_sched_step_supported(ga);
      if (ok) {
        SchedTables t{};
        t.items = (const int2*)(base_of(p) + p->sched_items_off);
        t.pred_off = (const int*)(base_of(p) + p->sched_pred_off_off);
        t.preds = (const int*)(base_of(p) + p->sched_preds_off);
        t.n_items = (int)p->sched_items.size();
        t.done = (int*)(base_of(p) + p->sched_done_off);
        if (++p->sched_epoch <= 0) p->sched_epoch = 1;
        t.epoch = p->sched_epoch;
        t.sched = h->d_status + 6;
        t.status = h->d_status;
        // test hook: the middle item's dependency wait runs out (failure detection without a fault)
        t.inject_item = std::getenv("THIN_ATTN_INJECT_SCHED_TIMEOUT") ? t.n_items / 2 : -1;
        cudaError_t e = launch_halving_sched(group.data(), (int)group.size(), t, st);
        if (e != cudaSuccess) return fail(THIN_ATTN_ECUDA, "halving scheduler: %s", cudaGetErrorString(e));
      } else {
        for (const StepArgs& ga : group) {
          cudaError_t e = launch_halving_step(ga, cf.dtype, use_tc_gram, st);
          if (e != cudaSuccess) return fail(THIN_ATTN_ECUDA, "halving step (n=%d): %s", ga.n, cudaGetErrorString(e));
        }
      }
      // per-step profile: one event after the group (drain_profile puts its time on the first step)
      if (!ev.empty()) CK(cudaEventRecord(ev[ev_steps + p->sched_s1 - 1], st));
    } else {
      cudaError_t e = sp.copy_only ? launch_copy_step(a, cf.dtype, st)
                                   : launch_halving_step(a, cf.dtype, use_tc_gram, st);
      if (e != cudaSuccess) return fail(THIN_ATTN_ECUDA, "halving step (n=%d): %s", sp.n, cudaGetErrorString(e));
      if (!ev.empty()) CK(cudaEventRecord(ev[ev_steps + si], st));
    }
    if (si + 1 < p->steps.size()) {
      ls = launch_waves_after((int)si);
      if (ls != THIN_ATTN_OK) return ls;
    }
  }
  if (!ev.empty()) {
    if (!merged_mark) CK(cudaEventRecord(ev[1], st));
    CK(cudaEventRecord(ev[2], st));
  }
  if (phase == 1) return THIN_ATTN_OK;
  if (fp8) {
    // e4m3 copies of q, k and the coreset keys for the attention's QK^T (timed with the attention)
    QkFp8Args fa{};
    fa.q = q;
    fa.k = k;
    fa.ck = p->fp8_ck_rows > 0 ? aa.ck : nullptr;
    fa.B = cf.B;
    fa.T = cf.T;
    fa.L = p->causal ? cf.T : cf.S;
    fa.H = cf.H;
    fa.E = cf.E;
    fa.ck_rows = p->fp8_ck_rows;
    fa.rows_per_bh = (int64_t)p->att_slots * p->att_slot_rows;
    fa.q8 = (uint8_t*)(base_of(p) + p->fp8_q_off);
    fa.k8 = (uint8_t*)(base_of(p) + p->fp8_k_off);
    fa.ck8 = (uint8_t*)(base_of(p) + p->fp8_ck_off);
    fa.amax = (unsigned*)(base_of(p) + p->fp8_amax_off);
    fa.scales = (float*)(base_of(p) + p->fp8_scales_off);
    fa.qk_inv = (float*)(base_of(p) + p->fp8_inv_off);
    if (!ev.empty()) CK(cudaEventRecord(ev[4], sa));
    cudaError_t e = launch_qk_fp8(fa, st);
    if (e != cudaSuccess) return fail(THIN_ATTN_ECUDA, "e4m3 copies of q and k: %s", cudaGetErrorString(e));
    aa.q8 = fa.q8;
    aa.k8 = fa.k8;
    aa.ck8 = p->fp8_ck_rows > 0 ? fa.ck8 : nullptr;
    aa.qk_inv = fa.qk_inv;
    aa.pairs = nullptr;   // the e4m3 S MMAs are in the two-CTA kernel
    aa.n_pairs = 0;
  }
  ls = launch_waves_after((int)p->steps.size());
  if (ls != THIN_ATTN_OK) return ls;
  if (cidx) {
    if (p->final_buf == BUF_TOKENS) {
      cudaError_t e = launch_iota(cidx, (int64_t)p->coreset_idx_elems, cf.S, st);
      if (e != cudaSuccess) return fail(THIN_ATTN_ECUDA, "iota: %s", cudaGetErrorString(e));
    } else if (p->coreset_idx_elems) {
      const void *dk, *dv;
      int32_t* didx;
      buf_ptrs(p, p->final_buf, k, v, &dk, &dv, &didx);
      CK(cudaMemcpyAsync(cidx, didx, p->coreset_idx_elems * 4, cudaMemcpyDeviceToDevice, st));
    }
  }
  if (side) {
    CK(cudaEventRecord(h->ev_join, sa));
    CK(cudaEventRecord(h->ev_join2, st));
    CK(cudaStreamWaitEvent(caller, h->ev_join, 0));
    CK(cudaStreamWaitEvent(caller, h->ev_join2, 0));
    st = caller;
  }
  if (!ev.empty()) {
    CK(cudaEventRecord(ev[3], st));
    h->prof_pending.push_back({ev, waves.size(), sched ? p->sched_s0 : 0, sched ? p->sched_s1 : 0});
    if (h->prof_step_ms.size() != p->steps.size()) {
      h->prof_step_ms.assign(p->steps.size(), 0.0);
      h->prof_step_inst.resize(p->steps.size());
      h->prof_step_n.resize(p->steps.size());
      h->prof_step_calls = 0;
    }
    for (size_t si = 0; si < p->steps.size(); ++si) {
      h->prof_step_inst[si] = (int)p->steps[si].inst.size();
      h->prof_step_n[si] = p->steps[si].n;
    }
  }
  return THIN_ATTN_OK;
}

}  // namespace

extern "C" {

const char* thin_attn_version(void) { return "thin_attn 0.1 (sm_100a)"; }

const char* thin_attn_last_error(void) { return g_err.c_str(); }

thin_attn_status thin_attn_create(thin_attn_t* out, const thin_attn_config* cfg) {
  if (!out) return fail(THIN_ATTN_EINVAL, "out is null");
  *out = nullptr;
  thin_attn_status s = check_cfg(cfg);
  if (s != THIN_ATTN_OK) return s;
  thin_attn_s* h = new thin_attn_s();
  h->cfg = *cfg;
  h->scale = cfg->scale > 0.f ? cfg->scale : (float)(1.0 / std::sqrt((double)cfg->E));
  *out = h;
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_destroy(thin_attn_t h) {
  if (!h) return THIN_ATTN_OK;
  const bool on_device = h->d_status || h->st_mem || h->side || h->main || h->hp_in || !h->prof_free.empty() ||
                         !h->prof_pending.empty();
  DeviceGuard dg(on_device ? h->cfg.device : -1);
  for (auto& kv : h->plans) {
    if (kv.second->d_mem) cudaFree(kv.second->d_mem);
    delete kv.second;
  }
  if (h->d_status) cudaFree(h->d_status);
  if (h->st_mem) cudaFree(h->st_mem);
  for (auto& pe : h->prof_pending)
    for (auto e : pe.ev) cudaEventDestroy(e);
  for (auto& ev : h->prof_free)
    for (auto e : ev) cudaEventDestroy(e);
  for (auto e : h->ev_dep) cudaEventDestroy(e);
  for (auto e : {h->ev_join, h->ev_join2, h->ev_fork})
    if (e) cudaEventDestroy(e);
  if (h->side) cudaStreamDestroy(h->side);
  if (h->main) cudaStreamDestroy(h->main);
  for (auto sub : h->hp_sub) thin_attn_destroy(sub);
  for (auto e : h->hp_ev) cudaEventDestroy(e);
  for (auto st : {h->hp_in, h->hp_comp, h->hp_out})
    if (st) cudaStreamDestroy(st);
  delete h;
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_sched_layout(thin_attn_t h, int causal, int g, int32_t* entry, int32_t* pred_off,
                                       int32_t* preds, size_t max_items, size_t max_preds, size_t* n_items,
                                       size_t* n_preds) {
  if (!h || !n_items || !n_preds) return fail(THIN_ATTN_EINVAL, "null argument");
  std::lock_guard<std::mutex> lk(h->mu);
  Plan* p = nullptr;
  thin_attn_status s = get_plan(h, causal, g, &p);
  if (s != THIN_ATTN_OK) return s;
  const size_t ni = p->sched_items.size(), np = p->sched_preds.size();
  *n_items = ni;
  *n_preds = np;
  if (max_items < ni || max_preds < np) return THIN_ATTN_OK;   // sizes only
  if ((ni && (!entry || !pred_off)) || (np && !preds)) return fail(THIN_ATTN_EINVAL, "null array");
  // first trace entry of every step (copy steps have none)
  std::vector<int64_t> first(p->steps.size(), -1);
  int64_t e = 0;
  for (size_t si = 0; si < p->steps.size(); ++si) {
    if (p->steps[si].copy_only) continue;
    first[si] = e;
    e += (int64_t)p->steps[si].inst.size();
  }
  for (size_t i = 0; i < ni; ++i) {
    const int2 it = p->sched_items[i];
    entry[i] = (int32_t)(first[p->sched_s0 + it.x] + it.y);
    pred_off[i] = p->sched_pred_off[i];
  }
  if (ni) pred_off[ni] = p->sched_pred_off[ni];
  for (size_t i = 0; i < np; ++i) preds[i] = p->sched_preds[i];
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_plan(thin_attn_t h, int causal, int g, thin_attn_plan_info* info) {
  if (!h || !info) return fail(THIN_ATTN_EINVAL, "null argument");
  std::lock_guard<std::mutex> lk(h->mu);
  Plan* p = nullptr;
  thin_attn_status s = get_plan(h, causal, g, &p);
  if (s != THIN_ATTN_OK) return s;
  std::memset(info, 0, sizeof *info);
  info->levels = p->sz.r;
  info->leaf = p->sz.L;
  info->subsampled = p->sz.S_sub;
  info->coreset_rows = causal ? p->c : (p->sz.r > 0 ? p->sz.C : h->cfg.S);
  info->n_batches = p->n_b;
  info->n_nodes = p->n_slots;
  info->n_halvings = (int)p->trace.size();
  int launches = 1;
  const bool sched = p->sched_s1 > p->sched_s0 && std::getenv("THIN_ATTN_SIMT_GRAM") == nullptr &&
                     std::getenv("THIN_ATTN_LEVELWISE") == nullptr;
  for (int si = 0; si < (int)p->steps.size(); ++si)
    if (!sched || si < p->sched_s0 || si >= p->sched_s1) launches += step_launches(h->cfg, p, p->steps[si]);
  if (sched) launches += 1;
  info->kernel_launches = launches;
  {
    const AttnTables& at = !p->tc.tiles.empty() ? p->tc : p->simt;
    int rows = 0;
    for (const AttnTile& tl : at.tiles) rows += tl.qlen;
    info->attn_rows = rows;
  }
  info->trace_words = p->trace_words;
  info->coreset_idx_elems = p->coreset_idx_elems;
  info->workspace_bytes = p->bytes;
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_reserve(thin_attn_t h, int causal, int g) {
  if (!h) return fail(THIN_ATTN_EINVAL, "null handle");
  std::lock_guard<std::mutex> lk(h->mu);
  DeviceGuard dg(h->cfg.device);
  Plan* p = nullptr;
  thin_attn_status s = get_plan(h, causal, g, &p);
  if (s != THIN_ATTN_OK) return s;
  return materialise(h, p);
}

thin_attn_status thin_attn_trace_layout(thin_attn_t h, int causal, int g, thin_attn_trace_entry* entries,
                                        size_t capacity, size_t* count) {
  if (!h || !count) return fail(THIN_ATTN_EINVAL, "null argument");
  std::lock_guard<std::mutex> lk(h->mu);
  Plan* p = nullptr;
  thin_attn_status s = get_plan(h, causal, g, &p);
  if (s != THIN_ATTN_OK) return s;
  *count = p->trace.size();
  if (entries)
    std::memcpy(entries, p->trace.data(), std::min(capacity, p->trace.size()) * sizeof(thin_attn_trace_entry));
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_forward(thin_attn_t h, const void* q, const void* k, const void* v, void* out,
                                   int causal, int g, uint64_t seed, float* lse_opt, int32_t* coreset_idx_opt,
                                   uint32_t* trace_opt, void* stream) {
  if (!h) return fail(THIN_ATTN_EINVAL, "null handle");
  if (!q || !k || !v || !out) return fail(THIN_ATTN_EINVAL, "q, k, v and out must be non-null");
  for (const void* ptr : {q, k, v, (const void*)out})
    if (((uintptr_t)ptr) % 16) return fail(THIN_ATTN_EINVAL, "tensor pointers must be 16-byte aligned");
  std::lock_guard<std::mutex> lk(h->mu);
  DeviceGuard dg(h->cfg.device);
  if (!dg.ok) return fail(THIN_ATTN_ECUDA, "cannot select device %d", h->cfg.device);
  Plan* p = nullptr;
  thin_attn_status s = get_plan(h, causal, g, &p);
  if (s != THIN_ATTN_OK) return s;
  s = materialise(h, p);
  if (s != THIN_ATTN_OK) return s;
  if (h->cfg.thin_split)
    return fail(THIN_ATTN_EINVAL, "a thin_split handle forwards in two phases (thin_attn_forward_phase)");
  return run_forward(h, p, q, k, v, out, seed, lse_opt, coreset_idx_opt, trace_opt, (cudaStream_t)stream);
}

thin_attn_status thin_attn_forward_phase(thin_attn_t h, const void* q, const void* k, const void* v, void* out,
                                         int causal, int g, uint64_t seed, float* lse_opt, int32_t* coreset_idx_opt,
                                         uint32_t* trace_opt, int phase, void* stream) {
  if (!h) return fail(THIN_ATTN_EINVAL, "null handle");
  if (!h->cfg.thin_split || causal != 1) return fail(THIN_ATTN_EINVAL, "phases need a thin_split handle and causal = 1");
  if (phase != 1 && phase != 2) return fail(THIN_ATTN_EINVAL, "phase %d: 1 (thinning) or 2 (merges and attention)", phase);
  if (!q || !k || !v || !out) return fail(THIN_ATTN_EINVAL, "q, k, v and out must be non-null");
  for (const void* ptr : {q, k, v, (const void*)out})
    if (((uintptr_t)ptr) % 16) return fail(THIN_ATTN_EINVAL, "tensor pointers must be 16-byte aligned");
  std::lock_guard<std::mutex> lk(h->mu);
  DeviceGuard dg(h->cfg.device);
  if (!dg.ok) return fail(THIN_ATTN_ECUDA, "cannot select device %d", h->cfg.device);
  Plan* p = nullptr;
  thin_attn_status s = get_plan(h, causal, g, &p);
  if (s != THIN_ATTN_OK) return s;
  s = materialise(h, p);
  if (s != THIN_ATTN_OK) return s;
  return run_forward(h, p, q, k, v, out, seed, lse_opt, coreset_idx_opt, trace_opt, (cudaStream_t)stream, phase);
}

thin_attn_status thin_attn_nodes_layout(thin_attn_t h, int causal, int g, int* own_begin, int* own_end, int* n_batches,
                                        uint64_t* bytes_per_batch) {
  if (!h || !own_begin || !own_end || !n_batches || !bytes_per_batch) return fail(THIN_ATTN_EINVAL, "null argument");
  if (causal != 1) return fail(THIN_ATTN_EINVAL, "batch coresets exist for causal = 1 only");
  std::lock_guard<std::mutex> lk(h->mu);
  Plan* p = nullptr;
  thin_attn_status s = get_plan(h, causal, g, &p);
  if (s != THIN_ATTN_OK) return s;
  const thin_attn_config& cf = h->cfg;
  *own_begin = p->own_k0;
  *own_end = p->own_k1;
  *n_batches = p->n_b;
  *bytes_per_batch = (uint64_t)cf.B * cf.H * p->c * ((uint64_t)(cf.E + cf.D) * elt(cf) + 4);
  return THIN_ATTN_OK;
}

}  // extern "C"

namespace {

// The level-0 nodes of batches [k0, k1) to or from exchange blocks (see thin_attn_nodes_layout): per
// batch, keys, values and token indices of every (b,h), each section (b,h)-major.
thin_attn_status nodes_copy(thin_attn_s* h, int causal, int g, void* blocks, int k0, int k1, bool to_blocks,
                            cudaStream_t st) {
  std::lock_guard<std::mutex> lk(h->mu);
  DeviceGuard dg(h->cfg.device);
  if (!dg.ok) return fail(THIN_ATTN_ECUDA, "cannot select device %d", h->cfg.device);
  Plan* p = nullptr;
  thin_attn_status s = get_plan(h, causal, g, &p);
  if (s != THIN_ATTN_OK) return s;
  s = materialise(h, p);
  if (s != THIN_ATTN_OK) return s;
  if (k0 < 0 || k1 > p->n_b || k0 > k1) return fail(THIN_ATTN_EINVAL, "batches [%d, %d) outside [0, %d)", k0, k1, p->n_b);
  if (((uintptr_t)blocks) % 16) return fail(THIN_ATTN_EINVAL, "the exchange buffer must be 16-byte aligned");
  const thin_attn_config& cf = h->cfg;
  const size_t es = elt(cf), BH = (size_t)cf.B * cf.H, c = p->c;
  const void *nk, *nv;
  int32_t* nidx;
  buf_ptrs(p, BUF_NODES, nullptr, nullptr, &nk, &nv, &nidx);
  const size_t kw = c * cf.E * es, vw = c * cf.D * es, iw = c * 4;   // bytes of one (b,h)'s node
  const size_t block = BH * (kw + vw + iw);
  const size_t slots = (size_t)p->n_slots;
  for (int kb = k0; kb < k1; ++kb) {
    char* blk = (char*)blocks + (size_t)(kb - k0) * block;
    struct Sec { char* node; size_t w; char* b; } secs[3] = {
        {(char*)nk + (size_t)kb * kw, kw, blk}, {(char*)nv + (size_t)kb * vw, vw, blk + BH * kw},
        {(char*)nidx + (size_t)kb * iw, iw, blk + BH * (kw + vw)}};
    for (const Sec& x : secs) {
      // node rows of batch kb for every (b,h): pitch = one (b,h)'s node slots
      if (to_blocks)
        CK(cudaMemcpy2DAsync(x.b, x.w, x.node, slots * x.w, x.w, BH, cudaMemcpyDeviceToDevice, st));
      else
        CK(cudaMemcpy2DAsync(x.node, slots * x.w, x.b, x.w, x.w, BH, cudaMemcpyDeviceToDevice, st));
    }
  }
  return THIN_ATTN_OK;
}

}  // namespace

extern "C" {

thin_attn_status thin_attn_nodes_export(thin_attn_t h, int causal, int g, void* dst, void* stream) {
  if (!h || !dst) return fail(THIN_ATTN_EINVAL, "null argument");
  if (causal != 1) return fail(THIN_ATTN_EINVAL, "batch coresets exist for causal = 1 only");
  int k0 = 0, k1 = 0, nb = 0;
  uint64_t bpb = 0;
  thin_attn_status s = thin_attn_nodes_layout(h, causal, g, &k0, &k1, &nb, &bpb);
  if (s != THIN_ATTN_OK) return s;
  return nodes_copy(h, causal, g, dst, k0, k1, true, (cudaStream_t)stream);
}

thin_attn_status thin_attn_nodes_import(thin_attn_t h, int causal, int g, const void* src, int batch_begin,
                                        int batch_end, void* stream) {
  if (!h || !src) return fail(THIN_ATTN_EINVAL, "null argument");
  if (causal != 1) return fail(THIN_ATTN_EINVAL, "batch coresets exist for causal = 1 only");
  return nodes_copy(h, causal, g, (void*)src, batch_begin, batch_end, false, (cudaStream_t)stream);
}

}  // extern "C"

namespace {

constexpr size_t kHostPipelineMin = 64u << 20;  // input bytes from which the host path pipelines

// Shards of the pipelined host path: 8 or 4 groups of heads, else of batch rows (0: no pipeline).
// The copy-in bounds the pipeline; more shards shorten the tail (the last shard's compute and
// copy-out).
void host_groups(const thin_attn_config& c, int* groups, bool* by_heads) {
  *groups = 0;
  *by_heads = true;
  for (int ng : {8, 4})
    if (c.H % ng == 0) {
      *groups = ng;
      return;
    }
  *by_heads = false;
  for (int ng : {8, 4})
    if (c.B % ng == 0) {
      *groups = ng;
      return;
    }
}

// Set up the pipelined host path once: one handle per group, each a shard (b0, h0, H_total) of this
// handle's problem, so their random streams, and so every output, are this handle's; three
// non-blocking streams and their events.
thin_attn_status host_pipeline_setup(thin_attn_s* h) {
  if (!h->hp_sub.empty()) return THIN_ATTN_OK;
  const thin_attn_config& c = h->cfg;
  int NG;
  bool by_heads;
  host_groups(c, &NG, &by_heads);
  const int Ht = c.H_total > 0 ? c.H_total : c.H;
  // all or nothing: everything is made first and kept only if every piece was made
  std::vector<thin_attn_s*> subs;
  std::vector<cudaEvent_t> evs;
  cudaStream_t sts[3] = {nullptr, nullptr, nullptr};
  auto undo = [&]() {
    for (auto sub : subs) thin_attn_destroy(sub);
    for (auto e : evs) cudaEventDestroy(e);
    for (auto st : sts)
      if (st) cudaStreamDestroy(st);
  };
  for (int gi = 0; gi < NG; ++gi) {
    thin_attn_config sc = c;
    if (by_heads) {
      sc.H = c.H / NG;
      sc.h0 = c.h0 + gi * sc.H;
    } else {
      sc.B = c.B / NG;
      sc.b0 = c.b0 + gi * sc.B;
    }
    sc.H_total = Ht;
    thin_attn_t sub = nullptr;
    thin_attn_status s = thin_attn_create(&sub, &sc);
    if (s != THIN_ATTN_OK) {
      undo();
      return s;
    }
    subs.push_back(sub);
  }
  DeviceGuard dg(c.device);
  for (auto& st : sts)
    if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) {
      st = nullptr;
      undo();
      return fail(THIN_ATTN_ECUDA, "host pipeline: %s", cudaGetErrorString(cudaGetLastError()));
    }
  for (int i = 0; i < 3 * NG + 1; ++i) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      undo();
      return fail(THIN_ATTN_ECUDA, "host pipeline: %s", cudaGetErrorString(cudaGetLastError()));
    }
    evs.push_back(e);
  }
  h->hp_sub = subs;
  h->hp_ev = evs;
  h->hp_in = sts[0];
  h->hp_comp = sts[1];
  h->hp_out = sts[2];
  h->hp_groups = NG;
  h->hp_by_heads = by_heads;
  return THIN_ATTN_OK;
}

}  // namespace

extern "C" {

thin_attn_status thin_attn_forward_host(thin_attn_t h, const void* q, const void* k, const void* v, void* out,
                                        int causal, int g, uint64_t seed, float* lse_opt, void* stream) {
  if (!h) return fail(THIN_ATTN_EINVAL, "null handle");
  if (!q || !k || !v || !out) return fail(THIN_ATTN_EINVAL, "q, k, v and out must be non-null");
  const thin_attn_config& c = h->cfg;
  if (c.q_begin != 0 || c.q_end != 0)
    return fail(THIN_ATTN_EUNSUPPORTED, "the host-buffer forward takes no query-row range (q_begin, q_end)");
  const size_t es = elt(c);
  const int64_t L = causal ? c.T : c.S;
  const size_t qb = (size_t)c.B * c.T * c.H * c.E * es, kb = (size_t)c.B * L * c.H * c.E * es,
               vb = (size_t)c.B * L * c.H * c.D * es, ob = (size_t)c.B * c.T * c.H * c.D * es,
               lb = (size_t)c.B * c.H * c.T * 4;
  cudaStream_t st = (cudaStream_t)stream;
  // Large problems run as shards in a pipeline: the copy-in of group i+1 and the copy-out of group
  // i-1 overlap the compute of group i (double-buffered staging).
  int groups;
  bool by_heads;
  host_groups(c, &groups, &by_heads);
  const bool pipeline = qb + kb + vb >= kHostPipelineMin && groups > 0;
  const int NG = pipeline ? groups : 1;
  const size_t gq = qb / NG, gk = kb / NG, gv = vb / NG, go = ob / NG, gl = lb / NG;
  const size_t slot = align256(gq) + align256(gk) + align256(gv) + align256(go) + align256(gl);
  const size_t need = (pipeline ? 2 : 1) * slot;
  {
    std::lock_guard<std::mutex> lk(h->mu);
    DeviceGuard dg(c.device);
    if (h->st_bytes < need) {
      if (h->st_mem) cudaFree(h->st_mem);
      h->st_mem = nullptr;
      h->st_bytes = 0;
      if (cudaMalloc(&h->st_mem, need) != cudaSuccess) {
        cudaGetLastError();
        return fail(THIN_ATTN_ENOMEM, "host-path staging of %zu bytes", need);
      }
      h->st_bytes = need;
    }
    if (pipeline) {
      thin_attn_status s = host_pipeline_setup(h);
      if (s != THIN_ATTN_OK) return s;
    }
  }
  auto slot_ptrs = [&](int sl, char** dq, char** dk, char** dv, char** dout, char** dl) {
    char* base = (char*)h->st_mem + sl * slot;
    *dq = base;
    *dk = *dq + align256(gq);
    *dv = *dk + align256(gk);
    *dout = *dv + align256(gv);
    *dl = *dout + align256(go);
  };
  DeviceGuard dg(c.device);
  if (!pipeline) {
    char *dq, *dk, *dv, *dout, *dl;
    slot_ptrs(0, &dq, &dk, &dv, &dout, &dl);
    CK(cudaMemcpyAsync(dq, q, qb, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(dk, k, kb, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(dv, v, vb, cudaMemcpyHostToDevice, st));
    thin_attn_status s = thin_attn_forward(h, dq, dk, dv, dout, causal, g, seed, lse_opt ? (float*)dl : nullptr,
                                           nullptr, nullptr, stream);
    if (s != THIN_ATTN_OK) return s;
    CK(cudaMemcpyAsync(out, dout, ob, cudaMemcpyDeviceToHost, st));
    if (lse_opt) CK(cudaMemcpyAsync(lse_opt, dl, lb, cudaMemcpyDeviceToHost, st));
    CK(cudaStreamSynchronize(st));
    return THIN_ATTN_OK;
  }
  // group gi: heads [gi G, (gi+1) G) of every (b, t) row -- a 2-D copy with the row pitch of the
  // whole tensor -- or batch rows [gi B', (gi+1) B') -- a contiguous range
  const int Gh = c.H / NG, Gb = c.B / NG;
  auto copy = [&](void* dst, const void* src, size_t row_elems, int64_t rows, int gi, bool to_dev, cudaStream_t s2) {
    const size_t full = row_elems * es;   // bytes of one (b, t) row of the whole tensor
    if (h->hp_by_heads) {
      const size_t w = full / NG, off = (size_t)gi * w;
      return to_dev ? cudaMemcpy2DAsync(dst, w, (const char*)src + off, full, w, rows, cudaMemcpyHostToDevice, s2)
                    : cudaMemcpy2DAsync((char*)dst + off, full, src, w, w, rows, cudaMemcpyDeviceToHost, s2);
    }
    const size_t bytes = full * rows / NG, off = (size_t)gi * bytes;
    return to_dev ? cudaMemcpyAsync(dst, (const char*)src + off, bytes, cudaMemcpyHostToDevice, s2)
                  : cudaMemcpyAsync((char*)dst + off, src, bytes, cudaMemcpyDeviceToHost, s2);
  };
  cudaEvent_t* ev = h->hp_ev.data();
  cudaEvent_t ev_start = ev[3 * NG];
  CK(cudaEventRecord(ev_start, st));
  for (cudaStream_t s2 : {h->hp_in, h->hp_comp, h->hp_out}) CK(cudaStreamWaitEvent(s2, ev_start, 0));
  for (int gi = 0; gi < NG; ++gi) {
    char *dq, *dk, *dv, *dout, *dl;
    slot_ptrs(gi & 1, &dq, &dk, &dv, &dout, &dl);
    cudaEvent_t in_done = ev[3 * gi], comp_done = ev[3 * gi + 1], out_done = ev[3 * gi + 2];
    // the slot's inputs are free once group gi-2 has computed
    if (gi >= 2) CK(cudaStreamWaitEvent(h->hp_in, ev[3 * (gi - 2) + 1], 0));
    const int64_t rows_q = (int64_t)c.B * c.T;
    const int64_t rows_kv = (int64_t)c.B * L;
    CK(copy(dq, q, (size_t)c.H * c.E, rows_q, gi, true, h->hp_in));
    CK(copy(dk, k, (size_t)c.H * c.E, rows_kv, gi, true, h->hp_in));
    CK(copy(dv, v, (size_t)c.H * c.D, rows_kv, gi, true, h->hp_in));
    CK(cudaEventRecord(in_done, h->hp_in));
    // compute once the inputs are in and the slot's outputs of group gi-2 are out
    CK(cudaStreamWaitEvent(h->hp_comp, in_done, 0));
    if (gi >= 2) CK(cudaStreamWaitEvent(h->hp_comp, ev[3 * (gi - 2) + 2], 0));
    thin_attn_status s = thin_attn_forward(h->hp_sub[gi], dq, dk, dv, dout, causal, g, seed,
                                           lse_opt ? (float*)dl : nullptr, nullptr, nullptr, h->hp_comp);
    if (s != THIN_ATTN_OK) return s;
    CK(cudaEventRecord(comp_done, h->hp_comp));
    CK(cudaStreamWaitEvent(h->hp_out, comp_done, 0));
    CK(copy(out, dout, (size_t)c.H * c.D, (int64_t)c.B * c.T, gi, false, h->hp_out));
    if (lse_opt) {
      // lse (B, H, T): group gi holds heads [gi G, (gi+1) G) of every b, or batch rows of it
      if (h->hp_by_heads)
        CK(cudaMemcpy2DAsync(lse_opt + (size_t)gi * Gh * c.T, (size_t)c.H * c.T * 4, dl, (size_t)Gh * c.T * 4,
                             (size_t)Gh * c.T * 4, c.B, cudaMemcpyDeviceToHost, h->hp_out));
      else
        CK(cudaMemcpyAsync(lse_opt + (size_t)gi * Gb * c.H * c.T, dl, gl, cudaMemcpyDeviceToHost, h->hp_out));
    }
    CK(cudaEventRecord(out_done, h->hp_out));
  }
  CK(cudaStreamWaitEvent(st, ev[3 * (NG - 1) + 2], 0));
  CK(cudaStreamSynchronize(st));
  // a bounded wait that gave up in a group's kernels is reported here, like thin_attn_check would
  for (auto sub : h->hp_sub) {
    thin_attn_status s = thin_attn_check(sub, st);
    if (s != THIN_ATTN_OK) return s;
  }
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_profile(thin_attn_t h, int enable) {
  if (!h) return fail(THIN_ATTN_EINVAL, "null handle");
  std::lock_guard<std::mutex> lk(h->mu);
  h->prof_on = enable != 0;
  return THIN_ATTN_OK;
}

}  // extern "C"

namespace {
// Wait for the recorded forwards and add their times to the phase and step sums (lock held).
thin_attn_status drain_profile(thin_attn_s* h) {
  DeviceGuard dg(h->prof_pending.empty() ? -1 : h->cfg.device);
  for (auto& pe : h->prof_pending) {
    auto& ev = pe.ev;
    CK(cudaEventSynchronize(ev[3]));
    float t;
    CK(cudaEventElapsedTime(&t, ev[0], ev[1]));
    h->prof_ms[0] += t;
    CK(cudaEventElapsedTime(&t, ev[1], ev[2]));
    h->prof_ms[1] += t;
    const size_t first_step = 4 + 2 * pe.waves;
    for (size_t w = 0; w < pe.waves; ++w) {
      CK(cudaEventElapsedTime(&t, ev[4 + 2 * w], ev[5 + 2 * w]));
      h->prof_ms[2] += t;
    }
    for (size_t si = 0; si < h->prof_step_ms.size() && first_step + si < ev.size(); ++si) {
      // a group's steps share the event recorded after it: its whole time goes on its first step
      if ((int)si > pe.group0 && (int)si < pe.group1) continue;
      const size_t end = (int)si == pe.group0 && pe.group1 > pe.group0 ? (size_t)pe.group1 - 1 : si;
      CK(cudaEventElapsedTime(&t, si ? ev[first_step + si - 1] : ev[0], ev[first_step + end]));
      h->prof_step_ms[si] += t;
    }
    CK(cudaEventElapsedTime(&t, ev[0], ev[3]));
    h->prof_total += t;
    h->prof_calls += 1;
    h->prof_step_calls += 1;
    h->prof_free.push_back(ev);
  }
  h->prof_pending.clear();
  return THIN_ATTN_OK;
}
}  // namespace

extern "C" {

thin_attn_status thin_attn_profile_steps(thin_attn_t h, int max_steps, double* ms, int* n_inst, int* n_points,
                                         int* n_steps, int* calls) {
  if (!h || !n_steps || !calls || max_steps < 0 || (max_steps > 0 && (!ms || !n_inst || !n_points)))
    return fail(THIN_ATTN_EINVAL, "null argument");
  std::lock_guard<std::mutex> lk(h->mu);
  thin_attn_status s = drain_profile(h);
  if (s != THIN_ATTN_OK) return s;
  const int ns = (int)h->prof_step_ms.size();
  for (int i = 0; i < ns && i < max_steps; ++i) {
    ms[i] = h->prof_step_ms[i];
    n_inst[i] = h->prof_step_inst[i];
    n_points[i] = h->prof_step_n[i];
    h->prof_step_ms[i] = 0;
  }
  *n_steps = ns;
  *calls = h->prof_step_calls;
  h->prof_step_calls = 0;
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_profile_read(thin_attn_t h, double* ms, int* calls) {
  if (!h || !ms || !calls) return fail(THIN_ATTN_EINVAL, "null argument");
  std::lock_guard<std::mutex> lk(h->mu);
  thin_attn_status s = drain_profile(h);
  if (s != THIN_ATTN_OK) return s;
  for (int i = 0; i < 3; ++i) ms[i] = h->prof_ms[i];
  ms[3] = h->prof_total;
  *calls = h->prof_calls;
  h->prof_ms[0] = h->prof_ms[1] = h->prof_ms[2] = h->prof_total = 0;
  h->prof_calls = 0;
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_check(thin_attn_t h, void* stream) {
  if (!h) return fail(THIN_ATTN_EINVAL, "null handle");
  DeviceGuard dg(h->cfg.device);
  CK(cudaStreamSynchronize((cudaStream_t)stream));
  if (!h->d_status) return THIN_ATTN_OK;
  int st[4] = {0, 0, 0, 0};
  CK(cudaMemcpy(st, h->d_status, sizeof st, cudaMemcpyDeviceToHost));
  if (st[0] != 0) {
    CK(cudaMemset(h->d_status, 0, 16));
    if (st[0] == 7)
      return fail(THIN_ATTN_ETIMEOUT, "device wait gave up (code 7: halving scheduler, work item %d waited for its inputs)",
                  st[1]);
    if (st[0] != 1)
      return fail(THIN_ATTN_ETIMEOUT, "device wait gave up (code %d: halving kernel, instance or CTA %d)", st[0], st[1]);
    return fail(THIN_ATTN_ETIMEOUT, "device wait gave up (code %d; query tile %d of (b,h) %d; wait %d at key tile %d)",
                st[0], st[1] >> 16, st[1] & 0xFFFF, st[2] / 1000, st[2] % 1000);
  }
  return THIN_ATTN_OK;
}

}  // extern "C"

// =============================================================================================
// Express decode cache ("EXPRESS ... operates as an updatable weighted cache object", Express
// Language Modeling, "The EXPRESS Meta-Procedure").  Token t of each (b,h) is appended, attended
// exactly as query t of the prefill (exact prefix + snapshot nodes + its own batch), and when a
// batch completes it is KH-Compressed into a level-0 node and the 4-ary counter's merges run --
// with the prefill's Philox rounds and pair indices, so the nodes equal the prefill's.  Raw
// tokens are kept for the exact prefix and the one batch in progress (rows ne .. ne+b-1).
// =============================================================================================
namespace {

struct CacheStep {
  StepPlan sp;
  int src_level = -1, dst_level = -1;   // intermediate level buffers (or -1)
};

}  // namespace

struct thin_attn_cache_s {
  thin_attn_config cf{};
  int g = 0;
  uint64_t seed = 0;
  float scale = 0.f;
  int ne = 0, bsz = 0, L = 0, c = 0, n_bmax = 0, n_slots = 0;
  Sizes sz{};
  std::vector<int> level_base;
  std::vector<std::vector<CacheStep>> batch_steps;               // [k]
  std::map<std::pair<int, int>, std::vector<CacheStep>> merges;   // (target level, node) -> 2 steps
  std::vector<BufSpec> levels;
  BufSpec raw, nodes, mtemp;
  AttnTables tab;
  size_t delta_off = 0, c2_off = 0, delta_floats = 0, c2_floats = 0, bytes = 0;
  void* d_mem = nullptr;
  int* d_status = nullptr;
  int64_t t = 0;
  bool use_tc = false;
  // split-key decode attention: keys of every position, chunks of the largest, partials buffer
  bool use_split = false;
  std::vector<int> pos_keys;
  int max_splits = 0;
  size_t part_off = 0, arrive_off = 0;
};

namespace {

void cache_add_step(thin_attn_cache_s* cc, CacheStep& st) {
  st.sp.sub_stride = sub_stride_of(st.sp);
  for (auto& in : st.sp.inst) in.ctr_bh = ctr_bh_of(cc->cf, in.bh);
  cc->delta_floats = std::max(cc->delta_floats, st.sp.inst.size() * (size_t)st.sp.m_pad * st.sp.m_pad);
  cc->c2_floats = std::max(cc->c2_floats, st.sp.inst.size());
}

thin_attn_status cache_build(thin_attn_cache_s* cc) {
  const thin_attn_config& cf = cc->cf;
  const int BH = cf.B * cf.H, T = cf.T;
  cc->ne = std::min(cf.n_exact, T);
  cc->bsz = cf.batch;
  cc->L = cc->ne + cc->bsz;
  cc->n_bmax = T > cc->ne ? (T - cc->ne) / cc->bsz : 0;
  cc->sz = compress_sizes(cc->bsz, cc->g);
  cc->c = cc->sz.C;
  for (int lv = 0; (cc->n_bmax >> (2 * lv)) > 0; ++lv) {
    cc->level_base.push_back(cc->n_slots);
    cc->n_slots += cc->n_bmax >> (2 * lv);
  }
  const Sizes& sz = cc->sz;
  // intermediate level buffers of one batch (all (b,h))
  for (int lv = 1; lv < sz.r; ++lv) {
    BufSpec b;
    b.rows = (int64_t)BH * (sz.S_sub >> lv);
    cc->levels.push_back(b);
  }
  cc->raw.rows = (int64_t)cf.B * cc->L * cf.H;
  cc->nodes.rows = (int64_t)BH * cc->n_slots * cc->c;
  cc->mtemp.rows = (int64_t)BH * 2 * cc->c;
  for (int k = 0; k < cc->n_bmax; ++k) {
    std::vector<CacheStep> steps;
    if (sz.r == 0) {
      CacheStep st;
      st.sp.copy_only = true;
      st.sp.n = cc->bsz;
      st.sp.src_buf = BUF_TOKENS;
      st.sp.dst_buf = BUF_NODES;
      st.sp.S_full = st.sp.S_sub = cc->bsz;
      for (int bh = 0; bh < BH; ++bh) {
        HalveInst in{};
        in.src_row = (int64_t)(bh / cf.H) * cc->L + cc->ne;
        in.dst_row = ((int64_t)bh * cc->n_slots + k) * cc->c;
        in.bh = (uint32_t)bh;
        in.tok0 = (uint32_t)(cc->ne + k * cc->bsz);
        st.sp.inst.push_back(in);
      }
      steps.push_back(std::move(st));
    }
    for (int lv = 1; lv <= sz.r; ++lv) {
      CacheStep st;
      st.sp.n = 4 * sz.L * (1 << (lv - 1));
      st.sp.m = st.sp.n / 2;
      st.sp.m_pad = (st.sp.m + 31) / 32 * 32;
      const int in_rows = sz.S_sub >> (lv - 1), G = in_rows / st.sp.n, out_rows = in_rows / 2;
      st.sp.src_buf = lv == 1 ? BUF_TOKENS : 0;
      st.src_level = lv == 1 ? -1 : lv - 2;
      st.sp.dst_buf = lv == sz.r ? BUF_NODES : 0;
      st.dst_level = lv == sz.r ? -1 : lv - 1;
      st.sp.S_full = cc->bsz;
      st.sp.S_sub = sz.S_sub;
      for (int bh = 0; bh < BH; ++bh)
        for (int gi = 0; gi < G; ++gi) {
          HalveInst in{};
          in.src_row = lv == 1 ? (int64_t)(bh / cf.H) * cc->L + cc->ne : (int64_t)bh * in_rows + (int64_t)gi * st.sp.n;
          in.dst_row = (lv == sz.r ? ((int64_t)bh * cc->n_slots + k) * cc->c : (int64_t)bh * out_rows) +
                       (int64_t)gi * st.sp.m;
          in.bh = (uint32_t)bh;
          in.round_id = round_batch(k, lv);
          in.pair0 = (uint32_t)(gi * st.sp.m);
          in.sub_round = round_subsample(k);
          in.tok0 = (uint32_t)(cc->ne + k * cc->bsz);
          st.sp.inst.push_back(in);
        }
      cache_add_step(cc, st);
      steps.push_back(std::move(st));
    }
    cc->batch_steps.push_back(std::move(steps));
  }
  for (int lv = 1; (cc->n_bmax >> (2 * lv)) > 0; ++lv)
    for (int j = 0; j < (cc->n_bmax >> (2 * lv)); ++j) {
      std::vector<CacheStep> two;
      for (int step = 0; step < 2; ++step) {
        CacheStep st;
        st.sp.phase = 1;
        st.sp.merge_level = lv;
        st.sp.n = (step == 0 ? 4 : 2) * cc->c;
        st.sp.m = st.sp.n / 2;
        st.sp.m_pad = (st.sp.m + 31) / 32 * 32;
        st.sp.src_buf = step == 0 ? BUF_NODES : BUF_MTEMP;
        st.sp.dst_buf = step == 0 ? BUF_MTEMP : BUF_NODES;
        st.sp.S_full = st.sp.S_sub = st.sp.n;
        for (int bh = 0; bh < BH; ++bh) {
          HalveInst in{};
          const int64_t mt = (int64_t)bh * 2 * cc->c;
          in.src_row = step == 0 ? ((int64_t)bh * cc->n_slots + cc->level_base[lv - 1] + 4 * j) * cc->c : mt;
          in.dst_row = step == 0 ? mt : ((int64_t)bh * cc->n_slots + cc->level_base[lv] + j) * cc->c;
          in.bh = (uint32_t)bh;
          in.round_id = round_merge(lv, j, step);
          st.sp.inst.push_back(in);
        }
        cache_add_step(cc, st);
        two.push_back(std::move(st));
      }
      cc->merges[{lv, j}] = std::move(two);
    }
  // attention table: one tile (one query) per position t
  AttnTables& t = cc->tab;
  for (int pos = 0; pos < T; ++pos) {
    const int seg0 = (int)t.segs.size();
    if (pos < cc->ne) {
      t.segs.push_back({SEG_TOKENS, 0, pos + 1, 0, 0.f, 0});
    } else {
      const int k = (pos - cc->ne) / cc->bsz, tin = (pos - cc->ne) % cc->bsz;
      if (cc->ne > 0) t.segs.push_back({SEG_TOKENS, 0, cc->ne, 0, 0.f, 0});
      for (int lv = 0; ((int64_t)1 << (2 * lv)) <= k; ++lv) {
        const int64_t p4 = (int64_t)1 << (2 * lv);
        const int d = (int)((k / p4) % 4), base = (int)((k / (p4 * 4)) * 4);
        const double w = std::ldexp((double)cc->bsz / cc->c, 2 * lv);
        for (int j = 0; j < d; ++j)
          t.segs.push_back({SEG_COMPACT, cc->level_base[lv] + base + j, cc->c, 0, (float)std::log(w), 0});
      }
      t.segs.push_back({SEG_TOKENS, cc->ne, tin + 1, 0, 0.f, 0});
    }
    t.tiles.push_back({0, 1, seg0, (int)t.segs.size() - seg0});
  }
  int max_segs = 0;
  cc->pos_keys.assign(T, 0);
  for (int pos = 0; pos < T; ++pos) {
    const AttnTile& tl = t.tiles[pos];
    max_segs = std::max(max_segs, tl.nseg);
    for (int q = 0; q < tl.nseg; ++q) cc->pos_keys[pos] += t.segs[tl.seg0 + q].len;
    cc->max_splits = std::max(cc->max_splits, (cc->pos_keys[pos] + decode_chunk_keys() - 1) / decode_chunk_keys());
  }
  // split-key kernels when few (b,h) rows would leave most SMs idle with one CTA per row
  cc->use_split = decode_attention_supported(cf.E, cf.D, max_segs, cc->max_splits) && BH <= 64 &&
                  std::getenv("THIN_ATTN_DECODE_TILES") == nullptr;
  // device layout
  size_t off = 0;
  for (auto& steps : cc->batch_steps)
    for (auto& st : steps) {
      st.sp.inst_off = off;
      off = align256(off + st.sp.inst.size() * sizeof(HalveInst));
    }
  for (auto& kv : cc->merges)
    for (auto& st : kv.second) {
      st.sp.inst_off = off;
      off = align256(off + st.sp.inst.size() * sizeof(HalveInst));
    }
  t.tiles_off = off;
  off = align256(off + t.tiles.size() * sizeof(AttnTile));
  t.segs_off = off;
  off = align256(off + t.segs.size() * sizeof(AttnSeg));
  const size_t table_end = off;
  const size_t es = elt(cf);
  auto place = [&](BufSpec& b) {
    b.k_off = off;
    off = align256(off + (size_t)b.rows * cf.E * es);
    b.v_off = off;
    off = align256(off + (size_t)b.rows * cf.D * es);
    b.idx_off = off;
    off = align256(off + (size_t)b.rows * 4);
  };
  for (auto& b : cc->levels) place(b);
  place(cc->raw);
  place(cc->nodes);
  place(cc->mtemp);
  cc->delta_off = off;
  off = align256(off + cc->delta_floats * 4);
  cc->c2_off = off;
  off = align256(off + std::max<size_t>(cc->c2_floats, 1) * 4);
  cc->part_off = off;
  if (cc->use_split) off = align256(off + (size_t)cc->max_splits * BH * (cf.D + 2) * 4);
  cc->arrive_off = off;
  if (cc->use_split) off = align256(off + (size_t)BH * 4);
  cc->bytes = off;
  cudaError_t e = cudaMalloc(&cc->d_mem, cc->bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(THIN_ATTN_ENOMEM, "decode cache of %zu bytes: %s", cc->bytes, cudaGetErrorString(e));
  }
  std::vector<char> host(table_end);
  auto put = [&](const std::vector<HalveInst>& v, size_t o) {
    if (!v.empty()) std::memcpy(host.data() + o, v.data(), v.size() * sizeof(HalveInst));
  };
  for (auto& steps : cc->batch_steps)
    for (auto& st : steps) put(st.sp.inst, st.sp.inst_off);
  for (auto& kv : cc->merges)
    for (auto& st : kv.second) put(st.sp.inst, st.sp.inst_off);
  set_key_tile_counts(t);
  std::memcpy(host.data() + t.tiles_off, t.tiles.data(), t.tiles.size() * sizeof(AttnTile));
  std::memcpy(host.data() + t.segs_off, t.segs.data(), t.segs.size() * sizeof(AttnSeg));
  CK(cudaMemcpy(cc->d_mem, host.data(), table_end, cudaMemcpyHostToDevice));
  CK(cudaMalloc(&cc->d_status, kStatusBytes));
  CK(cudaMemset(cc->d_status, 0, kStatusBytes));
  CK(cudaMemset((char*)cc->d_mem + cc->nodes.idx_off, 0xFF, (size_t)cc->nodes.rows * 4));
  if (cc->use_split) CK(cudaMemset((char*)cc->d_mem + cc->arrive_off, 0, (size_t)BH * 4));
  return THIN_ATTN_OK;
}

thin_attn_status cache_run_step(thin_attn_cache_s* cc, CacheStep& st, cudaStream_t s) {
  const thin_attn_config& cf = cc->cf;
  char* base = (char*)cc->d_mem;
  auto ptrs = [&](int buf, int level, const void** K, const void** V, int32_t** I, int64_t* rows) {
    const BufSpec& b = buf == BUF_TOKENS ? cc->raw : buf == BUF_NODES ? cc->nodes : buf == BUF_MTEMP ? cc->mtemp
                                                                                     : cc->levels[level];
    *K = base + b.k_off;
    *V = base + b.v_off;
    *I = (int32_t*)(base + b.idx_off);
    *rows = buf == BUF_TOKENS ? (int64_t)cf.B * cc->L : b.rows;
  };
  StepArgs a{};
  int64_t rows = 0;
  const void *sk, *sv, *dk, *dv;
  int32_t *sidx, *didx;
  int64_t drows;
  ptrs(st.sp.src_buf, st.src_level, &sk, &sv, &sidx, &rows);
  ptrs(st.sp.dst_buf, st.dst_level, &dk, &dv, &didx, &drows);
  a.src_kind = st.sp.src_buf == BUF_TOKENS ? SRC_TOKENS : SRC_COMPACT;
  a.srcK = sk;
  a.srcV = sv;
  a.srcIdx = st.sp.src_buf == BUF_TOKENS ? nullptr : sidx;
  a.H = cf.H;
  a.src_rows = rows;
  a.S_full = st.sp.S_full;
  a.S_sub = st.sp.S_sub;
  a.sub_stride = st.sp.sub_stride;
  a.dstK = (void*)dk;
  a.dstV = (void*)dv;
  a.dstIdx = didx;
  a.inst = (const HalveInst*)(base + st.sp.inst_off);
  a.n_inst = (int)st.sp.inst.size();
  a.n = st.sp.n;
  a.m = st.sp.m;
  a.m_pad = st.sp.m_pad;
  a.E = cf.E;
  a.D = cf.D;
  a.scale_log2e = (float)((double)cc->scale * 1.4426950408889634);
  a.C = st.sp.m > 0 ? (float)std::sqrt(2.0 * std::log(4.0 * st.sp.m)) : 0.f;
  a.seed = cc->seed;
  a.c2 = (float*)(base + cc->c2_off);
  a.delta = (float*)(base + cc->delta_off);
  a.status = cc->d_status;
  cudaError_t e = st.sp.copy_only ? launch_copy_step(a, cf.dtype, s) : launch_halving_step(a, cf.dtype, true, s);
  if (e != cudaSuccess) return fail(THIN_ATTN_ECUDA, "cache halving step (n=%d): %s", st.sp.n, cudaGetErrorString(e));
  return THIN_ATTN_OK;
}

}  // namespace

extern "C" {

thin_attn_status thin_attn_cache_create(thin_attn_cache_t* out, const thin_attn_config* cfg, int g, uint64_t seed) {
  if (!out) return fail(THIN_ATTN_EINVAL, "out is null");
  *out = nullptr;
  thin_attn_status s = check_cfg(cfg);
  if (s != THIN_ATTN_OK) return s;
  if (g < 0 || g > 6) return fail(THIN_ATTN_EINVAL, "g=%d outside 0..6", g);
  if (cfg->batch < 1 || cfg->n_exact < 0) return fail(THIN_ATTN_EINVAL, "the cache needs batch >= 1 and n_exact >= 0");
  if (cfg->q_begin != 0 || cfg->q_end != 0) return fail(THIN_ATTN_EINVAL, "the decode cache takes no query-row range");
  DeviceGuard dg(cfg->device);
  if (!dg.ok) return fail(THIN_ATTN_ECUDA, "cannot select device %d", cfg->device);
  thin_attn_cache_s* cc = new thin_attn_cache_s();
  cc->cf = *cfg;
  cc->cf.S = cfg->T;
  cc->g = g;
  cc->seed = seed;
  cc->scale = cfg->scale > 0.f ? cfg->scale : (float)(1.0 / std::sqrt((double)cfg->E));
  cc->use_tc = attention_tc_supported(cfg->dtype, cfg->E, cfg->D) && tensor_maps_available();
  s = cache_build(cc);
  if (s != THIN_ATTN_OK) {
    thin_attn_cache_destroy(cc);
    return s;
  }
  for (const auto& steps : cc->batch_steps)
    for (const auto& st : steps)
      if (!st.sp.copy_only && st.sp.m_pad > 2048) {
        thin_attn_cache_destroy(cc);
        return fail(THIN_ATTN_EUNSUPPORTED, "halving instance of %d points exceeds 4096", st.sp.n);
      }
  *out = cc;
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_cache_destroy(thin_attn_cache_t c) {
  if (!c) return THIN_ATTN_OK;
  DeviceGuard dg(c->d_mem || c->d_status ? c->cf.device : -1);
  if (c->d_mem) cudaFree(c->d_mem);
  if (c->d_status) cudaFree(c->d_status);
  delete c;
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_cache_length(thin_attn_cache_t c, int64_t* t) {
  if (!c || !t) return fail(THIN_ATTN_EINVAL, "null argument");
  *t = c->t;
  return THIN_ATTN_OK;
}

}  // extern "C"

namespace {
// One decoded token of every (b,h).  q, k, v, out point at the token's row of batch entry 0; entry b
// is `bstride` token rows further on (1 for (B,1,H,.) tensors, n for (B,n,H,.) ones); lse, if given,
// at the token's column of (b,h) 0, (b,h) i at lse + i * bstride.
thin_attn_status cache_decode_one(thin_attn_cache_s* c, const void* q, const void* k, const void* v, void* out,
                                  float* lse_opt, int64_t bstride, cudaStream_t st) {
  const thin_attn_config& cf = c->cf;
  if (c->t >= cf.T) return fail(THIN_ATTN_EINVAL, "the cache holds its capacity of %d tokens", cf.T);
  const int64_t pos = c->t;
  const size_t es = elt(cf);
  char* base = (char*)c->d_mem;
  // 1. the new key/value row: exact prefix row pos, or row ne + (pos - ne) mod b of the batch region
  const int64_t r = pos < c->ne ? pos : c->ne + (pos - c->ne) % c->bsz;
  if (!c->use_split) {   // (the split-key kernel reads the new row from k, v and appends it itself)
    const size_t krow = (size_t)cf.H * cf.E * es, vrow = (size_t)cf.H * cf.D * es;
    CK(cudaMemcpy2DAsync(base + c->raw.k_off + (size_t)r * krow, (size_t)c->L * krow, k, krow * bstride, krow, cf.B,
                         cudaMemcpyDeviceToDevice, st));
    CK(cudaMemcpy2DAsync(base + c->raw.v_off + (size_t)r * vrow, (size_t)c->L * vrow, v, vrow * bstride, vrow, cf.B,
                         cudaMemcpyDeviceToDevice, st));
  }
  // 2. attention of query pos against the cache as it stands (its own token included)
  AttnArgs aa{};
  aa.q = q;
  aa.k = base + c->raw.k_off;
  aa.v = base + c->raw.v_off;
  aa.ck = base + c->nodes.k_off;
  aa.cv = base + c->nodes.v_off;
  aa.out = out;
  aa.lse = lse_opt;
  aa.tiles = (const AttnTile*)(base + c->tab.tiles_off);
  aa.segs = (const AttnSeg*)(base + c->tab.segs_off);
  aa.tile0 = (int)pos;
  aa.n_tiles = 1;
  aa.B = cf.B;
  aa.T = (int)bstride;   // the query (and output) rows of batch entries b are bstride rows apart
  aa.L = c->L;
  aa.H = cf.H;
  aa.E = cf.E;
  aa.D = cf.D;
  aa.n_slots = std::max(1, c->n_slots);
  aa.slot_rows = c->c;
  aa.scale_log2e = (float)((double)c->scale * 1.4426950408889634);
  bool done = false;
  cudaError_t e = cudaSuccess;
  if (c->use_split) {
    const int n_splits = (c->pos_keys[pos] + decode_chunk_keys() - 1) / decode_chunk_keys();
    DecodeAppend ap;
    ap.new_k = k;
    ap.new_v = v;
    ap.row = (int)r;
    ap.arrive = (int*)(base + c->arrive_off);
    const AttnTile& tl = c->tab.tiles[pos];
    if (tl.nseg <= 32) {
      ap.nseg = tl.nseg;
      for (int s2 = 0; s2 < tl.nseg; ++s2) ap.segs[s2] = c->tab.segs[tl.seg0 + s2];
    }
    e = launch_decode_attention(aa, cf.dtype, n_splits, (float*)(base + c->part_off), ap, st);
    done = true;
  } else if (bstride != 1) {
    return fail(THIN_ATTN_EUNSUPPORTED, "several tokens per call need the split-key decode (B*H <= 64)");
  }
  if (e == cudaSuccess && !done && c->use_tc) e = launch_attention_tc(aa, c->d_status, st, &done);
  if (e == cudaSuccess && !done) e = launch_attention_simt(aa, cf.dtype, st);
  if (e != cudaSuccess) return fail(THIN_ATTN_ECUDA, "cache attention: %s", cudaGetErrorString(e));
  // 3. a completed batch becomes a level-0 node; the 4-ary counter merges equal levels
  if (pos >= c->ne && (pos - c->ne + 1) % c->bsz == 0) {
    const int kb = (int)((pos - c->ne) / c->bsz);
    for (auto& stp : c->batch_steps[kb]) {
      thin_attn_status s = cache_run_step(c, stp, st);
      if (s != THIN_ATTN_OK) return s;
    }
    const int64_t done_batches = kb + 1;
    for (int lv = 1; done_batches % ((int64_t)1 << (2 * lv)) == 0; ++lv) {
      const int j = (int)(done_batches >> (2 * lv)) - 1;
      auto it = c->merges.find({lv, j});
      if (it == c->merges.end()) break;
      for (auto& stp : it->second) {
        thin_attn_status s = cache_run_step(c, stp, st);
        if (s != THIN_ATTN_OK) return s;
      }
    }
  }
  c->t = pos + 1;
  return THIN_ATTN_OK;
}
}  // namespace

extern "C" {

thin_attn_status thin_attn_cache_decode(thin_attn_cache_t c, const void* q, const void* k, const void* v, void* out,
                                        float* lse_opt, void* stream) {
  if (!c) return fail(THIN_ATTN_EINVAL, "null cache");
  if (!q || !k || !v || !out) return fail(THIN_ATTN_EINVAL, "q, k, v and out must be non-null");
  for (const void* ptr : {q, k, v, (const void*)out})
    if (((uintptr_t)ptr) % 16) return fail(THIN_ATTN_EINVAL, "tensor pointers must be 16-byte aligned");
  DeviceGuard dg(c->cf.device);
  return cache_decode_one(c, q, k, v, out, lse_opt, 1, (cudaStream_t)stream);
}

thin_attn_status thin_attn_cache_decode_n(thin_attn_cache_t c, const void* q, const void* k, const void* v, void* out,
                                          float* lse_opt, int n, void* stream) {
  if (!c) return fail(THIN_ATTN_EINVAL, "null cache");
  if (n < 0) return fail(THIN_ATTN_EINVAL, "n = %d", n);
  if (n == 0) return THIN_ATTN_OK;
  if (!q || !k || !v || !out) return fail(THIN_ATTN_EINVAL, "q, k, v and out must be non-null");
  for (const void* ptr : {q, k, v, (const void*)out})
    if (((uintptr_t)ptr) % 16) return fail(THIN_ATTN_EINVAL, "tensor pointers must be 16-byte aligned");
  const thin_attn_config& cf = c->cf;
  if (c->t + n > cf.T) return fail(THIN_ATTN_EINVAL, "%d tokens would exceed the capacity of %d (holds %lld)", n, cf.T,
                                   (long long)c->t);
  if (n > 1 && !c->use_split)
    return fail(THIN_ATTN_EUNSUPPORTED, "several tokens per call need the split-key decode (B*H <= 64)");
  DeviceGuard dg(cf.device);
  const size_t es = elt(cf), krow = (size_t)cf.H * cf.E * es, vrow = (size_t)cf.H * cf.D * es;
  for (int i = 0; i < n; ++i) {
    thin_attn_status s = cache_decode_one(c, (const char*)q + i * krow, (const char*)k + i * krow,
                                          (const char*)v + i * vrow, (char*)out + i * vrow,
                                          lse_opt ? lse_opt + i : nullptr, n, (cudaStream_t)stream);
    if (s != THIN_ATTN_OK) return s;
  }
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_cache_nodes(thin_attn_cache_t c, int32_t* idx_out, void* stream) {
  if (!c || !idx_out) return fail(THIN_ATTN_EINVAL, "null argument");
  DeviceGuard dg(c->cf.device);
  if (c->nodes.rows)
    CK(cudaMemcpyAsync(idx_out, (char*)c->d_mem + c->nodes.idx_off, (size_t)c->nodes.rows * 4,
                       cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
  return THIN_ATTN_OK;
}

thin_attn_status thin_attn_cache_check(thin_attn_cache_t c, void* stream) {
  if (!c) return fail(THIN_ATTN_EINVAL, "null cache");
  DeviceGuard dg(c->cf.device);
  CK(cudaStreamSynchronize((cudaStream_t)stream));
  int sts[4] = {0, 0, 0, 0};
  CK(cudaMemcpy(sts, c->d_status, sizeof sts, cudaMemcpyDeviceToHost));
  if (sts[0] != 0) {
    CK(cudaMemset(c->d_status, 0, 16));
    return fail(THIN_ATTN_ETIMEOUT, "device wait gave up (code %d)", sts[0]);
  }
  return THIN_ATTN_OK;
}

}  // extern "C"
