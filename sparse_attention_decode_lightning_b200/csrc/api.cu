// Host side of the libdsa C ABI: argument checks, workspace carve-up and the
// launch sequence of each entry point.  Nothing here computes attention; every
// step of the path runs in the kernels of the sibling files.
#include "common.cuh"
#include "internal.h"

#include <mutex>

#include <nvtx3/nvToolsExt.h>

namespace dsa {

namespace {

constexpr int B200_SMS = 148;
constexpr int TAIL_PARTS = B200_SMS / 2;

// NVTX range over a scope (header-only NVTX v3: no library to link; the
// ranges cost nothing unless a profiler collects them)
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// Grouped IndexShare attention: `units` (layer, query) units of one split on
// the SM pairs.  When they leave a last wave that fills at most half of the
// pairs, the units of that wave (tail) run cut into tail_s splits; head units
// run whole.  Without such a tail: head = units, tail = 0, tail_s = 1.
void plan_group(int units, int topk, int* head, int* tail, int* tail_s) {
  const int pairs = TAIL_PARTS;
  const int waves = units / pairs, rest = units % pairs;
  int s = rest > 0 ? pairs / rest : 1;
  const int max_s = topk / 64 < DSA_MAX_SPLITS ? topk / 64 : DSA_MAX_SPLITS;
  if (s > max_s) s = max_s;
  const bool split = waves >= 1 && rest > 0 && s >= 2;
  *head = split ? waves * pairs : units;
  *tail = split ? rest : 0;
  *tail_s = split ? s : 1;
}

int choose_splits(int Q, int topk, int requested) {
  int S = requested;
  if (S <= 0) {
    // (query, split) units run on 2-SM clusters: pick the smallest S whose
    // units fill the 74 SM pairs to at least 85% over whole waves, keeping
    // >= 64 selected rows per split; otherwise the best-filling S.
    const int pairs = B200_SMS / 2;
    const int cap = topk / 64 > 0 ? (topk / 64 < 16 ? topk / 64 : 16) : 1;
    int best = 1;
    double best_eff = -1.0;
    S = 0;
    for (int s = 1; s <= cap; ++s) {
      const long units = static_cast<long>(Q) * s;
      const long waves = (units + pairs - 1) / pairs;
      const double eff = static_cast<double>(units) / (static_cast<double>(pairs) * waves);
      if (eff >= 0.85) { S = s; break; }
      if (eff > best_eff + 1e-9) { best_eff = eff; best = s; }
    }
    if (S == 0) S = best;
  }
  if (S < 1) S = 1;
  if (S > DSA_MAX_SPLITS) S = DSA_MAX_SPLITS;
  if (S > topk) S = topk;
  return S;
}

bool ws_layout(int Q, int max_len, int topk, int num_splits, WsLayout* L) {
  if (Q <= 0 || max_len <= 0 || topk <= 0 || topk > DSA_MAX_TOPK || num_splits < 0 ||
      num_splits > DSA_MAX_SPLITS)
    return false;
  WsLayout w;
  w.ld = static_cast<int>(align_up(static_cast<size_t>(max_len), 64));
  w.S = choose_splits(Q, topk, num_splits);
  size_t off = 0;
  w.err = off;      off = align_up(off + 256, 256);
  w.scores = off;   off = align_up(off + static_cast<size_t>(Q) * w.ld * 4, 256);
  // the split partials of Q x S units, plus room for the tail of a grouped
  // MLA launch (at most one partial per SM pair, see dsa_decode_step)
  w.parts = static_cast<size_t>(Q) * w.S + TAIL_PARTS;
  w.o_part = off;   off = align_up(off + w.parts * DSA_HEADS * DSA_DIM_V * 4, 256);
  w.l_part = off;   off = align_up(off + w.parts * DSA_HEADS * 4, 256);
  // fused indexer -> selector: a 4096-bin histogram and 4 counters per query,
  // and room for the threshold bin's candidates (about 1/16 of a row, at
  // least 4096, at most 65536; a larger bin is re-read from the scores)
  int cap = static_cast<int>(align_up(static_cast<size_t>(max_len / 16), 16));
  cap = cap < 4096 ? 4096 : (cap > 65536 ? 65536 : cap);
  w.cand_cap = cap;
  w.hist = off;     off = align_up(off + static_cast<size_t>(Q) * 4096 * 4, 256);
  w.ctr = off;      off = align_up(off + static_cast<size_t>(Q) * 16, 256);
  w.cand = off;     off = align_up(off + static_cast<size_t>(Q) * cap * 8, 256);
  w.total = off;
  *L = w;
  return true;
}

bool page_size_ok(int page_size, int num_pages) {
  if (page_size < 1 || page_size > 1024 || (page_size & (page_size - 1))) return false;
  return static_cast<int64_t>(num_pages) * page_size < (int64_t(1) << 31);
}

int device_sm_count() {
  static std::atomic<int> cache[64];   // 0 until looked up; racing lookups store the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return B200_SMS;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = B200_SMS;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

namespace {

template <typename T>
T* ws_ptr(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

dsa_status check_common(const int64_t* seq_offsets, const int32_t* q_offsets,
                        const int32_t* q_vis, int B, int Q, int max_len, int topk) {
  if (!seq_offsets || !q_offsets || !q_vis) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Q <= 0 || max_len <= 0 || topk <= 0) return DSA_ERR_INVALID_ARG;
  if (B > DSA_MAX_BATCH || Q > 65535 || topk > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  if (Q > B * DSA_MAX_Q_PER_SEQ) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

// head counts of the two model shapes: DeepSeek-V3.2 (128 MLA heads, 64
// indexer heads) and GLM-5.2 (64 and 32)
bool heads_ok(int heads) { return heads == DSA_HEADS || heads == DSA_HEADS_GLM; }
bool idx_heads_ok(int idx_heads) { return idx_heads == DSA_IDX_HEADS || idx_heads == DSA_IDX_HEADS_GLM; }

dsa_status indexer_checks(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                          int64_t total_keys, int idx_heads) {
  if (!q_idx || !w || !k_idx) return DSA_ERR_INVALID_ARG;
  if (!idx_heads_ok(idx_heads)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q_idx) || !aligned16(w) || !aligned16(k_idx)) return DSA_ERR_INVALID_ARG;
  if (total_keys <= 0) return DSA_ERR_INVALID_ARG;
  if (total_keys >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

dsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

dsa_status do_indexer_topk(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                           int64_t total_keys, const int64_t* seq_offsets,
                           const int32_t* q_offsets, const int32_t* q_vis, int B, int Q,
                           int idx_heads, int max_len, int topk, int first_only, int32_t* out_idx,
                           float* out_scores, void* ws, const WsLayout& L, cudaStream_t st,
                           bool fused = false) {
  uint32_t* err = ws_ptr<uint32_t>(ws, L.err);
  float* scores = ws_ptr<float>(ws, L.scores);
  cudaError_t e;
  if (fused) {
    // the indexer fills per-query first-digit histograms (zeroed here, with
    // the selector's counters that follow them) and the selector starts from
    // them, launched while the indexer drains
    uint32_t* hist = ws_ptr<uint32_t>(ws, L.hist);
    e = cudaMemsetAsync(hist, 0, L.ctr - L.hist + static_cast<size_t>(Q) * 16, st);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
    e = launch_indexer(q_idx, w, k_idx, total_keys, seq_offsets, q_offsets, q_vis, B, Q,
                       idx_heads, first_only, scores, L.ld, err, st, hist);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
    e = launch_topk_hist(scores, L.ld, q_offsets, q_vis, B, Q, max_len, topk, first_only, hist,
                         ws_ptr<uint32_t>(ws, L.ctr), ws_ptr<uint64_t>(ws, L.cand), L.cand_cap,
                         out_idx, out_scores, err, st, true);
  } else {
    e = launch_indexer(q_idx, w, k_idx, total_keys, seq_offsets, q_offsets, q_vis, B, Q,
                       idx_heads, first_only, scores, L.ld, err, st);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
    // the selector starts while the indexer drains (its scores are waited for)
    e = launch_topk(scores, L.ld, q_offsets, q_vis, B, Q, max_len, topk, first_only, out_idx,
                    out_scores, err, st, true);
  }
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  if (first_only) {
    e = launch_expand_idx(q_offsets, B, Q, topk, out_idx, out_scores, st);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

dsa_status do_sparse_mla(const void* q, const void* kv_pool, int num_pages, int page_size,
                         const int32_t* page_table, int max_pages, const int32_t* q_offsets,
                         const int32_t* q_vis, const int32_t* idx, int B, int Q, int H,
                         int topk, float scale, int S, float* out, float* lse, void* ws,
                         const WsLayout& L, cudaStream_t st, bool pdl,
                         const int32_t* win_page_table = nullptr, int win_max_pages = 0,
                         const int32_t* win_vis = nullptr, int window = 0, bool kv8 = false,
                         float kv_scale = 1.f) {
  uint32_t* err = ws_ptr<uint32_t>(ws, L.err);
  float* o_part = ws_ptr<float>(ws, L.o_part);
  float* l_part = ws_ptr<float>(ws, L.l_part);
  cudaError_t e = launch_sparse_mla(static_cast<const __nv_bfloat16*>(q),
                                    static_cast<const __nv_bfloat16*>(kv_pool), num_pages,
                                    page_size, page_table, max_pages, q_offsets, q_vis, idx, B, Q,
                                    H, topk, scale, S, out, lse, o_part, l_part, err, st, pdl,
                                    win_page_table, win_max_pages, win_vis, window, kv8, kv_scale);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  if (S > 1) {
    e = launch_combine(o_part, l_part, Q, S, H, out, lse, st, true);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

dsa_status mla_checks(const void* q, const void* kv_pool, int num_pages, int page_size,
                      const int32_t* page_table, int max_pages, const int32_t* idx, float* out,
                      float* lse, float scale, int heads) {
  if (!q || !kv_pool || !page_table || !idx || !out || !lse) return DSA_ERR_INVALID_ARG;
  if (!heads_ok(heads)) return DSA_ERR_UNSUPPORTED;
  if (!page_size_ok(page_size, num_pages > 0 ? num_pages : 1)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(kv_pool) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  if (num_pages <= 0 || max_pages <= 0) return DSA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || scale != scale) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

}  // namespace

cudaError_t launch_sparse_mla(const __nv_bfloat16* q, const __nv_bfloat16* pool, int num_pages,
                              int page_size, const int32_t* page_table, int max_pages,
                              const int32_t* q_offsets, const int32_t* q_vis,
                              const int32_t* idx, int B, int Q, int H, int topk, float scale, int S,
                              float* out, float* lse, float* o_part, float* l_part,
                              uint32_t* err, cudaStream_t st, bool pdl,
                              const int32_t* win_page_table, int win_max_pages,
                              const int32_t* win_vis, int window, bool kv8, float kv_scale) {
  return launch_sparse_mla_tc(q, pool, num_pages, page_size, page_table, max_pages, q_offsets,
                              q_vis, idx, B, Q, H, topk, scale, S, out, lse, o_part, l_part, err,
                              st, pdl, win_page_table, win_max_pages, win_vis, window, kv8,
                              kv_scale);
}

}  // namespace dsa

using namespace dsa;

extern "C" {

const char* dsa_status_string(int s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_DEVICE_BOUNDS: return "DSA_ERR_DEVICE_BOUNDS";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    default: return "DSA_ERR_UNKNOWN";
  }
}

int dsa_version(void) { return 300; }

int dsa_mla_group_plan(int units, int topk, int* head_units, int* tail_units, int* tail_splits) {
  if (units <= 0 || topk <= 0 || topk > DSA_MAX_TOPK || !head_units || !tail_units || !tail_splits)
    return 0;
  plan_group(units, topk, head_units, tail_units, tail_splits);
  return 1;
}

int dsa_choose_splits(int Q, int topk, int num_splits) {
  if (Q <= 0 || topk <= 0 || topk > DSA_MAX_TOPK || num_splits < 0 || num_splits > DSA_MAX_SPLITS)
    return 0;
  return choose_splits(Q, topk, num_splits);
}

size_t dsa_workspace_bytes(int Q, int max_len, int topk, int num_splits) {
  WsLayout L;
  if (!ws_layout(Q, max_len, topk, num_splits, &L)) return 0;
  return L.total;
}

dsa_status dsa_indexer_scores(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                              int64_t total_keys, const int64_t* seq_offsets,
                              const int32_t* q_offsets, const int32_t* q_vis, int B, int Q,
                              int idx_heads, int max_len, int first_only, float* scores,
                              int ld_scores, void* ws, size_t ws_bytes, void* stream) {
  dsa_status s = check_common(seq_offsets, q_offsets, q_vis, B, Q, max_len, 1);
  if (s != DSA_OK) return s;
  if ((s = indexer_checks(q_idx, w, k_idx, total_keys, idx_heads)) != DSA_OK) return s;
  if (!scores || !ws || ld_scores < max_len || (ld_scores & 3) || !aligned16(scores))
    return DSA_ERR_INVALID_ARG;
  if (ws_bytes < 256) return DSA_ERR_WORKSPACE;
  return cuda_status(launch_indexer(q_idx, w, k_idx, total_keys, seq_offsets, q_offsets, q_vis,
                                    B, Q, idx_heads, first_only, scores, ld_scores,
                                    static_cast<uint32_t*>(ws), static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_topk_select(const float* scores, int ld_scores, const int32_t* q_offsets,
                           const int32_t* q_vis, int B, int Q, int max_len, int topk,
                           int first_only, int32_t* out_idx, float* out_scores, void* ws,
                           size_t ws_bytes, void* stream) {
  if (!scores || !q_offsets || !q_vis || !out_idx || !ws) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Q <= 0 || max_len <= 0 || topk <= 0) return DSA_ERR_INVALID_ARG;
  if (B > DSA_MAX_BATCH || Q > 65535 || topk > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  if (ld_scores < max_len || (ld_scores & 3) || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  // the selector keeps its working set on chip; the workspace holds the error flag
  if (ws_bytes < 256) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_topk(scores, ld_scores, q_offsets, q_vis, B, Q, max_len, topk,
                              first_only, out_idx, out_scores, static_cast<uint32_t*>(ws), st,
                              false);
  return cuda_status(e);
}

dsa_status dsa_indexer_topk(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                            int64_t total_keys, const int64_t* seq_offsets,
                            const int32_t* q_offsets, const int32_t* q_vis, int B, int Q,
                            int idx_heads, int max_len, int topk, int first_only,
                            int32_t* out_idx, float* out_scores, void* ws, size_t ws_bytes,
                            void* stream) {
  dsa_status s = check_common(seq_offsets, q_offsets, q_vis, B, Q, max_len, topk);
  if (s != DSA_OK) return s;
  if ((s = indexer_checks(q_idx, w, k_idx, total_keys, idx_heads)) != DSA_OK) return s;
  if (!out_idx || !ws) return DSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!ws_layout(Q, max_len, topk, 1, &L)) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return DSA_ERR_WORKSPACE;
  return do_indexer_topk(q_idx, w, k_idx, total_keys, seq_offsets, q_offsets, q_vis, B, Q,
                         idx_heads, max_len, topk, first_only, out_idx, out_scores, ws, L,
                         static_cast<cudaStream_t>(stream));
}

dsa_status dsa_indexer_topk_fused(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                                  int64_t total_keys, const int64_t* seq_offsets,
                                  const int32_t* q_offsets, const int32_t* q_vis, int B, int Q,
                                  int idx_heads, int max_len, int topk, int first_only,
                                  int32_t* out_idx, float* out_scores, void* ws, size_t ws_bytes,
                                  void* stream) {
  dsa_status s = check_common(seq_offsets, q_offsets, q_vis, B, Q, max_len, topk);
  if (s != DSA_OK) return s;
  if ((s = indexer_checks(q_idx, w, k_idx, total_keys, idx_heads)) != DSA_OK) return s;
  if (!out_idx || !ws) return DSA_ERR_INVALID_ARG;
  WsLayout L;
  if (!ws_layout(Q, max_len, topk, 1, &L)) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return DSA_ERR_WORKSPACE;
  return do_indexer_topk(q_idx, w, k_idx, total_keys, seq_offsets, q_offsets, q_vis, B, Q,
                         idx_heads, max_len, topk, first_only, out_idx, out_scores, ws, L,
                         static_cast<cudaStream_t>(stream), true);
}

dsa_status dsa_sparse_mla_decode(const void* q, const void* kv_pool, int num_pages, int page_size,
                                 const int32_t* page_table, int max_pages,
                                 const int32_t* q_offsets, const int32_t* q_vis,
                                 const int32_t* idx, int B, int Q, int heads, int topk,
                                 float scale, int num_splits, float* out, float* lse, void* ws,
                                 size_t ws_bytes, void* stream) {
  if (!q_offsets || !q_vis || !ws) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Q <= 0 || topk <= 0) return DSA_ERR_INVALID_ARG;
  if (B > DSA_MAX_BATCH || Q > 65535 || topk > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  if (num_splits < 0 || num_splits > DSA_MAX_SPLITS) return DSA_ERR_UNSUPPORTED;
  dsa_status s = mla_checks(q, kv_pool, num_pages, page_size, page_table, max_pages, idx, out, lse,
                            scale, heads);
  if (s != DSA_OK) return s;
  WsLayout L;
  if (!ws_layout(Q, 1, topk, num_splits, &L)) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return DSA_ERR_WORKSPACE;
  return do_sparse_mla(q, kv_pool, num_pages, page_size, page_table, max_pages, q_offsets, q_vis,
                       idx, B, Q, heads, topk, scale, L.S, out, lse, ws, L,
                       static_cast<cudaStream_t>(stream), false);
}

dsa_status dsa_sparse_mla_decode_window(const void* q, const void* kv_pool, int num_pages,
                                        int page_size, const int32_t* page_table, int max_pages,
                                        const int32_t* win_page_table, int win_max_pages,
                                        const int32_t* q_offsets, const int32_t* q_vis,
                                        const int32_t* win_vis, const int32_t* idx, int B, int Q,
                                        int heads, int topk, int window, float scale,
                                        int num_splits, float* out, float* lse, void* ws,
                                        size_t ws_bytes, void* stream) {
  if (!q_offsets || !q_vis || !ws) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Q <= 0 || topk <= 0 || window < 0) return DSA_ERR_INVALID_ARG;
  if (window > 0 && (!win_page_table || !win_vis || win_max_pages <= 0)) return DSA_ERR_INVALID_ARG;
  if (B > DSA_MAX_BATCH || Q > 65535 || topk + window > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  if (num_splits < 0 || num_splits > DSA_MAX_SPLITS) return DSA_ERR_UNSUPPORTED;
  dsa_status s = mla_checks(q, kv_pool, num_pages, page_size, page_table, max_pages, idx, out, lse,
                            scale, heads);
  if (s != DSA_OK) return s;
  WsLayout L;
  if (!ws_layout(Q, 1, topk + window, num_splits, &L)) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return DSA_ERR_WORKSPACE;
  return do_sparse_mla(q, kv_pool, num_pages, page_size, page_table, max_pages, q_offsets, q_vis,
                       idx, B, Q, heads, topk, scale, L.S, out, lse, ws, L,
                       static_cast<cudaStream_t>(stream), false, win_page_table, win_max_pages,
                       win_vis, window);
}

dsa_status dsa_sparse_mla_decode_fp8(const void* q, const void* kv_pool, float kv_scale,
                                     int num_pages, int page_size, const int32_t* page_table,
                                     int max_pages, const int32_t* q_offsets, const int32_t* q_vis,
                                     const int32_t* idx, int B, int Q, int heads, int topk,
                                     float scale, int num_splits, float* out, float* lse, void* ws,
                                     size_t ws_bytes, void* stream) {
  if (!q_offsets || !q_vis || !ws) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Q <= 0 || topk <= 0) return DSA_ERR_INVALID_ARG;
  if (!(kv_scale > 0.f) || kv_scale != kv_scale || kv_scale > 3.0e38f) return DSA_ERR_INVALID_ARG;
  if (B > DSA_MAX_BATCH || Q > 65535 || topk > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  if (num_splits < 0 || num_splits > DSA_MAX_SPLITS) return DSA_ERR_UNSUPPORTED;
  dsa_status s = mla_checks(q, kv_pool, num_pages, page_size, page_table, max_pages, idx, out, lse,
                            scale, heads);
  if (s != DSA_OK) return s;
  WsLayout L;
  if (!ws_layout(Q, 1, topk, num_splits, &L)) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return DSA_ERR_WORKSPACE;
  return do_sparse_mla(q, kv_pool, num_pages, page_size, page_table, max_pages, q_offsets, q_vis,
                       idx, B, Q, heads, topk, scale, L.S, out, lse, ws, L,
                       static_cast<cudaStream_t>(stream), false, nullptr, 0, nullptr, 0, true,
                       kv_scale);
}

dsa_status dsa_lse_combine(const float* o_parts, const float* lse_parts, int Q, int S, int heads,
                           float* out, float* lse, void* stream) {
  if (!o_parts || !lse_parts || !out || !lse) return DSA_ERR_INVALID_ARG;
  if (Q <= 0 || S <= 0) return DSA_ERR_INVALID_ARG;
  if (!heads_ok(heads)) return DSA_ERR_UNSUPPORTED;
  if (Q > 65535 * 8 || S > 1024) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(o_parts) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  return cuda_status(launch_combine(o_parts, lse_parts, Q, S, heads, out, lse,
                                    static_cast<cudaStream_t>(stream), false));
}

dsa_status dsa_decode_step(int n_layers, int index_share, int mtp_index_share,
                           const uint8_t* const* q_idx_layers, const float* const* w_layers,
                           const uint8_t* const* k_idx_layers, int64_t total_keys,
                           const int64_t* seq_offsets, const int32_t* q_offsets,
                           const int32_t* q_vis, int B, int Q, int heads, int idx_heads,
                           int max_len, int topk,
                           const void* const* q_layers, const void* const* pool_layers,
                           int num_pages, int page_size, const int32_t* const* page_table_layers,
                           int max_pages, float scale, int num_splits,
                           float* const* out_layers, float* const* lse_layers,
                           int32_t* idx_out, void* ws, size_t ws_bytes, void* stream) {
  if (n_layers <= 0 || index_share <= 0) return DSA_ERR_INVALID_ARG;
  if (!q_idx_layers || !w_layers || !k_idx_layers || !q_layers || !pool_layers ||
      !page_table_layers || !out_layers || !lse_layers || !idx_out || !ws)
    return DSA_ERR_INVALID_ARG;
  dsa_status s = check_common(seq_offsets, q_offsets, q_vis, B, Q, max_len, topk);
  if (s != DSA_OK) return s;
  if (num_splits < 0 || num_splits > DSA_MAX_SPLITS) return DSA_ERR_UNSUPPORTED;
  for (int l = 0; l < n_layers; ++l) {
    if (l % index_share == 0 &&
        (s = indexer_checks(q_idx_layers[l], w_layers[l], k_idx_layers[l], total_keys,
                            idx_heads)) != DSA_OK)
      return s;
    if ((s = mla_checks(q_layers[l], pool_layers[l], num_pages, page_size, page_table_layers[l],
                        max_pages, idx_out, out_layers[l], lse_layers[l], scale, heads)) != DSA_OK)
      return s;
  }
  WsLayout L;
  if (!ws_layout(Q, max_len, topk, num_splits, &L)) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < L.total) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // host-side ranges: they mark when each stage's launches are enqueued
  NvtxRange step_range("dsa_decode_step");
  for (int l0 = 0; l0 < n_layers; l0 += index_share) {
    const int g = l0 / index_share;
    const int l1 = l0 + index_share < n_layers ? l0 + index_share : n_layers;
    int32_t* idx_g = idx_out + static_cast<size_t>(g) * Q * topk;
    {
      NvtxRange r("dsa_indexer_topk");
      s = do_indexer_topk(q_idx_layers[l0], w_layers[l0], k_idx_layers[l0], total_keys,
                          seq_offsets, q_offsets, q_vis, B, Q, idx_heads, max_len, topk,
                          mtp_index_share, idx_g, nullptr, ws, L, st);
      if (s != DSA_OK) return s;
    }
    NvtxRange r("dsa_sparse_mla");
    if (L.S == 1) {
      // The layers that share this index set run as one grid over (layer,
      // query) units, each on an SM pair.  When the units leave a last wave
      // that fills at most half of the pairs, those tail units run as a
      // second grid cut into splits (merged by LSE), so the last wave takes
      // a fraction of a unit's time instead of a whole one.
      for (int c0 = l0; c0 < l1; c0 += MLA_MAX_LAYERS_PER_LAUNCH) {
        const int n = l1 - c0 < MLA_MAX_LAYERS_PER_LAUNCH ? l1 - c0 : MLA_MAX_LAYERS_PER_LAUNCH;
        MlaLayerPtrs lp[MLA_MAX_LAYERS_PER_LAUNCH];
        for (int i = 0; i < n; ++i)
          lp[i] = {static_cast<const __nv_bfloat16*>(q_layers[c0 + i]),
                   static_cast<const __nv_bfloat16*>(pool_layers[c0 + i]),
                   page_table_layers[c0 + i], out_layers[c0 + i], lse_layers[c0 + i]};
        int head = 0, tail = 0, tail_s = 1;
        plan_group(n * Q, topk, &head, &tail, &tail_s);
        const bool split_tail = tail > 0;
        uint32_t* err = ws_ptr<uint32_t>(ws, L.err);
        if (launch_sparse_mla_layers(lp, n, num_pages, page_size, max_pages, q_offsets, q_vis,
                                     idx_g, B, Q, heads, topk, scale, 1, nullptr, nullptr, err, st,
                                     true, nullptr, 0, nullptr, 0, false, 1.f, 0,
                                     head) != cudaSuccess)
          return DSA_ERR_CUDA;
        if (split_tail) {
          float* o_part = ws_ptr<float>(ws, L.o_part);
          float* l_part = ws_ptr<float>(ws, L.l_part);
          if (launch_sparse_mla_layers(lp, n, num_pages, page_size, max_pages, q_offsets, q_vis,
                                       idx_g, B, Q, heads, topk, scale, tail_s, o_part, l_part,
                                       err, st, true, nullptr, 0, nullptr, 0, false, 1.f, head,
                                       tail) != cudaSuccess ||
              launch_combine_layers(o_part, l_part, tail, tail_s, heads, head, Q, lp, n, st,
                                    true) != cudaSuccess)
            return DSA_ERR_CUDA;
        }
      }
      continue;
    }
    // with split-K the partial buffers hold one layer at a time
    for (int l = l0; l < l1; ++l) {
      s = do_sparse_mla(q_layers[l], pool_layers[l], num_pages, page_size, page_table_layers[l],
                        max_pages, q_offsets, q_vis, idx_g, B, Q, heads, topk, scale, L.S,
                        out_layers[l], lse_layers[l], ws, L, st, true);
      if (s != DSA_OK) return s;
    }
  }
  return DSA_OK;
}

dsa_status dsa_check_error(void* ws, void* stream) {
  if (!ws) return DSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  uint32_t flag = 0;
  if (cudaMemcpy(&flag, ws, sizeof(flag), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (flag) {
    const uint32_t zero = 0;
    if (cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return DSA_ERR_CUDA;
  }
  if (flag & DEVERR_TIMEOUT) return DSA_ERR_TIMEOUT;
  if (flag & DEVERR_CAPACITY) return DSA_ERR_UNSUPPORTED;   // the cause of any bounds flag after it
  if (flag & DEVERR_BOUNDS) return DSA_ERR_DEVICE_BOUNDS;
  return DSA_OK;
}

}  // extern "C"
