// Host-side declarations shared by the libdsa translation units: the
// workspace carve-up and the kernel launchers.
#pragma once

#include <atomic>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stddef.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

// Byte offsets of the workspace regions (all 256-byte aligned).
struct WsLayout {
  size_t err = 0;      // uint32 error flag (+ padding)
  size_t scores = 0;   // fp32 [Q, ld]
  size_t o_part = 0;   // fp32 [parts, 128, 512]
  size_t l_part = 0;   // fp32 [parts, 128]
  size_t hist = 0;     // u32 [Q, 4096]: the indexer's first-digit histograms
  size_t ctr = 0;      // u32 [Q, 4]: the histogram selector's counters (follows hist;
                       // both are zeroed together before each indexer launch)
  size_t cand = 0;     // u64 [Q, cand_cap]: its threshold-bin candidates
  size_t total = 0;
  int cand_cap = 0;
  int ld = 0;          // score row stride (elements)
  int S = 0;           // split-K parts chosen for Q queries
  size_t parts = 0;    // (unit, split) partials the buffers hold: Q * S + one per SM pair
};

// 2-D tensor map, 128-byte swizzle, no OOB fill value (zeros)
bool encode_tiled_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                     uint64_t inner_elems, uint64_t rows, uint64_t row_stride_bytes,
                     uint32_t box_inner, uint32_t box_rows);

// Runs `set` (cudaFuncSetAttribute calls) once per device and remembers the
// success in `done` (device ids below 64; other ids run `set` on every call).
// Safe from several host threads: a race at most runs the idempotent `set`
// twice.
template <typename F>
inline cudaError_t set_once_per_device(std::atomic<bool> (&done)[64], F&& set) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const bool tracked = dev >= 0 && dev < 64;
  if (tracked && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  const cudaError_t e = set();
  if (e == cudaSuccess && tracked) done[dev].store(true, std::memory_order_release);
  return e;
}

bool ws_layout(int Q, int max_len, int topk, int num_splits, WsLayout* out);
// a latent-cache page of page_size tokens: a power of two from 1 to 1024, and
// every pool row index (num_pages * page_size) fits in int32
bool page_size_ok(int page_size, int num_pages);
int device_sm_count();
int choose_splits(int Q, int topk, int requested);

// kernel launchers (return cudaSuccess or the launch error)
cudaError_t launch_indexer(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                           int64_t total_keys, const int64_t* seq_offsets,
                           const int32_t* q_offsets, const int32_t* q_vis, int B, int Q,
                           int idx_heads, int first_only, float* scores, int ld, uint32_t* err,
                           cudaStream_t st, uint32_t* hist = nullptr);

cudaError_t launch_topk(const float* scores, int ld, const int32_t* q_offsets,
                        const int32_t* q_vis, int B, int Q, int max_len, int topk,
                        int first_only, int32_t* out_idx, float* out_scores, uint32_t* err,
                        cudaStream_t st, bool pdl);

cudaError_t launch_topk_hist(const float* scores, int ld, const int32_t* q_offsets,
                             const int32_t* q_vis, int B, int Q, int max_len, int topk,
                             int first_only, const uint32_t* hist, uint32_t* ctr, uint64_t* cand,
                             int cand_cap, int32_t* out_idx, float* out_scores, uint32_t* err,
                             cudaStream_t st, bool pdl);

cudaError_t launch_expand_idx(const int32_t* q_offsets, int B, int Q, int topk,
                              int32_t* out_idx, float* out_scores, cudaStream_t st);

cudaError_t launch_sparse_mla(const __nv_bfloat16* q, const __nv_bfloat16* pool, int num_pages,
                              int page_size, const int32_t* page_table, int max_pages,
                              const int32_t* q_offsets, const int32_t* q_vis,
                              const int32_t* idx, int B, int Q, int H, int topk, float scale, int S,
                              float* out, float* lse, float* o_part, float* l_part,
                              uint32_t* err, cudaStream_t st, bool pdl,
                              const int32_t* win_page_table = nullptr, int win_max_pages = 0,
                              const int32_t* win_vis = nullptr, int window = 0,
                              bool kv8 = false, float kv_scale = 1.f);

// the sparse MLA kernel itself (sparse_mla_sm100.cu): o_part / l_part hold
// the split partials when S > 1; err may be null (nothing is reported)
cudaError_t launch_sparse_mla_tc(const __nv_bfloat16* q, const __nv_bfloat16* pool, int num_pages,
                                 int page_size, const int32_t* page_table, int max_pages,
                                 const int32_t* q_offsets, const int32_t* q_vis,
                                 const int32_t* idx, int B, int Q, int H, int topk, float scale,
                                 int S, float* out, float* lse, float* o_part, float* l_part,
                                 uint32_t* err, cudaStream_t st, bool pdl,
                                 const int32_t* win_page_table = nullptr, int win_max_pages = 0,
                                 const int32_t* win_vis = nullptr, int window = 0,
                                 bool kv8 = false, float kv_scale = 1.f);

// Several layers that share one index set (IndexShare) in one grid: units
// gi = layer * Q + query for gi in [g0, g0 + n_units) (default: all L * Q),
// each cut into S splits.  With S == 1 every unit writes its layer's O and
// LSE; with S > 1 the partials of unit gi, split c go to row
// ((gi - g0) * S + c) of o_part [n_units, S, H, 512] / l_part [n_units, S, H].
struct MlaLayerPtrs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* pool;
  const int32_t* page_table;
  float* out;
  float* lse;
};
constexpr int MLA_MAX_LAYERS_PER_LAUNCH = 4;
cudaError_t launch_sparse_mla_layers(const MlaLayerPtrs* layers, int L, int num_pages,
                                     int page_size, int max_pages, const int32_t* q_offsets,
                                     const int32_t* q_vis, const int32_t* idx, int B, int Q, int H,
                                     int topk, float scale, int S, float* o_part, float* l_part,
                                     uint32_t* err, cudaStream_t st, bool pdl,
                                     const int32_t* win_page_table = nullptr, int win_max_pages = 0,
                                     const int32_t* win_vis = nullptr, int window = 0,
                                     bool kv8 = false, float kv_scale = 1.f, int g0 = 0,
                                     int n_units = -1);
// The split merge for partial rows laid out as above: row i is unit g0 + i,
// written to its layer's O and LSE
cudaError_t launch_combine_layers(const float* o_part, const float* l_part, int n_units, int S,
                                  int H, int g0, int Q, const MlaLayerPtrs* layers, int L,
                                  cudaStream_t st, bool pdl);

cudaError_t launch_combine(const float* o_part, const float* l_part, int Q, int S, int H,
                           float* out, float* lse, cudaStream_t st, bool pdl);

// pdl = true: the kernel may start before the previous kernel on the stream
// ends (programmatic dependent launch); it waits for it in pdl_wait().  Only
// set where the previous kernel is one of this library's, launched by the same
// entry point, so everything older on the stream has finished before it.
inline void add_pdl_attr(cudaLaunchAttribute* attrs, unsigned int* n, bool pdl) {
  if (!pdl) return;
  attrs[*n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[*n].val.programmaticStreamSerializationAllowed = 1;
  ++*n;
}

}  // namespace dsa
