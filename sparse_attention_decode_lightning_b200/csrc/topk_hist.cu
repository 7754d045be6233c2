// Token selector fed by the indexer's histograms (the fused indexer -> top-k
// path; "大语言模型结构总览", section 2.2: the selector keeps the k = 2048
// best-scoring tokens).  Same result as topk.cu: the topk highest scores of a
// row, ties to the lower position, as a set.
//
// With the composite key of position s
//     V(s) = (u(s) << pb) | s,   u(s) = ~key(I[s]),   pb = bits(vis - 1)
// (a smaller V is a better position), the first 12-bit digit of V is the top
// 12 bits of u.  The indexer adds every score it writes to a per-row
// histogram of that digit, so this kernel starts from the threshold digit t
// (the smallest d with count(digits <= d) >= topk) without a first pass:
//   collect  any number of CTAs per row scan the row (L2-resident: the
//            indexer has just written it), stage in shared memory the
//            positions with digit < t and the bin-t keys V, then reserve
//            their output slots and candidate-list entries with one atomic
//            per CTA and list and write them out;
//   finish   the last CTA of the row picks the need = topk - count(< t)
//            smallest V of bin t by 11-bit radix passes that stop as soon as
//            the rest of the group is needed whole, over the candidate list
//            (in shared memory when it holds at most 8192 keys) or, if bin t
//            overflowed the list, over the row itself, and writes them.
// The histograms and counters are zeroed by the caller before the indexer.
// Output slots come from atomic counters, so the row is unordered.  Rows
// with vis <= topk take every visible position and -1 padding.
// The candidates and counters are written by other CTAs of this grid, and
// the histograms and scores by the indexer that this kernel overlaps as a
// programmatic dependent, so all of them are read with ld_l2_* (L2 only, and
// kept after the grid-dependency wait by a memory clobber).
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int THREADS = 1024;
constexpr int DIGIT = 12;
constexpr int BINS = 1 << DIGIT;
constexpr int LIST_SMEM = 8192;                 // finisher: candidate lists kept in shared memory
constexpr int STAGE_BYTES = LIST_SMEM * 8;      // dynamic shared memory: histogram / staging / list
constexpr int TAKE_CAP = DSA_MAX_TOPK;          // staged positions below the threshold digit
constexpr int MID_CAP = (STAGE_BYTES - TAKE_CAP * 4) / 8;   // staged threshold-bin keys (u64)
constexpr int FDIGIT = 11;                      // finisher radix digit
constexpr int UNROLL = 4;                       // float4 loads a thread keeps in flight
static_assert(BINS * 4 <= STAGE_BYTES, "the histogram fits the staging space");
static_assert(BINS % THREADS == 0, "histogram load");

struct HistTopkArgs {
  const float* scores;
  int ld;
  const int32_t* q_offsets;
  const int32_t* q_vis;
  int B, Q, topk, first_only;
  const uint32_t* hist; // [Q][BINS], filled by the indexer
  uint32_t* ctr;        // [Q][4]: output slots, candidates, finished CTAs; zero on entry
  uint64_t* cand;       // [Q][cand_cap]
  int cand_cap;
  int32_t* out_idx;
  float* out_scores;
  uint32_t* err;
};

__device__ __forceinline__ int hist_row_query(const HistTopkArgs& a, int y) {
  if (!a.first_only) return y;
  const int q0 = a.q_offsets[y];
  return (a.q_offsets[y + 1] > q0 && q0 >= 0 && q0 < a.Q) ? q0 : -1;
}

// The smallest digit d of hist[0..nb) with count(<= d) >= need; *below =
// count(< d).  Block-wide; nb <= BINS, 4 bins per thread.
__device__ void find_digit(const uint32_t* hist, int nb, uint32_t need, uint32_t* s_warp,
                           uint32_t* s_d, uint32_t* s_below) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {                               // if no bin qualifies (inconsistent counts)
    *s_d = static_cast<uint32_t>(nb - 1);
    *s_below = 0;
  }
  uint32_t c[4], sum = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = 4 * tid + k;
    c[k] = i < nb ? hist[i] : 0u;
    sum += c[k];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w0 = s_warp[lane];
    uint32_t w = w0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += y;
    }
    s_warp[lane] = w - w0;
  }
  __syncthreads();
  uint32_t acc = s_warp[warp] + incl - sum;     // count below this thread's bins
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (acc < need && acc + c[k] >= need) {
      *s_d = static_cast<uint32_t>(4 * tid + k);
      *s_below = acc;
    }
    acc += c[k];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(THREADS, 2) topk_hist_kernel(HistTopkArgs a) {
  // s_dyn holds the row's histogram until the threshold digit is known, then
  // this CTA's staged output: positions below the threshold digit (TAKE_CAP,
  // at least any row's count of them, which is < topk) and keys of the
  // threshold bin (MID_CAP; more spill to the global list one by one), and
  // in the finishing CTA the row's candidate list
  extern __shared__ __align__(16) uint8_t s_dyn[];   // STAGE_BYTES
  uint32_t* s_h = reinterpret_cast<uint32_t*>(s_dyn);
  __shared__ uint32_t s_bins[1 << FDIGIT];
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_t, s_below, s_last, s_nt, s_nm, s_bt, s_bm;
  uint32_t* s_take = s_h;
  uint64_t* s_mid = reinterpret_cast<uint64_t*>(s_h + TAKE_CAP);
  const int tid = threadIdx.x;
  const int cpr = static_cast<int>(gridDim.x);  // CTAs of this row
  pdl_trigger();
  const int q = hist_row_query(a, blockIdx.y);
  if (q < 0) return;
  pdl_wait();                                   // the scores and histograms of the indexer
  int vis = a.q_vis[q];
  if (vis < 0 || vis > a.ld) {
    if (tid == 0 && blockIdx.x == 0) raise_error(a.err, DEVERR_BOUNDS);
    vis = vis < 0 ? 0 : a.ld;
  }
  const int topk = a.topk;
  const float* row = a.scores + static_cast<size_t>(q) * a.ld;
  int32_t* oi = a.out_idx + static_cast<size_t>(q) * topk;
  float* os = a.out_scores ? a.out_scores + static_cast<size_t>(q) * topk : nullptr;
  const uint32_t* hist = a.hist + static_cast<size_t>(q) * BINS;
  uint32_t* ctr = a.ctr + static_cast<size_t>(q) * 4;
  uint64_t* cand = a.cand + static_cast<size_t>(q) * a.cand_cap;

  if (vis <= topk) {                            // every visible position, then padding
    for (int i = blockIdx.x * THREADS + tid; i < topk; i += cpr * THREADS) {
      oi[i] = i < vis ? i : -1;
      if (os) os[i] = i < vis ? ld_l2_f32(&row[i]) : -INFINITY;
    }
    return;
  }
  const int pb = 32 - __clz(vis - 1);           // vis >= 2 here
  const int R0 = 32 - DIGIT + pb;               // bits of V below the first digit
  const uint64_t pos_mask = (uint64_t(1) << pb) - 1;

  // ---- threshold digit from the histogram (every CTA of the row)
  {
    // all of a thread's loads in flight before the first store (the L2 loads
    // are ordered asm, so a store between them would wait for each in turn)
    uint32_t h[BINS / THREADS];
#pragma unroll
    for (int k = 0; k < BINS / THREADS; ++k) h[k] = ld_l2_u32(&hist[k * THREADS + tid]);
#pragma unroll
    for (int k = 0; k < BINS / THREADS; ++k) s_h[k * THREADS + tid] = h[k];
  }
  __syncthreads();
  find_digit(s_h, BINS, static_cast<uint32_t>(topk), s_warp, &s_t, &s_below);
  const uint32_t t = s_t;
  const uint32_t n_bin = s_h[t];                // positions with digit t
  uint32_t need = static_cast<uint32_t>(topk) - s_below;
  if (tid == 0) {
    s_nt = 0;
    s_nm = 0;
  }
  __syncthreads();                              // s_h is staging space from here

  // ---- collect over this CTA's slice (whole float4 groups) into shared memory
  const int n4 = (vis + 3) >> 2;
  const int per = (n4 + cpr - 1) / cpr;
  const int g0 = blockIdx.x * per, g1 = min(n4, g0 + per);
  const float4* row4 = reinterpret_cast<const float4*>(row);
  for (int base = g0; base < g1; base += UNROLL * THREADS) {
    float4 vv[UNROLL];                          // UNROLL loads in flight per thread
#pragma unroll
    for (int r = 0; r < UNROLL; ++r) {
      const int g = base + r * THREADS + tid;
      vv[r] = g < g1 ? ld_l2_f32x4(&row4[g]) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int r = 0; r < UNROLL; ++r) {
      const int g = base + r * THREADS + tid;
      const float e[4] = {vv[r].x, vv[r].y, vv[r].z, vv[r].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // about one score in twenty is kept: a lane that keeps one takes its
        // staging slot with a shared-memory atomic of its own
        const int p = 4 * g + k;
        const uint32_t u = ~float_key(e[k]);
        const uint32_t d = u >> (32 - DIGIT);
        if (g < g1 && p < vis && d <= t) {
          if (d < t) {
            const uint32_t slot = atomicAdd(&s_nt, 1u);
            if (slot < static_cast<uint32_t>(TAKE_CAP)) s_take[slot] = static_cast<uint32_t>(p);
          } else {
            const uint64_t V = (static_cast<uint64_t>(u) << pb) | static_cast<uint64_t>(p);
            const uint32_t c = atomicAdd(&s_nm, 1u);
            if (c < static_cast<uint32_t>(MID_CAP)) {
              s_mid[c] = V;
            } else {                            // a crowded bin: straight to the global list
              const uint32_t gc = atomicAdd(&ctr[1], 1u);
              if (gc < static_cast<uint32_t>(a.cand_cap)) cand[gc] = V;
            }
          }
        }
      }
    }
  }
  __syncthreads();
  if (tid == 0) {                               // one reservation per CTA and list
    const uint32_t nt = min(s_nt, static_cast<uint32_t>(TAKE_CAP));
    const uint32_t nm = min(s_nm, static_cast<uint32_t>(MID_CAP));
    s_nt = nt;
    s_nm = nm;
    s_bt = nt ? atomicAdd(&ctr[0], nt) : 0u;
    s_bm = nm ? atomicAdd(&ctr[1], nm) : 0u;
  }
  __syncthreads();
  for (uint32_t i = tid; i < s_nt; i += THREADS) {
    const uint32_t slot = s_bt + i;
    if (slot < static_cast<uint32_t>(topk)) {   // bounded even if the histogram is stale
      const int p = static_cast<int>(s_take[i]);
      oi[slot] = p;
      if (os) os[slot] = ld_l2_f32(&row[p]);
    }
  }
  for (uint32_t i = tid; i < s_nm; i += THREADS)
    if (s_bm + i < static_cast<uint32_t>(a.cand_cap)) cand[s_bm + i] = s_mid[i];

  // ---- the last CTA of the row finishes it
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    s_last = atomicAdd(&ctr[2], 1u) == static_cast<uint32_t>(cpr - 1);
    if (s_last) {
      // every other CTA of the row has added its entries: one thread reads
      // the row's totals and hands them to the block, so every thread takes
      // the same branches (and barriers) below
      __threadfence();
      s_bm = ld_l2_u32(&ctr[1]);                // candidates of bin t
      s_bt = ld_l2_u32(&ctr[0]);                // positions below the threshold digit
      s_nt = 0;
    }
  }
  __syncthreads();
  if (!s_last) return;
  const uint32_t n_cand = s_bm;
  const bool from_list = n_cand <= static_cast<uint32_t>(a.cand_cap);
  if (n_cand != n_bin && tid == 0) raise_error(a.err, DEVERR_BOUNDS);   // histogram and row disagree
  // bin t's keys take the slots after the row's positions below the
  // threshold digit, numbered by a shared counter
  const uint32_t base0 = s_bt;
  __syncthreads();                              // s_h (staging) is reused below

  // the need smallest V of bin t, by radix passes of FDIGIT bits over the
  // bits below the first digit.  A pass keeps the group of keys that share
  // the prefix found so far; once the keys still needed are the whole group
  // it is taken without further passes (typically after one or two passes).
  // Keys come from the candidate list (in shared memory when it fits) or, if
  // bin t overflowed the list, from the row itself.
  const bool smem_list = from_list && n_cand <= static_cast<uint32_t>(LIST_SMEM);
  uint64_t* s_list = reinterpret_cast<uint64_t*>(s_dyn);
  if (smem_list) {
    for (uint32_t i = tid; i < n_cand; i += THREADS) s_list[i] = ld_l2_u64(&cand[i]);
    __syncthreads();
  }
  auto fetch = [&](int i, uint64_t* V) -> bool {   // i < n_src
    if (smem_list) {
      *V = s_list[i];
      return true;
    }
    if (from_list) {
      *V = ld_l2_u64(&cand[i]);
      return true;
    }
    const uint32_t u = ~float_key(ld_l2_f32(&row[i]));
    if ((u >> (32 - DIGIT)) != t) return false;
    *V = (static_cast<uint64_t>(u) << pb) | static_cast<uint64_t>(i);
    return true;
  };
  const int n_src = from_list ? static_cast<int>(n_cand) : vis;
  uint64_t prefix = static_cast<uint64_t>(t) << R0;
  int R = R0;
  uint32_t left = need, group = n_cand;
  while (R > 0 && left < group) {
    const int w = R < FDIGIT ? R : FDIGIT;
    const int shift = R - w;
    for (int i = tid; i < (1 << w); i += THREADS) s_bins[i] = 0;
    __syncthreads();
    for (int i = tid; i < n_src; i += THREADS) {
      uint64_t V;
      if (fetch(i, &V) && (V >> R) == (prefix >> R))
        atomicAdd(&s_bins[static_cast<uint32_t>(V >> shift) & ((1u << w) - 1u)], 1u);
    }
    __syncthreads();
    find_digit(s_bins, 1 << w, left, s_warp, &s_t, &s_below);
    const uint32_t d = s_t;
    left -= s_below;
    group = s_bins[d];
    prefix |= static_cast<uint64_t>(d) << shift;
    R = shift;
    __syncthreads();                            // every thread has read s_bins
  }
  // taken: every key of bin t whose bits above R are at most the prefix's
  for (int i = tid; i < n_src; i += THREADS) {
    uint64_t V = 0;
    if (fetch(i, &V) && (V >> R) <= (prefix >> R)) {
      const uint32_t slot = base0 + atomicAdd(&s_nt, 1u);
      if (slot < static_cast<uint32_t>(topk)) {
        const int p = static_cast<int>(V & pos_mask);
        oi[slot] = p;
        if (os) os[slot] = ld_l2_f32(&row[p]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_topk_hist(const float* scores, int ld, const int32_t* q_offsets,
                             const int32_t* q_vis, int B, int Q, int max_len, int topk,
                             int first_only, const uint32_t* hist, uint32_t* ctr, uint64_t* cand,
                             int cand_cap, int32_t* out_idx, float* out_scores, uint32_t* err,
                             cudaStream_t st, bool pdl) {
  const int rows = first_only ? B : Q;
  if (rows <= 0) return cudaSuccess;
  if (rows > 65535 || topk > DSA_MAX_TOPK) return cudaErrorInvalidValue;
  // CTAs per row: cover the SMs about twice, at least 16K scores a CTA
  const int sms = device_sm_count();
  int cpr = (2 * sms + rows - 1) / rows;
  const int by_len = (max_len + 16383) / 16384;
  if (cpr > by_len) cpr = by_len;
  if (cpr < 1) cpr = 1;
  // the same shared-memory carve-out as the indexer it overlaps, so that an SM
  // need not drain to change its L1/shared split when this kernel arrives
  static std::atomic<bool> attr_done[64];
  const cudaError_t ea = set_once_per_device(attr_done, [] {
    const cudaError_t e = cudaFuncSetAttribute(topk_hist_kernel,
                                               cudaFuncAttributePreferredSharedMemoryCarveout,
                                               cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(topk_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                STAGE_BYTES);
  });
  if (ea != cudaSuccess) return ea;
  HistTopkArgs a{scores, ld, q_offsets, q_vis, B, Q, topk, first_only, hist, ctr, cand, cand_cap,
                 out_idx, out_scores, err};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cpr), static_cast<unsigned>(rows), 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = STAGE_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  unsigned int na = 0;
  add_pdl_attr(attr, &na, pdl);
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, topk_hist_kernel, a);
}

}  // namespace dsa
