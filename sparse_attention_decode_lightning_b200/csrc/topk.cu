// Token selector: the topk highest indexer scores of each query, ties to the
// lower position ("大语言模型结构总览", section 2.2: the token selector keeps the
// k = 2048 best-scoring tokens; section 7.2: causal top-2048).
//
// Exact radix select over 64-bit keys  (order-preserving u32 of the fp32
// score) << 32 | (0xFFFFFFFF - position), which are all distinct, so "the k
// largest keys" is exactly the top-k with the lower-position tie rule.
//   pass 1 (hist):    many CTAs per query build a 4096-bin histogram of the top
//                     12 key bits (shared-memory atomics, merged in global).
//   pass 2 (filter):  every CTA finds the bin holding the k-th key; keys above
//                     it are written out, keys inside it become candidates.
//   pass 3 (resolve): one CTA per query refines the candidates 8 bits at a
//                     time until the remaining candidates are exactly needed.
// Scores are read twice (from L2 when the indexer just wrote them); the
// candidate set is the small slice of the distribution at the threshold.
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int CHUNK = 8192;     // scores per CTA in passes 1 and 2
constexpr int PT = 512;         // threads for passes 1 and 2
constexpr int RT = 1024;        // threads for pass 3

struct TopkArgs {
  const float* scores;
  int ld;
  const int32_t* q_offsets;
  const int32_t* q_vis;
  int B, Q, max_len, topk, first_only;
  int32_t* out_idx;
  float* out_scores;
  uint32_t* hist;
  uint32_t* meta;
  uint64_t* cand;
  uint64_t* cand2;
  uint32_t* err;
};

// query handled by grid row y, or -1
__device__ __forceinline__ int row_query(const TopkArgs& a, int y) {
  if (!a.first_only) return y;
  const int q0 = a.q_offsets[y];
  return (a.q_offsets[y + 1] > q0 && q0 >= 0 && q0 < a.Q) ? q0 : -1;
}

__device__ __forceinline__ int clamped_vis(const TopkArgs& a, int q) {
  int v = a.q_vis[q];
  if (v < 0 || v > a.max_len) {
    raise_error(a.err, DEVERR_BOUNDS);
    v = v < 0 ? 0 : a.max_len;
  }
  return v;
}

__global__ void __launch_bounds__(PT) topk_hist_kernel(TopkArgs a) {
  __shared__ uint32_t h[TOPK_BINS];
  const int q = row_query(a, blockIdx.y);
  if (q < 0) return;
  const int vis = clamped_vis(a, q);
  if (vis <= a.topk) return;                         // every visible key is kept
  const int beg = blockIdx.x * CHUNK;
  if (beg >= vis) return;
  const int end = min(vis, beg + CHUNK);
  for (int i = threadIdx.x; i < TOPK_BINS; i += PT) h[i] = 0;
  __syncthreads();
  const float* row = a.scores + static_cast<size_t>(q) * a.ld;
  for (int i = beg + 4 * threadIdx.x; i < end; i += 4 * PT) {
    const float4 v = *reinterpret_cast<const float4*>(row + i);
    atomicAdd(&h[float_key(v.x) >> 20], 1u);
    if (i + 1 < end) atomicAdd(&h[float_key(v.y) >> 20], 1u);
    if (i + 2 < end) atomicAdd(&h[float_key(v.z) >> 20], 1u);
    if (i + 3 < end) atomicAdd(&h[float_key(v.w) >> 20], 1u);
  }
  __syncthreads();
  uint32_t* g = a.hist + static_cast<size_t>(q) * TOPK_BINS;
  for (int i = threadIdx.x; i < TOPK_BINS; i += PT)
    if (h[i]) atomicAdd(&g[i], h[i]);
}

// threshold bin of a histogram: largest bin b with count(bins >= b) >= k;
// returns b and count(bins > b) through shared memory.  nthreads*per == bins.
template <int NT, int BINS>
__device__ void find_threshold(const uint32_t* hist, uint32_t k, uint32_t* s_bin,
                               uint32_t* s_above, uint32_t* s_tmp) {
  constexpr int PER = BINS / NT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // thread t owns bins [BINS - PER*(t+1), BINS - PER*t), i.e. counted from the top
  const int hi = BINS - PER * tid;
  uint32_t c[PER];
  uint32_t sum = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) { c[j] = hist[hi - 1 - j]; sum += c[j]; }
  uint32_t incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) s_tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    constexpr int NW = NT / 32;
    const uint32_t v = lane < NW ? s_tmp[lane] : 0;
    uint32_t vi = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, vi, off);
      if (lane >= off) vi += y;
    }
    if (lane < NW) s_tmp[lane] = vi - v;
  }
  __syncthreads();
  uint32_t run = s_tmp[warp] + incl - sum;     // count in bins above this thread's range
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if (run < k && run + c[j] >= k) { *s_bin = static_cast<uint32_t>(hi - 1 - j); *s_above = run; }
    run += c[j];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(PT, 2) topk_filter_kernel(TopkArgs a) {
  __shared__ uint32_t s_tmp[32];
  __shared__ uint32_t s_bin, s_above;
  const int q = row_query(a, blockIdx.y);
  if (q < 0) return;
  const int vis = clamped_vis(a, q);
  const int beg = blockIdx.x * CHUNK;
  const float* row = a.scores + static_cast<size_t>(q) * a.ld;
  int32_t* oi = a.out_idx + static_cast<size_t>(q) * a.topk;
  float* os = a.out_scores ? a.out_scores + static_cast<size_t>(q) * a.topk : nullptr;
  if (vis <= a.topk) {                               // keep all visible positions
    const int end = min(vis, beg + CHUNK);
    for (int i = beg + threadIdx.x; i < end; i += PT) {
      oi[i] = i;
      if (os) os[i] = row[i];
    }
    return;
  }
  if (beg >= vis) return;
  const int end = min(vis, beg + CHUNK);
  find_threshold<PT, TOPK_BINS>(a.hist + static_cast<size_t>(q) * TOPK_BINS,
                                static_cast<uint32_t>(a.topk), &s_bin, &s_above, s_tmp);
  const uint32_t tb = s_bin;
  uint32_t* meta = a.meta + static_cast<size_t>(q) * TOPK_META;
  if (blockIdx.x == 0 && threadIdx.x == 0) { meta[2] = tb; meta[3] = s_above; }
  uint64_t* cand = a.cand + static_cast<size_t>(q) * a.ld;
  // each thread holds its CHUNK / PT scores in registers; slots are reserved
  // with one block scan and one global atomic per counter per CTA
  constexpr int PER4 = CHUNK / (4 * PT);
  float4 v[PER4];
  uint32_t na = 0, nc = 0;
#pragma unroll
  for (int k = 0; k < PER4; ++k) {
    const int i = beg + 4 * (threadIdx.x + k * PT);
    v[k] = i < end ? *reinterpret_cast<const float4*>(row + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float vv[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t bin = float_key(vv[e]) >> 20;
      const bool valid = i + e < end;
      na += (valid && bin > tb);
      nc += (valid && bin == tb);
    }
  }
  // block exclusive scan of (na << 16 | nc); totals stay below 2^16 per CTA
  const uint32_t packed = (na << 16) | nc;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = packed;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  __shared__ uint32_t s_warp[PT / 32];
  __shared__ uint32_t s_base_a, s_base_c;
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = lane < PT / 32 ? s_warp[lane] : 0;
    uint32_t xi = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, xi, off);
      if (lane >= off) xi += y;
    }
    if (lane < PT / 32) s_warp[lane] = xi - x;
    if (lane == 31) {
      s_base_a = (xi >> 16) ? atomicAdd(&meta[0], xi >> 16) : 0;
      s_base_c = (xi & 0xFFFFu) ? atomicAdd(&meta[1], xi & 0xFFFFu) : 0;
    }
  }
  __syncthreads();
  const uint32_t pre = s_warp[warp] + incl - packed;
  uint32_t pa = s_base_a + (pre >> 16), pc = s_base_c + (pre & 0xFFFFu);
#pragma unroll
  for (int k = 0; k < PER4; ++k) {
    const int i = beg + 4 * (threadIdx.x + k * PT);
    const float vv[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t key = float_key(vv[e]);
      const uint32_t bin = key >> 20;
      if (i + e < end) {
        if (bin > tb) {
          oi[pa] = i + e;
          if (os) os[pa] = vv[e];
          ++pa;
        } else if (bin == tb) {
          cand[pc++] = (static_cast<uint64_t>(key) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(i + e));
        }
      }
    }
  }
}

__global__ void __launch_bounds__(RT) topk_resolve_kernel(TopkArgs a) {
  __shared__ uint32_t h[256];
  __shared__ uint32_t s_tmp[32];
  __shared__ uint32_t s_digit, s_gt, s_out, s_n;
  const int q = row_query(a, blockIdx.x);
  if (q < 0) return;
  const int vis = clamped_vis(a, q);
  int32_t* oi = a.out_idx + static_cast<size_t>(q) * a.topk;
  float* os = a.out_scores ? a.out_scores + static_cast<size_t>(q) * a.topk : nullptr;
  if (vis <= a.topk) {
    for (int i = vis + threadIdx.x; i < a.topk; i += RT) {
      oi[i] = -1;
      if (os) os[i] = -INFINITY;
    }
    return;
  }
  const uint32_t* meta = a.meta + static_cast<size_t>(q) * TOPK_META;
  uint32_t base = meta[3];                     // positions already written
  uint32_t need = static_cast<uint32_t>(a.topk) - base;
  uint32_t n = meta[1];                        // candidates in the threshold bin
  uint64_t* src = a.cand + static_cast<size_t>(q) * a.ld;
  uint64_t* dst = a.cand2 + static_cast<size_t>(q) * a.ld;
  if (n < need || n > static_cast<uint32_t>(a.ld)) {   // inconsistent counters
    if (threadIdx.x == 0) raise_error(a.err, DEVERR_BOUNDS);
    n = min(n, need);
  }
  // 52 low bits remain undecided: 20 score bits below the 12-bit bin, 32 position bits
  for (int pass = 0; pass <= 7; ++pass) {
    if (n == need || pass == 7) {
      for (uint32_t j = threadIdx.x; j < n && j < need; j += RT) {
        const uint64_t e = src[j];
        oi[base + j] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(e));
        if (os) os[base + j] = key_float(static_cast<uint32_t>(e >> 32));
      }
      break;
    }
    // digit positions 44, 36, 28, 20, 12, 4 (8 bits each), then bits 3..0
    const int sh = pass < 6 ? 44 - 8 * pass : 0;
    const uint32_t mask = pass < 6 ? 0xFFu : 0xFu;
    for (int i = threadIdx.x; i < 256; i += RT) h[i] = 0;
    if (threadIdx.x == 0) { s_out = 0; s_n = 0; s_digit = 0; s_gt = 0; }
    __syncthreads();
    for (uint32_t j = threadIdx.x; j < n; j += RT)
      atomicAdd(&h[static_cast<uint32_t>(src[j] >> sh) & mask], 1u);
    __syncthreads();
    {
      // threshold digit: largest d with count(digits >= d) >= need
      uint32_t c = threadIdx.x < 256 ? h[255 - threadIdx.x] : 0;
      const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
      uint32_t incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (lane == 31) s_tmp[warp] = incl;
      __syncthreads();
      if (warp == 0) {
        const uint32_t v = s_tmp[lane];
        uint32_t vi = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, vi, off);
          if (lane >= off) vi += y;
        }
        s_tmp[lane] = vi - v;
      }
      __syncthreads();
      const uint32_t before = s_tmp[warp] + incl - c;   // count in digits above
      if (threadIdx.x < 256 && before < need && before + c >= need) {
        s_digit = 255u - threadIdx.x;
        s_gt = before;
      }
      __syncthreads();
    }
    const uint32_t d = s_digit, gt = s_gt;
    for (uint32_t j = threadIdx.x; j < n; j += RT) {
      const uint64_t e = src[j];
      const uint32_t dg = static_cast<uint32_t>(e >> sh) & mask;
      if (dg > d) {
        const uint32_t p = base + atomicAdd(&s_out, 1u);
        oi[p] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(e));
        if (os) os[p] = key_float(static_cast<uint32_t>(e >> 32));
      } else if (dg == d) {
        dst[atomicAdd(&s_n, 1u)] = e;
      }
    }
    __syncthreads();
    base += gt;
    need -= gt;
    n = h[d];
    uint64_t* t = src; src = dst; dst = t;
    __syncthreads();
  }
}

__global__ void expand_idx_kernel(const int32_t* q_offsets, int Q, int topk, int32_t* out_idx,
                                  float* out_scores) {
  const int b = blockIdx.x;
  const int q0 = q_offsets[b], q1 = q_offsets[b + 1];
  if (q0 < 0 || q1 > Q) return;
  for (int q = q0 + 1; q < q1; ++q) {
    for (int i = threadIdx.x; i < topk; i += blockDim.x) {
      out_idx[static_cast<size_t>(q) * topk + i] = out_idx[static_cast<size_t>(q0) * topk + i];
      if (out_scores)
        out_scores[static_cast<size_t>(q) * topk + i] = out_scores[static_cast<size_t>(q0) * topk + i];
    }
  }
}

}  // namespace

cudaError_t launch_topk(const float* scores, int ld, const int32_t* q_offsets,
                        const int32_t* q_vis, int B, int Q, int max_len, int topk,
                        int first_only, int32_t* out_idx, float* out_scores, uint32_t* hist,
                        uint32_t* meta, uint64_t* cand, uint64_t* cand2, uint32_t* err,
                        cudaStream_t st) {
  const int rows = first_only ? B : Q;
  if (rows <= 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(hist, 0, static_cast<size_t>(Q) * TOPK_BINS * sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(meta, 0, static_cast<size_t>(Q) * TOPK_META * sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  TopkArgs a{scores, ld, q_offsets, q_vis, B, Q, max_len, topk, first_only,
             out_idx, out_scores, hist, meta, cand, cand2, err};
  const dim3 grid((max_len + CHUNK - 1) / CHUNK, rows);
  topk_hist_kernel<<<grid, PT, 0, st>>>(a);
  topk_filter_kernel<<<grid, PT, 0, st>>>(a);
  topk_resolve_kernel<<<rows, RT, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_expand_idx(const int32_t* q_offsets, int B, int Q, int topk, int32_t* out_idx,
                              float* out_scores, cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  expand_idx_kernel<<<B, 256, 0, st>>>(q_offsets, Q, topk, out_idx, out_scores);
  return cudaGetLastError();
}

}  // namespace dsa
