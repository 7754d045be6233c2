// Sparse MLA decode, CUDA-core form (absorbed MQA over the selected tokens).
//
// Source: "大语言模型结构总览", section 2.2 (MLA in MQA mode over the tokens the
// selector keeps) and section 2.1 (576-d latent = 512 kv rank + 64 RoPE,
// 128 heads).  Per head h and selected token j:
//   z_j = scale * q[h,:576] . C[j,:576],  O[h] = sum_j softmax(z)_j C[j,:512],
//   LSE[h] = ln sum_j exp(z_j).
//
// One CTA = (query, split, 8 heads); one warp per head.  Tiles of 32 selected
// rows are gathered through the page table into shared memory; each warp
// keeps an online softmax (running max and sum) and its 512 output values in
// registers (16 per lane).  Out-of-range indices are skipped and flagged.
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int ROWS = 32;
constexpr int HPC = 8;                    // heads per CTA
constexpr int THREADS = HPC * 32;
constexpr int CH = DSA_DIM / 8;           // 16-byte chunks per latent row (72)

struct MlaArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* pool;
  int num_pages;
  const int32_t* page_table;
  int max_pages;
  const int32_t* q_offsets;
  const int32_t* q_vis;
  const int32_t* idx;
  int B, Q, topk;
  float scale;
  int S;
  float* out;
  float* lse;
  float* o_part;
  float* l_part;
  uint32_t* err;
};

__device__ __forceinline__ int seq_of_query(const int32_t* q_offsets, int B, int q) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (q_offsets[mid] <= q) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(THREADS) sparse_mla_simt_kernel(MlaArgs a) {
  __shared__ __align__(16) __nv_bfloat16 tile[ROWS * DSA_DIM];
  __shared__ int64_t row_off[ROWS];       // element offset of the row in the pool, -1 = skip
  const int q = blockIdx.x, split = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.z * HPC + warp;
  const int b = seq_of_query(a.q_offsets, a.B, q);
  const int vis = a.q_vis[q];
  const int per = (a.topk + a.S - 1) / a.S;
  const int r0 = split * per, r1 = min(a.topk, r0 + per);

  float qv[DSA_DIM / 32];
  const __nv_bfloat16* qh = a.q + (static_cast<size_t>(q) * DSA_HEADS + h) * DSA_DIM;
#pragma unroll
  for (int i = 0; i < DSA_DIM / 32; ++i) qv[i] = __bfloat162float(qh[lane + 32 * i]);

  float m = -INFINITY, l = 0.f;
  float o[DSA_DIM_V / 32];
#pragma unroll
  for (int i = 0; i < DSA_DIM_V / 32; ++i) o[i] = 0.f;

  for (int r = r0; r < r1; r += ROWS) {
    __syncthreads();
    if (threadIdx.x < ROWS) {
      const int j = r + threadIdx.x;
      int64_t off = -1;
      if (j < r1) {
        const int s = a.idx[static_cast<size_t>(q) * a.topk + j];
        if (s >= 0) {
          const int pg_slot = s / DSA_PAGE_SIZE;
          bool ok = s < vis && pg_slot < a.max_pages;
          int pg = ok ? a.page_table[static_cast<size_t>(b) * a.max_pages + pg_slot] : -1;
          ok = ok && pg >= 0 && pg < a.num_pages;
          if (ok) off = (static_cast<int64_t>(pg) * DSA_PAGE_SIZE + s % DSA_PAGE_SIZE) * DSA_DIM;
          else raise_error(a.err, DEVERR_BOUNDS);
        }
      }
      row_off[threadIdx.x] = off;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < ROWS * CH; c += THREADS) {
      const int rr = c / CH, ch = c % CH;
      const int64_t off = row_off[rr];
      uint4 v = make_uint4(0, 0, 0, 0);
      if (off >= 0) v = *reinterpret_cast<const uint4*>(a.pool + off + ch * 8);
      *reinterpret_cast<uint4*>(&tile[rr * DSA_DIM + ch * 8]) = v;
    }
    __syncthreads();
    // scores of the 32 rows; lane j keeps row j's
    float z_mine = -INFINITY;
    for (int j = 0; j < ROWS; ++j) {
      float p = 0.f;
#pragma unroll
      for (int i = 0; i < DSA_DIM / 32; ++i)
        p = fmaf(qv[i], __bfloat162float(tile[j * DSA_DIM + lane + 32 * i]), p);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
      if (lane == j && row_off[j] >= 0) z_mine = p * a.scale;
    }
    float tmax = z_mine;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
    const float m_new = fmaxf(m, tmax);
    if (m_new == -INFINITY) continue;
    const float alpha = (m == -INFINITY) ? 0.f : __expf(m - m_new);
    const float p_mine = (z_mine == -INFINITY) ? 0.f : expf(z_mine - m_new);
    float psum = p_mine;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    l = l * alpha + psum;
#pragma unroll
    for (int i = 0; i < DSA_DIM_V / 32; ++i) o[i] *= alpha;
    for (int j = 0; j < ROWS; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p_mine, j);
      if (pj != 0.f) {
#pragma unroll
        for (int i = 0; i < DSA_DIM_V / 32; ++i)
          o[i] = fmaf(pj, __bfloat162float(tile[j * DSA_DIM + lane + 32 * i]), o[i]);
      }
    }
    m = m_new;
  }

  float* oo;
  float* ll;
  if (a.S == 1) {
    oo = a.out + (static_cast<size_t>(q) * DSA_HEADS + h) * DSA_DIM_V;
    ll = a.lse + static_cast<size_t>(q) * DSA_HEADS + h;
  } else {
    oo = a.o_part + ((static_cast<size_t>(q) * a.S + split) * DSA_HEADS + h) * DSA_DIM_V;
    ll = a.l_part + (static_cast<size_t>(q) * a.S + split) * DSA_HEADS + h;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int i = 0; i < DSA_DIM_V / 32; ++i) oo[lane + 32 * i] = o[i] * inv;
  if (lane == 0) *ll = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_sparse_mla_simt(const __nv_bfloat16* q, const __nv_bfloat16* pool,
                                   int num_pages, const int32_t* page_table, int max_pages,
                                   const int32_t* q_offsets, const int32_t* q_vis,
                                   const int32_t* idx, int B, int Q, int topk, float scale,
                                   int S, float* out, float* lse, float* o_part, float* l_part,
                                   uint32_t* err, cudaStream_t st) {
  MlaArgs a{q, pool, num_pages, page_table, max_pages, q_offsets, q_vis, idx, B, Q, topk,
            scale, S, out, lse, o_part, l_part, err};
  const dim3 grid(Q, S, DSA_HEADS / HPC);
  sparse_mla_simt_kernel<<<grid, THREADS, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
