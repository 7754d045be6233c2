// Sparse MLA decode on sm_100a tensor cores (absorbed MQA over the selected
// latents).  Source: "大语言模型结构总览", section 2.2 (MLA in MQA mode over the
// k = 2048 selected tokens; paged and non-paged kernels) and section 2.1 (one
// 576-d latent per token = 512 kv rank + 64 RoPE; 128 heads).  Per head h:
//   z_j = scale * q[h,:] . C[j,:],  O[h] = sum_j softmax(z)_j C[j,:512],
//   LSE[h] = ln sum_j exp(z_j).
//
// Work unit: (query, split) on a cluster of two CTAs.  The 128 x 512 fp32
// output alone fills one SM's tensor memory, and the 128 x 576 bf16 query
// (147 KB) would crowd out the gather pipeline, so the pair divides both:
//   CTA 0 holds q[:, 0:256) and computes S0 = q[:,0:256) C[:,0:256)^T and
//         O[:, 0:256);
//   CTA 1 holds q[:, 256:576) and computes S1 = q[:,256:576) C[:,256:576)^T
//         and O[:, 256:512).
// Each CTA gathers only the latent columns it uses (0:256 or 256:576), so
// every latent byte crosses HBM once.  Per 32-row tile the CTAs swap their
// fp32 partial scores through distributed shared memory; both form
// S = S0 + S1 (bitwise equal on both sides), run the same online softmax and
// feed the same P to their half of O += P V.
//
// Roles per CTA (192 threads):
//   warp 0      producer: page-table lookups and TMA tile::gather4 row
//               gathers (4 rows x 128 B per op, 128-byte swizzle) into a
//               3-stage ring; the query slice once.
//   warp 1      tcgen05 issuer: S (M=128 heads, N=32 rows, K=256|320) into a
//               double-buffered TMEM slot; O += P V (M=128, N=256, V read
//               MN-major straight from the gathered tile).
//   warps 2..5  softmax: one head row per thread; exchange, online softmax
//               in the exp2 domain with a lazy rescale of O (only when the
//               running max grows by more than 2^8), P into shared memory as
//               a bf16 hi + lo pair (about 16 significant bits: a single bf16
//               P costs ~1% of the output RMS once the running max is stale),
//               final O / l and LSE.
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int NR = 32;                         // selected rows per tile
constexpr int NST = 3;                         // gather ring depth
constexpr int THREADS = 192;
constexpr int MAXCH = 5;                       // 64-column chunks per CTA (CTA 1)
constexpr int CHUNK_Q = DSA_HEADS * 128;       // 16 KB: 128 heads x 64 bf16
constexpr int CHUNK_T = NR * 128;              // 4 KB: 32 rows x 64 bf16
constexpr int STAGE_BYTES = MAXCH * CHUNK_T;
constexpr int P_BYTES = DSA_HEADS * 128;       // 128 rows of 32 bf16 hi + 32 bf16 lo
constexpr int X_BYTES = DSA_HEADS * NR * 4;    // one tile of fp32 partial scores
constexpr int OFF_Q = 0;
constexpr int OFF_ST = OFF_Q + MAXCH * CHUNK_Q;
constexpr int OFF_P = OFF_ST + NST * STAGE_BYTES;
constexpr int OFF_X = OFF_P + 2 * P_BYTES;
constexpr int OFF_CRD = OFF_X + 2 * X_BYTES;    // pool row of every entry of the split
constexpr int OFF_BAR = OFF_CRD + DSA_MAX_TOPK * 4;
constexpr int NBAR = 2 * NST + 5 * 2 + 3;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "sparse MLA shared memory exceeds the sm_100 limit");
static_assert(OFF_ST % 1024 == 0 && OFF_P % 1024 == 0 && OFF_X % 1024 == 0, "swizzle atoms");
constexpr uint32_t O_COL = 0;                  // TMEM columns [0,256): O half
constexpr uint32_t S_COL = 256;                // [256,320): two 32-column score slots
constexpr uint32_t TMEM_COLS = 512;

struct MlaTcArgs {
  const int32_t* page_table;
  int max_pages;
  int num_pages;
  const int32_t* q_offsets;
  const int32_t* q_vis;
  const int32_t* idx;
  int B, Q, topk, S;
  float scale_log2;
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

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
  const bool ok = mbar_wait(bar, parity, err);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    sparse_mla_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_kv, MlaTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qs = smem + OFF_Q;
  uint8_t* st = smem + OFF_ST;
  uint8_t* pb = smem + OFF_P;
  uint8_t* xb = smem + OFF_X;
  int* crd = reinterpret_cast<int*>(smem + OFF_CRD);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + NST;
  uint64_t* s_full = bars + 2 * NST;
  uint64_t* s_empty = s_full + 2;
  uint64_t* x_full = s_empty + 2;
  uint64_t* p_full = x_full + 2;
  uint64_t* p_empty = p_full + 2;
  uint64_t* o_done = p_empty + 2;
  uint64_t* o_final = o_done + 1;
  uint64_t* q_full = o_final + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int unit = blockIdx.x >> 1;
  const int q = unit / a.S, split = unit % a.S;
  const int nch = rank ? 5 : 4;                 // 64-column chunks gathered by this CTA
  const int gch0 = rank ? 4 : 0;                // first global chunk
  const int b = seq_of_query(a.q_offsets, a.B, q);
  int vis = a.q_vis[q];
  if (vis < 0) vis = 0;
  const int per = (a.topk + a.S - 1) / a.S;
  const int r0 = split * per;
  const int r1 = min(a.topk, r0 + per);
  const int ntiles = r1 > r0 ? (r1 - r0 + NR - 1) / NR : 0;

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);     // one arrival per softmax warp
      mbar_init(&x_full[i], 4);      // one remote arrival per peer softmax warp
      mbar_init(&p_full[i], 4);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    mbar_init(q_full, 1);
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();                 // the peer's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (tid == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_kv);
    mbar_arrive_expect_tx(q_full, nch * CHUNK_Q);
    for (int c = 0; c < nch; ++c)
      tma_load_2d(qs + c * CHUNK_Q, &tmap_q, (gch0 + c) * 64, q * DSA_HEADS, q_full);
  }
  // pool row of every entry of this split, resolved once by all threads with
  // many independent loads in flight (-1 = padding or out of range)
  {
    constexpr int PER = (DSA_MAX_TOPK + THREADS - 1) / THREADS;
    int sv[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int j = r0 + tid + k * THREADS;
      sv[k] = j < r1 ? a.idx[static_cast<size_t>(q) * a.topk + j] : -1;
    }
    int pg[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int sx = sv[k];
      const bool ok = sx >= 0 && sx < vis && (sx >> 6) < a.max_pages;
      pg[k] = ok ? a.page_table[static_cast<size_t>(b) * a.max_pages + (sx >> 6)] : -1;
    }
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int jj = tid + k * THREADS;
      if (r0 + jj < r1) {
        const int sx = sv[k];
        const bool ok = pg[k] >= 0 && pg[k] < a.num_pages;
        if (!ok && sx != -1 && rank == 0) raise_error(a.err, DEVERR_BOUNDS);
        crd[jj] = ok ? pg[k] * DSA_PAGE_SIZE + (sx & (DSA_PAGE_SIZE - 1)) : -1;
      }
    }
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = l2_policy_evict_first();
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % NST;
      if (!warp_wait(&empty[s], ((t / NST) & 1) ^ 1, a.err)) break;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], nch * CHUNK_T);
      __syncwarp();
      if (lane < NR / 4) {
        const int j = t * NR + 4 * lane;        // entry within the split
        const int n = r1 - r0;
        const int c0 = j + 0 < n ? crd[j + 0] : -1;
        const int c1 = j + 1 < n ? crd[j + 1] : -1;
        const int c2 = j + 2 < n ? crd[j + 2] : -1;
        const int c3 = j + 3 < n ? crd[j + 3] : -1;
        for (int c = 0; c < nch; ++c)
          tma_gather4(st + s * STAGE_BYTES + c * CHUNK_T + 4 * lane * 128, &tmap_kv,
                      (gch0 + c) * 64, c0, c1, c2, c3, &full[s], pol);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_s = umma_idesc(1 /*BF16*/, DSA_HEADS, NR);
      constexpr uint32_t idesc_pv = umma_idesc(1 /*BF16*/, DSA_HEADS, 256, 0, 1);
      bool ok = mbar_wait(q_full, 0, a.err);
      for (int t = 0; t <= ntiles && ok; ++t) {
        if (t < ntiles) {
          const int s = t % NST, sb = t & 1;
          if (!mbar_wait(&full[s], (t / NST) & 1, a.err)) break;
          if (!mbar_wait(&s_empty[sb], ((t >> 1) & 1) ^ 1, a.err)) break;
          tc_fence_after();
          const uint32_t qa = smem_u32(qs), ta = smem_u32(st + s * STAGE_BYTES);
          for (int c = 0; c < nch; ++c) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_f16(tmem + S_COL + sb * NR,
                      umma_desc_sw128(qa + c * CHUNK_Q + kk * 32, 1024, 16),
                      umma_desc_sw128(ta + c * CHUNK_T + kk * 32, 1024, 16), idesc_s,
                      (c | kk) != 0);
            }
          }
          mma_commit(&s_full[sb]);
        }
        if (t >= 1) {
          const int u = t - 1, ub = u & 1, us = u % NST;
          if (!mbar_wait(&p_full[ub], (u >> 1) & 1, a.err)) break;
          tc_fence_after();
          const uint32_t pa = smem_u32(pb + ub * P_BYTES), va = smem_u32(st + us * STAGE_BYTES);
          // k-steps 0,1: P_hi x V rows 0-15, 16-31; k-steps 2,3: P_lo x the same rows
#pragma unroll
          for (int kk = 0; kk < 2 * (NR / 16); ++kk) {
            mma_f16(tmem + O_COL, umma_desc_sw128(pa + kk * 32, 1024, 16),
                    umma_desc_sw128_mn(va + (kk % (NR / 16)) * 2048, CHUNK_T, 1024), idesc_pv,
                    (u > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&p_empty[ub]);
          mma_commit(o_done);
          mma_commit(&empty[us]);
          if (u == ntiles - 1) mma_commit(o_final);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t peer = rank ^ 1u;
    const uint32_t peer_x = map_to_rank(smem_u32(xb), peer);
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
      const int sb = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      const int jrow = t * NR + lane;
      const uint32_t vmask = __ballot_sync(0xffffffffu, jrow < r1 - r0 && crd[jrow] >= 0);
      if (!(ok = warp_wait(&s_full[sb], ph, a.err))) break;
      tc_fence_after();
      float v[NR];
      tmem_ld32(lane_base + S_COL + sb * NR, v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[sb]);
      // my partial scores -> the peer's exchange slot; the warp barrier orders
      // all lanes' stores before lane 0's cluster-scope release arrive
      const uint32_t dst = peer_x + sb * X_BYTES + h * NR * 4;
#pragma unroll
      for (int i = 0; i < NR / 4; ++i)
        st_cluster_v4(dst + 16 * i, v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_rank(smem_u32(&x_full[sb]), peer));
      const bool got = mbar_wait_cluster(&x_full[sb], ph, a.err);
      if (!(ok = __all_sync(0xffffffffu, got))) break;
      const float4* src = reinterpret_cast<const float4*>(xb + sb * X_BYTES + h * NR * 4);
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < NR / 4; ++i) {
        const float4 pv = src[i];
        const float s4[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = 4 * i + k;
          const float z = ((vmask >> r) & 1u) ? (v[r] + s4[k]) * a.scale_log2 : -INFINITY;
          v[r] = z;
          mt = fmaxf(mt, z);
        }
      }
      // running max, moved only when it grows by more than 8 (a factor 2^8)
      float alpha = 1.f;
      bool resc = false;
      if (mt > m_use + 8.f) {
        if (m_use != -INFINITY) {
          alpha = fast_exp2(m_use - mt);
          resc = true;
        }
        m_use = mt;
      }
      float ps = 0.f;
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        const float p = (v[r] == -INFINITY) ? 0.f : fast_exp2(v[r] - m_use);
        v[r] = p;
        ps += p;
      }
      l = l * alpha + ps;
      // the P slot is free once PV(t-2) is done
      if (!(ok = warp_wait(&p_empty[sb], ph ^ 1, a.err))) break;
      if (__any_sync(0xffffffffu, resc)) {
        // O must not move under a running PV: wait for PV(t-1)
        if (t >= 1 && !(ok = warp_wait(o_done, (t - 1) & 1, a.err))) break;
        tc_fence_after();
        for (int c = 0; c < 256 / 32; ++c) {
          float o[32];
          tmem_ld32(lane_base + O_COL + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(lane_base + O_COL + c * 32, o);
        }
        tmem_st_wait();
        tc_fence_before();
      }
      // P row h as bf16 hi + lo (p ~= hi + lo to ~16 bits): hi in 16-byte
      // chunks 0..3, lo in chunks 4..7 of the 128-byte row, 128-byte swizzle
      // (chunk u stored at u ^ (h & 7)).  PV then runs over K = 64 =
      // [P_hi | P_lo] against [V ; V].
      uint8_t* prow = pb + sb * P_BYTES + h * 128;
#pragma unroll
      for (int u = 0; u < NR / 8; ++u) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __nv_bfloat162 hv = __floats2bfloat162_rn(v[8 * u + 2 * k], v[8 * u + 2 * k + 1]);
          const float2 hf = __bfloat1622float2(hv);
          const __nv_bfloat162 lv =
              __floats2bfloat162_rn(v[8 * u + 2 * k] - hf.x, v[8 * u + 2 * k + 1] - hf.y);
          hw[k] = *reinterpret_cast<const uint32_t*>(&hv);
          lw[k] = *reinterpret_cast<const uint32_t*>(&lv);
        }
        *reinterpret_cast<uint4*>(prow + ((u ^ (h & 7)) * 16)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(prow + (((u + 4) ^ (h & 7)) * 16)) =
            make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    // ---- epilogue: O / l for this CTA's 256 value columns; LSE from CTA 0
    const bool have = ok && ntiles > 0 && warp_wait(o_final, 0, a.err);
    if (have) tc_fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* orow;
    float* lrow;
    if (a.S == 1) {
      orow = a.out + (static_cast<size_t>(q) * DSA_HEADS + h) * DSA_DIM_V + rank * 256;
      lrow = a.lse + static_cast<size_t>(q) * DSA_HEADS + h;
    } else {
      orow = a.o_part + ((static_cast<size_t>(q) * a.S + split) * DSA_HEADS + h) * DSA_DIM_V + rank * 256;
      lrow = a.l_part + (static_cast<size_t>(q) * a.S + split) * DSA_HEADS + h;
    }
    for (int c = 0; c < 256 / 32; ++c) {
      float o[32];
      if (have) {
        tmem_ld32(lane_base + O_COL + c * 32, o);
        tmem_ld_wait();
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 w = have && l > 0.f ? make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(orow + c * 32 + i) = w;
      }
    }
    if (rank == 0) *lrow = l > 0.f ? m_use * 0.69314718055994531f + logf(l) : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  cluster_sync();                 // no CTA leaves while its peer may still touch it
}

}  // namespace

cudaError_t launch_sparse_mla_tc(const __nv_bfloat16* q, const __nv_bfloat16* pool, int num_pages,
                                 const int32_t* page_table, int max_pages,
                                 const int32_t* q_offsets, const int32_t* q_vis,
                                 const int32_t* idx, int B, int Q, int topk, float scale, int S,
                                 float* out, float* lse, float* o_part, float* l_part,
                                 uint32_t* err, cudaStream_t st) {
  if (Q <= 0) return cudaSuccess;
  CUtensorMap tq, tkv;
  if (!encode_tiled_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, DSA_DIM,
                       static_cast<uint64_t>(Q) * DSA_HEADS, DSA_DIM * 2, 64, DSA_HEADS))
    return cudaErrorInvalidValue;
  if (!encode_tiled_2d(&tkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pool, DSA_DIM,
                       static_cast<uint64_t>(num_pages) * DSA_PAGE_SIZE, DSA_DIM * 2, 64, 1))
    return cudaErrorInvalidValue;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(sparse_mla_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  MlaTcArgs a{page_table, max_pages, num_pages, q_offsets, q_vis, idx, B, Q, topk, S,
              scale * 1.4426950408889634f, out, lse, o_part, l_part, err};
  sparse_mla_tc_kernel<<<2 * Q * S, THREADS, SMEM_BYTES, st>>>(tq, tkv, a);
  return cudaGetLastError();
}

}  // namespace dsa
