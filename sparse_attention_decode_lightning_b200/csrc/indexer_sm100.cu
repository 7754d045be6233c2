// Lightning indexer on sm_100a: I[q,s] = sum_h w[q,h] * ReLU(q_idx[q,h,:] . K[s,:]).
//
// Source: "大语言模型结构总览", section 2.2 DeepSeek-V3.2 -- the indexer is a
// light FP8 scorer (64 heads x 128 dims) that gives every prior token of a
// query one relevance scalar; it streams the whole key cache, which makes it
// the HBM-bound part of the decode step.
//
// Design (persistent, warp-specialised, one CTA per SM):
//   warp 0      TMA producer: 128-key x 128-byte e4m3 tiles (16 KB, 128-byte
//               swizzle) into an 8-stage shared-memory ring; the queries of the
//               current sequence (8 KB each) into a query buffer.
//   warps 1,2   two tcgen05 issuers, one per pipeline; pipeline p takes the
//               CTA's key tiles of parity p: for every query of the tile's
//               sequence, D[128 keys, 64 heads] = K_tile . q^T as 4 MMAs of
//               kind::f8f6f4 (M=128, N=64, K=32) into one of its 4 TMEM slots
//               (64 columns each, all 512 columns in use).  A single issuer
//               thread spends ~1500 cycles per tile on mbarrier waits, MMA
//               issue and commits, which alone caps a CTA near 25 GB/s; two
//               independent issuers double that.
//   warps 3..10 two epilogue warpgroups, one per pipeline: each thread reads
//               its key row (64 fp32 head dots) with tcgen05.ld and reduces
//               sum_h w_h * max(d_h, 0) in registers; 128 consecutive fp32
//               scores per warpgroup are written coalesced.
// Work: the flattened list of (sequence, 128-key tile) items is cut into
// equal contiguous ranges, one per CTA; a sequence's keys are read once for
// all of its queries (MTP verify positions share the tile).
#include "common.cuh"
#include "internal.h"


namespace dsa {
namespace {

constexpr int KT = 128;                                // keys per tile (MMA M)
constexpr int STAGES = 8;                              // key-tile ring depth
constexpr int NACC = 8;                                // TMEM accumulator slots (all 512 columns)
constexpr int ACC_COLS = DSA_IDX_HEADS;                // 64 fp32 columns per slot
constexpr int PIPES = 2;                               // MMA issuer + epilogue warpgroup pairs
constexpr int SLOTS_PER_PIPE = NACC / PIPES;
constexpr int THREADS = 32 + PIPES * 32 + PIPES * 128;
constexpr int KEY_TILE = KT * DSA_IDX_DIM;             // 16384 B
constexpr int Q_TILE = DSA_IDX_HEADS * DSA_IDX_DIM;    // 8192 B
constexpr int OFF_KEYS = 0;
constexpr int OFF_Q = OFF_KEYS + STAGES * KEY_TILE;
constexpr int OFF_PREFIX = OFF_Q + DSA_MAX_Q_PER_SEQ * Q_TILE;
constexpr int OFF_SCAN = OFF_PREFIX + ((DSA_MAX_BATCH + 1) * 4 + 15) / 16 * 16;
constexpr int OFF_BAR = OFF_SCAN + 64 * 4;
constexpr int NBAR = 2 * STAGES + 2 * NACC + 2 + PIPES;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_USED = OFF_MISC + 16;
constexpr int SMEM_BYTES = SMEM_USED + 1024;           // slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "indexer shared memory exceeds the sm_100 limit");

struct IdxArgs {
  const float* w;
  const int64_t* seq_offsets;
  const int32_t* q_offsets;
  const int32_t* q_vis;
  float* scores;
  int ld;
  int B;
  int first_only;
  uint32_t* err;
};

// queries of sequence b that this launch scores (0 if the entry is invalid)
__device__ __forceinline__ int seq_queries(const IdxArgs& a, int b) {
  const int n = a.q_offsets[b + 1] - a.q_offsets[b];
  if (n < 0 || n > DSA_MAX_Q_PER_SEQ) return -1;
  return a.first_only ? (n > 0 ? 1 : 0) : n;
}

// visible keys of query q, clamped to the sequence length and the score row
__device__ __forceinline__ int query_vis(const IdxArgs& a, int q, int64_t len, bool* bad) {
  int v = a.q_vis[q];
  const int64_t lim = len < a.ld ? len : a.ld;
  if (v < 0) { *bad = true; v = 0; }
  if (v > lim) { *bad = true; v = static_cast<int>(lim); }
  return v;
}

// exclusive scan of x[0..n) in place, x[n] = total; all threads participate
__device__ void block_exclusive_scan(int* x, int n, int* tmp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = blockDim.x >> 5;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int beg = min(n, tid * per), end = min(n, beg + per);
  int s = 0;
  for (int i = beg; i < end; ++i) s += x[i];
  int incl = s;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < nw ? tmp[lane] : 0;
    int vi = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, vi, off);
      if (lane >= off) vi += y;
    }
    if (lane < nw) tmp[lane] = vi - v;
    if (lane == 31) tmp[32] = vi;
  }
  __syncthreads();
  int base = tmp[warp] + incl - s;
  for (int i = beg; i < end; ++i) {
    const int t = x[i];
    x[i] = base;
    base += t;
  }
  __syncthreads();
  if (tid == 0) x[n] = tmp[32];
  __syncthreads();
}

__global__ void __launch_bounds__(THREADS, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_q, IdxArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* keys = smem + OFF_KEYS;
  uint8_t* qbuf = smem + OFF_Q;
  int* prefix = reinterpret_cast<int*>(smem + OFF_PREFIX);
  int* scan_tmp = reinterpret_cast<int*>(smem + OFF_SCAN);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = acc_full + NACC;
  uint64_t* q_full = acc_empty + NACC;
  uint64_t* q_empty = q_full + 1;
  uint64_t* mma_done = q_full + 2;        // one per pipeline
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = a.B;

  // ---- tiles per sequence -> exclusive prefix over the batch
  for (int b = tid; b < B; b += THREADS) {
    const int nq = seq_queries(a, b);
    bool bad = nq < 0;
    int mv = 0;
    const int64_t len = a.seq_offsets[b + 1] - a.seq_offsets[b];
    if (len < 0) bad = true;
    for (int j = 0; j < nq; ++j) mv = max(mv, query_vis(a, a.q_offsets[b] + j, len < 0 ? 0 : len, &bad));
    if (bad) raise_error(a.err, DEVERR_BOUNDS);
    prefix[b] = (nq <= 0 || len < 0) ? 0 : (mv + KT - 1) / KT;
  }
  __syncthreads();
  block_exclusive_scan(prefix, B, scan_tmp);

  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < NACC; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 4); }
    mbar_init(q_full, 1);
    mbar_init(q_empty, PIPES);        // every MMA issuer releases the query buffer
    for (int p = 0; p < PIPES; ++p) mbar_init(&mma_done[p], 1);
    mbar_fence_init();
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_q);
  }
  if (warp == 1) tmem_alloc(tmem_holder, NACC * ACC_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int total = prefix[B];
  const int t_begin = static_cast<int>(static_cast<int64_t>(total) * blockIdx.x / gridDim.x);
  const int t_end = static_cast<int>(static_cast<int64_t>(total) * (blockIdx.x + 1) / gridDim.x);

  // first sequence of this CTA's range: largest b with prefix[b] <= t_begin
  int b_first = 0;
  if (t_begin < t_end) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= t_begin) lo = mid; else hi = mid - 1;
    }
    b_first = lo;
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && t_begin < t_end) {
      const uint64_t pol = l2_policy_evict_first();
      int b = b_first, cur_b = -1;
      uint32_t stage = 0, phase = 0, qphase = 0, issued = 0, q_issued = 0;
      bool ok = true;
      for (int i = t_begin; i < t_end && ok; ++i) {
        while (prefix[b + 1] <= i) ++b;
        const int t = i - prefix[b];
        if (b != cur_b) {
          if (cur_b >= 0) {
            if (!mbar_wait(q_empty, qphase, a.err)) { ok = false; break; }
            qphase ^= 1;
          }
          const int nq = seq_queries(a, b);
          mbar_arrive_expect_tx(q_full, nq * Q_TILE);
          for (int j = 0; j < nq; ++j)
            tma_load_2d(qbuf + j * Q_TILE, &tmap_q, 0, (a.q_offsets[b] + j) * DSA_IDX_HEADS, q_full);
          ++q_issued;
          cur_b = b;
        }
        if (!mbar_wait(&empty[stage], phase ^ 1, a.err)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[stage], KEY_TILE);
        const int64_t row = a.seq_offsets[b] + static_cast<int64_t>(t) * KT;
        tma_load_2d_hint(keys + stage * KEY_TILE, &tmap_k, 0, static_cast<int>(row), &full[stage], pol);
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) {
        // drain the copies still in flight before the CTA's memory goes away
        const uint32_t n = issued < STAGES ? issued : STAGES;
        for (uint32_t k = 0; k < n; ++k) {
          const uint32_t it = issued - 1 - k;
          mbar_wait(&full[it % STAGES], (it / STAGES) & 1, a.err);
        }
        if (q_issued) mbar_wait(q_full, (q_issued - 1) & 1, a.err);
      }
    }
  } else if (warp <= 2) {
    // ------------------------------------------------------------ MMA issuers
    // pipeline p = warp - 1 owns the CTA's tiles of parity p and TMEM slots
    // 4p .. 4p+3; both walk every tile to keep the query-buffer hand-off in step
    const int pipe = warp - 1;
    if (lane == 0 && t_begin < t_end) {
      constexpr uint32_t idesc = umma_idesc(0 /*E4M3*/, KT, ACC_COLS);
      int b = b_first, cur_b = -1, nq = 0;
      uint32_t qphase = 0, n = 0;
      bool ok = true;
      for (int i = t_begin; i < t_end && ok; ++i) {
        while (prefix[b + 1] <= i) ++b;
        if (b != cur_b) {
          if (cur_b >= 0) mma_commit(q_empty);
          if (!mbar_wait(q_full, qphase, a.err)) { ok = false; break; }
          qphase ^= 1;
          nq = seq_queries(a, b);
          cur_b = b;
        }
        const int local = i - t_begin;
        if ((local & 1) != pipe) continue;
        const int stage = local % STAGES;
        if (!mbar_wait(&full[stage], (local / STAGES) & 1, a.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(keys + stage * KEY_TILE);
        for (int j = 0; j < nq; ++j, ++n) {
          const uint32_t slot = pipe * SLOTS_PER_PIPE + n % SLOTS_PER_PIPE;
          if (!mbar_wait(&acc_empty[slot], ((n / SLOTS_PER_PIPE) & 1) ^ 1, a.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t b_base = smem_u32(qbuf + j * Q_TILE);
#pragma unroll
          for (int kk = 0; kk < DSA_IDX_DIM / 32; ++kk) {
            mma_f8f6f4(tmem + slot * ACC_COLS, umma_desc_sw128(a_base + kk * 32, 1024, 16),
                       umma_desc_sw128(b_base + kk * 32, 1024, 16), idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&acc_full[slot]);
        }
        if (!ok) break;
        mma_commit(&empty[stage]);
      }
      // every MMA this thread issued must finish before TMEM is released
      mma_commit(&mma_done[pipe]);
      mbar_wait(&mma_done[pipe], 0, a.err);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    if (t_begin < t_end) {
      const int g = (warp - 3) >> 2;           // warpgroup = pipeline 0 / 1
      const int quarter = warp & 3;            // TMEM lanes this warp may read
      const int row = quarter * 32 + lane;     // key row of the tile
      int b = b_first;
      uint32_t n = 0;
      bool ok = true;
      for (int i = t_begin; i < t_end && ok; ++i) {
        while (prefix[b + 1] <= i) ++b;
        if (((i - t_begin) & 1) != g) continue;
        const int t = i - prefix[b];
        const int nq = seq_queries(a, b);
        const int q0 = a.q_offsets[b];
        const int64_t len = a.seq_offsets[b + 1] - a.seq_offsets[b];
        for (int j = 0; j < nq; ++j, ++n) {
          const uint32_t slot = g * SLOTS_PER_PIPE + n % SLOTS_PER_PIPE;
          if (!mbar_wait(&acc_full[slot], (n / SLOTS_PER_PIPE) & 1, a.err)) { ok = false; break; }
          tc_fence_after();
          float v[ACC_COLS];
          const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + slot * ACC_COLS;
          tmem_ld16(taddr + 0, v + 0);
          tmem_ld16(taddr + 16, v + 16);
          tmem_ld16(taddr + 32, v + 32);
          tmem_ld16(taddr + 48, v + 48);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[slot]);
          const int q = q0 + j;
          bool bad = false;
          const int vis = query_vis(a, q, len, &bad);
          const int s = t * KT + row;
          if (s < vis) {
            const float4* wp = reinterpret_cast<const float4*>(a.w + static_cast<size_t>(q) * DSA_IDX_HEADS);
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
            for (int h4 = 0; h4 < DSA_IDX_HEADS / 4; ++h4) {
              const float4 ww = __ldg(wp + h4);
              s0 = fmaf(ww.x, fmaxf(v[4 * h4 + 0], 0.f), s0);
              s1 = fmaf(ww.y, fmaxf(v[4 * h4 + 1], 0.f), s1);
              s2 = fmaf(ww.z, fmaxf(v[4 * h4 + 2], 0.f), s2);
              s3 = fmaf(ww.w, fmaxf(v[4 * h4 + 3], 0.f), s3);
            }
            a.scores[static_cast<size_t>(q) * a.ld + s] = (s0 + s1) + (s2 + s3);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, NACC * ACC_COLS);
  }
}

}  // namespace

cudaError_t launch_indexer(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                           int64_t total_keys, const int64_t* seq_offsets,
                           const int32_t* q_offsets, const int32_t* q_vis, int B, int Q,
                           int first_only, float* scores, int ld, uint32_t* err,
                           cudaStream_t st) {
  if (B <= 0 || Q <= 0 || total_keys <= 0) return cudaSuccess;
  CUtensorMap tk, tq;
  if (!encode_tiled_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_idx, DSA_IDX_DIM,
                       static_cast<uint64_t>(total_keys), DSA_IDX_DIM, DSA_IDX_DIM, KT))
    return cudaErrorInvalidValue;
  if (!encode_tiled_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_idx, DSA_IDX_DIM,
                       static_cast<uint64_t>(Q) * DSA_IDX_HEADS, DSA_IDX_DIM, DSA_IDX_DIM,
                       DSA_IDX_HEADS))
    return cudaErrorInvalidValue;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(indexer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  IdxArgs args{w, seq_offsets, q_offsets, q_vis, scores, ld, B, first_only, err};
  const int grid = device_sm_count();
  indexer_kernel<<<grid, THREADS, SMEM_BYTES, st>>>(tk, tq, args);
  return cudaGetLastError();
}

}  // namespace dsa
