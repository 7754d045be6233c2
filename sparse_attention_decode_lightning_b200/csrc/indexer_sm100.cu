// Lightning indexer on sm_100a: I[q,s] = sum_h w[q,h] * ReLU(q_idx[q,h,:] . K[s,:]).
//
// Source: "大语言模型结构总览", section 2.2 DeepSeek-V3.2 -- the indexer is a
// light FP8 scorer (64 heads x 128 dims) that gives every prior token of a
// query one relevance scalar; it streams the whole key cache, which makes it
// the HBM-bound part of the decode step.  Section 7.2 GLM-5.2 gives the same
// scorer with 32 heads; the kernel is instantiated for HI = 64 and HI = 32
// heads (the per-query MMA has N = HI).
//
// Design (persistent, one CTA per SM, two independent sub-pipelines):
// the CTA's contiguous range of (sequence, 128-key tile) items is cut in two
// halves, one per pipeline, and each pipeline has
//   a producer warp   TMA loads of 128-key x 128-byte e4m3 tiles (16 KB,
//                     128-byte swizzle, L2 evict-first) into its own ring,
//                     and the queries of its current sequence (8 KB each);
//   an issuer warp    for every query of the tile's sequence, D[128 keys, HI
//                     heads] = K_tile . q^T as 4 MMAs of kind::f8f6f4 (M=128,
//                     N=HI, K=32) into one of its 4 TMEM slots;
//   an epilogue warpgroup   each thread reads its key row (HI fp32 head
//                     dots) with tcgen05.ld and reduces sum_h w_h max(d_h, 0)
//                     in registers; scores are written coalesced.
// A single issuer thread spends ~1500 cycles per tile on mbarrier waits, MMA
// issue and commits (measured with per-role clock64 timelines), which alone
// caps a CTA near 25 GB/s; two issuers that never wait on each other double
// it.  The ring depth per pipeline is chosen at run time from the largest
// number of queries per sequence (the query buffer holds them all).
// A sequence's keys are read once for all of its queries (MTP verify
// positions share each tile).  With several queries a sequence the epilogue
// does 8 x HI ReLU-weighted sums per key and sets the pace; that case runs an
// instance with two epilogue warpgroups per pipeline that take alternate
// accumulator groups (640 threads, 96 registers: columns are read 32 at a
// time).  Measured on 16 sequences x 8 positions at 128K: 239 -> 218 us.
#include "common.cuh"
#include "internal.h"


namespace dsa {
namespace {

constexpr int KT = 128;                                // keys per tile (MMA M)
constexpr int PIPES = 2;                               // independent sub-pipelines per CTA
constexpr int SLOTS = 4;                               // TMEM accumulator slots per pipeline
constexpr int ACC_COLS = DSA_IDX_HEADS;                // TMEM columns per slot (64 heads at most)
// per pipeline: producer, MMA issuer and EPI epilogue warps (EPI = 4, or 8
// when sequences carry several queries: two warps per TMEM lane quarter, each
// taking one query of a pair)
constexpr int threads_for(int epi) { return 32 * (2 + epi) * PIPES; }
constexpr int KEY_TILE = KT * DSA_IDX_DIM;             // 16384 B
constexpr int Q_TILE = DSA_IDX_HEADS * DSA_IDX_DIM;    // 8192 B: one query's tile at 64 heads
constexpr int MAX_STAGES = 6;                          // per pipeline
constexpr int OFF_PREFIX = 0;
constexpr int OFF_SCAN = OFF_PREFIX + ((DSA_MAX_BATCH + 1) * 4 + 15) / 16 * 16;
constexpr int NBAR_PIPE = 2 * MAX_STAGES + 2 * SLOTS + 5;
constexpr int OFF_BAR = OFF_SCAN + 64 * 4;
constexpr int OFF_MISC = OFF_BAR + PIPES * NBAR_PIPE * 8;
// per pipeline: the current sequence's head weights [queries][64] fp32 and
// visible lengths, shared by its four epilogue warps
constexpr int WS_PIPE = DSA_MAX_Q_PER_SEQ * DSA_IDX_HEADS * 4 + DSA_MAX_Q_PER_SEQ * 4;
constexpr int OFF_WS = (OFF_MISC + 16 + 15) / 16 * 16;
constexpr int OFF_DATA = (OFF_WS + PIPES * WS_PIPE + 1023) / 1024 * 1024;   // rings + query buffers
constexpr int SMEM_BYTES = 230400;                     // dynamic shared memory requested
constexpr int DATA_BYTES = SMEM_BYTES - 1024 - OFF_DATA;
static_assert(SMEM_BYTES <= 232448, "indexer shared memory exceeds the sm_100 limit");
static_assert(DATA_BYTES >= PIPES * (2 * KEY_TILE + (DSA_MAX_Q_PER_SEQ + 1) / 2 * 2 * Q_TILE),
              "two stages and a full query buffer must fit per pipeline");

struct IdxArgs {
  const float* w;
  const int64_t* seq_offsets;
  const int32_t* q_offsets;
  const int32_t* q_vis;
  float* scores;
  int ld;
  uint32_t* hist;       // nullable: per query, counts of the top 12 bits of ~key(score)
  int B;
  int first_only;
  uint32_t* err;
};

// The written scores of a warp into their query's histogram of the
// selector's first radix digit (top 12 bits of ~key(score)); lanes that fall
// into the same bin add together.  Called by all 32 lanes from converged code
// (a mask taken inside a divergent branch is not a safe match set); lanes
// without a score pass valid = false.
__device__ __forceinline__ void hist_add(uint32_t* h, bool valid, float v) {
  const uint32_t bin = valid ? (~float_key(v)) >> 20 : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xffffffffu, bin);
  if (valid && static_cast<int>(threadIdx.x & 31) == __ffs(peers) - 1)
    atomicAdd(&h[bin], static_cast<uint32_t>(__popc(peers)));
}

// A pipeline's shared-memory histogram (one query per sequence) goes to its
// query's row in global memory and is cleared; each epilogue warp e takes
// every EPI-th group of 32 bins.  g == nullptr only clears.
template <int EPI>
__device__ __forceinline__ void hist_flush(uint32_t* s_hist, uint32_t* g, int e, int lane) {
  for (int bin = e * 32 + lane; bin < 4096; bin += 32 * EPI) {
    const uint32_t c = s_hist[bin];
    if (g && c) atomicAdd(&g[bin], c);
    s_hist[bin] = 0;
  }
}

// An epilogue warp's wait for an accumulator group.  With histograms the warp
// gives up as a whole (hist_add needs all 32 lanes), so a lane whose bounded
// wait ran out takes the others with it.
template <bool HIST>
__device__ __forceinline__ bool acc_wait(uint64_t* bar, uint32_t phase, uint32_t* err) {
  const bool ok = mbar_wait(bar, phase, err);
  if constexpr (HIST) return __all_sync(0xffffffffu, ok);
  return ok;
}

// queries of sequence b that this launch scores (-1 if the entry is invalid)
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

// largest b with prefix[b] <= t (prefix non-decreasing over [0, B])
__device__ __forceinline__ int seq_of_tile(const int* prefix, int B, int t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int HI, int EPI, bool HIST>
__global__ void __launch_bounds__(threads_for(EPI), 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_q, IdxArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  int* prefix = reinterpret_cast<int*>(smem + OFF_PREFIX);
  int* scan_tmp = reinterpret_cast<int*>(smem + OFF_SCAN);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  int* s_maxq = reinterpret_cast<int*>(smem + OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = a.B;
  pdl_trigger();   // the selector after this kernel may be scheduled as SMs free up

  // ---- tiles per sequence -> exclusive prefix over the batch; largest query count
  if (tid == 0) *s_maxq = 1;
  __syncthreads();
  constexpr int NT = threads_for(EPI);
  constexpr int WPP = 2 + EPI;                     // warps per pipeline
  for (int b = tid; b < B; b += NT) {
    const int nq = seq_queries(a, b);
    bool bad = nq < 0;
    int mv = 0;
    const int64_t len = a.seq_offsets[b + 1] - a.seq_offsets[b];
    if (len < 0) bad = true;
    for (int j = 0; j < nq; ++j) mv = max(mv, query_vis(a, a.q_offsets[b] + j, len < 0 ? 0 : len, &bad));
    if (bad) raise_error(a.err, DEVERR_BOUNDS);
    prefix[b] = (nq <= 0 || len < 0) ? 0 : (mv + KT - 1) / KT;
    if (nq > 1) atomicMax(s_maxq, nq);
  }
  __syncthreads();
  block_exclusive_scan(prefix, B, scan_tmp);
  const int maxq = *s_maxq;
  // Sequences with several queries (MTP verify) take their queries two at a
  // time: one MMA with N = 2 HI (two query tiles side by side) into one of 2
  // accumulator slots, instead of one N = HI MMA per query into 4 slots.
  // Halves the MMAs and commits per tile.
  constexpr int QT = HI * DSA_IDX_DIM;             // one query's e4m3 tile (bytes)
  const int G = maxq >= 2 ? 2 : 1;
  const int nslots = SLOTS / G;
  const uint32_t slot_cols = HI * G;
  const int qtiles = (maxq + G - 1) / G * G;      // the last pair may read one tile past nq
  // per-pipeline shared memory: [ring of `stages` key tiles][query buffer of
  // qtiles tiles][with histograms and one query per sequence: a 4096-bin
  // histogram of the running sequence, which costs the ring one stage]
  const bool smem_hist = HIST && maxq == 1;
  const int pipe_bytes = (DATA_BYTES / PIPES) / 1024 * 1024;
  const int stages =
      min(MAX_STAGES, (pipe_bytes - qtiles * QT - (smem_hist ? 4096 * 4 : 0)) / KEY_TILE);

  const int pipe = warp / WPP;                     // 0 / 1
  const int pw = warp % WPP;                       // role within the pipeline
  uint8_t* keys = smem + OFF_DATA + pipe * pipe_bytes;
  uint8_t* qbuf = keys + stages * KEY_TILE;
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(qbuf + qtiles * QT);   // used if smem_hist
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR) + pipe * NBAR_PIPE;
  uint64_t* full = bars;
  uint64_t* empty = bars + MAX_STAGES;
  uint64_t* acc_full = bars + 2 * MAX_STAGES;
  uint64_t* acc_empty = acc_full + SLOTS;
  uint64_t* q_full = acc_empty + SLOTS;
  uint64_t* q_empty = q_full + 1;
  uint64_t* mma_done = q_full + 2;
  uint64_t* w_free = q_full + 3;                   // epilogue warps left the previous sequence
  uint64_t* w_full = q_full + 4;                   // the sequence's weights are in w_s
  float* w_s = reinterpret_cast<float*>(smem + OFF_WS + pipe * WS_PIPE);
  int* vis_s = reinterpret_cast<int*>(w_s + DSA_MAX_Q_PER_SEQ * DSA_IDX_HEADS);

  if (tid < PIPES) {
    uint64_t* pb = reinterpret_cast<uint64_t*>(smem + OFF_BAR) + tid * NBAR_PIPE;
    for (int i = 0; i < MAX_STAGES; ++i) { mbar_init(&pb[i], 1); mbar_init(&pb[MAX_STAGES + i], 1); }
    for (int i = 0; i < SLOTS; ++i) {
      mbar_init(&pb[2 * MAX_STAGES + i], 1);
      mbar_init(&pb[2 * MAX_STAGES + SLOTS + i], 4);   // one lane quarter each: 4 warps
    }
    mbar_init(&pb[2 * MAX_STAGES + 2 * SLOTS + 0], 1);   // q_full
    mbar_init(&pb[2 * MAX_STAGES + 2 * SLOTS + 1], 1);   // q_empty
    mbar_init(&pb[2 * MAX_STAGES + 2 * SLOTS + 2], 1);   // mma_done
    mbar_init(&pb[2 * MAX_STAGES + 2 * SLOTS + 3], EPI);   // w_free: the epilogue warps
    mbar_init(&pb[2 * MAX_STAGES + 2 * SLOTS + 4], EPI);   // w_full
    mbar_fence_init();
    if (tid == 0) {
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_q);
    }
  }
  if (warp == 1) tmem_alloc(tmem_holder, PIPES * SLOTS * ACC_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder + pipe * SLOTS * ACC_COLS;

  // this CTA's tiles, then this pipeline's contiguous half of them
  const int total = prefix[B];
  const int c_begin = static_cast<int>(static_cast<int64_t>(total) * blockIdx.x / gridDim.x);
  const int c_end = static_cast<int>(static_cast<int64_t>(total) * (blockIdx.x + 1) / gridDim.x);
  const int c_mid = c_begin + (c_end - c_begin + 1) / 2;
  const int t_begin = pipe == 0 ? c_begin : c_mid;
  const int t_end = pipe == 0 ? c_mid : c_end;
  const int b_first = t_begin < t_end ? seq_of_tile(prefix, B, t_begin) : 0;

  if (pw == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && t_begin < t_end) {
      const uint64_t pol = l2_policy_evict_first();
      int b = b_first, cur_b = -1;
      uint32_t issued = 0, q_issued = 0, qphase = 0;
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
          mbar_arrive_expect_tx(q_full, nq * QT);
          for (int j = 0; j < nq; ++j)
            tma_load_2d(qbuf + j * QT, &tmap_q, 0, (a.q_offsets[b] + j) * HI, q_full);
          ++q_issued;
          cur_b = b;
        }
        const uint32_t s = issued % stages;
        if (!mbar_wait(&empty[s], ((issued / stages) & 1) ^ 1, a.err)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[s], KEY_TILE);
        const int64_t row = a.seq_offsets[b] + static_cast<int64_t>(t) * KT;
        tma_load_2d_hint(keys + s * KEY_TILE, &tmap_k, 0, static_cast<int>(row), &full[s], pol);
        ++issued;
      }
      if (!ok) {
        // drain the copies still in flight before the CTA's memory goes away
        const uint32_t n = issued < static_cast<uint32_t>(stages) ? issued : stages;
        for (uint32_t k = 0; k < n; ++k) {
          const uint32_t it = issued - 1 - k;
          mbar_wait(&full[it % stages], (it / stages) & 1, a.err);
        }
        if (q_issued) mbar_wait(q_full, (q_issued - 1) & 1, a.err);
      }
    }
  } else if (pw == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && t_begin < t_end) {
      const uint32_t idesc = umma_idesc(0 /*E4M3*/, KT, static_cast<int>(slot_cols));
      int b = b_first, cur_b = -1, nq = 0;
      uint32_t qphase = 0, n = 0, k = 0;
      bool ok = true;
      for (int i = t_begin; i < t_end && ok; ++i, ++k) {
        while (prefix[b + 1] <= i) ++b;
        if (b != cur_b) {
          if (cur_b >= 0) mma_commit(q_empty);
          if (!mbar_wait(q_full, qphase, a.err)) { ok = false; break; }
          qphase ^= 1;
          nq = seq_queries(a, b);
          cur_b = b;
        }
        const uint32_t s = k % stages;
        if (!mbar_wait(&full[s], (k / stages) & 1, a.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(keys + s * KEY_TILE);
        for (int j0 = 0; j0 < nq; j0 += G, ++n) {
          const uint32_t slot = n % nslots;
          if (!mbar_wait(&acc_empty[slot], ((n / nslots) & 1) ^ 1, a.err)) { ok = false; break; }
          tc_fence_after();
          // G consecutive HI-row query tiles form one HI*G-row B operand (the
          // 128-byte swizzle atoms continue every 1024 bytes across tiles)
          const uint32_t b_base = smem_u32(qbuf + j0 * QT);
#pragma unroll
          for (int kk = 0; kk < DSA_IDX_DIM / 32; ++kk) {
            mma_f8f6f4(tmem + slot * slot_cols, umma_desc_sw128(a_base + kk * 32, 1024, 16),
                       umma_desc_sw128(b_base + kk * 32, 1024, 16), idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&acc_full[slot]);
        }
        if (!ok) break;
        mma_commit(&empty[s]);
      }
      // every MMA this thread issued must finish before TMEM is released
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, a.err);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    if (t_begin < t_end) {
      const int quarter = warp & 3;            // TMEM lanes this warp may read
      const int row = quarter * 32 + lane;     // key row of the tile
      int b = b_first, cur_b = -1, nq = 0, q0 = 0;
      uint32_t n = 0, wph = 0;
      bool ok = true;
      for (int i = t_begin; i < t_end && ok; ++i) {
        while (prefix[b + 1] <= i) ++b;
        if (b != cur_b) {
          // new sequence: once all the epilogue warps are past the previous
          // one, they copy its weights and visible lengths into w_s / vis_s
          // (bounded mbarrier waits, not bar.sync, so a timed-out warp cannot
          // leave the others waiting for ever)
          __syncwarp();
          if (lane == 0) mbar_arrive(w_free);
          if (!(ok = mbar_wait(w_free, wph, a.err))) break;
          if (smem_hist)   // the previous sequence's counts out, zeros for this one
            hist_flush<EPI>(s_hist, cur_b >= 0 ? a.hist + static_cast<size_t>(q0) * 4096 : nullptr,
                            pw - 2, lane);
          nq = seq_queries(a, b);
          q0 = a.q_offsets[b];
          const int64_t len = a.seq_offsets[b + 1] - a.seq_offsets[b];
          const int e = pw - 2;                  // 0..EPI-1
          for (int x = e * 32 + lane; x < nq * HI; x += 32 * EPI)
            w_s[x] = __ldg(a.w + static_cast<size_t>(q0) * HI + x);
          if (e == 0 && lane < nq) {
            bool bad = false;
            vis_s[lane] = query_vis(a, q0 + lane, len, &bad);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(w_full);
          if (!(ok = mbar_wait(w_full, wph, a.err))) break;
          wph ^= 1;
          cur_b = b;
        }
        const int t = i - prefix[b];
        // 8 epilogue warps: the two warps of a lane quarter take alternate
        // accumulator groups (group n to half n % 2; the slot count is even, so
        // a slot always belongs to one half).  Each warp runs half the groups,
        // reading a query's columns 32 at a time (96 registers a thread at 640
        // threads); a group is released when its last column is in registers.
        if constexpr (EPI == 8) {
          const int half = (pw - 2) >> 2;
          for (int j0 = 0; j0 < nq; j0 += G, ++n) {
            if (static_cast<int>(n & 1u) != half) continue;
            const uint32_t slot = n % nslots;
            if (!acc_wait<HIST>(&acc_full[slot], (n / nslots) & 1, a.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + slot * slot_cols;
            float r[2] = {0.f, 0.f};
            for (int jj = 0; jj < G && j0 + jj < nq; ++jj) {
              const float4* wp = reinterpret_cast<const float4*>(w_s + (j0 + jj) * HI);
              float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll 1
              for (int c = 0; c < HI / 32; ++c) {
                float v[32];
                tmem_ld32(taddr + static_cast<uint32_t>(jj * HI + 32 * c), v);
                tmem_ld_wait();
#pragma unroll
                for (int h4 = 0; h4 < 8; ++h4) {
                  const float4 ww = wp[8 * c + h4];
                  s0 = fmaf(ww.x, fmaxf(v[4 * h4 + 0], 0.f), s0);
                  s1 = fmaf(ww.y, fmaxf(v[4 * h4 + 1], 0.f), s1);
                  s2 = fmaf(ww.z, fmaxf(v[4 * h4 + 2], 0.f), s2);
                  s3 = fmaf(ww.w, fmaxf(v[4 * h4 + 3], 0.f), s3);
                }
              }
              r[jj] = (s0 + s1) + (s2 + s3);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[slot]);
            const int s = t * KT + row;
            for (int jj = 0; jj < G && j0 + jj < nq; ++jj) {
              const bool in = s < vis_s[j0 + jj];
              if (in) a.scores[static_cast<size_t>(q0 + j0 + jj) * a.ld + s] = r[jj];
              if constexpr (HIST) hist_add(a.hist + static_cast<size_t>(q0 + j0 + jj) * 4096, in, r[jj]);
            }
          }
          continue;
        }
        // query pairs: both queries' 2 HI columns are read with a single wait
        // (the wait covers every outstanding TMEM load, so reading the second
        // query later would cost a second full load latency)
        if (G == 2) {
          for (int j0 = 0; j0 < nq; j0 += 2, ++n) {
            const uint32_t slot = n % nslots;
            const bool two = j0 + 1 < nq;
            if (!acc_wait<HIST>(&acc_full[slot], (n / nslots) & 1, a.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            float v[2 * HI];
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + slot * slot_cols;
            // the second query's columns are past nq for an odd last query: not used
#pragma unroll
            for (int c = 0; c < 2 * HI / 32; ++c) tmem_ld32(taddr + 32 * c, v + 32 * c);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[slot]);
            const int s = t * KT + row;
            float r0 = 0.f, r1 = 0.f;
            {
              const float4* w0 = reinterpret_cast<const float4*>(w_s + j0 * HI);
              const float4* w1 = reinterpret_cast<const float4*>(w_s + (two ? j0 + 1 : j0) * HI);
              float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
              for (int h4 = 0; h4 < HI / 4; ++h4) {
                const float4 x = w0[h4];
                const float4 y = w1[h4];
                a0 = fmaf(x.x, fmaxf(v[4 * h4 + 0], 0.f), a0);
                a1 = fmaf(x.y, fmaxf(v[4 * h4 + 1], 0.f), a1);
                a0 = fmaf(x.z, fmaxf(v[4 * h4 + 2], 0.f), a0);
                a1 = fmaf(x.w, fmaxf(v[4 * h4 + 3], 0.f), a1);
                b0 = fmaf(y.x, fmaxf(v[HI + 4 * h4 + 0], 0.f), b0);
                b1 = fmaf(y.y, fmaxf(v[HI + 4 * h4 + 1], 0.f), b1);
                b0 = fmaf(y.z, fmaxf(v[HI + 4 * h4 + 2], 0.f), b0);
                b1 = fmaf(y.w, fmaxf(v[HI + 4 * h4 + 3], 0.f), b1);
              }
              r0 = a0 + a1;
              r1 = b0 + b1;
            }
            const bool in0 = s < vis_s[j0], in1 = two && s < vis_s[j0 + 1];
            if (in0) a.scores[static_cast<size_t>(q0 + j0) * a.ld + s] = r0;
            if (in1) a.scores[static_cast<size_t>(q0 + j0 + 1) * a.ld + s] = r1;
            if constexpr (HIST) {
              hist_add(a.hist + static_cast<size_t>(q0 + j0) * 4096, in0, r0);
              if (two) hist_add(a.hist + static_cast<size_t>(q0 + j0 + 1) * 4096, in1, r1);
            }
          }
          continue;
        }
        for (int j = 0; j < nq; ++j) {
          const uint32_t slot = n % nslots;
          const int jj = j % G;                    // query within the slot's pair
          if (jj == 0) {
            if (!acc_wait<HIST>(&acc_full[slot], (n / nslots) & 1, a.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          float v[HI];
          const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + slot * slot_cols +
                                 static_cast<uint32_t>(jj * HI);
#pragma unroll
          for (int c = 0; c < HI / 16; ++c) tmem_ld16(taddr + 16 * c, v + 16 * c);
          tmem_ld_wait();
          if (jj == G - 1 || j == nq - 1) {        // last query of the slot: release it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[slot]);
            ++n;
          }
          const int q = q0 + j;
          const int vis = vis_s[j];
          const int s = t * KT + row;
          const bool in = s < vis;
          float sc = 0.f;
          if (in) {
            const float4* wp = reinterpret_cast<const float4*>(w_s + j * HI);
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
            for (int h4 = 0; h4 < HI / 4; ++h4) {
              const float4 ww = wp[h4];
              s0 = fmaf(ww.x, fmaxf(v[4 * h4 + 0], 0.f), s0);
              s1 = fmaf(ww.y, fmaxf(v[4 * h4 + 1], 0.f), s1);
              s2 = fmaf(ww.z, fmaxf(v[4 * h4 + 2], 0.f), s2);
              s3 = fmaf(ww.w, fmaxf(v[4 * h4 + 3], 0.f), s3);
            }
            sc = (s0 + s1) + (s2 + s3);
            a.scores[static_cast<size_t>(q) * a.ld + s] = sc;
          }
          if constexpr (HIST) {
            if (smem_hist) {
              if (in) atomicAdd(&s_hist[(~float_key(sc)) >> 20], 1u);
            } else {
              hist_add(a.hist + static_cast<size_t>(q) * 4096, in, sc);
            }
          }
        }
      }
      // the last sequence's counts, once every epilogue warp has added its own
      if (smem_hist && ok && cur_b >= 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(w_free);
        if (mbar_wait(w_free, wph, a.err))
          hist_flush<EPI>(s_hist, a.hist + static_cast<size_t>(q0) * 4096, pw - 2, lane);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*tmem_holder, PIPES * SLOTS * ACC_COLS);
  }
}

}  // namespace

namespace {

template <int HI, int EPI, bool HIST>
cudaError_t launch_indexer_h(const CUtensorMap& tk, const CUtensorMap& tq, const IdxArgs& args,
                             cudaStream_t st) {
  static std::atomic<bool> attr_done[64];
  const cudaError_t e = set_once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(indexer_kernel<HI, EPI, HIST>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  if (e != cudaSuccess) return e;
  indexer_kernel<HI, EPI, HIST><<<device_sm_count(), threads_for(EPI), SMEM_BYTES, st>>>(tk, tq, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_indexer(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                           int64_t total_keys, const int64_t* seq_offsets,
                           const int32_t* q_offsets, const int32_t* q_vis, int B, int Q,
                           int idx_heads, int first_only, float* scores, int ld, uint32_t* err,
                           cudaStream_t st, uint32_t* hist) {
  if (B <= 0 || Q <= 0 || total_keys <= 0) return cudaSuccess;
  if (idx_heads != 64 && idx_heads != 32) return cudaErrorInvalidValue;
  CUtensorMap tk, tq;
  if (!encode_tiled_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_idx, DSA_IDX_DIM,
                       static_cast<uint64_t>(total_keys), DSA_IDX_DIM, DSA_IDX_DIM, KT))
    return cudaErrorInvalidValue;
  if (!encode_tiled_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_idx, DSA_IDX_DIM,
                       static_cast<uint64_t>(Q) * idx_heads, DSA_IDX_DIM, DSA_IDX_DIM,
                       static_cast<uint32_t>(idx_heads)))
    return cudaErrorInvalidValue;
  IdxArgs args{w, seq_offsets, q_offsets, q_vis, scores, ld, hist, B, first_only, err};
  // several queries in a sequence (MTP verify): the 8-epilogue-warp instance
  const bool multi = Q > B && !first_only;
  if (hist) {
    if (idx_heads == 64)
      return multi ? launch_indexer_h<64, 8, true>(tk, tq, args, st)
                   : launch_indexer_h<64, 4, true>(tk, tq, args, st);
    return multi ? launch_indexer_h<32, 8, true>(tk, tq, args, st)
                 : launch_indexer_h<32, 4, true>(tk, tq, args, st);
  }
  if (idx_heads == 64)
    return multi ? launch_indexer_h<64, 8, false>(tk, tq, args, st)
                 : launch_indexer_h<64, 4, false>(tk, tq, args, st);
  return multi ? launch_indexer_h<32, 8, false>(tk, tq, args, st)
               : launch_indexer_h<32, 4, false>(tk, tq, args, st);
}

}  // namespace dsa
