// Token selector: the topk highest indexer scores of each query, ties to the
// lower position ("大语言模型结构总览", section 2.2: the token selector keeps the
// k = 2048 best-scoring tokens; section 7.2: causal top-2048).
//
// One kernel launch, one thread-block cluster of C CTAs per query row.  The
// row's visible positions are cut into C contiguous slices; every CTA loads
// its slice into shared memory as order-preserving u32 keys (a slice longer
// than SLICE_CAP keeps its head there and re-reads the rest from global
// memory).
//
// Exact radix select on the composite key of position s
//     V(s) = (u(s) << pb) | s,   u(s) = ~key(I[s]),   pb = bits(vis - 1)
// (u measures the key down from the largest possible key).  V is distinct
// per position and a smaller V is a better position (higher score, then
// lower position), so the topk smallest V are exactly the top-k with the
// lower-position tie rule.  The first 12-bit digit of V is the sign, exponent
// and top three mantissa bits of the score: relative bins of 1/8 of an
// octave, the same in every CTA without first agreeing on the row's range,
// so the first histogram is built while the copies land.  (Measuring u from
// the row's own maximum instead narrowed the bins but cost a cluster-wide
// min/max round and a separate histogram pass.)  Rows whose scores sit in a
// band narrower than a bin take the rescan path below.
//
// Steps ('|' is a cluster barrier):
//   load, keys and the pass-1 histogram (4096 bins, top digit of V) |
//           every CTA sums the C histograms through distributed shared
//           memory (1024 bins at a time, stopping at the chunk that holds the
//           threshold digit t: the smallest d with count(digits <= d) >= k)
//   then one of
//   exact:  bin t holds exactly the positions still needed: every CTA writes
//           its positions with digit <= t to the output | done
//   gather: bin t has at most CAND_CAP positions over the row: every CTA
//           writes its positions with digit < t to the output and pushes its
//           bin-t positions into rank 0's shared memory | rank 0 finishes the
//           selection among them alone (12-bit passes, block barriers only)
//   rescan: (degenerate score sets) further 12-bit passes over the slices
//           with a cluster merge each, then as "exact".
// Output slots are handed out by an atomic on a counter in rank 0's shared
// memory, so the index row is in no particular order.
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int THREADS = 1024;
constexpr int DIGIT = 12;                     // bits per radix pass
constexpr int BINS = 1 << DIGIT;
constexpr int CHUNK = 4 * THREADS;            // scores per load round: one float4 per thread
constexpr int NCHUNK = 10;
constexpr int SLICE_CAP = NCHUNK * CHUNK;     // 40960 scores a CTA keeps in shared memory
constexpr int CAND_CAP = 4096;                // bin-t positions rank 0 gathers
constexpr int MAX_CLUSTER = 8;                // portable cluster size
constexpr int MAX_CLUSTER_NP = 16;            // non-portable size for a few long rows
constexpr int MIN_SLICE = 2048;               // rows are not cut finer than this
constexpr int RS_MIN_CLUSTER = 8;             // clusters this large merge by parts (see below)
static_assert(BINS == 4 * THREADS, "bins are merged THREADS at a time, scanned 4 per thread");

constexpr size_t smem_bytes(int scap) {
  return static_cast<size_t>(scap) * 4 + 2 * BINS * 4 + CAND_CAP * 8;
}

struct TopkArgs {
  const float* scores;
  int ld;
  const int32_t* q_offsets;
  const int32_t* q_vis;
  int B, Q, max_len, topk, first_only;
  int32_t* out_idx;
  float* out_scores;
  uint32_t* err;
  int scap;             // slice elements held in shared memory (multiple of 4)
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

// Calls f(position, key, valid) for every element of the slice, in the same
// order on every call.  Groups of four that lie wholly inside the on-chip copy
// take the first loop, where valid is the constant true; the rest (the
// ragged tail and any part beyond scap, read from global memory and
// converted) take the second.
template <class F>
__device__ __forceinline__ void for_slice(const uint32_t* s_key, const float* grow, int beg, int n,
                                          int scap, F&& f) {
  const int full = min(n, scap) & ~(4 * THREADS - 1);   // whole steps of 4*THREADS on chip
  const int j0 = 4 * static_cast<int>(threadIdx.x);
  for (int base = 0; base < full; base += 4 * THREADS) {
    const int j = base + j0;
    const uint4 k = *reinterpret_cast<const uint4*>(s_key + j);
    f(beg + j, k.x, true);
    f(beg + j + 1, k.y, true);
    f(beg + j + 2, k.z, true);
    f(beg + j + 3, k.w, true);
  }
  for (int j = full + j0; j < n; j += 4 * THREADS) {
    uint4 k;
    if (j < scap) {
      k = *reinterpret_cast<const uint4*>(s_key + j);
    } else {
      const float4 v = __ldg(reinterpret_cast<const float4*>(grow + j));
      k = make_uint4(float_key(v.x), float_key(v.y), float_key(v.z), float_key(v.w));
    }
    f(beg + j, k.x, true);
    f(beg + j + 1, k.y, j + 1 < n);
    f(beg + j + 2, k.z, j + 2 < n);
    f(beg + j + 3, k.w, j + 3 < n);
  }
}

// Exclusive prefix sum of x over the CTA in thread order, and the CTA total.
// Every thread calls it; s_warp holds one word per warp.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t x, uint32_t* s_warp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  const uint32_t wt = s_warp[lane];            // THREADS / 32 == 32 warp totals
  uint32_t wi = wt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, wi, off);
    if (lane >= off) wi += y;
  }
  *total = __shfl_sync(0xffffffffu, wi, 31);
  const uint32_t wbase = __shfl_sync(0xffffffffu, wi - wt, warp);
  __syncthreads();                             // s_warp may be reused after this
  return wbase + incl - x;
}

// Threshold digit of a histogram whose bins 4*tid .. 4*tid+3 this thread
// holds in c: the smallest d with count(digits <= d) >= need.  Publishes d,
// the count below it and its count through s_t, s_cb, s_cnt.
__device__ __forceinline__ void find_threshold4(const uint32_t c[4], uint32_t need, uint32_t* s_warp,
                                                uint32_t* s_t, uint32_t* s_cb, uint32_t* s_cnt) {
  const uint32_t tot = c[0] + c[1] + c[2] + c[3];
  uint32_t all;
  uint32_t before = block_excl_scan(tot, s_warp, &all);
  if (before < need && before + tot >= need) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (before < need && before + c[k] >= need) {
        *s_t = 4 * threadIdx.x + k;
        *s_cb = before;
        *s_cnt = c[k];
      }
      before += c[k];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(THREADS, 1) topk_cluster_kernel(TopkArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* s_key = reinterpret_cast<uint32_t*>(smem);                  // scores, then keys
  uint32_t* s_hist = s_key + a.scap;                                     // [2][BINS]
  uint64_t* s_cand = reinterpret_cast<uint64_t*>(s_hist + 2 * BINS);    // rank 0: gathered V
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_t, s_cb, s_cnt;         // threshold digit, count below it, its count
  __shared__ __align__(8) uint64_t s_ctr;      // rank 0: output slots | gathered candidates << 32
  __shared__ uint32_t s_obase, s_cbase;
  __shared__ uint32_t s_sum[BINS / RS_MIN_CLUSTER];   // this CTA's part of the summed histogram
  __shared__ uint32_t s_part, s_pidx, s_pbefore;   // its total; the part holding the threshold

  const int tid = threadIdx.x;
  const int C = static_cast<int>(gridDim.x);    // cluster = one grid row
  const uint32_t rank = cluster_ctarank();
  pdl_trigger();
  // q_offsets and q_vis are inputs of the whole step; the scores, the
  // outputs and the error word belong to the kernels before this one
  const int q = row_query(a, blockIdx.y);
  if (q < 0) return;                            // the whole cluster leaves
  pdl_wait();
  const int vis = clamped_vis(a, q);
  const int topk = a.topk;
  const float* row = a.scores + static_cast<size_t>(q) * a.ld;
  int32_t* oi = a.out_idx + static_cast<size_t>(q) * topk;
  float* os = a.out_scores ? a.out_scores + static_cast<size_t>(q) * topk : nullptr;

  if (vis <= topk) {                            // every visible position, then padding
    for (int i = static_cast<int>(rank) * THREADS + tid; i < topk; i += C * THREADS) {
      oi[i] = i < vis ? i : -1;
      if (os) os[i] = i < vis ? row[i] : -INFINITY;
    }
    return;                                     // the whole cluster leaves
  }

  // This CTA's slice [beg, beg + n), beg a multiple of 4.  Every float4 read
  // ends at round_up(beg + n, 4) <= ld, since beg and ld are multiples of 4
  // and beg + n <= vis <= ld.
  const int L = (((vis + C - 1) / C) + 3) & ~3;
  const int beg = min(vis, static_cast<int>(rank) * L);
  const int n = max(0, min(vis, beg + L) - beg);
  const float* grow = row + beg;
  const int nsm = min(n, a.scap);               // elements copied on chip
  const int nch = (nsm + CHUNK - 1) / CHUNK;

  if (tid == 0) s_ctr = 0;
  for (int i = tid; i < 2 * BINS; i += THREADS) s_hist[i] = 0;
  __syncthreads();                              // histograms clear before any add

  // ---- keys on chip and the pass-1 histogram: every thread loads one float4
  // of each 4*THREADS-score chunk (five chunks' loads in flight at a time),
  // turns it into keys, stores them and bins them.  (One thread setting up
  // bulk copies of the chunks took ~1,200 cycles longer, for the same copy
  // time.)  V measures a key down from the largest possible key (u = ~key),
  // so the pass-1 digit is the top DIGIT bits of ~key (sign, exponent and
  // three mantissa bits of the score): every CTA bins alike with no
  // agreement on the row's range first.
  auto hist4 = [&](uint4 k, int j, int lim) {
    const uint32_t e[4] = {k.x, k.y, k.z, k.w};
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (j + t < lim) atomicAdd(&s_hist[(~e[t]) >> (32 - DIGIT)], 1u);
  };
  constexpr int LB = 5;                         // chunks whose loads are in flight together
  for (int c0 = 0; c0 < nch; c0 += LB) {
    float4 v[LB];
#pragma unroll
    for (int u = 0; u < LB; ++u) {
      const int j = (c0 + u) * CHUNK + 4 * tid;
      if (c0 + u < nch && j < nsm) v[u] = __ldg(reinterpret_cast<const float4*>(grow + j));
    }
#pragma unroll
    for (int u = 0; u < LB; ++u) {
      const int j = (c0 + u) * CHUNK + 4 * tid;
      if (c0 + u < nch && j < nsm) {
        const uint4 k = make_uint4(float_key(v[u].x), float_key(v[u].y), float_key(v[u].z), float_key(v[u].w));
        *reinterpret_cast<uint4*>(s_key + j) = k;
        hist4(k, j, nsm);
      }
    }
  }
  for (int j = a.scap + 4 * tid; j < n; j += 4 * THREADS) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(grow + j));
    hist4(make_uint4(float_key(v.x), float_key(v.y), float_key(v.z), float_key(v.w)), j, n);
  }
  cluster_sync();            // every CTA's keys and pass-1 histogram; counters zeroed
  const uint32_t gmax = 0xFFFFFFFFu;                    // u = gmax - key = ~key
  const uint32_t range = gmax;
  const int pb = 32 - __clz(vis - 1);                   // vis >= 2 here
  const uint64_t pos_mask = (1ull << pb) - 1ull;
  auto make_v = [&](int pos, uint32_t key) -> uint64_t {
    return (static_cast<uint64_t>(gmax - key) << pb) | static_cast<uint64_t>(pos);
  };
  // pass 1 took the top DIGIT bits of V = (~key << pb) | pos: with 32 + pb
  // significant bits, sh0 - pb = 32 - DIGIT and every later test on the
  // digit is a comparison of the key with a bound
  const int tb = (range ? 32 - __clz(range) : 0) + pb;  // significant bits of V
  const int w0 = min(DIGIT, tb);
  const int sh0 = tb - w0;
  const uint32_t dmask0 = (1u << w0) - 1u;
  const bool fast0 = sh0 >= pb;
  const int us0 = fast0 ? sh0 - pb : 0;
  auto digit0 = [&](int pos, uint32_t key) -> uint32_t {   // general form
    return (((gmax - key) << (pb - sh0)) | (static_cast<uint32_t>(pos) >> sh0)) & dmask0;
  };

  // threshold digit of the cluster's summed histograms; h = this pass's buffer
  auto merged_threshold = [&](const uint32_t* h, uint32_t need) {
    if (C >= RS_MIN_CLUSTER) {
      // By parts: CTA r sums bins [lo_r, hi_r) over the cluster (BINS remote
      // loads a CTA, instead of C per bin up to the threshold's chunk), the
      // part totals locate the part that holds the threshold, and every CTA
      // scans that part's sums.  One cluster barrier more, 1/C of the
      // distributed shared memory traffic.
      const int lo = static_cast<int>(rank) * BINS / C, hi = (static_cast<int>(rank) + 1) * BINS / C;
      uint32_t m = 0;
      if (tid < hi - lo) {
        const uint32_t a0 = smem_u32(h + lo + tid);
        for (int r = 0; r < C; ++r) m += ld_cluster_u32(map_to_rank(a0, static_cast<uint32_t>(r)));
        s_sum[tid] = m;
      }
      uint32_t tot;
      block_excl_scan(m, s_warp, &tot);
      if (tid == 0) s_part = tot;
      cluster_sync();          // every part summed
      if (tid < 32) {
        const uint32_t pt = tid < C ? ld_cluster_u32(map_to_rank(smem_u32(&s_part), static_cast<uint32_t>(tid))) : 0u;
        uint32_t incl = pt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
          if (tid >= off) incl += y;
        }
        const uint32_t before = incl - pt;
        if (tid < C && before < need && incl >= need) {
          s_pidx = static_cast<uint32_t>(tid);
          s_pbefore = before;
        }
      }
      __syncthreads();
      const int p = static_cast<int>(s_pidx);
      const int plo = p * BINS / C, phi = (p + 1) * BINS / C;
      const uint32_t pb = s_pbefore;
      const uint32_t v = tid < phi - plo
                             ? ld_cluster_u32(map_to_rank(smem_u32(&s_sum[tid]), static_cast<uint32_t>(p)))
                             : 0u;
      const uint32_t ex = pb + block_excl_scan(v, s_warp, &tot);
      if (tid < phi - plo && ex < need && ex + v >= need) {
        s_t = static_cast<uint32_t>(plo + tid);
        s_cb = ex;
        s_cnt = v;
      }
      __syncthreads();
      return;
    }
    uint32_t carry = 0;
    for (int c0 = 0; c0 < BINS; c0 += THREADS) {
      const uint32_t a0 = smem_u32(h + c0 + tid);
      uint32_t m = 0;
      for (int r = 0; r < C; ++r) m += ld_cluster_u32(map_to_rank(a0, static_cast<uint32_t>(r)));
      uint32_t tot;
      const uint32_t ex = carry + block_excl_scan(m, s_warp, &tot);
      if (ex < need && ex + m >= need) {
        s_t = static_cast<uint32_t>(c0 + tid);
        s_cb = ex;
        s_cnt = m;
      }
      carry += tot;
      if (carry >= need) break;
    }
    __syncthreads();
  };
  // "exact" / "rescan" ending: every slice position with sel(pos, key) is
  // written to the output; slots from rank 0's counter, then a cluster barrier
  auto write_selected = [&](auto sel) {
    uint32_t cnt = 0;
    for_slice(s_key, grow, beg, n, a.scap, [&](int pos, uint32_t key, bool valid) {
      cnt += valid && sel(pos, key);
    });
    uint32_t tot;
    const uint32_t pre = block_excl_scan(cnt, s_warp, &tot);
    if (tid == 0)
      s_obase = static_cast<uint32_t>(atom_add_cluster_u64(map_to_rank(smem_u32(&s_ctr), 0u), tot));
    __syncthreads();
    uint32_t o = s_obase + pre;
    for_slice(s_key, grow, beg, n, a.scap, [&](int pos, uint32_t key, bool valid) {
      if (valid && sel(pos, key)) {
        if (o < static_cast<uint32_t>(topk)) {
          oi[o] = pos;
          if (os) os[o] = key_float(key);
        } else {
          raise_error(a.err, DEVERR_BOUNDS);
        }
        ++o;
      }
    });
    cluster_sync();          // rank 0's counter stays alive until every CTA took its slots
  };

  reinterpret_cast<uint4*>(s_hist + BINS)[tid] = make_uint4(0u, 0u, 0u, 0u);
  uint32_t need = static_cast<uint32_t>(topk);
  merged_threshold(s_hist, need);
  const uint32_t t0 = s_t;
  need -= s_cb;
  const uint32_t cnt0 = s_cnt;

  // digit < t0 ("better") and digit <= t0 ("in"): in the fast form
  // key >= kb1 and key >= kin1, from u < t0 << us0 and u < (t0 + 1) << us0
  // (64-bit: with t0 = 0 the bound is 2^32 and no key is better)
  const uint64_t kb1 = static_cast<uint64_t>(gmax) - (static_cast<uint64_t>(t0) << us0) + 1u;
  const uint64_t u2 = static_cast<uint64_t>(t0 + 1u) << us0;
  const uint32_t kin1 = u2 > gmax ? 0u : static_cast<uint32_t>(gmax - u2 + 1u);
  auto fast_better = [&](int, uint32_t key) { return static_cast<uint64_t>(key) >= kb1; };
  auto fast_in = [&](int, uint32_t key) { return key >= kin1; };
  auto gen_better = [&](int pos, uint32_t key) { return digit0(pos, key) < t0; };
  auto gen_in = [&](int pos, uint32_t key) { return digit0(pos, key) <= t0; };

  if (cnt0 == need) {
    // ---- exact: positions with digit <= t0
    if (fast0) write_selected(fast_in);
    else write_selected(gen_in);
    return;
  }

  if (cnt0 <= static_cast<uint32_t>(CAND_CAP)) {
    // ---- gather: digit < t0 goes out now, digit == t0 goes to rank 0
    auto gather = [&](auto better, auto in) {
      // One pass over the slice records which of this thread's elements are
      // "in" and which of those are "better" as bits of two masks (bit c is
      // the thread's c-th element in for_slice order, element j(c) below);
      // the writes then visit only the set bits.  Slices of up to
      // 64 * MASK_WORDS elements a thread; longer ones read the slice twice.
      constexpr int MASK_WORDS = 2;               // (the adds below name both words)
      const bool masked = n <= 64 * MASK_WORDS * THREADS;
      uint64_t m_in[MASK_WORDS] = {}, m_better[MASK_WORDS] = {};
      uint32_t nb = 0, ni = 0;
      if (masked) {
        int c = 0;
        for_slice(s_key, grow, beg, n, a.scap, [&](int pos, uint32_t key, bool valid) {
          if (valid && in(pos, key)) {
            // words picked by comparison, not by index, to stay in registers
            const uint64_t bit = 1ull << (c & 63);
            const bool bt = better(pos, key);
            if (c < 64) {
              m_in[0] |= bit;
              if (bt) m_better[0] |= bit;
            } else {
              m_in[1] |= bit;
              if (bt) m_better[1] |= bit;
            }
          }
          ++c;
        });
#pragma unroll
        for (int w = 0; w < MASK_WORDS; ++w) {
          nb += static_cast<uint32_t>(__popcll(m_better[w]));
          ni += static_cast<uint32_t>(__popcll(m_in[w]));
        }
      } else {
        for_slice(s_key, grow, beg, n, a.scap, [&](int pos, uint32_t key, bool valid) {
          nb += valid && better(pos, key);
          ni += valid && in(pos, key);
        });
      }
      // per CTA nb < topk and ni - nb <= cnt0 <= CAND_CAP: both halves stay below 2^16
      uint32_t tot;
      const uint32_t pre = block_excl_scan((nb << 16) | (ni - nb), s_warp, &tot);
      const uint32_t nb_cta = tot >> 16;
      if (tid == 0) {
        // rank 0 also takes the slots of the `need` positions it will pick from bin t0
        const uint64_t add =
            (static_cast<uint64_t>(tot & 0xFFFFu) << 32) | (nb_cta + (rank == 0 ? need : 0u));
        const uint64_t old = atom_add_cluster_u64(map_to_rank(smem_u32(&s_ctr), 0u), add);
        s_obase = static_cast<uint32_t>(old) + (rank == 0 ? nb_cta : 0u);   // rank 0: its picks
        s_cbase = static_cast<uint32_t>(old >> 32);
      }
      __syncthreads();
      uint32_t o = s_obase - (rank == 0 ? nb_cta : 0u) + (pre >> 16);
      uint32_t ci = s_cbase + (pre & 0xFFFFu);
      const uint32_t cand0 = map_to_rank(smem_u32(s_cand), 0u);
      auto emit = [&](int pos, uint32_t key, bool is_better) {
        if (is_better) {
          if (o < static_cast<uint32_t>(topk)) {
            oi[o] = pos;
            if (os) os[o] = key_float(key);
          } else {
            raise_error(a.err, DEVERR_BOUNDS);
          }
          ++o;
        } else {
          if (ci < static_cast<uint32_t>(CAND_CAP)) st_cluster_u64(cand0 + ci * 8u, make_v(pos, key));
          else raise_error(a.err, DEVERR_BOUNDS);
          ++ci;
        }
      };
      if (masked) {
        // element c of this thread: j = (c / 4) * 4 * THREADS + 4 * tid + c % 4
        // (for_slice's order); visited in increasing c, as the first pass saw them
#pragma unroll
        for (int w = 0; w < MASK_WORDS; ++w) {
          for (uint64_t m = m_in[w]; m; m &= m - 1) {
            const int b = __ffsll(static_cast<long long>(m)) - 1;
            const int c = 64 * w + b;
            const int j = (c >> 2) * (4 * THREADS) + 4 * tid + (c & 3);
            const uint32_t key = j < a.scap ? s_key[j] : float_key(__ldg(grow + j));
            emit(beg + j, key, (m_better[w] >> b) & 1ull);
          }
        }
      } else {
        for_slice(s_key, grow, beg, n, a.scap, [&](int pos, uint32_t key, bool valid) {
          if (valid && in(pos, key)) emit(pos, key, better(pos, key));
        });
      }
    };
    if (fast0) gather(fast_better, fast_in);
    else gather(gen_better, gen_in);
    cluster_sync();          // bin t0 gathered in rank 0; the other CTAs are done
    if (rank != 0) return;

    // rank 0: the `need` smallest V among the cnt0 gathered candidates
    const uint32_t picks = need;
    uint64_t P = t0;
    int rem = sh0;
    for (;;) {
      const int w = min(DIGIT, rem);
      const int sh = rem - w;
      const uint32_t dmask = (1u << w) - 1u;
      reinterpret_cast<uint4*>(s_hist)[tid] = make_uint4(0u, 0u, 0u, 0u);
      __syncthreads();
      for (uint32_t i = tid; i < cnt0; i += THREADS) {
        const uint64_t V = s_cand[i];
        if ((V >> rem) == P) atomicAdd(&s_hist[static_cast<uint32_t>(V >> sh) & dmask], 1u);
      }
      __syncthreads();
      const uint4 h4 = reinterpret_cast<const uint4*>(s_hist)[tid];
      const uint32_t c4[4] = {h4.x, h4.y, h4.z, h4.w};
      find_threshold4(c4, need, s_warp, &s_t, &s_cb, &s_cnt);
      need -= s_cb;
      P = (P << w) | s_t;
      rem = sh;
      if (s_cnt == need || rem == 0) break;   // rem == 0 implies s_cnt == need == 1
    }
    const uint64_t VT = (P << rem) | ((1ull << rem) - 1ull);
    uint32_t c = 0;
    for (uint32_t i = tid; i < cnt0; i += THREADS) c += s_cand[i] <= VT;
    uint32_t picked;
    uint32_t op = s_obase + block_excl_scan(c, s_warp, &picked);
    for (uint32_t i = tid; i < cnt0; i += THREADS) {
      const uint64_t V = s_cand[i];
      if (V <= VT) {
        if (op < static_cast<uint32_t>(topk)) {
          oi[op] = static_cast<int32_t>(V & pos_mask);
          if (os) os[op] = key_float(gmax - static_cast<uint32_t>(V >> pb));
        } else {
          raise_error(a.err, DEVERR_BOUNDS);
        }
        ++op;
      }
    }
    if (tid == 0 && picked != picks) raise_error(a.err, DEVERR_BOUNDS);
    return;
  }

  // ---- rescan (bin t0 holds more than CAND_CAP positions): further passes
  // over the slices, positions alive while V's decided bits equal P
  uint64_t P = t0;
  int rem = sh0;
  for (int pass = 1;; ++pass) {
    const int w = min(DIGIT, rem);
    const int sh = rem - w;
    const uint32_t dmask = (1u << w) - 1u;
    uint32_t* h = s_hist + (pass & 1) * BINS;
    for_slice(s_key, grow, beg, n, a.scap, [&](int pos, uint32_t key, bool valid) {
      if (valid) {
        const uint64_t V = make_v(pos, key);
        if ((V >> rem) == P) atomicAdd(&h[static_cast<uint32_t>(V >> sh) & dmask], 1u);
      }
    });
    cluster_sync();          // every CTA's histogram of this pass is complete
    // the other buffer was last read remotely before this barrier
    reinterpret_cast<uint4*>(s_hist + ((pass + 1) & 1) * BINS)[tid] = make_uint4(0u, 0u, 0u, 0u);
    merged_threshold(h, need);
    need -= s_cb;
    P = (P << w) | s_t;
    rem = sh;
    if (s_cnt == need || rem == 0) break;     // rem == 0 implies s_cnt == need == 1
  }
  // V <= V_T as (u, position) <= (uT, pT); uT fits 32 bits since V_T < 2^(32 + pb)
  const uint64_t VT = (P << rem) | ((1ull << rem) - 1ull);
  const uint32_t uT = static_cast<uint32_t>(VT >> pb);
  const uint32_t pT = static_cast<uint32_t>(VT & pos_mask);
  write_selected([&](int pos, uint32_t key) {
    const uint32_t u = gmax - key;
    return u < uT || (u == uT && static_cast<uint32_t>(pos) <= pT);
  });
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

// CTAs per query row: enough clusters to cover the SMs once, at most `cap`
// and no slice shorter than MIN_SLICE
int topk_cluster_size(int rows, int max_len, int cap) {
  int C = device_sm_count() / (rows > 0 ? rows : 1);
  C = C < 1 ? 1 : (C > cap ? cap : C);
  const int by_len = max_len / MIN_SLICE;
  if (C > by_len) C = by_len < 1 ? 1 : by_len;
  return C;
}

// Largest cluster size the device schedules for this kernel: 16 (opt-in,
// non-portable) when at least one such cluster fits, else 8.  Queried once
// per device; a handful of long rows (1M context) then gets twice the CTAs.
int max_cluster_for_device(size_t smem) {
  static std::atomic<int> cached[64];  // 0 until queried; racing queries store the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MAX_CLUSTER;
  const int known = cached[dev].load(std::memory_order_relaxed);
  if (known) return known;
  int cap = MAX_CLUSTER;
  if (cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(MAX_CLUSTER_NP, 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = MAX_CLUSTER_NP;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel, &cfg) == cudaSuccess && n > 0)
      cap = MAX_CLUSTER_NP;
  }
  cudaGetLastError();   // a refused query leaves no sticky error behind
  cached[dev].store(cap, std::memory_order_relaxed);
  return cap;
}

}  // namespace

cudaError_t launch_topk(const float* scores, int ld, const int32_t* q_offsets,
                        const int32_t* q_vis, int B, int Q, int max_len, int topk,
                        int first_only, int32_t* out_idx, float* out_scores, uint32_t* err,
                        cudaStream_t st, bool pdl) {
  const int rows = first_only ? B : Q;
  if (rows <= 0) return cudaSuccess;
  if (rows > 65535 || topk > DSA_MAX_TOPK) return cudaErrorInvalidValue;
  static std::atomic<bool> attr_done[64];
  const cudaError_t ea = set_once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smem_bytes(SLICE_CAP)));
  });
  if (ea != cudaSuccess) return ea;
  // beyond the portable 8 CTAs only when 8 would leave slices longer than the
  // on-chip copy (merging 16 histograms costs more than it saves otherwise)
  int C = topk_cluster_size(rows, max_len, MAX_CLUSTER);
  if (C == MAX_CLUSTER && (max_len + C - 1) / C > SLICE_CAP)
    C = topk_cluster_size(rows, max_len, max_cluster_for_device(smem_bytes(SLICE_CAP)));
  const int slice = (((max_len + C - 1) / C) + 3) & ~3;
  const int scap = slice < SLICE_CAP ? slice : SLICE_CAP;
  TopkArgs a{scores, ld, q_offsets, q_vis, B, Q, max_len, topk, first_only,
             out_idx, out_scores, err, scap};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(C), static_cast<unsigned>(rows), 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes(scap);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  unsigned int na = 1;
  add_pdl_attr(attr, &na, pdl);
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel, a);
}

cudaError_t launch_expand_idx(const int32_t* q_offsets, int B, int Q, int topk, int32_t* out_idx,
                              float* out_scores, cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  expand_idx_kernel<<<B, 256, 0, st>>>(q_offsets, Q, topk, out_idx, out_scores);
  return cudaGetLastError();
}

}  // namespace dsa
