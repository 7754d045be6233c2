// Two-tier latent cache (HiSparse).  Source: "GLM-5.2 推理部署" (inference
// deployment), section "HiSparse 的通信路径：GPU↔CPU KV swap": at 1M context the
// full KV cache stays in pinned host memory and HBM keeps a buffer of hot
// slots (4096-6144 slots of 16 tokens, host:device 8-10x).  Per step:
//   1. miss detection -- the indexer's top-K positions are compared with the
//      device buffer;
//   2. LRU eviction   -- victims come from the device buffer, least recently
//      used first;
//   3. H2D fetch      -- the page table is updated and the missing entries are
//      pulled from host memory.
//
// Steps 1-2 are host bookkeeping over one step's index rows (dsa_tier_plan):
// plain C++ on caller-owned state, no device work, costing the pages a step
// touches (not the slots or the pages of the whole context).  Step 3 is one
// kernel (dsa_tier_fetch) that reads the planned pages straight from pinned
// host memory (mapped into the device address space), writes them into their
// device slots and patches the device page table: a single launch whatever
// the number of misses, instead of one copy call per 18 KB page and an
// upload of the whole table.
//
// Readings where the page is silent: a slot holds one 16-token page of one
// sequence; each sequence owns dev_slots slots; "recently used" counts plan
// calls (every page a step selects is used at that step), ties between
// equally old slots go to the lower slot index, and never-used slots count
// as oldest; the misses of a step are placed in ascending page order into
// the victims in ascending (last use, slot) order; a step that selects more
// distinct pages of a sequence than it has slots is refused.
#include "common.cuh"
#include "internal.h"

#include <algorithm>
#include <cstring>
#include <vector>

namespace dsa {
namespace {

constexpr uint32_t TIER_MAGIC = 0x54495231u;   // "TIR1"
constexpr int TIER_ROW_BYTES = DSA_DIM * 2;    // one bf16 latent row
constexpr int TIER_PAGE_BYTES = DSA_TIER_PAGE * TIER_ROW_BYTES;   // 18432 B

struct TierHeader {
  uint32_t magic;
  int32_t B, dev_slots, max_pages;
  int64_t step;                 // plan calls so far
  int64_t hits, misses, evictions;   // totals over all steps
};

// Per-sequence arrays after the header.  The slots form one list in the order
// they would be evicted: oldest use first, never-used slots ahead of used
// ones, equal ages by ascending slot index.  A step moves every slot it uses
// to the tail in ascending slot order, which keeps that order; the victims of
// a step are the first slots of the list whose page the step did not select.
struct TierSeq {
  int64_t* stamp;          // [max_pages]  step at which the page was last selected
  int32_t* slot_of_page;   // [max_pages]  device slot or -1
  int32_t* page_of_slot;   // [dev_slots]  logical page or -1
  int32_t* prev;           // [dev_slots]  LRU list links (-1 = none)
  int32_t* next;           // [dev_slots]
  int32_t* ends;           // [2]          list head, tail
};

size_t seq_bytes(int dev_slots, int max_pages) {
  const size_t n = static_cast<size_t>(max_pages) * (8 + 4) + static_cast<size_t>(dev_slots) * 12 + 8;
  return (n + 63) / 64 * 64;
}

size_t header_bytes() { return (sizeof(TierHeader) + 63) / 64 * 64; }

TierSeq seq_view(void* state, int b) {
  TierHeader* h = static_cast<TierHeader*>(state);
  uint8_t* p = static_cast<uint8_t*>(state) + header_bytes() + b * seq_bytes(h->dev_slots, h->max_pages);
  TierSeq s;
  s.stamp = reinterpret_cast<int64_t*>(p);
  p += static_cast<size_t>(h->max_pages) * 8;
  s.slot_of_page = reinterpret_cast<int32_t*>(p);
  p += static_cast<size_t>(h->max_pages) * 4;
  s.page_of_slot = reinterpret_cast<int32_t*>(p);
  p += static_cast<size_t>(h->dev_slots) * 4;
  s.prev = reinterpret_cast<int32_t*>(p);
  p += static_cast<size_t>(h->dev_slots) * 4;
  s.next = reinterpret_cast<int32_t*>(p);
  p += static_cast<size_t>(h->dev_slots) * 4;
  s.ends = reinterpret_cast<int32_t*>(p);
  return s;
}

void list_unlink(TierSeq& s, int32_t x) {
  const int32_t a = s.prev[x], c = s.next[x];
  if (a >= 0) s.next[a] = c; else s.ends[0] = c;
  if (c >= 0) s.prev[c] = a; else s.ends[1] = a;
  s.prev[x] = s.next[x] = -1;
}

void list_append(TierSeq& s, int32_t x) {
  const int32_t tail = s.ends[1];
  s.prev[x] = tail;
  s.next[x] = -1;
  if (tail >= 0) s.next[tail] = x; else s.ends[0] = x;
  s.ends[1] = x;
}

bool tier_sizes_ok(int B, int dev_slots, int max_pages) {
  return B > 0 && B <= DSA_MAX_BATCH && dev_slots > 0 && max_pages > 0 &&
         static_cast<int64_t>(B) * dev_slots < (int64_t(1) << 31) &&
         static_cast<int64_t>(B) * max_pages < (int64_t(1) << 31);
}

// Grid-stride over the planned copies; copy i = (host page, device page,
// evicted host page or -1).  A CTA copies one 18 KB page: every thread
// issues its (up to) five 16-byte loads from the pinned host cache before
// storing any, so a page's reads are all in flight over the host link at
// once.  With a device page table the kernel also patches it: the evicted
// page loses its slot and the fetched page gets its own.  A step's evicted
// pages and fetched pages are disjoint, so no two CTAs write one entry.
// Entries outside either cache are skipped and flagged.
__global__ void __launch_bounds__(256) tier_fetch_kernel(const uint4* __restrict__ host,
                                                         uint4* __restrict__ dev,
                                                         const int32_t* __restrict__ copies, int n,
                                                         const int32_t* n_dev,
                                                         int64_t host_pages, int64_t dev_pages,
                                                         int32_t* __restrict__ page_table,
                                                         uint32_t* err) {
  constexpr int V = TIER_PAGE_BYTES / 16;      // 1152 uint4 per page
  constexpr int PER = (V + 255) / 256;         // 5 per thread
  if (n_dev) n = min(n, *n_dev);               // the count the device planner wrote
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const int64_t src = copies[3 * i], dst = copies[3 * i + 1], gone = copies[3 * i + 2];
    if (src < 0 || src >= host_pages || dst < 0 || dst >= dev_pages || gone >= host_pages) {
      if (threadIdx.x == 0) raise_error(err, DEVERR_BOUNDS);
      continue;
    }
    const uint4* s = host + src * V;
    uint4* d = dev + dst * V;
    uint4 v[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int e = threadIdx.x + k * 256;
      if (e < V) v[k] = s[e];
    }
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int e = threadIdx.x + k * 256;
      if (e < V) d[e] = v[k];
    }
    if (page_table && threadIdx.x == 0) {
      if (gone >= 0) page_table[gone] = -1;
      page_table[src] = static_cast<int32_t>(dst);
    }
  }
}

// ---------------------------------------------------------------- device planner
// The same plan as dsa_tier_plan, computed on the device so that a tiered
// step needs no host round trip (and can be captured in a graph).  Device
// state, each region 256-byte aligned:
//   hdr   int32 [16]: n_copies, hits, misses, evictions of the last step; step; done
//   stamp int32 [B,P], page_of_slot int32 [B,D], last_use int32 [B,D], copies int32 [B*D,3]
// The device page table (int32 [B,P], pool page b*D + slot or -1) is the
// page -> slot map itself.
constexpr int DEV_MAX_SLOTS = 8192;            // slots per sequence the planner sorts on chip
constexpr int PLAN_THREADS = 1024;

struct DevLayout {
  size_t hdr, stamp, page_of_slot, last_use, copies, total;
};

DevLayout dev_layout(int B, int D, int P) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  DevLayout L;
  size_t off = 0;
  L.hdr = off;          off = up(off + 64);
  L.stamp = off;        off = up(off + static_cast<size_t>(B) * P * 4);
  L.page_of_slot = off; off = up(off + static_cast<size_t>(B) * D * 4);
  L.last_use = off;     off = up(off + static_cast<size_t>(B) * D * 4);
  L.copies = off;       off = up(off + static_cast<size_t>(B) * D * 12);
  L.total = off;
  return L;
}

int pow2_at_least(int x) {
  int n = 1;
  while (n < x) n <<= 1;
  return n;
}

__device__ __forceinline__ int pow2_dev(int x) {
  int n = 1;
  while (n < x) n <<= 1;
  return n;
}

// ascending bitonic sort of a[0..N) in shared memory, N a power of two; every
// thread of the block calls it
template <typename T>
__device__ void block_bitonic_sort(T* a, int N) {
  for (int k = 2; k <= N; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < N; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const T x = a[i], y = a[ixj];
          if ((x > y) == ((i & k) == 0)) {
            a[i] = y;
            a[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// One CTA per sequence.  1. the distinct selected pages (a page's stamp is
// swapped to this step; the thread that changed it lists the page);
// 2. hits refresh their slot's last use, misses are listed; 3. every slot
// gets the key (last use + 1, slot), or the largest key if its page is
// selected now; the nmiss oldest are found by a radix select on the age
// (ties to the lower slot) and only they, and the misses, are sorted on
// chip; 4. miss i goes to the slot of victim i, evicting its page, and the
// page table and copy list are written.  The last CTA to finish advances the step.
__global__ void __launch_bounds__(PLAN_THREADS) tier_plan_kernel(
    int32_t* __restrict__ hdr, int32_t* __restrict__ stamp, int32_t* __restrict__ page_of_slot,
    int32_t* __restrict__ last_use, int32_t* __restrict__ copies, const int32_t* __restrict__ idx,
    int Q, int topk, const int32_t* __restrict__ q_offsets, int D, int P,
    int32_t* __restrict__ page_table, uint32_t* err) {
  extern __shared__ __align__(16) uint8_t tsm[];
  const int N = pow2_dev(D);
  uint64_t* keys = reinterpret_cast<uint64_t*>(tsm);               // [N]
  uint32_t* need = reinterpret_cast<uint32_t*>(keys + N);          // [D]
  uint32_t* miss = need + D;                                       // [N]
  __shared__ int s_nneed, s_nmiss, s_hits, s_base, s_digit, s_below, s_nvict;
  __shared__ int s_hist[256], s_wsum[32];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int t = hdr[4];
  if (tid == 0) { s_nneed = 0; s_nmiss = 0; s_hits = 0; }
  __syncthreads();
  int32_t* stamp_b = stamp + static_cast<size_t>(b) * P;
  int32_t* table_b = page_table + static_cast<size_t>(b) * P;
  int q0 = q_offsets[b], q1 = q_offsets[b + 1];
  if (q0 < 0 || q1 > Q || q1 < q0) {            // rows outside idx: none of them is read
    if (tid == 0) raise_error(err, DEVERR_BOUNDS);
    q0 = q1 = 0;
  }
  for (int q = q0; q < q1; ++q) {
    const int32_t* row = idx + static_cast<size_t>(q) * topk;
    for (int j = tid; j < topk; j += PLAN_THREADS) {
      const int32_t pos = row[j];
      if (pos < 0) continue;
      const int pg = pos / DSA_TIER_PAGE;
      if (pg >= P) {
        raise_error(err, DEVERR_BOUNDS);
        continue;
      }
      if (atomicExch(&stamp_b[pg], t) != t) {
        const int k = atomicAdd(&s_nneed, 1);
        if (k < D) need[k] = static_cast<uint32_t>(pg);
      }
    }
  }
  __syncthreads();
  const int nneed = s_nneed;
  if (nneed > D) {
    // more distinct pages than slots: this sequence's step cannot be served
    if (tid == 0) raise_error(err, DEVERR_CAPACITY);
  } else {
    for (int i = tid; i < nneed; i += PLAN_THREADS) {
      const int pg = static_cast<int>(need[i]);
      const int e = table_b[pg];
      if (e >= 0) {
        last_use[e] = t;
        atomicAdd(&s_hits, 1);
      } else {
        miss[atomicAdd(&s_nmiss, 1)] = static_cast<uint32_t>(pg);
      }
    }
    __syncthreads();
    const int nmiss = s_nmiss;
    if (nmiss > 0) {
      uint32_t* age = need;      // the page list is spent once hits and misses are known
      // 3. every slot's age: last use + 1 (0 = never used), or the largest
      // value for the slots whose page this step selected (never victims)
      {
        constexpr int SPT = DEV_MAX_SLOTS / PLAN_THREADS;
        int own[SPT], stp[SPT], lu[SPT];
#pragma unroll
        for (int k = 0; k < SPT; ++k) {
          const int x = tid + k * PLAN_THREADS;
          own[k] = x < D ? page_of_slot[static_cast<size_t>(b) * D + x] : -1;
          lu[k] = x < D ? last_use[static_cast<size_t>(b) * D + x] : 0;
        }
#pragma unroll
        for (int k = 0; k < SPT; ++k) stp[k] = own[k] >= 0 ? stamp_b[own[k]] : -1;
#pragma unroll
        for (int k = 0; k < SPT; ++k) {
          const int x = tid + k * PLAN_THREADS;
          if (x < D)
            age[x] = (own[k] >= 0 && stp[k] == t) ? 0xFFFFFFFFu : static_cast<uint32_t>(lu[k] + 1);
        }
      }
      // 4. the nmiss-th smallest age T, 8 bits at a time from the top: every
      // slot whose age is below T is a victim, and so are the `remaining`
      // lowest-indexed slots whose age equals T
      uint32_t prefix = 0, mask = 0;
      int remaining = nmiss;
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += PLAN_THREADS) s_hist[i] = 0;
        __syncthreads();
        for (int x = tid; x < D; x += PLAN_THREADS) {
          const uint32_t a = age[x];
          if ((a & mask) == prefix) atomicAdd(&s_hist[(a >> shift) & 255u], 1);
        }
        __syncthreads();
        if (tid < 32) {
          int c[8], sum = 0;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            c[k] = s_hist[tid * 8 + k];
            sum += c[k];
          }
          int incl = sum;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (tid >= off) incl += y;
          }
          const int excl = incl - sum;
          if (excl < remaining && remaining <= incl) {
            int acc = excl;
            for (int k = 0; k < 8; ++k) {
              if (acc + c[k] >= remaining) {
                s_digit = tid * 8 + k;
                s_below = acc;
                break;
              }
              acc += c[k];
            }
          }
        }
        __syncthreads();
        remaining -= s_below;
        prefix |= static_cast<uint32_t>(s_digit) << shift;
        mask |= 0xFFu << shift;
        __syncthreads();                       // s_digit and s_below are rewritten next pass
      }
      // 5. the victims' keys (age, slot): ties at T ranked in slot order by a
      // block scan over contiguous slot ranges
      {
        const int chunk = (D + PLAN_THREADS - 1) / PLAN_THREADS;
        const int x0 = min(D, tid * chunk), x1 = min(D, x0 + chunk);
        int eq = 0;
        for (int x = x0; x < x1; ++x) eq += age[x] == prefix;
        const int lane = tid & 31, warp = tid >> 5;
        int v = eq;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, v, off);
          if (lane >= off) v += y;
        }
        if (lane == 31) s_wsum[warp] = v;
        if (tid == 0) s_nvict = 0;
        __syncthreads();
        if (warp == 0) {
          const int w0 = s_wsum[lane];
          int w = w0;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
          }
          s_wsum[lane] = w - w0;
        }
        __syncthreads();
        int rank = s_wsum[warp] + v - eq;
        for (int x = x0; x < x1; ++x) {
          const uint32_t a = age[x];
          bool take = a < prefix;
          if (a == prefix) take = rank++ < remaining;
          if (take) keys[atomicAdd(&s_nvict, 1)] = (static_cast<uint64_t>(a) << 32) | static_cast<uint32_t>(x);
        }
      }
      const int Nv = pow2_dev(nmiss);
      __syncthreads();
      for (int i = nmiss + tid; i < Nv; i += PLAN_THREADS) {
        keys[i] = ~0ull;
        miss[i] = 0xFFFFFFFFu;
      }
      __syncthreads();
      block_bitonic_sort(keys, Nv);
      block_bitonic_sort(miss, Nv);
      if (tid == 0) s_base = atomicAdd(&hdr[0], nmiss);
      __syncthreads();
      for (int i = tid; i < nmiss; i += PLAN_THREADS) {
        const int x = static_cast<int>(keys[i] & 0xFFFFFFFFu);
        const int pg = static_cast<int>(miss[i]);
        const int gs = b * D + x;
        const int old = page_of_slot[gs];
        if (old >= 0) {
          table_b[old] = -1;
          atomicAdd(&hdr[3], 1);
        }
        page_of_slot[gs] = pg;
        table_b[pg] = gs;
        last_use[gs] = t;
        const int c = s_base + i;
        copies[3 * c] = b * P + pg;
        copies[3 * c + 1] = gs;
        copies[3 * c + 2] = old >= 0 ? b * P + old : -1;
      }
    }
    if (tid == 0) {
      atomicAdd(&hdr[1], s_hits);
      atomicAdd(&hdr[2], nmiss);
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(&hdr[5], 1) == static_cast<int>(gridDim.x) - 1) {
      hdr[4] = t + 1;
      hdr[5] = 0;
    }
  }
}

// pinned host memory the device can address over [p, p + pages * page bytes)
bool host_cache_device_ptr(const void* p, int64_t pages, const void** dptr) {
  cudaPointerAttributes a0, a1;
  const uint8_t* first = static_cast<const uint8_t*>(p);
  const uint8_t* last = first + pages * static_cast<int64_t>(TIER_PAGE_BYTES) - 1;
  if (cudaPointerGetAttributes(&a0, first) != cudaSuccess ||
      cudaPointerGetAttributes(&a1, last) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (a0.type != cudaMemoryTypeHost || a1.type != cudaMemoryTypeHost || !a0.devicePointer ||
      !a1.devicePointer ||
      static_cast<const uint8_t*>(a1.devicePointer) - static_cast<const uint8_t*>(a0.devicePointer) !=
          last - first)
    return false;
  *dptr = a0.devicePointer;
  return true;
}

bool is_device_memory(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

size_t dsa_tier_state_bytes(int B, int dev_slots, int max_pages) {
  if (!tier_sizes_ok(B, dev_slots, max_pages)) return 0;
  return header_bytes() + static_cast<size_t>(B) * seq_bytes(dev_slots, max_pages);
}

dsa_status dsa_tier_init(void* state, size_t state_bytes, int B, int dev_slots, int max_pages) {
  if (!state || (reinterpret_cast<uintptr_t>(state) & 7u)) return DSA_ERR_INVALID_ARG;
  if (!tier_sizes_ok(B, dev_slots, max_pages)) return DSA_ERR_INVALID_ARG;
  if (state_bytes < dsa_tier_state_bytes(B, dev_slots, max_pages)) return DSA_ERR_WORKSPACE;
  TierHeader* h = static_cast<TierHeader*>(state);
  std::memset(h, 0, header_bytes());
  h->magic = TIER_MAGIC;
  h->B = B;
  h->dev_slots = dev_slots;
  h->max_pages = max_pages;
  for (int b = 0; b < B; ++b) {
    TierSeq s = seq_view(state, b);
    std::fill(s.stamp, s.stamp + max_pages, int64_t(-1));
    std::fill(s.slot_of_page, s.slot_of_page + max_pages, -1);
    std::fill(s.page_of_slot, s.page_of_slot + dev_slots, -1);
    for (int x = 0; x < dev_slots; ++x) {      // every slot empty, in slot order
      s.prev[x] = x - 1;
      s.next[x] = x + 1 < dev_slots ? x + 1 : -1;
    }
    s.ends[0] = 0;
    s.ends[1] = dev_slots - 1;
  }
  return DSA_OK;
}

dsa_status dsa_tier_plan(void* state, const int32_t* idx, int Q, int topk,
                         const int32_t* q_offsets, int32_t* page_table, int32_t* copies,
                         int cap_copies, int* n_copies, int64_t* stats) {
  if (!state || !idx || !q_offsets || !n_copies || (cap_copies > 0 && !copies))
    return DSA_ERR_INVALID_ARG;
  TierHeader* h = static_cast<TierHeader*>(state);
  if (h->magic != TIER_MAGIC) return DSA_ERR_INVALID_ARG;
  const int B = h->B, D = h->dev_slots, P = h->max_pages;
  if (Q <= 0 || topk <= 0 || topk > DSA_MAX_TOPK || cap_copies < 0) return DSA_ERR_INVALID_ARG;
  if (q_offsets[0] != 0 || q_offsets[B] != Q) return DSA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (q_offsets[b + 1] < q_offsets[b]) return DSA_ERR_INVALID_ARG;
  const int64_t t = h->step;

  // 1. miss detection (no state change but the per-page stamps, which a
  // refused step puts back): the distinct pages each sequence selects and the
  // ones not resident; refuse the step if a sequence overflows its slots, a
  // position lies beyond the sequence's pages, or the copy list is too short
  std::vector<std::vector<int32_t>> need(B), miss(B);
  std::vector<std::vector<int64_t>> old_stamp(B);
  auto undo = [&](int upto) {
    for (int c = 0; c <= upto && c < B; ++c) {
      TierSeq sc = seq_view(state, c);
      for (size_t i = 0; i < need[c].size(); ++i) sc.stamp[need[c][i]] = old_stamp[c][i];
    }
  };
  int64_t total_miss = 0;
  for (int b = 0; b < B; ++b) {
    TierSeq s = seq_view(state, b);
    for (int q = q_offsets[b]; q < q_offsets[b + 1]; ++q) {
      const int32_t* row = idx + static_cast<size_t>(q) * topk;
      for (int j = 0; j < topk; ++j) {
        const int32_t pos = row[j];
        if (pos < 0) continue;
        const int64_t pg = pos / DSA_TIER_PAGE;
        if (pg >= P) {
          undo(b);
          return DSA_ERR_DEVICE_BOUNDS;
        }
        if (s.stamp[pg] == t) continue;      // already counted in this step
        old_stamp[b].push_back(s.stamp[pg]);
        s.stamp[pg] = t;
        need[b].push_back(static_cast<int32_t>(pg));
        if (s.slot_of_page[pg] < 0) miss[b].push_back(static_cast<int32_t>(pg));
      }
    }
    if (static_cast<int>(need[b].size()) > D) {
      undo(b);
      return DSA_ERR_UNSUPPORTED;
    }
    total_miss += static_cast<int64_t>(miss[b].size());
  }
  if (total_miss > cap_copies) {
    undo(B - 1);
    return DSA_ERR_WORKSPACE;
  }

  // 2. LRU eviction and the fetch plan: the misses, in ascending page order,
  // take the first slots of the eviction list whose page is not selected now;
  // then every slot this step used moves to the tail in ascending slot order
  int n = 0;
  int64_t hits = 0, evictions = 0;
  std::vector<int32_t> used;
  for (int b = 0; b < B; ++b) {
    TierSeq s = seq_view(state, b);
    used.clear();
    for (int32_t pg : need[b])
      if (s.slot_of_page[pg] >= 0) used.push_back(s.slot_of_page[pg]);
    hits += static_cast<int64_t>(used.size());
    std::sort(miss[b].begin(), miss[b].end());
    size_t k = 0;
    for (int32_t x = s.ends[0]; x >= 0 && k < miss[b].size(); x = s.next[x]) {
      const int32_t owner = s.page_of_slot[x];
      if (owner >= 0 && s.stamp[owner] == t) continue;   // selected at this step
      const int32_t pg = miss[b][k++];
      if (owner >= 0) {
        s.slot_of_page[owner] = -1;
        ++evictions;
      }
      s.page_of_slot[x] = pg;
      s.slot_of_page[pg] = x;
      copies[3 * n] = b * P + pg;
      copies[3 * n + 1] = b * D + x;
      copies[3 * n + 2] = owner >= 0 ? b * P + owner : -1;
      ++n;
      used.push_back(x);
    }
    std::sort(used.begin(), used.end());
    for (int32_t x : used) {
      list_unlink(s, x);
      list_append(s, x);
    }
  }
  if (page_table) {
    for (int b = 0; b < B; ++b) {
      TierSeq s = seq_view(state, b);
      for (int pg = 0; pg < P; ++pg)
        page_table[static_cast<size_t>(b) * P + pg] =
            s.slot_of_page[pg] >= 0 ? b * D + s.slot_of_page[pg] : -1;
    }
  }
  h->step = t + 1;
  h->hits += hits;
  h->misses += total_miss;
  h->evictions += evictions;
  *n_copies = n;
  if (stats) {
    stats[0] = hits;
    stats[1] = total_miss;
    stats[2] = evictions;
  }
  return DSA_OK;
}

dsa_status dsa_tier_fetch(const void* host_cache, int64_t host_pages, void* dev_pool,
                          int64_t dev_pages, const int32_t* copies, int n, int32_t* page_table,
                          void* ws, void* stream) {
  if (!host_cache || !dev_pool || !ws || (n > 0 && !copies)) return DSA_ERR_INVALID_ARG;
  if (host_pages <= 0 || dev_pages <= 0 || n < 0) return DSA_ERR_INVALID_ARG;
  if (host_pages >= (int64_t(1) << 31) || dev_pages >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(host_cache) & 15u) || (reinterpret_cast<uintptr_t>(dev_pool) & 15u))
    return DSA_ERR_INVALID_ARG;
  if (n == 0) return DSA_OK;
  // the host cache must be pinned host memory the device can address, over
  // its whole extent (a pageable pointer would fault the kernel)
  const void* hdev = nullptr;
  if (!host_cache_device_ptr(host_cache, host_pages, &hdev) || !is_device_memory(dev_pool))
    return DSA_ERR_INVALID_ARG;
  const int grid = std::min(n, 8 * device_sm_count());
  tier_fetch_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(hdev), static_cast<uint4*>(dev_pool), copies, n, nullptr,
      host_pages, dev_pages, page_table, static_cast<uint32_t*>(ws));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

size_t dsa_tier_dev_state_bytes(int B, int dev_slots, int max_pages) {
  if (!tier_sizes_ok(B, dev_slots, max_pages) || dev_slots > DEV_MAX_SLOTS) return 0;
  return dev_layout(B, dev_slots, max_pages).total;
}

dsa_status dsa_tier_dev_init(void* dev_state, size_t state_bytes, int B, int dev_slots,
                             int max_pages, int32_t* page_table, void* stream) {
  if (!dev_state || !page_table) return DSA_ERR_INVALID_ARG;
  if (!tier_sizes_ok(B, dev_slots, max_pages) || dev_slots > DEV_MAX_SLOTS)
    return DSA_ERR_UNSUPPORTED;
  const DevLayout L = dev_layout(B, dev_slots, max_pages);
  if (state_bytes < L.total) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(dev_state);
  // counters and step 0; every stamp, slot owner and last use -1; every page absent
  if (cudaMemsetAsync(base + L.hdr, 0, 64, st) != cudaSuccess ||
      cudaMemsetAsync(base + L.stamp, 0xFF, L.copies - L.stamp, st) != cudaSuccess ||
      cudaMemsetAsync(page_table, 0xFF, static_cast<size_t>(B) * max_pages * 4, st) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status dsa_tier_swap_in(void* dev_state, size_t state_bytes, int B, int dev_slots,
                            int max_pages, const int32_t* idx, int Q, int topk,
                            const int32_t* q_offsets, int32_t* page_table,
                            const void* host_cache, void* dev_pool, void* ws, void* stream) {
  if (!dev_state || !idx || !q_offsets || !page_table || !host_cache || !dev_pool || !ws)
    return DSA_ERR_INVALID_ARG;
  if (!tier_sizes_ok(B, dev_slots, max_pages) || dev_slots > DEV_MAX_SLOTS)
    return DSA_ERR_UNSUPPORTED;
  if (Q <= 0 || topk <= 0 || topk > DSA_MAX_TOPK) return DSA_ERR_INVALID_ARG;
  const DevLayout L = dev_layout(B, dev_slots, max_pages);
  if (state_bytes < L.total) return DSA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(host_cache) & 15u) || (reinterpret_cast<uintptr_t>(dev_pool) & 15u))
    return DSA_ERR_INVALID_ARG;
  const int64_t host_pages = static_cast<int64_t>(B) * max_pages;
  const int64_t dev_pages = static_cast<int64_t>(B) * dev_slots;
  const void* hdev = nullptr;
  if (!host_cache_device_ptr(host_cache, host_pages, &hdev) || !is_device_memory(dev_pool) ||
      !is_device_memory(dev_state))
    return DSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(dev_state);
  int32_t* hdr = reinterpret_cast<int32_t*>(base + L.hdr);
  int32_t* copies = reinterpret_cast<int32_t*>(base + L.copies);
  const int N = pow2_at_least(dev_slots);
  const size_t smem = static_cast<size_t>(N) * 8 + static_cast<size_t>(dev_slots) * 4 + static_cast<size_t>(N) * 4;
  static std::atomic<bool> attr_done[64];
  if (set_once_per_device(attr_done, [] {
        return cudaFuncSetAttribute(tier_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(DEV_MAX_SLOTS) * 16);
      }) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaMemsetAsync(hdr, 0, 16, st) != cudaSuccess) return DSA_ERR_CUDA;   // this step's counters
  tier_plan_kernel<<<B, PLAN_THREADS, smem, st>>>(
      hdr, reinterpret_cast<int32_t*>(base + L.stamp), reinterpret_cast<int32_t*>(base + L.page_of_slot),
      reinterpret_cast<int32_t*>(base + L.last_use), copies, idx, Q, topk, q_offsets, dev_slots,
      max_pages, page_table, static_cast<uint32_t*>(ws));
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  tier_fetch_kernel<<<8 * device_sm_count(), 256, 0, st>>>(
      static_cast<const uint4*>(hdev), static_cast<uint4*>(dev_pool), copies,
      static_cast<int>(dev_pages), hdr, host_pages, dev_pages, nullptr, static_cast<uint32_t*>(ws));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_tier_dev_stats(const void* dev_state, int64_t* stats, void* stream) {
  if (!dev_state || !stats) return DSA_ERR_INVALID_ARG;
  int32_t h[5];
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess ||
      cudaMemcpy(h, dev_state, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DSA_ERR_CUDA;
  for (int i = 0; i < 5; ++i) stats[i] = h[i];
  return DSA_OK;
}

const int32_t* dsa_tier_dev_copies(const void* dev_state, int B, int dev_slots, int max_pages) {
  if (!dev_state || !tier_sizes_ok(B, dev_slots, max_pages)) return nullptr;
  return reinterpret_cast<const int32_t*>(static_cast<const uint8_t*>(dev_state) +
                                          dev_layout(B, dev_slots, max_pages).copies);
}

}  // extern "C"
