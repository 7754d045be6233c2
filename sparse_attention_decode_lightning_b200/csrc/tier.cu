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
                                                         int64_t host_pages, int64_t dev_pages,
                                                         int32_t* __restrict__ page_table,
                                                         uint32_t* err) {
  constexpr int V = TIER_PAGE_BYTES / 16;      // 1152 uint4 per page
  constexpr int PER = (V + 255) / 256;         // 5 per thread
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
  cudaPointerAttributes a0, a1;
  const uint8_t* first = static_cast<const uint8_t*>(host_cache);
  const uint8_t* last = first + host_pages * static_cast<int64_t>(TIER_PAGE_BYTES) - 1;
  if (cudaPointerGetAttributes(&a0, first) != cudaSuccess ||
      cudaPointerGetAttributes(&a1, last) != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_INVALID_ARG;
  }
  if (a0.type != cudaMemoryTypeHost || a1.type != cudaMemoryTypeHost || !a0.devicePointer ||
      !a1.devicePointer ||
      static_cast<const uint8_t*>(a1.devicePointer) - static_cast<const uint8_t*>(a0.devicePointer) !=
          last - first)
    return DSA_ERR_INVALID_ARG;
  cudaPointerAttributes ad;
  if (cudaPointerGetAttributes(&ad, dev_pool) != cudaSuccess || ad.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    return DSA_ERR_INVALID_ARG;
  }
  const int grid = std::min(n, 8 * device_sm_count());
  tier_fetch_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(a0.devicePointer), static_cast<uint4*>(dev_pool), copies, n,
      host_pages, dev_pages, page_table, static_cast<uint32_t*>(ws));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // extern "C"
