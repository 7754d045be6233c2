// Sparse MLA decode for callers that cannot allocate device memory.
//
// Some callers cannot hand this library a workspace: their device memory is
// owned by another allocator (a serving engine that reserves the whole HBM up
// front for its paged KV cache and weights has nothing left to give out), or
// they must not call cudaMalloc at all because it synchronises the device and
// would stall every stream in flight.  For them this entry point keeps the
// split-K partial outputs in a fixed array of device memory that the library
// itself owns, so the call allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds its NOALLOC_SCRATCH_BYTES until the process exits.  In host
// code its name is only a host-side stand-in, not a device address, so the
// address is looked up once per device with cudaGetSymbolAddress (with that
// device current) and cached; the first call on a device does that set-up.
// Its first 256 bytes hold the device error word (zero when the library is
// loaded, cleared again by dsa_noalloc_check_error); the split-K partials
// follow.
#include "common.cuh"
#include "internal.h"

#include <mutex>

namespace dsa {

namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(16) << 20;   // 16 MiB per device
constexpr size_t PART_O_BYTES = size_t(DSA_DIM_V) * 4;   // one head of one (query, split) output
constexpr size_t PART_L_BYTES = 4;
constexpr size_t ERR_BYTES = 256;                         // the error word, padded

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// device address of g_noalloc_scratch, per device (nullptr until looked up)
void* scratch_ptr(dsa_status* st) {
  static void* ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *st = DSA_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      *st = DSA_ERR_CUDA;
      return nullptr;
    }
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" dsa_status dsa_sparse_mla_decode_noalloc(const void* q, const void* kv_pool,
                                                    int num_pages, int page_size,
                                                    const int32_t* page_table,
                                                    int max_pages, const int32_t* q_offsets,
                                                    const int32_t* q_vis, const int32_t* idx,
                                                    int B, int Q, int heads, int topk, float scale,
                                                    int num_splits, float* out, float* lse,
                                                    void* stream) {
  if (!q || !kv_pool || !page_table || !q_offsets || !q_vis || !idx || !out || !lse)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv_pool) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Q <= 0 || topk <= 0 || num_pages <= 0 || max_pages <= 0) return DSA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (!page_size_ok(page_size, num_pages)) return DSA_ERR_UNSUPPORTED;
  if (B > DSA_MAX_BATCH || Q > 65535 || topk > DSA_MAX_TOPK) return DSA_ERR_UNSUPPORTED;
  if (heads != DSA_HEADS && heads != DSA_HEADS_GLM) return DSA_ERR_UNSUPPORTED;
  if (num_splits < 0 || num_splits > DSA_MAX_SPLITS) return DSA_ERR_UNSUPPORTED;
  const int S = choose_splits(Q, topk, num_splits);
  const size_t parts = static_cast<size_t>(Q) * S * heads;      // (query, split, head) partials
  const size_t need = S > 1 ? parts * (PART_O_BYTES + PART_L_BYTES) : 0;
  if (need > NOALLOC_SCRATCH_BYTES - ERR_BYTES) return DSA_ERR_UNSUPPORTED;   // beyond the fixed array
  dsa_status st = DSA_OK;
  uint8_t* scratch = static_cast<uint8_t*>(scratch_ptr(&st));
  if (!scratch) return st;
  uint32_t* err = reinterpret_cast<uint32_t*>(scratch);
  float* o_part = reinterpret_cast<float*>(scratch + ERR_BYTES);
  float* l_part = reinterpret_cast<float*>(scratch + ERR_BYTES + parts * PART_O_BYTES);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // every partial is written by the kernel before the merge reads it, so only
  // the error word needs to start at zero (it does when the library loads,
  // and dsa_noalloc_check_error clears it after reading)
  if (launch_sparse_mla_tc(static_cast<const __nv_bfloat16*>(q),
                           static_cast<const __nv_bfloat16*>(kv_pool), num_pages, page_size, page_table,
                           max_pages, q_offsets, q_vis, idx, B, Q, heads, topk, scale, S, out, lse,
                           o_part, l_part, err, s, false) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (S > 1 && launch_combine(o_part, l_part, Q, S, heads, out, lse, s, true) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

extern "C" dsa_status dsa_noalloc_check_error(void* stream) {
  dsa_status st = DSA_OK;
  uint8_t* scratch = static_cast<uint8_t*>(scratch_ptr(&st));
  if (!scratch) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
  uint32_t flag = 0;
  if (cudaMemcpy(&flag, scratch, sizeof(flag), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (flag) {
    const uint32_t zero = 0;
    if (cudaMemcpy(scratch, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  if (flag & DEVERR_TIMEOUT) return DSA_ERR_TIMEOUT;
  if (flag & DEVERR_BOUNDS) return DSA_ERR_DEVICE_BOUNDS;
  return DSA_OK;
}
