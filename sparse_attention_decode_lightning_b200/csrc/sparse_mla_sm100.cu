// Sparse MLA decode on sm_100a tensor cores (absorbed MQA over the selected
// latents).  Source: "大语言模型结构总览", section 2.2 (MLA in MQA mode over the
// k = 2048 selected tokens; paged and non-paged kernels) and section 2.1 (one
// 576-d latent per token = 512 kv rank + 64 RoPE; 128 heads; section 7.2
// gives GLM-5.2's 64 heads over the same absorbed latent).  Per head h:
//   z_j = scale * q[h,:] . C[j,:],  O[h] = sum_j softmax(z)_j C[j,:512],
//   LSE[h] = ln sum_j exp(z_j).
//
// H = 128 or 64 heads.  The MMAs always have M = 128 (the tensor core's full
// rate shape); with H = 64 the upper 64 TMEM lanes hold the same 64 heads
// again, and each copy of a head takes half of every tile's rows (see
// softmax_dup64), so all eight softmax warps work on 16 scores a thread and
// the partial-score exchange moves about half the bytes.
//
// Work unit: (query, split) on a cluster of two CTAs that divide the
// contraction dims and the output:
//   CTA 0: S0 = q[:, 0:256) C[:, 0:256)^T + q[:, 512:544) C[:, 512:544)^T, O[:, 0:256)
//   CTA 1: S1 = q[:, 256:512) C[:, 256:512)^T + q[:, 544:576) C[:, 544:576)^T, O[:, 256:512)
// so each CTA gathers the latent columns it uses (the 64 RoPE columns go to
// both; each contracts half of them, which keeps the pair in balance).  Per tile of 64 selected rows the CTAs swap their partial
// scores (16-bit codes with a scale per 32 values) through distributed
// shared memory; both form S0 + S1
// (bitwise equal on both sides), run the same online softmax and apply the
// same P to their half of O.
//
// Tensor memory (512 columns): O half [0,256) | S/P slot 0 [256,320) |
// S/P slot 1 [320,384) | the CTA's 256 latent query dims [384,512) (bf16
// pairs).  The scores MMA reads those from tensor memory and the RoPE query
// dims from shared memory; the softmax overwrites a slot's scores with P as
// fp16 (11 significant bits; a single bf16 P cost ~1.6% of the output RMS
// once the running max is stale, fp16 ~0.3% in a CPU model), which the PV MMA
// reads from tensor memory against V (MN-major, N = 256) in shared memory.
// The tile's value dims are bf16 for the scores MMA and are rewritten in
// place as fp16 (exact in fp16's normal range) by the producer warps between
// the two MMAs, since both operands of an MMA share one type.
//
// Latent rows are gathered through the page table with 16-byte cp.async by
// four producer warps (4 rows x 128 bytes per warp instruction, written in
// the 128-byte swizzle the MMA descriptors expect; a single warp cannot keep
// enough copies in flight) into a 3-stage ring; completion is signalled by
// cp.async.mbarrier.arrive so no producer ever waits for its own copies
// (waiting for them coupled a tile's arrival to the PV of an earlier tile).  Each stage holds one tile
// (64 rows x 256 or 320 dims) until its PV is done.  The partial scores are
// pushed into the peer with st.async, whose bytes complete the peer's
// mbarrier directly.  Measured on a cluster pair swapping 32 KB each way:
// st.async ~2300 cycles, remote loads after a release-arrive ~4700, bulk
// copies ~3000; the link moves ~16 bytes per cycle per direction, so the
// exchange, not the tensor core, sets the pace of a tile.
//
// Roles (416 threads): warps 0, 10..12 producers, warp 1 tcgen05 issuer,
// warps 2..9 softmax + epilogue as two warpgroups that take rows 0..31 and
// 32..63 of each tile (one head per thread, TMEM lane = head; the row maxima
// meet through shared memory).  A single warp per scheduler left the
// softmax arithmetic latency-bound on the critical path.
#include "common.cuh"
#include "internal.h"

#include <cuda_fp16.h>
#include <cuda_fp8.h>

namespace dsa {
namespace {

constexpr int NR = 64;                         // selected rows per tile
constexpr int NST = 3;                         // tile ring depth
constexpr int PRODUCERS = 4;                   // gather warps (cp.async parallelism)
constexpr int SMX_WARPS = 8;                   // softmax warps (two warpgroups)
constexpr int THREADS = 32 * (2 + SMX_WARPS + PRODUCERS - 1);   // warp 0 + warps 10.. produce
constexpr int MAXCH = 5;                       // 64-dim chunks per CTA (CTA 1)
constexpr int CHUNK_T = NR * 128;              // 8 KB: 64 rows x 64 bf16
constexpr int STAGE_BYTES = MAXCH * CHUNK_T;   // 40 KB
constexpr int QROPE_BYTES = DSA_HEADS * 128;   // 16 KB: 128 heads x 64 bf16
constexpr int X_CODE_BYTES = DSA_HEADS * NR * 2;           // 16 KB of 16-bit codes
constexpr int X_BYTES = X_CODE_BYTES + DSA_HEADS * 2 * 4;   // + a scale per (head, 32 rows): 17 KB
constexpr int OBOX_BYTES = DSA_HEADS * 128;    // 16 KB: output box of 128 heads x 32 fp32
constexpr int OFF_QR = 0;
constexpr int OFF_ST = OFF_QR + QROPE_BYTES;
constexpr int OFF_X = OFF_ST + NST * STAGE_BYTES;
constexpr int OFF_MX = OFF_X + 2 * X_BYTES;    // [2 tiles][2 warpgroups][128 heads] partial maxima
constexpr int OFF_CRD = OFF_MX + 2 * 2 * DSA_HEADS * 4;
constexpr int OFF_BAR = OFF_CRD + DSA_MAX_TOPK * 4;
constexpr int NBAR = 3 * NST + 5 * 2 + 2;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "sparse MLA shared memory exceeds the sm_100 limit");
static_assert(OFF_ST % 1024 == 0 && OFF_X % 1024 == 0, "swizzle atoms");
static_assert(8 * OBOX_BYTES <= OFF_MX - OFF_ST, "output boxes reuse the stage ring and exchange slots");
constexpr uint32_t O_COL = 0;
constexpr uint32_t S_COL = 256;
constexpr uint32_t Q_COL = 384;
constexpr uint32_t TMEM_COLS = 512;

// Layers of one launch (IndexShare: the layers that share an index set run
// as one grid; their units are (layer, query, split))
constexpr int MAX_LAYERS = MLA_MAX_LAYERS_PER_LAUNCH;

struct MlaTcArgs {
  const __nv_bfloat16* q[MAX_LAYERS];
  const __nv_bfloat16* pool[MAX_LAYERS];
  const int32_t* page_table[MAX_LAYERS];
  int L;                                       // layers whose pointers this launch holds
  int g0;                                      // first (layer, query) unit of this launch
  int max_pages;
  int num_pages;
  int page_shift;                              // log2 of the tokens per cache page
  // sliding window (DeepSeek-V4 CSA): the `window` most recent raw tokens of
  // the query, from a second page table into the same pool, follow the topk
  // selected entries (window = 0: none)
  const int32_t* win_page_table;
  int win_max_pages;
  const int32_t* win_vis;
  int window;
  const int32_t* q_offsets;
  const int32_t* q_vis;
  const int32_t* idx;
  int B, Q, topk, S;
  float scale_log2;
  float out_scale;                             // e4m3 cache: its per-tensor scale, else 1
  float* out[MAX_LAYERS];
  float* lse[MAX_LAYERS];
  float* o_part;
  float* l_part;
  uint32_t* err;
};

// Sequence of query q: the largest b < B with q_offsets[b] <= q, found by a
// full warp in rounds of 32 parallel probes (one round for B <= 32, three
// for B = 2048) instead of a chain of dependent loads.
__device__ __forceinline__ int seq_of_query_warp(const int32_t* q_offsets, int B, int q, int lane) {
  int lo = 0, hi = B;                  // q_offsets[lo] <= q; the answer lies in [lo, hi)
  while (hi - lo > 1) {
    const int step = (hi - lo + 31) / 32;
    const int i = lo + lane * step;
    const uint32_t m = __ballot_sync(0xffffffffu, i < hi && __ldg(q_offsets + i) <= q);
    lo += (31 - __clz(m)) * step;      // lane 0 probes lo itself, so m != 0
    hi = min(hi, lo + step);
  }
  return lo;
}



__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
  const bool ok = mbar_wait(bar, parity, err);
  return __all_sync(0xffffffffu, ok);
}

// the same for a barrier that the peer CTA arrives on (acquire at cluster scope)
__device__ __forceinline__ bool warp_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t* err) {
  const bool ok = mbar_wait_cluster(bar, parity, err);
  return __all_sync(0xffffffffu, ok);
}

// Partial scores cross the cluster link as 16-bit integers with one fp32
// scale per block of 32 (one thread's rows of one head): code = rint(s * qs)
// with qs = 32760 / amax, value = code * (amax / 32760).  The absolute error
// is at most amax / 65520 = 1.5e-5 amax, the bound a 15-bit mantissa float
// has for the block's largest value (the softmax is sensitive to absolute
// score error alone); a CPU simulation against the exact scores moves rms(O)
// by < 1e-3 and LSE by < 4e-4.  Invalid rows travel as code 0.
// The conversions stay on the FMA and integer pipes (float-to-int and back
// go through the narrow conversion unit, which the softmax's exp2 also
// needs): s * qs + (2^23 + 2^15) is a float in [2^23, 2^24), where the ulp
// is 1, so its low 16 mantissa bits hold code + 2^15; decoding ORs those
// bits under the exponent of 2^23 and subtracts 2^23 + 2^15 exactly.
constexpr float CODE_BIAS = 8421376.f;            // 2^23 + 2^15
__device__ __forceinline__ float block_scale_of(float amax) { return amax * (1.f / 32760.f); }

__device__ __forceinline__ float code_lo(uint32_t w) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7610)) - CODE_BIAS;
}
__device__ __forceinline__ float code_hi(uint32_t w) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7632)) - CODE_BIAS;
}

// two fp32 -> fp16 pair (lo in the low half), round to nearest even
__device__ __forceinline__ uint32_t f16x2_bits(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// two bf16 (low half first) -> two fp16: exact for magnitudes 2^-14 .. 65504
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  return f16x2_bits(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat162 v) {
  return *reinterpret_cast<uint32_t*>(&v);
}

// two e4m3 codes (low byte first) -> two bf16, exactly: every e4m3 value has
// at most 4 significant bits and an exponent inside bf16's range
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t pair) {
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(pair), __NV_E4M3);
  __half2 h;
  h = *reinterpret_cast<const __half2*>(&hr);
  const float2 f = __half22float2(h);
  return bf16x2_bits(__floats2bfloat162_rn(f.x, f.y));
}

__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint2 v) {
  return make_uint4(e4m3x2_to_bf16x2(v.x & 0xFFFFu), e4m3x2_to_bf16x2(v.x >> 16),
                    e4m3x2_to_bf16x2(v.y & 0xFFFFu), e4m3x2_to_bf16x2(v.y >> 16));
}

// two e4m3 codes -> two fp16, exactly (one cvt: an e4m3 value is an fp16
// value, its smallest subnormal 2^-9 above fp16's normal minimum)
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t pair) {
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(pair), __NV_E4M3);
  return static_cast<uint32_t>(hr.x) | (static_cast<uint32_t>(hr.y) << 16);
}

__device__ __forceinline__ uint4 e4m3x8_to_f16x8(uint2 v) {
  return make_uint4(e4m3x2_to_f16x2(v.x & 0xFFFFu), e4m3x2_to_f16x2(v.x >> 16),
                    e4m3x2_to_f16x2(v.y & 0xFFFFu), e4m3x2_to_f16x2(v.y >> 16));
}

// a bf16 pair with a finite element of magnitude >= 65536, which fp16 cannot hold
// (no bf16 value lies between fp16's maximum 65504 and 65536)
__device__ __forceinline__ bool bf16x2_beyond_f16(uint32_t w) {
  const uint32_t lo = w & 0x7FFFu, hi = (w >> 16) & 0x7FFFu;
  return (lo >= 0x4780u && lo < 0x7F80u) || (hi >= 0x4780u && hi < 0x7F80u);
}

// head h's 256 latent query dims of this CTA -> its TMEM lane at columns
// [Q_COL, Q_COL + 128): bf16 pairs as given, or (FP8 cache) fp16 pairs, since
// both operands of the scores MMA take one type.  bf16 -> fp16 is exact for
// magnitudes 2^-14 .. 65504; below, fp16's subnormal spacing 2^-24 rounds; an
// element beyond fp16's range is flagged as out of range.
template <bool F16>
__device__ __forceinline__ void load_query_tmem(const __nv_bfloat16* qh, uint32_t lane_addr,
                                                uint32_t* err) {
  const uint4* src = reinterpret_cast<const uint4*>(qh);
  bool bad = false;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float w[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint4 v = __ldg(src + c * 8 + i);
      if constexpr (F16) {
        bad |= bf16x2_beyond_f16(v.x) | bf16x2_beyond_f16(v.y) | bf16x2_beyond_f16(v.z) |
               bf16x2_beyond_f16(v.w);
        v = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z),
                       bf16x2_to_f16x2(v.w));
      }
      w[4 * i + 0] = __uint_as_float(v.x);
      w[4 * i + 1] = __uint_as_float(v.y);
      w[4 * i + 2] = __uint_as_float(v.z);
      w[4 * i + 3] = __uint_as_float(v.w);
    }
    tmem_st32(lane_addr + Q_COL + c * 32, w);
  }
  if (F16 && bad) raise_error(err, DEVERR_BOUNDS);
}

// the per-layer tensor maps: RoPE query dims, and the output
struct MlaMaps {
  CUtensorMap q[MAX_LAYERS];
  CUtensorMap o[MAX_LAYERS];
};

// Softmax and epilogue for 64 heads (GLM-5.2).  The MMAs keep M = 128, so
// the query heads are duplicated: TMEM lanes 64..127 hold heads 0..63 again,
// and the two copies of a head split each tile's rows.  Warp (g, quarter)
// owns head (quarter & 1) * 32 + lane and the row block blk = 2g +
// (quarter >> 1) of 16 rows: lanes 0..63 take blocks 0 and 2, lanes 64..127
// blocks 1 and 3.  Each copy writes P for its own rows and zeros for the
// rows of the other copy, so O[h] + O[h + 64] is the head's output; the
// epilogue adds the two through shared memory.  All eight softmax warps work,
// 16 scores a thread, where the plain layout leaves lanes 64..127 idle.
constexpr int DUP_HEADS = 64;
constexpr int DUP_BLOCKS = 4;                                  // 16-row blocks of a tile
constexpr int DUP_CODE_BYTES = DUP_HEADS * NR * 2;            // 8 KB of codes a tile
static_assert(DUP_CODE_BYTES + DUP_HEADS * DUP_BLOCKS * 4 <= X_BYTES, "exchange slot");

template <bool KV8>
__device__ __forceinline__ void softmax_dup64(
    const MlaTcArgs& a, const MlaMaps& maps, uint8_t* smem, uint32_t tmem, int layer, int q,
    int split, int gu, int ntiles, int nrows, const int* crd, uint8_t* xb, float* mx,
    uint64_t* s_full, uint64_t* p_full, uint64_t* slot_free, uint64_t* x_full, uint64_t* x_free,
    uint64_t* o_final, uint64_t* q_ready, int warp, int lane, int tid, uint32_t rank) {
  constexpr int NH = DUP_HEADS;
  const int g = (warp - 2) >> 2;
  const int gt = tid - 64;
  const int quarter = warp & 3;
  const int h = (quarter & 1) * 32 + lane;                     // head of this lane
  const int blk = 2 * g + (quarter >> 1);                      // its 16 rows of a tile
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  const uint32_t peer = rank ^ 1u;
  const uint32_t peer_x = map_to_rank(smem_u32(xb), peer);
  const uint32_t peer_xfull = map_to_rank(smem_u32(x_full), peer);
  const uint32_t peer_xfree = map_to_rank(smem_u32(x_free), peer);
  if (g == 0) {
    // head h's 256 latent query dims of this CTA -> both of its TMEM lanes
    load_query_tmem<KV8>(a.q[layer] + (static_cast<size_t>(q) * NH + h) * DSA_DIM + (rank ? 256 : 0),
                         lane_base, a.err);
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(q_ready);
  }
  float m_use = -INFINITY, l = 0.f;                            // l: this block's rows only
  bool ok = true;
  const float sl = a.scale_log2;
  const float zeros[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int t = 0; t < ntiles; ++t) {
    const int sb = t & 1;
    const uint32_t ph = (t >> 1) & 1;
    const int j = t * NR + 16 * blk + lane;
    const uint32_t vm = __ballot_sync(0xffffffffu, lane < 16 && j < nrows && crd[j] >= 0);
    float z[16];
    // my receive slot of tile t-1 has been read: the peer may push tile t+1
    if (t >= 1) {
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_relaxed(peer_xfree + ((t - 1) & 1) * 8);
    }
    if (g == 0 && quarter == 0 && lane == 0)
      mbar_arrive_expect_tx(&x_full[sb], static_cast<uint32_t>(NH) * DUP_BLOCKS * (16 * 2 + 4));
    if (ok) ok = warp_wait(&s_full[sb], ph, a.err);
    tc_fence_after();
    tmem_ld16(lane_base + S_COL + sb * NR + 16 * blk, z);
    tmem_ld_wait();
    // 16-bit codes with one scale per block (as block_scale_of describes);
    // rows that select nothing were gathered as zeros
    float am[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      am[i] = fmaxf(fmaxf(fabsf(z[4 * i]), fabsf(z[4 * i + 1])), fmaxf(fabsf(z[4 * i + 2]), fabsf(z[4 * i + 3])));
    const float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
    const float qs = amax > 0.f ? __fdividef(32760.f, amax) : 0.f;
    uint32_t cw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      z[2 * i] = fmaf(z[2 * i], qs, CODE_BIAS);
      z[2 * i + 1] = fmaf(z[2 * i + 1], qs, CODE_BIAS);
      cw[i] = __byte_perm(__float_as_uint(z[2 * i]), __float_as_uint(z[2 * i + 1]), 0x5410);
    }
    // slot layout [16-byte chunk k][block][head], then the scales [block][head]
    const uint32_t xoff = sb * X_BYTES + (blk * NH + h) * 16;
    const uint32_t soff = sb * X_BYTES + DUP_CODE_BYTES + (blk * NH + h) * 4;
    if (ok && t >= 2) ok = warp_wait_cluster(&x_free[sb], ((t >> 1) - 1) & 1, a.err);
    if (ok) {
#pragma unroll
      for (int k = 0; k < 2; ++k)
        st_async_v4(peer_x + xoff + k * (DUP_BLOCKS * NH * 16), __uint_as_float(cw[4 * k]),
                    __uint_as_float(cw[4 * k + 1]), __uint_as_float(cw[4 * k + 2]),
                    __uint_as_float(cw[4 * k + 3]), peer_xfull + sb * 8);
      st_async_b32(peer_x + soff, __float_as_uint(amax), peer_xfull + sb * 8);
    }
    if (ok) ok = warp_wait_cluster(&x_full[sb], ph, a.err);
    uint32_t pw[8];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint4 v = *reinterpret_cast<const uint4*>(xb + xoff + k * (DUP_BLOCKS * NH * 16));
      pw[4 * k] = v.x; pw[4 * k + 1] = v.y; pw[4 * k + 2] = v.z; pw[4 * k + 3] = v.w;
    }
    // z = (S0 + S1) * sl, evaluated alike on both CTAs (c0, k0 from rank 0)
    const float k_own = block_scale_of(amax) * sl;
    const float k_peer = block_scale_of(*reinterpret_cast<const float*>(xb + soff)) * sl;
    if (rank == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        z[2 * i] = fmaf(z[2 * i] - CODE_BIAS, k_own, code_lo(pw[i]) * k_peer);
        z[2 * i + 1] = fmaf(z[2 * i + 1] - CODE_BIAS, k_own, code_hi(pw[i]) * k_peer);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        z[2 * i] = fmaf(code_lo(pw[i]), k_peer, (z[2 * i] - CODE_BIAS) * k_own);
        z[2 * i + 1] = fmaf(code_hi(pw[i]), k_peer, (z[2 * i + 1] - CODE_BIAS) * k_own);
      }
    }
    if (vm != 0xFFFFu) {
#pragma unroll
      for (int r = 0; r < 16; ++r) z[r] = ((vm >> r) & 1u) ? z[r] : -INFINITY;
    }
    float m4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) m4[i] = fmaxf(fmaxf(z[4 * i], z[4 * i + 1]), fmaxf(z[4 * i + 2], z[4 * i + 3]));
    // tile maximum of head h over the four blocks (both copies of the head)
    float* mxt = mx + (t & 1) * DUP_BLOCKS * NH;
    mxt[blk * NH + h] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
    named_barrier(1, 32 * SMX_WARPS);
    const float mtile = fmaxf(fmaxf(mxt[h], mxt[NH + h]), fmaxf(mxt[2 * NH + h], mxt[3 * NH + h]));
    // running max, moved only when it grows by more than 8; identical in
    // every warp holding head h and in both CTAs
    float alpha = 1.f;
    bool resc = false;
    if (mtile > m_use + 8.f) {
      if (m_use != -INFINITY) {
        alpha = fast_exp2(m_use - mtile);
        resc = true;
      }
      m_use = mtile;
    }
    const float m_eff = m_use == -INFINITY ? 0.f : m_use;
    float ps0 = 0.f, ps1 = 0.f, ps2 = 0.f, ps3 = 0.f;
#pragma unroll
    for (int r = 0; r < 16; r += 4) {
      z[r + 0] = fast_exp2(z[r + 0] - m_eff);
      z[r + 1] = fast_exp2(z[r + 1] - m_eff);
      z[r + 2] = fast_exp2(z[r + 2] - m_eff);
      z[r + 3] = fast_exp2(z[r + 3] - m_eff);
      ps0 += z[r + 0];
      ps1 += z[r + 1];
      ps2 += z[r + 2];
      ps3 += z[r + 3];
    }
    l = l * alpha + ((ps0 + ps1) + (ps2 + ps3));
    // both copies' O lanes are rescaled (by the g == 0 warps, every lane)
    // after PV(t-1), as in the 128-head layout
    if (g == 0 && __any_sync(0xffffffffu, resc)) {
      if (ok && t >= 1) ok = warp_wait(&slot_free[(t - 1) & 1], ((t - 1) >> 1) & 1, a.err);
      tc_fence_after();
      for (int c = 0; c < 256 / 32; ++c) {
        float o[32];
        tmem_ld32(lane_base + O_COL + c * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= alpha;
        tmem_st32(lane_base + O_COL + c * 32, o);
      }
    }
    // P (fp16 pairs) for my 16 rows, zeros for the other copy's block
    float pk[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) pk[jj] = __uint_as_float(f16x2_bits(z[2 * jj], z[2 * jj + 1]));
    tmem_st8(lane_base + S_COL + sb * NR + 8 * blk, pk);
    tmem_st8(lane_base + S_COL + sb * NR + 8 * (blk ^ 1), zeros);
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&p_full[sb]);
  }
  // ---- epilogue: l over the four blocks; O = (O[h] + O[h + 64]) / l
  // (group g writes columns [128g, 128g+128) of this CTA's 256); LSE from CTA 0
  float* lsum = mx;                                            // reuse: [4][64]
  named_barrier(1, 32 * SMX_WARPS);
  lsum[blk * NH + h] = l;
  named_barrier(1, 32 * SMX_WARPS);
  const float lt = (lsum[h] + lsum[NH + h]) + (lsum[2 * NH + h] + lsum[3 * NH + h]);
  const bool have = ok && ntiles > 0 && warp_wait(o_final, 0, a.err);
  if (have) tc_fence_after();
  const float inv = lt > 0.f ? a.out_scale / lt : 0.f;
  float* lrow = a.S == 1 ? a.lse[layer] + static_cast<size_t>(q) * NH + h
                         : a.l_part + (static_cast<size_t>(gu) * a.S + split) * NH + h;
  const int orow0 = (a.S == 1 ? q : gu * a.S + split) * NH;
  uint8_t* box0 = smem + OFF_ST + g * 4 * OBOX_BYTES;
  const bool second = quarter >= 2;                            // lanes 64..127: the copies
  const int brow = quarter * 32 + lane;                        // this lane's box row
  for (int c = 0; c < 128 / 32; ++c) {
    uint8_t* box = box0 + c * OBOX_BYTES;
    float o[32];
    if (have) {
      tmem_ld32(lane_base + O_COL + 128 * g + c * 32, o);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = 0.f;
    }
    // the copies park their raw O in box rows 64..127
    if (second) {
#pragma unroll
      for (int jb = 0; jb < 8; ++jb)
        *reinterpret_cast<float4*>(box + brow * 128 + ((jb ^ (brow & 7)) << 4)) =
            make_float4(o[4 * jb], o[4 * jb + 1], o[4 * jb + 2], o[4 * jb + 3]);
    }
    named_barrier(2 + g, 128);
    if (!second) {
      const int prow = brow + 64;                              // the same head's copy
#pragma unroll
      for (int jb = 0; jb < 8; ++jb) {
        const float4 u = *reinterpret_cast<const float4*>(box + prow * 128 + ((jb ^ (prow & 7)) << 4));
        const float4 w = have && lt > 0.f
                             ? make_float4((o[4 * jb] + u.x) * inv, (o[4 * jb + 1] + u.y) * inv,
                                           (o[4 * jb + 2] + u.z) * inv, (o[4 * jb + 3] + u.w) * inv)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(box + brow * 128 + ((jb ^ (brow & 7)) << 4)) = w;
      }
    }
    fence_proxy_async_smem();
    named_barrier(2 + g, 128);
    if (gt == 128 * g) {
      tma_store_2d(&maps.o[layer], box, static_cast<int>(rank) * 256 + 128 * g + 32 * c, orow0);
      bulk_commit_group();
    }
  }
  if (gt == 128 * g) bulk_wait_all_read();
  if (rank == 0 && g == 0 && !second)
    *lrow = lt > 0.f ? m_use * 0.69314718055994531f + logf(lt) : -INFINITY;
}

template <int NH, bool KV8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    sparse_mla_tc_kernel(const __grid_constant__ MlaMaps maps, const __grid_constant__ MlaTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* qrope = smem + OFF_QR;
  uint8_t* st = smem + OFF_ST;
  uint8_t* xb = smem + OFF_X;
  int* crd = reinterpret_cast<int*>(smem + OFF_CRD);
  float* mx = reinterpret_cast<float*>(smem + OFF_MX);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + NST;
  uint64_t* s_full = bars + 2 * NST;     // [2] scores of a tile are in its slot
  uint64_t* p_full = s_full + 2;         // [2] P of a tile is in its slot
  uint64_t* slot_free = p_full + 2;      // [2] PV of the slot's tile is done
  uint64_t* x_full = slot_free + 2;      // [2] the peer's partial scores arrived
  uint64_t* x_free = x_full + 2;         // [2] the peer has read my partial from its slot
  uint64_t* o_final = x_free + 2;        // last PV
  uint64_t* q_ready = o_final + 1;       // query slice in TMEM / shared memory
  uint64_t* v_ready = q_ready + 1;       // [NST] a stage's value dims are fp16
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + OFF_MISC);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  pdl_trigger();
  const int unit = blockIdx.x >> 1;
  // (layer, query) unit gi = layer * Q + q, split `split` of it; with split-K
  // the partials of this launch's units are numbered from g0
  const int gu = unit / a.S, split = unit % a.S;
  const int gi = a.g0 + gu;
  const int layer = gi / a.Q;
  const int q = gi % a.Q;
  const int b = seq_of_query_warp(a.q_offsets, a.B, q, lane);
  int vis = a.q_vis[q];
  if (vis < 0) vis = 0;
  const int total = a.topk + a.window;             // selected entries, then the window
  const int per = (total + a.S - 1) / a.S;
  const int r0 = split * per;
  const int r1 = min(total, r0 + per);
  const int nrows = r1 > r0 ? r1 - r0 : 0;
  const int ntiles = (nrows + NR - 1) / NR;

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 32 * PRODUCERS);   // one copy-completion arrival per producer lane
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], SMX_WARPS);  // one arrival per softmax warp
      mbar_init(&slot_free[i], 1);
      mbar_init(&x_full[i], 1);   // armed with the tile's bytes; the peer's st.async complete them
      mbar_init(&x_free[i], SMX_WARPS);      // remote arrivals of the peer's softmax warps
    }
    mbar_init(o_final, 1);
    mbar_init(q_ready, 5);             // 4 query-loading warps + thread 0 with the RoPE bytes
    for (int i = 0; i < NST; ++i) mbar_init(&v_ready[i], PRODUCERS);   // one per producer warp
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();                 // the peer's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (tid == 0) {
    tma_prefetch_desc(&maps.q[layer]);
    if constexpr (NH == 64) {
      // 64 heads: rows 64..127 repeat rows 0..63 (TMEM lanes 64..127 carry
      // the same heads; see the softmax)
      mbar_arrive_expect_tx(q_ready, 2 * NH * 128);
      tma_load_2d(qrope, &maps.q[layer], 8 * 64, q * NH, q_ready);
      tma_load_2d(qrope + NH * 128, &maps.q[layer], 8 * 64, q * NH, q_ready);
    } else {
      mbar_arrive_expect_tx(q_ready, NH * 128);
      tma_load_2d(qrope, &maps.q[layer], 8 * 64, q * NH, q_ready);
    }
  }
  // the selected indices (and the error word) come from the kernel before
  pdl_wait();
  // pool row of every entry of this split, resolved once by all threads with
  // many independent loads in flight (-1 = padding or out of range)
  {
    constexpr int PER = (DSA_MAX_TOPK + THREADS - 1) / THREADS;
    int wvis = a.window > 0 ? a.win_vis[q] : 0;
    if (wvis < 0) wvis = 0;
    int sv[PER];
    bool win[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int j = r0 + tid + k * THREADS;
      win[k] = j >= a.topk;
      if (j >= r1) sv[k] = -1;
      else if (!win[k]) sv[k] = a.idx[static_cast<size_t>(q) * a.topk + j];
      else sv[k] = max(-1, wvis - a.window + (j - a.topk));   // before token 0: none
    }
    int pg[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int sx = sv[k];
      const int32_t* tab = win[k] ? a.win_page_table : a.page_table[layer];
      const int mp = win[k] ? a.win_max_pages : a.max_pages;
      const bool ok = sx >= 0 && sx < (win[k] ? wvis : vis) && (sx >> a.page_shift) < mp;
      pg[k] = ok ? tab[static_cast<size_t>(b) * mp + (sx >> a.page_shift)] : -1;
    }
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int jj = tid + k * THREADS;
      if (jj < nrows) {
        const int sx = sv[k];
        const bool ok = pg[k] >= 0 && pg[k] < a.num_pages;
        if (!ok && sx != -1 && rank == 0) raise_error(a.err, DEVERR_BOUNDS);
        crd[jj] = ok ? (pg[k] << a.page_shift) + (sx & ((1 << a.page_shift) - 1)) : -1;
      }
    }
  }
  __syncthreads();

  if (warp == 0 || warp >= 2 + SMX_WARPS) {
    // ------------------------------------------------------------ producers
    // producer p copies rows [16p, 16p+16) of every tile; its warp instruction
    // i copies row 16p + 4i + (lane >> 3), 16-byte piece (lane & 7); piece u
    // of row r lands at r*128 + ((u ^ (r & 7)) * 16)
    const int pw = warp == 0 ? 0 : warp - (1 + SMX_WARPS);
    const int pu = lane & 7;
    const uint8_t* pool = reinterpret_cast<const uint8_t*>(a.pool[layer]);
    bool ok = true;
    // Between its scores MMA and its PV MMA, tile t's value dims (this CTA's
    // 256 latent columns) are rewritten in place as fp16, the type of P; the
    // producers do it two tiles behind the copies they issue, each for its own
    // rows.  bf16 -> fp16 is exact for magnitudes 2^-14 .. 65504; smaller
    // values keep fp16's subnormal spacing 2^-24.
    // gather tile k into its stage (after that stage's last PV)
    auto gather = [&](int k) -> bool {
      const int s = k % NST;
      if (!warp_wait(&empty[s], ((k / NST) & 1) ^ 1, a.err)) return false;
      uint8_t* stage = st + s * STAGE_BYTES;
      if constexpr (KV8) {
        // e4m3 rows of 576 bytes: a lane loads all its 8-byte pieces (8 dims
        // of each of its 5 chunks of its 4 rows) before it widens them exactly
        // and stores them where the bf16 path's copies land: the 256 latent
        // dims as fp16 (the type of P and of the fp16 query, so no later
        // rewrite), the RoPE dims as bf16 (the type of the RoPE query)
        constexpr int RI = NR / (4 * PRODUCERS);
        uint2 v[RI][MAXCH];
#pragma unroll
        for (int i = 0; i < RI; ++i) {
          const int r = (NR / PRODUCERS) * pw + 4 * i + (lane >> 3);
          const int j = k * NR + r;
          const int row = j < nrows ? crd[j] : -1;
          const uint8_t* src = pool + static_cast<size_t>(row < 0 ? 0 : row) * DSA_DIM + pu * 8;
#pragma unroll
          for (int c = 0; c < MAXCH; ++c) {
            const int off = c < 4 ? (4 * static_cast<int>(rank) + c) * 64 : 512;
            v[i][c] = row >= 0 ? __ldg(reinterpret_cast<const uint2*>(src + off)) : make_uint2(0u, 0u);
          }
        }
#pragma unroll
        for (int i = 0; i < RI; ++i) {
          const int r = (NR / PRODUCERS) * pw + 4 * i + (lane >> 3);
          uint8_t* dst = stage + r * 128 + ((pu ^ (r & 7)) * 16);
#pragma unroll
          for (int c = 0; c < MAXCH; ++c)
            *reinterpret_cast<uint4*>(dst + c * CHUNK_T) =
                c < 4 ? e4m3x8_to_f16x8(v[i][c]) : e4m3x8_to_bf16x8(v[i][c]);
        }
        fence_proxy_async_smem();      // generic-proxy stores, read by the tensor core
        mbar_arrive(&full[s]);
      } else {
#pragma unroll
      for (int i = 0; i < NR / (4 * PRODUCERS); ++i) {
        const int r = (NR / PRODUCERS) * pw + 4 * i + (lane >> 3);
        const int j = k * NR + r;
        const int row = j < nrows ? crd[j] : -1;
        const uint8_t* src = row >= 0 ? pool + static_cast<size_t>(row) * (DSA_DIM * 2) + pu * 16 : pool;
        const uint32_t nb = row >= 0 ? 16u : 0u;
        const int sh = row >= 0 ? 1 : 0;      // address step only for real rows
        uint8_t* dst = stage + r * 128 + ((pu ^ (r & 7)) * 16);
#pragma unroll
        for (int c = 0; c < 4; ++c) cp_async16(dst + c * CHUNK_T, src + sh * (4 * rank + c) * 128, nb);
        cp_async16(dst + 4 * CHUNK_T, src + sh * 8 * 128, nb);
      }
      // arrives once this lane's copies of the tile have landed; the producer
      // never blocks on its own copies
      cp_async_arrive_noinc(&full[s]);
      }
      return true;
    };
    // tile t's value dims -> fp16, between its scores MMA and its PV
    auto convert = [&](int t) -> bool {
        const int s = t % NST;
        // the scores MMA has read the tile (its copies are complete too)
        if (!warp_wait(&s_full[t & 1], (t >> 1) & 1, a.err)) return false;
        if (!warp_wait(&full[s], (t / NST) & 1, a.err)) return false;
        uint8_t* stage = st + s * STAGE_BYTES;
#pragma unroll 4
        for (int i = lane; i < (NR / PRODUCERS) * 4 * 8; i += 32) {
          // piece i of this producer's rows: chunk i / (rows * 8), row, 16-byte piece
          const int c = i / ((NR / PRODUCERS) * 8);
          const int rr = (i / 8) % (NR / PRODUCERS);
          uint4* pc = reinterpret_cast<uint4*>(stage + c * CHUNK_T +
                                               ((NR / PRODUCERS) * pw + rr) * 128 + (i % 8) * 16);
          const uint4 v = *pc;
          *pc = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z),
                           bf16x2_to_f16x2(v.w));
        }
        fence_proxy_async_smem();      // generic-proxy stores, read by the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&v_ready[s]);
        return true;
    };
    // The copies run ahead: the first NST tiles are issued before any
    // conversion; later, tile k-2 (whose scores MMA is long done) is
    // converted before tile k waits for its stage.
    for (int k = 0; k < ntiles + 2 && ok; ++k) {
      if (k < NST && k < ntiles) ok = gather(k);
      if (!KV8 && ok && k >= 2) ok = convert(k - 2);
      if (ok && k >= NST && k < ntiles) ok = gather(k);
    }
    cp_async_wait<0>();                 // nothing in flight when the CTA retires
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      // latent dims: bf16, or fp16 over an FP8 cache; RoPE dims: bf16
      constexpr uint32_t idesc_s = umma_idesc(KV8 ? 0 /*F16*/ : 1 /*BF16*/, DSA_HEADS, NR);
      constexpr uint32_t idesc_r = umma_idesc(1 /*BF16*/, DSA_HEADS, NR);
      constexpr uint32_t idesc_pv = umma_idesc(0 /*F16*/, DSA_HEADS, 256, 0, 1);
      bool ok = mbar_wait(q_ready, 0, a.err);
      tc_fence_after();
      const uint32_t qra = smem_u32(qrope);
      for (int u = 0; u <= ntiles && ok; ++u) {
        if (u < ntiles) {
          const int sb = u & 1, s = u % NST;
          if (!(ok = mbar_wait(&slot_free[sb], ((u >> 1) & 1) ^ 1, a.err))) break;
          if (!(ok = mbar_wait(&full[s], (u / NST) & 1, a.err))) break;
          // the tile was written by cp.async (generic proxy); order it before
          // the tensor core's shared-memory reads (async proxy)
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t ta = smem_u32(st + s * STAGE_BYTES);
          const uint32_t d = tmem + S_COL + sb * NR;
          // 256 dims with q from tensor memory: k-step kk reads chunk kk/4
#pragma unroll
          for (int kk = 0; kk < 16; ++kk)
            mma_f16_ts(d, tmem + Q_COL + kk * 8,
                       umma_desc_sw128(ta + (kk >> 2) * CHUNK_T + (kk & 3) * 32, 1024, 16),
                       idesc_s, kk > 0);
          // this CTA's 32 of the 64 RoPE dims: q from shared memory
#pragma unroll
          for (int kk = 2 * rank; kk < 2 * rank + 2; ++kk)
            mma_f16(d, umma_desc_sw128(qra + kk * 32, 1024, 16),
                    umma_desc_sw128(ta + 4 * CHUNK_T + kk * 32, 1024, 16), idesc_r, 1u);
          mma_commit(&s_full[sb]);
        }
        if (u >= 1) {
          const int t = u - 1, pbuf = t & 1, s = t % NST;
          if (!(ok = mbar_wait(&p_full[pbuf], (t >> 1) & 1, a.err))) break;
          if (!KV8 && !(ok = mbar_wait(&v_ready[s], (t / NST) & 1, a.err))) break;
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t pa = tmem + S_COL + pbuf * NR;   // P (fp16 pairs) in cols [0,32)
          const uint32_t va = smem_u32(st + s * STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < NR / 16; ++kk) {
            // k-step kk: P x rows 16kk .. 16kk+15 of V (fp16, MN-major)
            mma_f16_ts(tmem + O_COL, pa + kk * 8,
                       umma_desc_sw128_mn(va + kk * 2048, CHUNK_T, 1024), idesc_pv,
                       (t > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&slot_free[pbuf]);
          mma_commit(&empty[s]);
          if (t == ntiles - 1) mma_commit(o_final);
        }
      }
    }
  } else if constexpr (NH == 64) {
    softmax_dup64<KV8>(a, maps, smem, tmem, layer, q, split, gu, ntiles, nrows, crd, xb, mx, s_full,
                  p_full, slot_free, x_full, x_free, o_final, q_ready, warp, lane, tid, rank);
  } else {
    // ------------------------------------------------------------ softmax
    const int g = (warp - 2) >> 2;                 // warpgroup: tile rows [32g, 32g+32)
    const int gt = tid - 64;                       // 0..255 within the softmax warps
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    constexpr bool live = true;                  // 128 heads: every lane carries one
    const uint32_t peer = rank ^ 1u;
    const uint32_t peer_x = map_to_rank(smem_u32(xb), peer);
    const uint32_t peer_xfull = map_to_rank(smem_u32(x_full), peer);
    const uint32_t peer_xfree = map_to_rank(smem_u32(x_free), peer);
    // partial scores are exchanged by push: each CTA stores its partial into
    // the peer's shared memory with st.async and reads the peer's from its own
    if (g == 0) {
      if (live) {
        // head h's 256 latent query dims of this CTA -> tensor memory
        load_query_tmem<KV8>(
            a.q[layer] + (static_cast<size_t>(q) * NH + h) * DSA_DIM + (rank ? 256 : 0), lane_base,
            a.err);
        tmem_st_wait();
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    float m_use = -INFINITY, l = 0.f;                // l: this warpgroup's rows only
    bool ok = true;
    // A wait that runs out clears ok; the warp then skips its remaining waits
    // and data movement but keeps every barrier arrival, so no other warp of
    // the block is left waiting on it.
    for (int t = 0; t < ntiles; ++t) {
      const int sb = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      const int j = t * NR + 32 * g + lane;
      const uint32_t vm = __ballot_sync(0xffffffffu, j < nrows && crd[j] >= 0);
      float z[32];
      float mt0 = -INFINITY, mt1 = -INFINITY;
      const float sl = a.scale_log2;
      // my partial -> the peer's receive slot, pushed with st.async: every
      // store completes its bytes on the peer's x_full[sb], whose expected
      // count (the whole 17 KB tile) one thread of the peer arms.  The
      // partials travel as 16-bit codes with a scale per 32 values (see
      // block_scale_of); both CTAs decode their own partial from the codes too,
      // so they hold bitwise-equal scores.  Slot layout [16-byte chunk
      // k][warpgroup][head], then the scales [warpgroup][head]: a warp's chunk
      // k is 512 contiguous bytes, bank-conflict free; the peer fills mine
      // alike.  The peer's slot sb is written again only after the peer has
      // read tile t-2 from it (its remote arrival on x_free[sb]).
      // My receive slot of tile t-1 has been read (its values went into
      // tile t-1's softmax, which is finished): the peer may push tile t+1
      // into it.  The arrival needs no release fence, which would also wait
      // for this thread's own remote stores (measured ~9 us a launch against
      // ~2 us for this form).
      if (t >= 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive_remote_relaxed(peer_xfree + ((t - 1) & 1) * 8);
      }
      if (g == 0 && quarter == 0 && lane == 0)
        mbar_arrive_expect_tx(&x_full[sb], static_cast<uint32_t>(NH) * 2 * (32 * 2 + 4));
      if (live) {
        if (ok) ok = warp_wait(&s_full[sb], ph, a.err);
        tc_fence_after();
        tmem_ld32(lane_base + S_COL + sb * NR + 32 * g, z);
        tmem_ld_wait();
        // rows that select nothing were gathered as zeros, so their partial
        // scores are exactly 0 and leave amax alone
        float am[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          am[i] = fmaxf(fmaxf(fabsf(z[4 * i]), fabsf(z[4 * i + 1])),
                        fmaxf(fabsf(z[4 * i + 2]), fabsf(z[4 * i + 3])));
        const float amax = fmaxf(fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3])),
                                 fmaxf(fmaxf(am[4], am[5]), fmaxf(am[6], am[7])));
        // |z * qs| <= 32760 (1 + 2^-21): the code never leaves [-32767, 32767]
        const float qs = amax > 0.f ? __fdividef(32760.f, amax) : 0.f;
        uint32_t cw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          z[2 * i] = fmaf(z[2 * i], qs, CODE_BIAS);
          z[2 * i + 1] = fmaf(z[2 * i + 1], qs, CODE_BIAS);
          cw[i] = __byte_perm(__float_as_uint(z[2 * i]), __float_as_uint(z[2 * i + 1]), 0x5410);
        }
        const uint32_t xoff = sb * X_BYTES + (g * DSA_HEADS + h) * 16;
        const uint32_t soff = sb * X_BYTES + X_CODE_BYTES + (g * DSA_HEADS + h) * 4;
        if (ok && t >= 2) ok = warp_wait_cluster(&x_free[sb], ((t >> 1) - 1) & 1, a.err);
        if (ok) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            st_async_v4(peer_x + xoff + k * (2 * DSA_HEADS * 16), __uint_as_float(cw[4 * k]),
                        __uint_as_float(cw[4 * k + 1]), __uint_as_float(cw[4 * k + 2]),
                        __uint_as_float(cw[4 * k + 3]), peer_xfull + sb * 8);
          st_async_b32(peer_x + soff, __float_as_uint(amax), peer_xfull + sb * 8);
        }
        if (ok) ok = warp_wait_cluster(&x_full[sb], ph, a.err);
        uint32_t pw[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 v = *reinterpret_cast<const uint4*>(xb + xoff + k * (2 * DSA_HEADS * 16));
          pw[4 * k] = v.x; pw[4 * k + 1] = v.y; pw[4 * k + 2] = v.z; pw[4 * k + 3] = v.w;
        }
        // z = (S0 + S1) * sl with S_i = code_i * scale_i: both CTAs evaluate
        // fma(c0, k0, c1 * k1), c0 and k0 from rank 0's partial, so they hold
        // bitwise-equal z.  My own codes are still in z as code + CODE_BIAS.
        const float k_own = block_scale_of(amax) * sl;
        const float k_peer = block_scale_of(*reinterpret_cast<const float*>(xb + soff)) * sl;
        if (rank == 0) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            z[2 * i] = fmaf(z[2 * i] - CODE_BIAS, k_own, code_lo(pw[i]) * k_peer);
            z[2 * i + 1] = fmaf(z[2 * i + 1] - CODE_BIAS, k_own, code_hi(pw[i]) * k_peer);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            z[2 * i] = fmaf(code_lo(pw[i]), k_peer, (z[2 * i] - CODE_BIAS) * k_own);
            z[2 * i + 1] = fmaf(code_hi(pw[i]), k_peer, (z[2 * i + 1] - CODE_BIAS) * k_own);
          }
        }
        if (vm != 0xffffffffu) {
#pragma unroll
          for (int r = 0; r < 32; ++r) z[r] = ((vm >> r) & 1u) ? z[r] : -INFINITY;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          mt0 = fmaxf(mt0, fmaxf(z[4 * i + 0], z[4 * i + 1]));
          mt1 = fmaxf(mt1, fmaxf(z[4 * i + 2], z[4 * i + 3]));
        }
      }
      // tile maximum over both warpgroups' rows
      float* mxt = mx + (t & 1) * 2 * DSA_HEADS;
      mxt[g * DSA_HEADS + h] = fmaxf(mt0, mt1);
      named_barrier(1, 32 * SMX_WARPS);
      if (live) {
        const float mt = fmaxf(mxt[h], mxt[DSA_HEADS + h]);
        // running max, moved only when it grows by more than 8 (a factor 2^8);
        // identical in both warpgroups and both CTAs
        float alpha = 1.f;
        bool resc = false;
        if (mt > m_use + 8.f) {
          if (m_use != -INFINITY) {
            alpha = fast_exp2(m_use - mt);
            resc = true;
          }
          m_use = mt;
        }
        const float m_eff = m_use == -INFINITY ? 0.f : m_use;   // exp2(-inf - m_eff) = 0
        float ps0 = 0.f, ps1 = 0.f, ps2 = 0.f, ps3 = 0.f;
#pragma unroll
        for (int r = 0; r < 32; r += 4) {
          z[r + 0] = fast_exp2(z[r + 0] - m_eff);
          z[r + 1] = fast_exp2(z[r + 1] - m_eff);
          z[r + 2] = fast_exp2(z[r + 2] - m_eff);
          z[r + 3] = fast_exp2(z[r + 3] - m_eff);
          ps0 += z[r + 0];
          ps1 += z[r + 1];
          ps2 += z[r + 2];
          ps3 += z[r + 3];
        }
        l = l * alpha + ((ps0 + ps1) + (ps2 + ps3));
        // O is rescaled (rarely: only when the running max moves) after PV(t-1)
        // has finished, which completes phase (t-1)/2 of slot_free[(t-1)&1];
        // PV(t+1) needs P(t+1), so that barrier cannot have moved further.
        // Without a rescale P(t) is published at once, and PV(t-1) runs
        // behind the scores MMA of tile t+1 without holding up the softmax.
        if (g == 0 && __any_sync(0xffffffffu, resc)) {
          if (ok && t >= 1) ok = warp_wait(&slot_free[(t - 1) & 1], ((t - 1) >> 1) & 1, a.err);
          tc_fence_after();
          for (int c = 0; c < 256 / 32; ++c) {
            float o[32];
            tmem_ld32(lane_base + O_COL + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(lane_base + O_COL + c * 32, o);
          }
        }
        // P as fp16 (slot columns [16g, 16g+16)), two rows per column; P
        // <= 2^8 under the lazy maximum, inside fp16's range, with 11
        // significant bits (a single bf16 P cost ~1.6% of rms(O), fp16 ~0.3%)
        float pk[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj)
          pk[jj] = __uint_as_float(f16x2_bits(z[2 * jj], z[2 * jj + 1]));
        tmem_st16(lane_base + S_COL + sb * NR + 16 * g, pk);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    // ---- epilogue: l over both warpgroups, then O / l (warpgroup g writes
    // columns [128g, 128g+128) of this CTA's 256); LSE from CTA 0
    float* lsum = mx;                               // reuse: [2][128]
    named_barrier(1, 32 * SMX_WARPS);
    lsum[g * DSA_HEADS + h] = l;
    named_barrier(1, 32 * SMX_WARPS);
    const float lt = lsum[h] + lsum[DSA_HEADS + h];
    const bool have = ok && live && ntiles > 0 && warp_wait(o_final, 0, a.err);
    if (have) tc_fence_after();
    const float inv = lt > 0.f ? a.out_scale / lt : 0.f;
    // O / l leaves through shared memory: warpgroup g fills four boxes of
    // [128 heads x 32 fp32] (its columns [128g, 128g+128) of this CTA's 256)
    // in the 128-byte swizzle, then one thread stores them with TMA.  The
    // stage ring and the exchange slots are idle once the last PV is done.
    float* lrow = a.S == 1 ? a.lse[layer] + static_cast<size_t>(q) * NH + h
                           : a.l_part + (static_cast<size_t>(gu) * a.S + split) * NH + h;
    const int orow0 = (a.S == 1 ? q : gu * a.S + split) * NH;
    uint8_t* box0 = smem + OFF_ST + g * 4 * OBOX_BYTES;
    // box by box: the TMA store of box c reads shared memory while box c+1
    // is filled
    for (int c = 0; c < 128 / 32; ++c) {
      if (live) {
        float o[32];
        if (have) {
          tmem_ld32(lane_base + O_COL + 128 * g + c * 32, o);
          tmem_ld_wait();
        }
        uint8_t* row = box0 + c * OBOX_BYTES + h * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 w = have && lt > 0.f ? make_float4(o[4 * j] * inv, o[4 * j + 1] * inv,
                                                          o[4 * j + 2] * inv, o[4 * j + 3] * inv)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(row + ((j ^ (h & 7)) << 4)) = w;
        }
      }
      fence_proxy_async_smem();
      named_barrier(2 + g, 128);
      if (gt == 128 * g) {
        tma_store_2d(&maps.o[layer], box0 + c * OBOX_BYTES,
                     static_cast<int>(rank) * 256 + 128 * g + 32 * c, orow0);
        bulk_commit_group();
      }
    }
    // the shared-memory boxes may be released; the grid's end publishes O
    if (gt == 128 * g) bulk_wait_all_read();
    if (rank == 0 && g == 0 && live)
      *lrow = lt > 0.f ? m_use * 0.69314718055994531f + logf(lt) : -INFINITY;
    (void)gt;
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

cudaError_t launch_sparse_mla_layers(const MlaLayerPtrs* layers, int L, int num_pages,
                                     int page_size, int max_pages, const int32_t* q_offsets,
                                     const int32_t* q_vis, const int32_t* idx, int B, int Q, int H,
                                     int topk, float scale, int S, float* o_part, float* l_part,
                                     uint32_t* err, cudaStream_t st, bool pdl,
                                     const int32_t* win_page_table, int win_max_pages,
                                     const int32_t* win_vis, int window, bool kv8, float kv_scale,
                                     int g0, int n_units) {
  if (Q <= 0) return cudaSuccess;
  if (H != 128 && H != 64) return cudaErrorInvalidValue;
  if (L < 1 || L > MAX_LAYERS || S < 1) return cudaErrorInvalidValue;
  if (n_units < 0) n_units = L * Q - g0;
  if (g0 < 0 || n_units <= 0 || g0 + n_units > L * Q) return cudaErrorInvalidValue;
  int page_shift = 0;
  while ((1 << page_shift) < page_size) ++page_shift;
  if (page_size <= 0 || (1 << page_shift) != page_size) return cudaErrorInvalidValue;
  MlaMaps maps;
  for (int l = 0; l < L; ++l) {
    // RoPE query dims: boxes of H heads x 64 bf16 (rows past H in shared
    // memory are never read into a head's result)
    if (!encode_tiled_2d(&maps.q[l], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, layers[l].q, DSA_DIM,
                         static_cast<uint64_t>(Q) * H, DSA_DIM * 2, 64, static_cast<uint32_t>(H)))
      return cudaErrorInvalidValue;
    // output boxes of H heads x 32 fp32 into O [Q, H, 512] (S = 1) or the
    // split partials [n_units, S, H, 512]
    if (!encode_tiled_2d(&maps.o[l], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, S == 1 ? layers[l].out : o_part,
                         DSA_DIM_V, static_cast<uint64_t>(S == 1 ? Q : n_units * S) * H,
                         DSA_DIM_V * 4, 32, static_cast<uint32_t>(H)))
      return cudaErrorInvalidValue;
  }
  for (int l = L; l < MAX_LAYERS; ++l) {
    maps.q[l] = maps.q[0];
    maps.o[l] = maps.o[0];
  }
  // one instance per (head count, cache type)
  auto kernel = H == 128 ? (kv8 ? sparse_mla_tc_kernel<128, true> : sparse_mla_tc_kernel<128, false>)
                         : (kv8 ? sparse_mla_tc_kernel<64, true> : sparse_mla_tc_kernel<64, false>);
  static std::atomic<bool> attr_done[4][64];
  const int inst = (H == 128 ? 0 : 2) + (kv8 ? 1 : 0);
  const cudaError_t ea = set_once_per_device(attr_done[inst], [kernel] {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  if (ea != cudaSuccess) return ea;
  MlaTcArgs a = {};
  for (int l = 0; l < MAX_LAYERS; ++l) {
    const MlaLayerPtrs& y = layers[l < L ? l : 0];
    a.q[l] = y.q;
    a.pool[l] = y.pool;
    a.page_table[l] = y.page_table;
    a.out[l] = y.out;
    a.lse[l] = y.lse;
  }
  a.L = L;
  a.g0 = g0;
  a.max_pages = max_pages;
  a.num_pages = num_pages;
  a.page_shift = page_shift;
  a.win_page_table = win_page_table;
  a.win_max_pages = win_max_pages;
  a.win_vis = win_vis;
  a.window = window;
  a.q_offsets = q_offsets;
  a.q_vis = q_vis;
  a.idx = idx;
  a.B = B;
  a.Q = Q;
  a.topk = topk;
  a.S = S;
  a.scale_log2 = scale * kv_scale * 1.4426950408889634f;
  a.out_scale = kv_scale;
  a.o_part = o_part;
  a.l_part = l_part;
  a.err = err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * n_units * S), 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  unsigned int na = 0;
  add_pdl_attr(attr, &na, pdl);
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, maps, a);
}

cudaError_t launch_sparse_mla_tc(const __nv_bfloat16* q, const __nv_bfloat16* pool, int num_pages,
                                 int page_size, const int32_t* page_table, int max_pages,
                                 const int32_t* q_offsets, const int32_t* q_vis,
                                 const int32_t* idx, int B, int Q, int H, int topk, float scale,
                                 int S, float* out, float* lse, float* o_part, float* l_part,
                                 uint32_t* err, cudaStream_t st, bool pdl,
                                 const int32_t* win_page_table, int win_max_pages,
                                 const int32_t* win_vis, int window, bool kv8, float kv_scale) {
  const MlaLayerPtrs one = {q, pool, page_table, out, lse};
  return launch_sparse_mla_layers(&one, 1, num_pages, page_size, max_pages, q_offsets, q_vis, idx,
                                  B, Q, H, topk, scale, S, o_part, l_part, err, st, pdl,
                                  win_page_table, win_max_pages, win_vis, window, kv8, kv_scale,
                                  0, Q);
}

}  // namespace dsa
