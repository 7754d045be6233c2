// Split-K merge of partial attentions by log-sum-exp:
//   LSE = ln sum_c exp(LSE_c),  O = sum_c exp(LSE_c - LSE) O_c,
// parts with LSE_c = -inf (no selected token) get weight 0; if every part is
// empty O = 0 and LSE = -inf.  H heads per query (128, or GLM-5.2's 64).
// One CTA of 256 threads per (query, 8 heads, part of the 512 outputs): a
// warp per head; the split weights are recomputed by every thread from the S
// partial LSEs (L1-resident).  With few queries the outputs are cut into 2 or
// 4 parts (grid.y) so that the grid still covers the SMs: 4 queries x 64
// heads were 32 CTAs, each reading 16 partials of 8 x 512 floats.  One CTA per
// head (4096 CTAs of 128 threads for 32 queries) spent its time in CTA
// scheduling.
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int HEADS_PER_CTA = 8;               // 8 heads x 512 outputs, 16 per thread
constexpr int CTHREADS = HEADS_PER_CTA * DSA_DIM_V / 16;
constexpr int MAX_OUT = MLA_MAX_LAYERS_PER_LAUNCH;

// Partial row i (of n) belongs to unit gi = g0 + i, i.e. query gi % Q of the
// output layer gi / Q (a single output: g0 = 0, Q = n).
struct CombineArgs {
  const float* o_part;
  const float* l_part;
  int S, H, g0, Q;
  float* out[MAX_OUT];
  float* lse[MAX_OUT];
};

__global__ void __launch_bounds__(CTHREADS) lse_combine_kernel(const __grid_constant__ CombineArgs a) {
  pdl_trigger();
  pdl_wait();                                   // the partials come from the previous kernel
  // CTA: partial unit i, heads [h0, h0 + 8), 128-float quarters [k0, k1) of
  // the 512 outputs; thread: head h0 + tid / 32, float4 column tid % 32 of
  // each quarter
  const int S = a.S, H = a.H;
  const int k0 = blockIdx.y * 4 / gridDim.y, k1 = (blockIdx.y + 1) * 4 / gridDim.y;
  const int i = blockIdx.x / (H / HEADS_PER_CTA);
  const int h = (blockIdx.x % (H / HEADS_PER_CTA)) * HEADS_PER_CTA + (threadIdx.x >> 5);
  const int c4 = threadIdx.x & 31;              // float4 column within each 128-float quarter
  const int gi = a.g0 + i;
  const int layer = gi / a.Q;
  const size_t qh = static_cast<size_t>(gi % a.Q) * H + h;
  float* const out = a.out[layer];
  float* const lse = a.lse[layer];
  const float* lp = a.l_part + static_cast<size_t>(i) * S * H + h;
  float m = -INFINITY;
  for (int c = 0; c < S; ++c) m = fmaxf(m, lp[static_cast<size_t>(c) * H]);
  float4* o = reinterpret_cast<float4*>(out + qh * DSA_DIM_V) + c4;
  if (m == -INFINITY) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k >= k0 && k < k1) o[32 * k] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c4 == 0 && blockIdx.y == 0) lse[qh] = -INFINITY;
    return;
  }
  float tot = 0.f;
  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int c = 0; c < S; ++c) {
    const float lc = lp[static_cast<size_t>(c) * H];
    if (lc == -INFINITY) continue;
    const float wc = expf(lc - m);
    tot += wc;
    const float4* v = reinterpret_cast<const float4*>(
                          a.o_part + ((static_cast<size_t>(i) * S + c) * H + h) * DSA_DIM_V) + c4;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k < k0 || k >= k1) continue;
      const float4 x = v[32 * k];
      acc[k].x = fmaf(wc, x.x, acc[k].x);
      acc[k].y = fmaf(wc, x.y, acc[k].y);
      acc[k].z = fmaf(wc, x.z, acc[k].z);
      acc[k].w = fmaf(wc, x.w, acc[k].w);
    }
  }
  const float inv = 1.f / tot;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (k >= k0 && k < k1)
      o[32 * k] = make_float4(acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv);
  if (c4 == 0 && blockIdx.y == 0) lse[qh] = m + logf(tot);
}

}  // namespace

namespace {

cudaError_t launch_combine_args(const CombineArgs& args, int n, cudaStream_t st, bool pdl) {
  if (n <= 0) return cudaSuccess;
  const int H = args.H;
  if (H <= 0 || H % HEADS_PER_CTA) return cudaErrorInvalidValue;
  // cut the 512 outputs into parts until the grid covers twice the SMs
  const int ctas = n * (H / HEADS_PER_CTA);
  const int sms = device_sm_count();
  const int parts = ctas >= 2 * sms ? 1 : (2 * ctas >= 2 * sms ? 2 : 4);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas), static_cast<unsigned>(parts), 1);
  cfg.blockDim = dim3(CTHREADS, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  unsigned int na = 0;
  add_pdl_attr(attr, &na, pdl);
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, lse_combine_kernel, args);
}

}  // namespace

cudaError_t launch_combine(const float* o_part, const float* l_part, int Q, int S, int H,
                           float* out, float* lse, cudaStream_t st, bool pdl) {
  CombineArgs args = {};
  args.o_part = o_part;
  args.l_part = l_part;
  args.S = S;
  args.H = H;
  args.g0 = 0;
  args.Q = Q > 0 ? Q : 1;
  for (int l = 0; l < MAX_OUT; ++l) {
    args.out[l] = out;
    args.lse[l] = lse;
  }
  return launch_combine_args(args, Q, st, pdl);
}

cudaError_t launch_combine_layers(const float* o_part, const float* l_part, int n_units, int S,
                                  int H, int g0, int Q, const MlaLayerPtrs* layers, int L,
                                  cudaStream_t st, bool pdl) {
  if (L < 1 || L > MAX_OUT || Q <= 0 || g0 < 0 || g0 + n_units > L * Q)
    return cudaErrorInvalidValue;
  CombineArgs args = {};
  args.o_part = o_part;
  args.l_part = l_part;
  args.S = S;
  args.H = H;
  args.g0 = g0;
  args.Q = Q;
  for (int l = 0; l < MAX_OUT; ++l) {
    args.out[l] = layers[l < L ? l : 0].out;
    args.lse[l] = layers[l < L ? l : 0].lse;
  }
  return launch_combine_args(args, n_units, st, pdl);
}

}  // namespace dsa
