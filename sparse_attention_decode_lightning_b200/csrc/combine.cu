// Split-K merge of partial attentions by log-sum-exp:
//   LSE = ln sum_c exp(LSE_c),  O = sum_c exp(LSE_c - LSE) O_c,
// parts with LSE_c = -inf (no selected token) get weight 0; if every part is
// empty O = 0 and LSE = -inf.  One CTA of 128 threads per (query, head): the
// 512 outputs are one float4 per thread, the split weights are recomputed by
// every thread from the S partial LSEs (S <= 32, L1-resident).
#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

__global__ void __launch_bounds__(128) lse_combine_kernel(const float* __restrict__ o_part,
                                                          const float* __restrict__ l_part,
                                                          int S, float* __restrict__ out,
                                                          float* __restrict__ lse) {
  pdl_trigger();
  pdl_wait();                                   // the partials come from the previous kernel
  const int qh = blockIdx.x;                    // q * 128 + h
  const int q = qh / DSA_HEADS, h = qh % DSA_HEADS;
  const float* lp = l_part + static_cast<size_t>(q) * S * DSA_HEADS + h;
  float m = -INFINITY;
  for (int c = 0; c < S; ++c) m = fmaxf(m, lp[static_cast<size_t>(c) * DSA_HEADS]);
  float4* o = reinterpret_cast<float4*>(out + static_cast<size_t>(qh) * DSA_DIM_V) + threadIdx.x;
  if (m == -INFINITY) {
    *o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (threadIdx.x == 0) lse[qh] = -INFINITY;
    return;
  }
  float tot = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c = 0; c < S; ++c) {
    const float lc = lp[static_cast<size_t>(c) * DSA_HEADS];
    if (lc == -INFINITY) continue;
    const float wc = expf(lc - m);
    tot += wc;
    const float4 v = reinterpret_cast<const float4*>(
        o_part + ((static_cast<size_t>(q) * S + c) * DSA_HEADS + h) * DSA_DIM_V)[threadIdx.x];
    acc.x = fmaf(wc, v.x, acc.x);
    acc.y = fmaf(wc, v.y, acc.y);
    acc.z = fmaf(wc, v.z, acc.z);
    acc.w = fmaf(wc, v.w, acc.w);
  }
  const float inv = 1.f / tot;
  *o = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (threadIdx.x == 0) lse[qh] = m + logf(tot);
}

}  // namespace

cudaError_t launch_combine(const float* o_part, const float* l_part, int Q, int S, float* out,
                           float* lse, cudaStream_t st, bool pdl) {
  if (Q <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(Q) * DSA_HEADS, 1, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  unsigned int na = 0;
  add_pdl_attr(attr, &na, pdl);
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, lse_combine_kernel, o_part, l_part, S, out, lse);
}

}  // namespace dsa
