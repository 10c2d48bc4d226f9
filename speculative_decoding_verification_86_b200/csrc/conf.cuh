// Confidence head ("Speculative decoding becomes standard: DSpark and
// multi-token drafters", section "What DSpark adds"): a linear projection with
// a sigmoid estimates, for each drafted position, the probability that its
// token survives verification given that the earlier ones did.  The chance
// that the first j positions all survive is the prefix product; the request's
// budget is the number of leading positions whose prefix product stays at or
// above the threshold.
//
// One CTA per request, one warp per position: the bf16 x bf16 products are
// exact in fp32 and are summed in fp64, so the budget decision is made on an
// fp64 prefix product.
#pragma once
#include "common.cuh"

namespace sv {

__global__ void __launch_bounds__(kThreads) k_conf(ConfParams cp) {
  __shared__ double s_surv[kMaxK];
  const int i = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = warp; j < cp.kb; j += kWarps) {
    const uint16_t* h = cp.hidden + (static_cast<int64_t>(i) * cp.kb + j) * cp.H;
    double z = 0.0;
    for (int c = lane; c < cp.H; c += 32) {
      const float wf = __uint_as_float(static_cast<uint32_t>(__ldg(cp.w + c)) << 16);
      const float hf = __uint_as_float(static_cast<uint32_t>(__ldg(h + c)) << 16);
      z += static_cast<double>(wf * hf);
    }
    z = warp_sum_d(z);
    if (lane == 0) s_surv[j] = 1.0 / (1.0 + exp(-(z + static_cast<double>(cp.bias))));
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double prefix = 1.0;
    int budget = 0;
    bool counting = true;
    for (int j = 0; j < cp.kb; ++j) {
      prefix *= s_surv[j];
      if (counting && prefix >= static_cast<double>(cp.threshold)) ++budget;
      else counting = false;
      if (cp.out_survival) cp.out_survival[static_cast<int64_t>(i) * cp.kb + j] = static_cast<float>(s_surv[j]);
    }
    cp.out_len[i] = budget;
  }
}

}  // namespace sv
