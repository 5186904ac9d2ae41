// route_dev.cuh -- per-token top-k routing by one warp (shared by the routing kernel and
// the fused small-batch routing + permutation kernel).
//
// TileScale PR #70 (distributed FP8 MegaMoE), "Design": each token is routed to its top-k
// experts; FlashInfer PR #6465 runs top-k 10 over 512 experts.  Slot j receives the j-th
// largest logit, equal logits go to the lower expert index.  Weights: softmax over the
// selected logits (renormalised top-k) or over all E, or the sigmoid of the selected logit.
#pragma once

#include <float.h>
#include <limits.h>
#include <math.h>

namespace moe {

// Lane l of the calling warp receives slot l's expert id and weight (for l < k).  Each lane
// holds the logits of experts lane, lane+32, ... (E <= 32*VPT) in registers, so the k
// selection rounds are a register scan plus a 5-step warp arg-max each.
template <int VPT>
__device__ __forceinline__ void route_token_warp(const float* __restrict__ row, int E, int k,
                                                 int score, int renorm, int lane, int& my_id,
                                                 float& my_w) {
  float v[VPT];
  uint32_t taken = 0;  // bit i: expert lane + 32*i already selected or absent
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      v[i] = __ldg(row + e);
    } else {
      v[i] = -FLT_MAX;
      taken |= 1u << i;
    }
  }
  float my_val = 0.0f;
  my_id = 0;
  for (int j = 0; j < k; ++j) {
    // best untaken value of this lane; ascending i means ascending expert index, so a
    // strict comparison keeps the lower index on ties
    float bv = -FLT_MAX;
    int bi = INT_MAX;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      if (!((taken >> i) & 1u) && (bi == INT_MAX || v[i] > bv)) {
        bv = v[i];
        bi = lane + 32 * i;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      const bool better = oi != INT_MAX && (bi == INT_MAX || ov > bv || (ov == bv && oi < bi));
      if (better) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) {
      my_val = bv;
      my_id = bi;
    }
  }
  if (score == 0) {
    const float m = __shfl_sync(0xffffffffu, my_val, 0);  // slot 0 holds the maximum logit
    const float ex = lane < k ? expf(my_val - m) : 0.0f;
    float den;
    if (renorm) {
      den = ex;
    } else {
      den = 0.0f;
#pragma unroll
      for (int i = 0; i < VPT; ++i)
        if (lane + 32 * i < E) den += expf(v[i] - m);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    my_w = ex / den;
  } else {
    float sg = lane < k ? 1.0f / (1.0f + expf(-my_val)) : 0.0f;
    if (renorm) {
      float sum = sg;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      sg = sg / sum;
    }
    my_w = sg;
  }
}

}  // namespace moe
