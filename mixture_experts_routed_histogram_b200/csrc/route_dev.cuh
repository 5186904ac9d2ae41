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

// Order-preserving map of a float onto uint32 (a < b  <=>  key(a) < key(b)); -0 is folded
// onto +0 first so that equal values get equal keys.  Every real logit, -inf included, has a
// key above 0, which marks "taken or absent".
__device__ __forceinline__ uint32_t route_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float route_key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Lane l of the calling warp receives slot l's expert id and weight (for l < k).  Each lane
// holds the logits of experts lane, lane+32, ... (E <= 32*VPT) in registers.  A selection
// round is a register scan for the lane's best untaken key, one warp max-reduction of the
// keys and one min-reduction of the expert indices that reach that maximum, so equal logits
// go to the lower expert index.
template <int VPT>
__device__ __forceinline__ void route_token_warp(const float* __restrict__ row, int E, int k,
                                                 int score, int renorm, int lane, int& my_id,
                                                 float& my_w) {
  float v[VPT];
  uint32_t key[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldg(row + e) : -FLT_MAX;
    key[i] = e < E ? route_key(v[i]) : 0u;
  }
  float my_val = 0.0f;
  my_id = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0u;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      if (key[i] > bk) {  // strict: the lower i (lower expert index) keeps a tie
        bk = key[i];
        bi = i;
      }
    }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t cand = bk == m ? static_cast<uint32_t>(lane + 32 * bi) : 0xffffffffu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
    if (static_cast<int>(win & 31u) == lane) {
#pragma unroll
      for (int i = 0; i < VPT; ++i)
        if (i == static_cast<int>(win >> 5)) key[i] = 0u;
    }
    if (lane == j) {
      my_val = route_key_value(m);
      my_id = static_cast<int>(win);
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
