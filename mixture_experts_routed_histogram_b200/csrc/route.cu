// route.cu -- top-k routing, one warp per token.
//
// TileScale PR #70 (distributed FP8 MegaMoE), "Design": the routed MLP starts from
// routing each token to its top-k experts; FlashInfer PR #6465 runs top-k 10 over 512
// experts.  Slot j receives the j-th largest logit, equal logits go to the lower expert
// index.  Weights: softmax over the selected logits (renormalised top-k) or over all E,
// or the sigmoid of the selected logit.
//
// Each lane holds the logits of experts lane, lane+32, ... in registers (E <= 1024), so
// the k selection rounds are a register scan plus a 5-step warp arg-max each.
#include <float.h>
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kRouteWarps = 8;

template <int VPT>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_kernel(const float* __restrict__ logits, int32_t* __restrict__ ids,
                 float* __restrict__ w, int64_t T, int E, int k, int score, int renorm) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + t * E;

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
  int my_id = 0;
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

  float wt;
  if (score == 0) {
    const float m = __shfl_sync(0xffffffffu, my_val, 0);  // slot 0 holds the maximum logit
    float ex = lane < k ? expf(my_val - m) : 0.0f;
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
    wt = ex / den;
  } else {
    float s = lane < k ? 1.0f / (1.0f + expf(-my_val)) : 0.0f;
    if (renorm) {
      float sum = s;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      s = s / sum;
    }
    wt = s;
  }
  if (lane < k) {
    ids[t * k + lane] = my_id;
    w[t * k + lane] = wt;
  }
}

template <int VPT>
cudaError_t launch_vpt(const float* logits, int32_t* ids, float* w, int64_t T, int E, int k,
                       int score, int renorm, cudaStream_t stream) {
  const int64_t blocks = (T + kRouteWarps - 1) / kRouteWarps;
  route_kernel<VPT><<<static_cast<unsigned>(blocks), kRouteWarps * 32, 0, stream>>>(
      logits, ids, w, T, E, k, score, renorm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const float* logits, int32_t* ids, float* w, int64_t T, int E, int k,
                         int score, int renorm, cudaStream_t stream, int* launches) {
  if (T == 0) return cudaSuccess;
  ++*launches;
  const int need = (E + 31) / 32;
  if (need <= 1) return launch_vpt<1>(logits, ids, w, T, E, k, score, renorm, stream);
  if (need <= 2) return launch_vpt<2>(logits, ids, w, T, E, k, score, renorm, stream);
  if (need <= 4) return launch_vpt<4>(logits, ids, w, T, E, k, score, renorm, stream);
  if (need <= 8) return launch_vpt<8>(logits, ids, w, T, E, k, score, renorm, stream);
  if (need <= 16) return launch_vpt<16>(logits, ids, w, T, E, k, score, renorm, stream);
  return launch_vpt<32>(logits, ids, w, T, E, k, score, renorm, stream);
}

}  // namespace moe
