// route.cu -- top-k routing, one warp per token (the per-token work is route_token_warp in
// route_dev.cuh: TileScale PR #70 "Design" routing, FlashInfer PR #6465 top-k 10).
#include "kernels.h"
#include "launch.cuh"
#include "route_dev.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kRouteWarps = 8;

template <int VPT>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_kernel(const float* __restrict__ logits, int32_t* __restrict__ ids,
                 float* __restrict__ w, int64_t T, int E, int k, int ns, int score, int renorm) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteWarps + (threadIdx.x >> 5);
  pdl_wait();
  pdl_launch_dependents();
  if (t >= T) return;
  int id;
  float wt;
  route_token_warp<VPT>(logits + t * E, E, k, score, renorm, lane, id, wt);
  const int ks = k + ns;  // slots per token: the top-k, then the shared experts
  if (lane < k) {
    ids[t * ks + lane] = id;
    w[t * ks + lane] = wt;
  } else if (lane < ks) {
    ids[t * ks + lane] = E + (lane - k);
    w[t * ks + lane] = 1.0f;
  }
}

template <int VPT>
cudaError_t launch_vpt(const float* logits, int32_t* ids, float* w, int64_t T, int E, int k,
                       int ns, int score, int renorm, cudaStream_t stream) {
  const int64_t blocks = (T + kRouteWarps - 1) / kRouteWarps;
  return launch_k(route_kernel<VPT>, dim3(static_cast<unsigned>(blocks)), dim3(kRouteWarps * 32), 0,
                  stream, logits, ids, w, T, E, k, ns, score, renorm);
}

}  // namespace

cudaError_t launch_route(const float* logits, int32_t* ids, float* w, int64_t T, int E, int k,
                         int ns, int score, int renorm, cudaStream_t stream, int* launches) {
  if (T == 0) return cudaSuccess;
  ++*launches;
  const int need = (E + 31) / 32;
  if (need <= 1) return launch_vpt<1>(logits, ids, w, T, E, k, ns, score, renorm, stream);
  if (need <= 2) return launch_vpt<2>(logits, ids, w, T, E, k, ns, score, renorm, stream);
  if (need <= 4) return launch_vpt<4>(logits, ids, w, T, E, k, ns, score, renorm, stream);
  if (need <= 8) return launch_vpt<8>(logits, ids, w, T, E, k, ns, score, renorm, stream);
  if (need <= 16) return launch_vpt<16>(logits, ids, w, T, E, k, ns, score, renorm, stream);
  return launch_vpt<32>(logits, ids, w, T, E, k, ns, score, renorm, stream);
}

}  // namespace moe
