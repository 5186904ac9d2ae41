// combine_quant.cu -- the HBM-bound elementwise stages: top-k weighted combine, the 1x128
// e4m3 activation quantiser and the MXFP4 weight preparation.
//
// Combine: TileScale PR #70 (distributed FP8 MegaMoE), kernel 2 "L2 + scatter + reduce":
// the expert outputs of a token's k slots are summed with their routing weights in a
// fixed slot order.  Here the k rows are read from the expert-sorted y through
// assign2row (FlashInfer PR #5129, sorted I/O: the combine itself is unchanged).
//
// Activation quantiser: TileScale PR #70, "Design": FP8 E4M3 with fp32 scales per 128
// elements; the scale is the smallest power of two keeping the group's amax within 448
// (so it is also an exact UE8M0 value for the block-scaled MMA).
//
// Weight preparation: FlashInfer PR #6465, MXFP4 weights with K32 UE8M0 scaling; the
// scale follows the OCP MX rule 2^(floor(log2 amax) - 2).
#include <algorithm>

#include "kernels.h"
#include "launch.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const uint16_t* __restrict__ y, const float* __restrict__ w,
                   const int32_t* __restrict__ assign2row, uint16_t* __restrict__ out, int H,
                   int k) {
  __shared__ float sw[kMaxTopK];
  __shared__ int64_t srow[kMaxTopK];
  const int64_t t = blockIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x < k) {
    sw[threadIdx.x] = __ldg(w + t * k + threadIdx.x);
    srow[threadIdx.x] = static_cast<int64_t>(__ldg(assign2row + t * k + threadIdx.x)) * H;
  }
  __syncthreads();
  for (int c = threadIdx.x * 8; c < H; c += kCombineThreads * 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll 4
    for (int j = 0; j < k; ++j) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(y + srow[j] + c));
      const float wj = sw[j];
      acc[0] = fmaf(wj, bf16_lo(v.x), acc[0]);
      acc[1] = fmaf(wj, bf16_hi(v.x), acc[1]);
      acc[2] = fmaf(wj, bf16_lo(v.y), acc[2]);
      acc[3] = fmaf(wj, bf16_hi(v.y), acc[3]);
      acc[4] = fmaf(wj, bf16_lo(v.z), acc[4]);
      acc[5] = fmaf(wj, bf16_hi(v.z), acc[5]);
      acc[6] = fmaf(wj, bf16_lo(v.w), acc[6]);
      acc[7] = fmaf(wj, bf16_hi(v.w), acc[7]);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(out + t * H + c) = o;
  }
}

// The combine when GEMM2 split K: the k rows' partial sums are added slice by slice (in
// slice order) before the routing weights are applied (slot order), all in fp32.  Decode
// batches are a few tokens, so each token's columns are spread over blockIdx.y (one 4-column
// chunk per thread) and a slot's slice loads are all issued before the first add.
__global__ void __launch_bounds__(kCombineThreads)
    combine_parts_kernel(const float* __restrict__ part, const int* __restrict__ splits_dev,
                         int64_t R, const float* __restrict__ w,
                         const int32_t* __restrict__ assign2row,
                         uint16_t* __restrict__ out, int H, int k) {
  __shared__ float sw[kMaxTopK];
  __shared__ int64_t srow[kMaxTopK];
  const int64_t t = blockIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x < k) {
    sw[threadIdx.x] = __ldg(w + t * k + threadIdx.x);
    srow[threadIdx.x] = static_cast<int64_t>(__ldg(assign2row + t * k + threadIdx.x)) * H;
  }
  __syncthreads();
  const int splits = *splits_dev;  // written by the GEMM2 this kernel follows
  const int64_t slice = R * H;
  const int c = (blockIdx.y * kCombineThreads + threadIdx.x) * 4;
  if (c < H) {
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int j = 0; j < k; ++j) {
      float4 v[kMaxSplits];
#pragma unroll
      for (int s = 0; s < kMaxSplits; ++s)
        if (s < splits)
          v[s] = __ldcs(reinterpret_cast<const float4*>(part + s * slice + srow[j] + c));
      float y[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int s = 0; s < kMaxSplits; ++s) {
        if (s < splits) {
          y[0] += v[s].x; y[1] += v[s].y; y[2] += v[s].z; y[3] += v[s].w;
        }
      }
      const float wj = sw[j];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(wj, y[i], acc[i]);
    }
    uint2 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    *reinterpret_cast<uint2*>(out + t * H + c) = o;
  }
}

// Two (token, 128-column group)s per warp iteration, one per half-warp; each lane owns 8
// consecutive columns (one 16-byte load, one 8-byte store).  Warps stride over the groups
// so that a few thousand CTAs cover any T.
__global__ void __launch_bounds__(256)
    quant_x_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ xq,
                   float* __restrict__ sx, uint32_t* __restrict__ sxw, int64_t groups, int H) {
  const int lane = threadIdx.x & 31;
  const int hl = lane & 15;
  pdl_wait();
  pdl_launch_dependents();
  const int G = H / 128;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); w * 2 < groups;
       w += nwarps) {  // warp-uniform condition: both halves stay in the loop together
    const int64_t gid = w * 2 + (lane >> 4);
    const bool ok = gid < groups;
    const int64_t t = gid / G;
    const int g = static_cast<int>(gid - t * G);
    const int64_t base = t * H + g * 128 + hl * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (ok) v = __ldg(reinterpret_cast<const uint4*>(x + base));
    const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
    for (int off = 8; off > 0; off >>= 1)  // within the half-warp
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const int sc = fp8_scale_exponent(amax);
    const float inv = pow2f(-sc);
    uint2 q;
    q.x = static_cast<uint32_t>(cvt_e4m3x2(f[0] * inv, f[1] * inv)) |
          (static_cast<uint32_t>(cvt_e4m3x2(f[2] * inv, f[3] * inv)) << 16);
    q.y = static_cast<uint32_t>(cvt_e4m3x2(f[4] * inv, f[5] * inv)) |
          (static_cast<uint32_t>(cvt_e4m3x2(f[6] * inv, f[7] * inv)) << 16);
    if (ok) {
      *reinterpret_cast<uint2*>(xq + base) = q;
      if (hl == 0) {
        sx[t * G + g] = pow2f(sc);
        if (sxw) sxw[t * G + g] = static_cast<uint32_t>(sc + 127) * 0x01010101u;
      }
    }
  }
}

// One thread per (row, 32-element group).
__global__ void __launch_bounds__(256)
    quant_w_kernel(const uint16_t* __restrict__ w, uint8_t* __restrict__ packed,
                   uint8_t* __restrict__ sf, int64_t groups, int K) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (gid >= groups) return;
  const int G = K / 32;
  const int64_t r = gid / G;
  const int g = static_cast<int>(gid % G);
  const uint4* src = reinterpret_cast<const uint4*>(w + r * K + g * 32);
  float f[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = __ldg(src + q);
    f[8 * q + 0] = bf16_lo(v.x); f[8 * q + 1] = bf16_hi(v.x);
    f[8 * q + 2] = bf16_lo(v.y); f[8 * q + 3] = bf16_hi(v.y);
    f[8 * q + 4] = bf16_lo(v.z); f[8 * q + 5] = bf16_hi(v.z);
    f[8 * q + 6] = bf16_lo(v.w); f[8 * q + 7] = bf16_hi(v.w);
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(f[i]));
  int byte = 0;
  if (amax > 0.0f) {
    int e;
    frexpf(amax, &e);            // amax = m * 2^e, m in [0.5, 1): floor(log2 amax) = e - 1
    byte = (e - 1) - 2 + 127;
    byte = byte < 0 ? 0 : (byte > 254 ? 254 : byte);
  }
  const float inv = pow2f(127 - byte);
  uint32_t words[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t wv = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int i = 8 * q + 2 * b;
      wv |= cvt_e2m1x2(f[i] * inv, f[i + 1] * inv) << (8 * b);
    }
    words[q] = wv;
  }
  *reinterpret_cast<uint4*>(packed + r * (K / 2) + g * 16) =
      make_uint4(words[0], words[1], words[2], words[3]);
  sf[r * G + g] = static_cast<uint8_t>(byte);
}

}  // namespace

cudaError_t launch_combine(const uint16_t* y, const float* w, const int32_t* assign2row,
                           uint16_t* out, int64_t T, int H, int k, cudaStream_t stream,
                           int* launches) {
  if (T == 0) return cudaSuccess;
  ++*launches;
  return launch_k(combine_kernel, dim3(static_cast<unsigned>(T)), dim3(kCombineThreads), 0, stream,
                  y, w, assign2row, out, H, k);
}

cudaError_t launch_combine_parts(const float* part, const int* splits, int64_t R, const float* w,
                                 const int32_t* assign2row, uint16_t* out, int64_t T, int H,
                                 int k, cudaStream_t stream, int* launches) {
  if (T == 0) return cudaSuccess;
  ++*launches;
  const unsigned cblocks =
      static_cast<unsigned>((H + 4 * kCombineThreads - 1) / (4 * kCombineThreads));
  return launch_k(combine_parts_kernel, dim3(static_cast<unsigned>(T), cblocks),
                  dim3(kCombineThreads), 0, stream, part, splits, R, w, assign2row, out, H, k);
}

cudaError_t launch_quant_x(const uint16_t* x, uint8_t* xq, float* sx, uint32_t* sxw, int64_t T,
                           int H, cudaStream_t stream, int* launches) {
  const int64_t groups = T * (H / 128);
  if (groups == 0) return cudaSuccess;
  ++*launches;
  const int64_t blocks = std::min<int64_t>((groups + 15) / 16, 16 * num_sms());
  return launch_k(quant_x_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, x, xq,
                  sx, sxw, groups, H);
}

cudaError_t launch_quant_w_mxfp4(const uint16_t* w, uint8_t* packed, uint8_t* sf, int64_t rows,
                                 int K, cudaStream_t stream, int* launches) {
  const int64_t groups = rows * (K / 32);
  if (groups == 0) return cudaSuccess;
  ++*launches;
  quant_w_kernel<<<static_cast<unsigned>((groups + 255) / 256), 256, 0, stream>>>(w, packed, sf,
                                                                                groups, K);
  return cudaGetLastError();
}

}  // namespace moe
