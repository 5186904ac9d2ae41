// permute.cu -- per-expert histogram, exclusive prefix sum and stable scatter of the
// T*k (token, slot) assignments into an expert-sorted row space.
//
// FlashInfer PR #5129 (cuTile BF16 fused MoE), "sorted I/O": GEMM1 writes its output in
// an expert-sorted row space that GEMM2 then reads contiguously.  TileScale PR #70, first
// listed change: a flat m-task queue replaces a per-tile rescan of the experts; the
// offsets produced here are what the GEMM kernels turn into that queue.
//
// Two launches, both deterministic (no atomics decide an order):
//   1. chunk_hist_kernel: one CTA per chunk of consecutive assignments counts the
//      assignments of each expert in its chunk (shared-memory histogram).
//   2. scatter_kernel:    one CTA per chunk reads every chunk's histogram (a few hundred
//      KB at most, L2-resident), forms offsets[e] = exclusive scan over experts of the
//      totals, and the chunk's starting row for each expert = offsets[e] + the counts of
//      the earlier chunks.  It then walks its chunk in order, 256 assignments per round,
//      ranking equal experts inside a warp with __match_any_sync and across the 8 warps
//      with round-stamped per-warp counts, so the row of assignment a is offsets[e] +
//      #{a' < a : ids[a'] == e}: the stable order.
#include <mutex>

#include "kernels.h"
#include "launch.cuh"
#include "route_dev.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kDefaultChunk = 2048;
constexpr int kMaxChunks = 256;

__global__ void __launch_bounds__(kThreads)
    chunk_hist_kernel(const int32_t* __restrict__ ids, int64_t R, int E, int chunk,
                      int32_t* __restrict__ chunk_counts, int* status) {
  __shared__ int h[kMaxExperts];
  pdl_wait();
  pdl_launch_dependents();
  for (int e = threadIdx.x; e < E; e += kThreads) h[e] = 0;
  __syncthreads();
  const int64_t a0 = static_cast<int64_t>(blockIdx.x) * chunk;
  const int64_t a1 = min(a0 + chunk, R);
  for (int64_t a = a0 + threadIdx.x; a < a1; a += kThreads) {
    const int e = __ldg(ids + a);
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E))
      atomicAdd(&h[e], 1);
    else
      set_status(status, kStatusBadIndex);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads)
    chunk_counts[static_cast<int64_t>(blockIdx.x) * E + e] = h[e];
}

// In-place exclusive scan of s[0..n) (n <= 4 * kThreads) by the whole block; returns
// the total.
__device__ int block_exclusive_scan(int* s, int n, int* warp_sums) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + kThreads - 1) / kThreads;  // <= 4
  const int begin = tid * per;
  int local[4];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = begin + i;
    local[i] = (i < per && idx < n) ? s[idx] : 0;
    sum += local[i];
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  int warp_off = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int v = warp_sums[w];
    if (w < warp) warp_off += v;
    total += v;
  }
  int run = warp_off + incl - sum;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = begin + i;
    if (i < per && idx < n) {
      s[idx] = run;
      run += local[i];
    }
  }
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kThreads)
    scatter_kernel(const int32_t* __restrict__ ids, int64_t R, int E, int chunk, int nchunks,
                   const int32_t* __restrict__ chunk_counts, int32_t* __restrict__ counts,
                   int32_t* __restrict__ offsets, int32_t* __restrict__ row2assign,
                   int32_t* __restrict__ assign2row) {
  __shared__ int cursor[kMaxExperts];
  __shared__ int scan[kMaxExperts];
  __shared__ int wcnt[kWarps][kMaxExperts];
  __shared__ int warp_sums[kWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int me = blockIdx.x;
  pdl_wait();
  pdl_launch_dependents();

  for (int e = tid; e < E; e += kThreads) {
    int before = 0, total = 0;
#pragma unroll 8
    for (int c = 0; c < nchunks; ++c) {
      const int v = __ldg(chunk_counts + static_cast<int64_t>(c) * E + e);
      total += v;
      before += (c < me) ? v : 0;
    }
    cursor[e] = before;
    scan[e] = total;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) wcnt[w][e] = -1;
  }
  __syncthreads();
  const int grand = block_exclusive_scan(scan, E, warp_sums);
  for (int e = tid; e < E; e += kThreads) {
    cursor[e] += scan[e];
    if (me == 0) {
      offsets[e] = scan[e];
      counts[e] = (e + 1 < E ? scan[e + 1] : grand) - scan[e];
    }
  }
  if (me == 0 && tid == 0) offsets[E] = grand;
  __syncthreads();

  const int64_t a0 = static_cast<int64_t>(me) * chunk;
  const int64_t a1 = min(a0 + chunk, R);
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; a0 + static_cast<int64_t>(r) * kThreads < a1; ++r) {
    const int64_t a = a0 + static_cast<int64_t>(r) * kThreads + tid;
    int e = -1;
    if (a < a1) {
      e = __ldg(ids + a);
      if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt);
    const int grp = __popc(peers);
    const bool leader = (__ffs(peers) - 1) == lane;
    if (e >= 0 && leader) wcnt[warp][e] = (r << 8) | grp;
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int w = 0; w < warp; ++w) {
        const int v = wcnt[w][e];
        if ((v >> 8) == r) before += v & 255;
      }
      const int row = cursor[e] + before + rank;
      row2assign[row] = static_cast<int32_t>(a);
      assign2row[a] = row;
    }
    __syncthreads();
    if (e >= 0 && leader) atomicAdd(&cursor[e], grp);
  }
}

int chunk_size(int64_t R) {
  int64_t c = kDefaultChunk;
  if ((R + c - 1) / c > kMaxChunks) {
    c = (R + kMaxChunks - 1) / kMaxChunks;
    c = (c + kThreads - 1) / kThreads * kThreads;
  }
  return static_cast<int>(c);
}

}  // namespace

size_t permute_scratch_bytes(int64_t R, int E) {
  const int64_t c = chunk_size(R);
  const int64_t n = R > 0 ? (R + c - 1) / c : 1;
  return static_cast<size_t>(n) * E * sizeof(int32_t);
}

cudaError_t launch_permute(const int32_t* ids, int64_t R, int E, int32_t* counts,
                           int32_t* offsets, int32_t* row2assign, int32_t* assign2row,
                           int32_t* scratch, int* status, cudaStream_t stream, int* launches) {
  if (R == 0) {
    ++*launches;
    cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), stream);
    return cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream);
  }
  const int chunk = chunk_size(R);
  const int nchunks = static_cast<int>((R + chunk - 1) / chunk);
  *launches += 2;
  cudaError_t e = launch_k(chunk_hist_kernel, dim3(nchunks), dim3(kThreads), 0, stream, ids, R, E,
                           chunk, scratch, status);
  if (e != cudaSuccess) return e;
  return launch_k(scatter_kernel, dim3(nchunks), dim3(kThreads), 0, stream, ids, R, E, chunk,
                  nchunks, static_cast<const int32_t*>(scratch), counts, offsets, row2assign,
                  assign2row);
}

// ---------------------------------------------------------------- small batches, one launch
//
// For decode-sized batches (T <= 64, E <= 256) the whole front end runs in one CTA of 1024
// threads: warps route the tokens (route_token_warp), the ids stay in shared memory, a
// shared-memory histogram and one exclusive scan give counts/offsets, and the stable
// scatter walks the assignments in rounds of 1024 with the same warp-match + round-stamp
// ranking as scatter_kernel.  It replaces three launches on the latency-bound decode path.

constexpr int kSmallMaxT = 64;
constexpr int kSmallMaxE = 256;
constexpr int kSmallThreads = 1024;
constexpr int kSmallWarps = kSmallThreads / 32;

namespace {

template <int VPT>
__global__ void __launch_bounds__(kSmallThreads)
    route_permute_small_kernel(const float* __restrict__ logits, int T, int E, int k, int score,
                               int renorm, int32_t* __restrict__ ids, float* __restrict__ w,
                               int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                               int32_t* __restrict__ row2assign,
                               int32_t* __restrict__ assign2row) {
  __shared__ int s_ids[kSmallMaxT * kMaxTopK];
  __shared__ int scan[kSmallMaxE];
  __shared__ int cursor[kSmallMaxE];
  __shared__ int wcnt[kSmallWarps][kSmallMaxE];
  __shared__ int warp_sums[kSmallWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = T * k;
  pdl_wait();
  pdl_launch_dependents();

  for (int t = warp; t < T; t += kSmallWarps) {
    int id;
    float wt;
    route_token_warp<VPT>(logits + static_cast<int64_t>(t) * E, E, k, score, renorm, lane, id,
                          wt);
    if (lane < k) {
      ids[t * k + lane] = id;
      w[t * k + lane] = wt;
      s_ids[t * k + lane] = id;
    }
  }
  for (int e = tid; e < E; e += kSmallThreads) {
    scan[e] = 0;
#pragma unroll 4
    for (int ww = 0; ww < kSmallWarps; ++ww) wcnt[ww][e] = -1;
  }
  __syncthreads();
  for (int a = tid; a < R; a += kSmallThreads) atomicAdd(&scan[s_ids[a]], 1);
  __syncthreads();
  // exclusive scan of the E counts: one per thread, warp scans, then the warp totals
  const int cnt = tid < E ? scan[tid] : 0;
  int incl = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int ww = 0; ww < warp; ++ww) before += warp_sums[ww];
  const int excl = before + incl - cnt;
  if (tid < E) {
    cursor[tid] = excl;
    offsets[tid] = excl;
    counts[tid] = cnt;
  }
  if (tid == 0) offsets[E] = R;
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; r * kSmallThreads < R; ++r) {
    const int a = r * kSmallThreads + tid;
    const int e = a < R ? s_ids[a] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt);
    const int grp = __popc(peers);
    const bool leader = (__ffs(peers) - 1) == lane;
    if (e >= 0 && leader) wcnt[warp][e] = (r << 8) | grp;
    __syncthreads();
    if (e >= 0) {
      int bw = 0;
      for (int ww = 0; ww < warp; ++ww) {
        const int v = wcnt[ww][e];
        if ((v >> 8) == r) bw += v & 255;
      }
      const int row = cursor[e] + bw + rank;
      row2assign[row] = a;
      assign2row[a] = row;
    }
    __syncthreads();
    if (e >= 0 && leader) atomicAdd(&cursor[e], grp);
  }
}

template <int VPT>
cudaError_t launch_small(const float* logits, int T, int E, int k, int score, int renorm,
                         int32_t* ids, float* w, int32_t* counts, int32_t* offsets,
                         int32_t* row2assign, int32_t* assign2row, cudaStream_t stream) {
  return launch_k(route_permute_small_kernel<VPT>, dim3(1), dim3(kSmallThreads), 0, stream, logits,
                  T, E, k, score, renorm, ids, w, counts, offsets, row2assign, assign2row);
}

}  // namespace

bool use_route_permute_small(int64_t T, int E, int k) {
  return T > 0 && T <= kSmallMaxT && E <= kSmallMaxE && k <= kMaxTopK;
}

cudaError_t launch_route_permute_small(const float* logits, int64_t T, int E, int k, int score,
                                       int renorm, int32_t* ids, float* w, int32_t* counts,
                                       int32_t* offsets, int32_t* row2assign,
                                       int32_t* assign2row, cudaStream_t stream, int* launches) {
  ++*launches;
  const int t = static_cast<int>(T);
  const int need = (E + 31) / 32;
  if (need <= 1)
    return launch_small<1>(logits, t, E, k, score, renorm, ids, w, counts, offsets, row2assign,
                           assign2row, stream);
  if (need <= 2)
    return launch_small<2>(logits, t, E, k, score, renorm, ids, w, counts, offsets, row2assign,
                           assign2row, stream);
  if (need <= 4)
    return launch_small<4>(logits, t, E, k, score, renorm, ids, w, counts, offsets, row2assign,
                           assign2row, stream);
  return launch_small<8>(logits, t, E, k, score, renorm, ids, w, counts, offsets, row2assign,
                         assign2row, stream);
}

// ---------------------------------------------------------------- allocation-free variant
//
// For callers that cannot hand the library a workspace: the per-chunk histograms live in
// this file-scope device array instead (256 KB, held on every device that loads the
// library until the process exits).  Every call shares it, so two calls whose kernels
// overlap on the GPU (different streams, or different host threads) race on it; calls
// serialised on one stream are safe.  The histogram kernel overwrites every entry a call
// reads, so nothing has to be cleared between calls.

constexpr int kNoAllocScratchInts = 1 << 16;
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchInts];

namespace {
std::mutex g_noalloc_mu;
constexpr int kMaxDevices = 64;
int32_t* g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

// Device address of g_noalloc_scratch on the current device.  In host code the array's
// name is only a host-side stand-in, so the address is looked up once per device (with
// that device current) and cached.
static cudaError_t noalloc_scratch(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

bool permute_noalloc_fits(int64_t R, int E) {
  if (R == 0) return true;
  const int64_t c = chunk_size(R);
  const int64_t n = (R + c - 1) / c;
  return n * E <= kNoAllocScratchInts;
}

cudaError_t launch_permute_noalloc(const int32_t* ids, int64_t R, int E, int32_t* counts,
                                   int32_t* offsets, int32_t* row2assign, int32_t* assign2row,
                                   cudaStream_t stream, int* launches) {
  if (R == 0) {
    ++*launches;
    cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), stream);
    return cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream);
  }
  int32_t* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  const int chunk = chunk_size(R);
  const int nchunks = static_cast<int>((R + chunk - 1) / chunk);
  *launches += 2;
  chunk_hist_kernel<<<nchunks, kThreads, 0, stream>>>(ids, R, E, chunk, scratch, nullptr);
  scatter_kernel<<<nchunks, kThreads, 0, stream>>>(ids, R, E, chunk, nchunks, scratch, counts,
                                                   offsets, row2assign, assign2row);
  return cudaGetLastError();
}

}  // namespace moe
