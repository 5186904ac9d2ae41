// permute.cu -- per-expert histogram, exclusive prefix sum and stable scatter of the
// T*k (token, slot) assignments into an expert-sorted row space.
//
// FlashInfer PR #5129 (cuTile BF16 fused MoE), "sorted I/O": GEMM1 writes its output in
// an expert-sorted row space that GEMM2 then reads contiguously.  TileScale PR #70, first
// listed change: a flat m-task queue replaces a per-tile rescan of the experts; the
// offsets produced here are what the GEMM kernels turn into that queue.
//
// Three launches, all deterministic (no atomics decide an order).  Chunks are 64 tokens'
// assignments (larger once there would be more than 128 chunks), so each launch has one CTA
// per chunk or per expert and every SM has work at T = 8192:
//   1. chunk_hist_kernel: one CTA per chunk counts the assignments of each expert in its
//      chunk (shared-memory histogram) into cc[e][chunk].
//   2. chunk_scan_kernel: one CTA per expert scans its row of cc over the chunks:
//      base[e][chunk] = the expert's assignments in earlier chunks, tot[e] = all of them.
//   3. scatter_kernel:    one CTA per chunk forms offsets[e] = exclusive scan over experts of
//      tot, so the chunk's first row for expert e is offsets[e] + base[e][chunk].  It then
//      walks its chunk in order, 256 assignments per round, ranking equal experts inside a
//      warp with __match_any_sync and across the 8 warps with round-stamped per-warp
//      counts, so the row of assignment a is offsets[e] + #{a' < a : ids[a'] == e}: the
//      stable order.
#include <mutex>

#include "kernels.h"
#include "launch.cuh"
#include "route_dev.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxChunks = 128;          // chunks per call (one scan CTA thread each)
constexpr int kMinChunkTokens = 64;

// Tokens per chunk: 64, doubled until there are at most kMaxChunks chunks.
int chunk_tokens(int64_t T) {
  int64_t t = kMinChunkTokens;
  while ((T + t - 1) / t > kMaxChunks) t *= 2;
  return static_cast<int>(t);
}

int num_chunks(int64_t T) {
  const int64_t t = chunk_tokens(T);
  return T > 0 ? static_cast<int>((T + t - 1) / t) : 1;
}

// Scratch: per-chunk counts cc[E][nch], their exclusive scan over chunks base[E][nch], and
// the expert totals tot[E] (ints).
size_t scratch_ints(int64_t T, int E) {
  return static_cast<size_t>(2) * E * num_chunks(T) + E;
}

// Histogram of one chunk of consecutive assignments: cc[e][chunk].
__global__ void __launch_bounds__(kThreads)
    chunk_hist_kernel(const int32_t* __restrict__ ids, int64_t R, int E, int chunk, int nch,
                      int32_t* __restrict__ cc, int* status) {
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
    else if (status)
      set_status(status, kStatusBadIndex);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads)
    cc[static_cast<int64_t>(e) * nch + blockIdx.x] = h[e];
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

// One CTA per expert: base[e][c] = sum of cc[e][c'] over the chunks c' < c, tot[e] = all.
__global__ void __launch_bounds__(kThreads)
    chunk_scan_kernel(const int32_t* __restrict__ cc, int nch, int32_t* __restrict__ base,
                      int32_t* __restrict__ tot) {
  __shared__ int s[kThreads];
  __shared__ int warp_sums[kWarps];
  const int e = blockIdx.x, tid = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  s[tid] = tid < nch ? __ldg(cc + static_cast<int64_t>(e) * nch + tid) : 0;
  __syncthreads();
  const int total = block_exclusive_scan(s, nch, warp_sums);
  if (tid < nch) base[static_cast<int64_t>(e) * nch + tid] = s[tid];
  if (tid == 0) tot[e] = total;
}

// One CTA per chunk: offsets[e] = exclusive scan over experts of tot[e]; the chunk's first
// row for expert e is offsets[e] + base[e][chunk].  The chunk is then walked in order, 256
// assignments per round, ranking equal experts inside a warp with __match_any_sync and
// across the 8 warps with round-stamped per-warp counts, so the row of assignment a is
// offsets[e] + #{a' < a : ids[a'] == e}: the stable order.
__global__ void __launch_bounds__(kThreads)
    scatter_kernel(const int32_t* __restrict__ ids, int64_t R, int E, int chunk, int nch,
                   const int32_t* __restrict__ base, const int32_t* __restrict__ tot,
                   int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                   int32_t* __restrict__ row2assign, int32_t* __restrict__ assign2row) {
  __shared__ int cursor[kMaxExperts];
  __shared__ int scan[kMaxExperts];
  __shared__ int wcnt[kWarps][kMaxExperts];
  __shared__ int warp_sums[kWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int me = blockIdx.x;
  for (int e = tid; e < E; e += kThreads) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) wcnt[w][e] = -1;
  }
  pdl_wait();
  pdl_launch_dependents();

  for (int e = tid; e < E; e += kThreads) {
    cursor[e] = __ldg(base + static_cast<int64_t>(e) * nch + me);
    scan[e] = __ldg(tot + e);
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

// Scan + scatter after the chunk histograms are in `scratch`.
cudaError_t launch_scan_scatter(const int32_t* ids, int64_t T, int k, int E, int32_t* counts,
                                int32_t* offsets, int32_t* row2assign, int32_t* assign2row,
                                int32_t* scratch, cudaStream_t stream, int* launches) {
  const int tpc = chunk_tokens(T);
  const int nch = num_chunks(T);
  const int64_t R = T * k;
  int32_t* cc = scratch;
  int32_t* base = cc + static_cast<int64_t>(E) * nch;
  int32_t* tot = base + static_cast<int64_t>(E) * nch;
  *launches += 2;
  cudaError_t e = launch_k(chunk_scan_kernel, dim3(E), dim3(kThreads), 0, stream,
                           static_cast<const int32_t*>(cc), nch, base, tot);
  if (e != cudaSuccess) return e;
  return launch_k(scatter_kernel, dim3(nch), dim3(kThreads), 0, stream, ids, R, E, tpc * k, nch,
                  static_cast<const int32_t*>(base), static_cast<const int32_t*>(tot), counts,
                  offsets, row2assign, assign2row);
}

cudaError_t permute_empty(int E, int32_t* counts, int32_t* offsets, cudaStream_t stream,
                          int* launches) {
  ++*launches;
  cudaError_t e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), stream);
  if (e != cudaSuccess) return e;
  return cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream);
}

}  // namespace

size_t permute_scratch_bytes(int64_t T, int E) { return scratch_ints(T, E) * sizeof(int32_t); }

cudaError_t launch_permute(const int32_t* ids, int64_t T, int k, int E, int32_t* counts,
                           int32_t* offsets, int32_t* row2assign, int32_t* assign2row,
                           int32_t* scratch, int* status, cudaStream_t stream, int* launches) {
  if (T == 0) return permute_empty(E, counts, offsets, stream, launches);
  const int tpc = chunk_tokens(T);
  const int nch = num_chunks(T);
  ++*launches;
  cudaError_t e = launch_k(chunk_hist_kernel, dim3(nch), dim3(kThreads), 0, stream, ids, T * k, E,
                           tpc * k, nch, scratch, status);
  if (e != cudaSuccess) return e;
  return launch_scan_scatter(ids, T, k, E, counts, offsets, row2assign, assign2row, scratch,
                             stream, launches);
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
    route_permute_small_kernel(const float* __restrict__ logits, int T, int E, int k, int ns,
                               int score, int renorm, int32_t* __restrict__ ids,
                               float* __restrict__ w,
                               int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                               int32_t* __restrict__ row2assign,
                               int32_t* __restrict__ assign2row) {
  __shared__ int s_ids[kSmallMaxT * kMaxTopK];
  __shared__ int scan[kSmallMaxE];
  __shared__ int cursor[kSmallMaxE];
  __shared__ int wcnt[kSmallWarps][kSmallMaxE];
  __shared__ int warp_sums[kSmallWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ks = k + ns;        // slots per token: the top-k, then the shared experts
  const int Ea = E + ns;        // experts of the permutation
  const int R = T * ks;
  pdl_wait();
  pdl_launch_dependents();

  for (int t = warp; t < T; t += kSmallWarps) {
    int id;
    float wt;
    route_token_warp<VPT>(logits + static_cast<int64_t>(t) * E, E, k, score, renorm, lane, id,
                          wt);
    if (lane >= k) {
      id = E + (lane - k);
      wt = 1.0f;
    }
    if (lane < ks) {
      ids[t * ks + lane] = id;
      w[t * ks + lane] = wt;
      s_ids[t * ks + lane] = id;
    }
  }
  for (int e = tid; e < Ea; e += kSmallThreads) {
    scan[e] = 0;
#pragma unroll 4
    for (int ww = 0; ww < kSmallWarps; ++ww) wcnt[ww][e] = -1;
  }
  __syncthreads();
  for (int a = tid; a < R; a += kSmallThreads) atomicAdd(&scan[s_ids[a]], 1);
  __syncthreads();
  // exclusive scan of the Ea counts: one per thread, warp scans, then the warp totals
  const int cnt = tid < Ea ? scan[tid] : 0;
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
  if (tid < Ea) {
    cursor[tid] = excl;
    offsets[tid] = excl;
    counts[tid] = cnt;
  }
  if (tid == 0) offsets[Ea] = R;
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
cudaError_t launch_small(const float* logits, int T, int E, int k, int ns, int score, int renorm,
                         int32_t* ids, float* w, int32_t* counts, int32_t* offsets,
                         int32_t* row2assign, int32_t* assign2row, cudaStream_t stream) {
  return launch_k(route_permute_small_kernel<VPT>, dim3(1), dim3(kSmallThreads), 0, stream, logits,
                  T, E, k, ns, score, renorm, ids, w, counts, offsets, row2assign, assign2row);
}

}  // namespace

bool use_route_permute_small(int64_t T, int E_all, int k_all) {
  return T > 0 && T <= kSmallMaxT && E_all <= kSmallMaxE && k_all <= kMaxTopK;
}

cudaError_t launch_route_permute_small(const float* logits, int64_t T, int E, int k, int ns,
                                       int score, int renorm, int32_t* ids, float* w,
                                       int32_t* counts, int32_t* offsets, int32_t* row2assign,
                                       int32_t* assign2row, cudaStream_t stream, int* launches) {
  ++*launches;
  const int t = static_cast<int>(T);
  const int need = (E + 31) / 32;
  if (need <= 1)
    return launch_small<1>(logits, t, E, k, ns, score, renorm, ids, w, counts, offsets,
                           row2assign, assign2row, stream);
  if (need <= 2)
    return launch_small<2>(logits, t, E, k, ns, score, renorm, ids, w, counts, offsets,
                           row2assign, assign2row, stream);
  if (need <= 4)
    return launch_small<4>(logits, t, E, k, ns, score, renorm, ids, w, counts, offsets,
                           row2assign, assign2row, stream);
  return launch_small<8>(logits, t, E, k, ns, score, renorm, ids, w, counts, offsets,
                         row2assign, assign2row, stream);
}

// ---------------------------------------------------------------- allocation-free variant
//
// For callers that cannot hand the library a workspace: the per-chunk histograms and their
// scans live in this file-scope device array instead (512 KB, held on every device that
// loads the library until the process exits).  Every call shares it, so two calls whose
// kernels overlap on the GPU (different streams, or different host threads) race on it;
// calls serialised on one stream are safe.  The kernels overwrite every entry a call reads,
// so nothing has to be cleared between calls.

constexpr int kNoAllocScratchInts = 1 << 17;
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

bool permute_noalloc_fits(int64_t T, int E) {
  return T == 0 || scratch_ints(T, E) <= static_cast<size_t>(kNoAllocScratchInts);
}

cudaError_t launch_permute_noalloc(const int32_t* ids, int64_t T, int k, int E, int32_t* counts,
                                   int32_t* offsets, int32_t* row2assign, int32_t* assign2row,
                                   cudaStream_t stream, int* launches) {
  if (T == 0) return permute_empty(E, counts, offsets, stream, launches);
  int32_t* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  return launch_permute(ids, T, k, E, counts, offsets, row2assign, assign2row, scratch, nullptr,
                        stream, launches);
}

}  // namespace moe
