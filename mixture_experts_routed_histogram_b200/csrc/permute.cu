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
#include <cuda.h>

#include <algorithm>
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

// ---------------------------------------------------------------- larger batches, one launch
//
// The forward pass's front end for batches beyond the single-CTA kernel: routing, the
// per-block histograms, the prefix sums and the stable scatter in one cooperative launch
// (every CTA is resident, so the CTAs may wait for one another): nb CTAs of 32 warps (as
// many as are resident, at most one per 32 tokens), CTA b owning tokens
// [b * tpc, (b+1) * tpc).
//   phase 1  warps route their tokens (route_token_warp), write ids and w, keep the ids in
//            shared memory and count the CTA's assignments per expert -> cc[e][b];
//   barrier  grid-wide: an arrival count and a generation word in the workspace's status
//            block, bounded wait;
//   phase 2  tot[e] (all blocks' counts) and base[e] (those of the blocks before this
//            one): with few experts x blocks (<= 32768 cells) every CTA sums cc itself --
//            integer sums, so the order does not matter; with more, one warp per expert
//            (spread over the CTAs) scans its row of cc into base and tot in global memory
//            and a second barrier precedes the reads.  Then each CTA scans tot over the
//            experts (offsets; CTA 0 writes counts and offsets) and scatters its
//            assignments in order with the warp-match and round-stamp ranking of
//            scatter_kernel: row = offsets[e] + #{a' < a : ids[a'] == e}.
// Each step waits on global memory about once.  At T = 8192, E = 128, k = 8 the kernel takes
// about 18 us on the device (routing ~7, barrier ~2.5, column sums ~3, scan and scatter
// ~5; globaltimer stamps per CTA), against ~28 us for the four separate kernels it
// replaces.  It is launched with programmatic dependent launch as well as cooperatively,
// so its launch overlaps the previous kernel's tail.  Same outputs as launch_route
// followed by launch_permute, bit for bit.

constexpr int kFusedThreads = 1024;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedMaxBlocks = 1024;
constexpr int kFusedIdsSmem = 8192;   // assignments of a CTA kept in shared memory
constexpr int64_t kSinglePassCells = 32768;   // experts x blocks summed by every CTA itself

int fused_blocks_cap(int64_t T) {
  return static_cast<int>(std::min<int64_t>((T + kFusedWarps - 1) / kFusedWarps, kFusedMaxBlocks));
}

// In-place exclusive scan of s[0..n) (n <= 4 * kFusedThreads); returns the total.
__device__ int fused_exclusive_scan(int* s, int n, int* warp_sums) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + kFusedThreads - 1) / kFusedThreads;  // <= 4
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
  for (int w = 0; w < kFusedWarps; ++w) {
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

// Grid-wide barrier of a cooperative launch: gbar[0] counts arrivals (the last one resets it
// and advances gbar[1]); the others wait, bounded, for the generation to move.  `extra`
// arrivals more than the grid are awaited (a test hook that makes the wait run out).
// Returns false (every thread of the CTA) if the wait gave up.
__device__ bool grid_barrier(unsigned* gbar, int* s_ok, uint64_t limit_ns, unsigned extra) {
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile unsigned* vgen = gbar + 1;
    const unsigned gen = *vgen;
    __threadfence();
    bool ok = true;
    if (atomicAdd(gbar, 1u) == gridDim.x - 1 + extra) {
      atomicExch(gbar, 0u);
      __threadfence();
      atomicAdd(gbar + 1, 1u);
    } else {
      // poll with a short sleep between reads, so the waiting CTAs do not keep the line's
      // L2 slice busy while the last arrivals are still on their way
      const uint64_t start = globaltimer_ns();
      for (uint32_t i = 0; *vgen == gen; ++i) {
        __nanosleep(64);
        if ((i & 15u) == 15u && globaltimer_ns() - start > limit_ns) {
          ok = false;
          break;
        }
      }
    }
    __threadfence();
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

template <int VPT>
__global__ void __launch_bounds__(kFusedThreads)
    route_permute_kernel(const float* __restrict__ logits, int64_t T, int E, int k, int ns,
                         int score, int renorm, int tpc, int32_t* __restrict__ ids,
                         float* __restrict__ w, int32_t* __restrict__ cc,
                         int32_t* __restrict__ base, int32_t* __restrict__ tot,
                         int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                         int32_t* __restrict__ row2assign, int32_t* __restrict__ assign2row,
                         unsigned* gbar, int* status, uint64_t limit_ns, int inject_stall) {
  extern __shared__ int fsm[];
  const int Ea = E + ns, ks = k + ns;
  const int nb = gridDim.x;
  int* hist = fsm;                 // [Ea]: the block's histogram, later tot and its scan
  int* cursor = hist + Ea;         // [Ea]: base, then the block's first row per expert
  int* wcnt = cursor + Ea;         // [kFusedWarps][Ea]: round-stamped per-warp counts
  int* s_ids = wcnt + kFusedWarps * Ea;   // [min(tpc * ks, kFusedIdsSmem)]: the block's ids
  __shared__ int warp_sums[kFusedWarps];
  __shared__ int s_ok;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int me = blockIdx.x;
  const int64_t t0 = min(static_cast<int64_t>(me) * tpc, T);
  const int64_t t1 = min(t0 + tpc, T);
  const int64_t a0 = t0 * ks, a1 = t1 * ks;
  const bool ids_in_smem = a1 - a0 <= kFusedIdsSmem;
  for (int e = tid; e < Ea; e += kFusedThreads) {
    hist[e] = 0;
    cursor[e] = 0;
    for (int ww = 0; ww < kFusedWarps; ++ww) wcnt[ww * Ea + e] = -1;
  }
  pdl_wait();
  pdl_launch_dependents();
  __syncthreads();

  // ---- phase 1: route the block's tokens, count its assignments per expert; a warp with a
  // second token asks for that token's logits (into L2) before routing the first
  for (int64_t t = t0 + warp; t < t1; t += kFusedWarps) {
    if (t + kFusedWarps < t1) {
      const float* nxt = logits + (t + kFusedWarps) * E;
      for (int e = lane * 32; e < E; e += 32 * 32)   // one 128-byte line per lane
        asm volatile("prefetch.global.L2 [%0];" ::"l"(nxt + e));
    }
    int id;
    float wt;
    route_token_warp<VPT>(logits + t * E, E, k, score, renorm, lane, id, wt);
    if (lane >= k) {
      id = E + (lane - k);
      wt = 1.0f;
    }
    if (lane < ks) {
      ids[t * ks + lane] = id;
      w[t * ks + lane] = wt;
      if (ids_in_smem) s_ids[(t - t0) * ks + lane] = id;
      atomicAdd(&hist[id], 1);
    }
  }
  __syncthreads();
  for (int e = tid; e < Ea; e += kFusedThreads) cc[static_cast<int64_t>(e) * nb + me] = hist[e];

  if (!grid_barrier(gbar, &s_ok, limit_ns, inject_stall ? 1u : 0u)) {
    // the wait gave up (status recorded; outputs undefined): leave no expert any rows, so
    // the GEMMs after this kernel read no permutation entry
    if (tid == 0) set_status(status, kStatusTimeout);
    for (int e = tid; e <= Ea; e += kFusedThreads) {
      offsets[e] = 0;
      if (e < Ea) counts[e] = 0;
    }
    return;
  }

  // ---- phase 2: tot[e] = all blocks' counts, base[e] = those of the blocks before this one
  if (static_cast<int64_t>(Ea) * nb <= kSinglePassCells) {
    // few cells: every CTA sums them itself; a group of g lanes (a power of two, g * Ea <=
    // kFusedThreads when Ea is small) shares an expert's row of cc, every load issued
    // before the sums
    int g = 1;
    while (g < 32 && 2 * g * Ea <= kFusedThreads) g *= 2;
    const int per_warp = 32 / g;   // experts a warp handles per pass (the loop is warp-uniform)
    for (int eb = warp * per_warp; eb < Ea; eb += kFusedWarps * per_warp) {
      const int e0 = eb + lane / g, sub = lane & (g - 1);
      int all = 0, before = 0;
      if (e0 < Ea) {
        const int32_t* row = cc + static_cast<int64_t>(e0) * nb;
#pragma unroll 8
        for (int c = sub; c < nb; c += g) {
          const int v = __ldcg(row + c);
          all += v;
          before += c < me ? v : 0;
        }
      }
      for (int off = g >> 1; off > 0; off >>= 1) {
        all += __shfl_xor_sync(0xffffffffu, all, off);
        before += __shfl_xor_sync(0xffffffffu, before, off);
      }
      if (e0 < Ea && sub == 0) {
        hist[e0] = all;
        cursor[e0] = before;
      }
    }
  } else {
    // many cells (many experts): one warp per expert, spread over the CTAs, scans its row of
    // cc into base[e][*] and tot[e]; after a second barrier each CTA reads its column
    constexpr int kPer = kFusedMaxBlocks / 32;
    for (int e = warp * nb + me; e < Ea; e += nb * kFusedWarps) {
      const int32_t* src = cc + static_cast<int64_t>(e) * nb;
      int32_t* dst = base + static_cast<int64_t>(e) * nb;
      int v[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int c = i * 32 + lane;
        v[i] = c < nb ? __ldcg(src + c) : 0;
      }
      int run = 0;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        if (i * 32 < nb) {
          int incl = v[i];
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
          }
          if (i * 32 + lane < nb) dst[i * 32 + lane] = run + incl - v[i];
          run += __shfl_sync(0xffffffffu, incl, 31);
        }
      }
      if (lane == 0) tot[e] = run;
    }
    if (!grid_barrier(gbar, &s_ok, limit_ns, 0u)) {
      if (tid == 0) set_status(status, kStatusTimeout);
      for (int e = tid; e <= Ea; e += kFusedThreads) {
        offsets[e] = 0;
        if (e < Ea) counts[e] = 0;
      }
      return;
    }
    for (int e = tid; e < Ea; e += kFusedThreads) {
      hist[e] = __ldcg(tot + e);
      cursor[e] = __ldcg(base + static_cast<int64_t>(e) * nb + me);
    }
  }
  __syncthreads();
  const int grand = fused_exclusive_scan(hist, Ea, warp_sums);
  for (int e = tid; e < Ea; e += kFusedThreads) {
    cursor[e] += hist[e];
    if (me == 0) {
      offsets[e] = hist[e];
      counts[e] = (e + 1 < Ea ? hist[e + 1] : grand) - hist[e];
    }
  }
  if (me == 0 && tid == 0) offsets[Ea] = grand;
  __syncthreads();

  // ---- stable scatter of the block's assignments, kFusedThreads per round
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; a0 + static_cast<int64_t>(r) * kFusedThreads < a1; ++r) {
    const int64_t a = a0 + static_cast<int64_t>(r) * kFusedThreads + tid;
    const int e = a < a1 ? (ids_in_smem ? s_ids[a - a0] : __ldcg(ids + a)) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lt);
    const int grp = __popc(peers);
    const bool leader = (__ffs(peers) - 1) == lane;
    if (e >= 0 && leader) wcnt[warp * Ea + e] = (r << 10) | grp;
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int ww = 0; ww < warp; ++ww) {
        const int v = wcnt[ww * Ea + e];
        if ((v >> 10) == r) before += v & 1023;
      }
      const int row = cursor[e] + before + rank;
      row2assign[row] = static_cast<int32_t>(a);
      assign2row[a] = row;
    }
    __syncthreads();
    if (e >= 0 && leader) atomicAdd(&cursor[e], grp);
  }
}

size_t route_permute_scratch_bytes(int64_t T, int E) {
  return (static_cast<size_t>(2) * E * fused_blocks_cap(T) + E) * sizeof(int32_t);
}

template <int VPT>
cudaError_t launch_fused(const float* logits, int64_t T, int E, int k, int ns, int score,
                         int renorm, int32_t* ids, float* w, int32_t* counts, int32_t* offsets,
                         int32_t* row2assign, int32_t* assign2row, int32_t* scratch,
                         unsigned* gbar, int* status, uint64_t limit_ns, cudaStream_t stream) {
  const int Ea = E + ns, ks = k + ns;
  auto kern = route_permute_kernel<VPT>;
  constexpr size_t kMaxSmem = sizeof(int) * (kMaxExperts * (2 + kFusedWarps) + kFusedIdsSmem);
  static cudaError_t attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (attr != cudaSuccess) return attr;
  // as many CTAs as can be resident (every one must be, they wait for each other), at most
  // one per 32 tokens; the shared memory depends on the ids a CTA keeps, so size the grid
  // for the largest
  const size_t fixed = sizeof(int) * static_cast<size_t>(Ea) * (2 + kFusedWarps);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, kern, kFusedThreads, fixed + sizeof(int) * kFusedIdsSmem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int nb = std::max(1, std::min(fused_blocks_cap(T), per_sm * num_sms()));
  const int tpc = static_cast<int>((T + nb - 1) / nb);
  const int nb_used = static_cast<int>((T + tpc - 1) / tpc);   // no empty CTA
  const size_t smem =
      fixed + sizeof(int) * static_cast<size_t>(std::min<int64_t>(static_cast<int64_t>(tpc) * ks,
                                                                   kFusedIdsSmem));
  int32_t* cc = scratch;
  int32_t* base = cc + static_cast<int64_t>(Ea) * nb_used;
  int32_t* tot = base + static_cast<int64_t>(Ea) * nb_used;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(nb_used);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: they wait for each other
  at[0].val.cooperative = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // as launch_k
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, logits, T, E, k, ns, score, renorm, tpc, ids, w, cc, base,
                            tot, counts, offsets, row2assign, assign2row, gbar, status, limit_ns,
                            g_inject_stall);
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
struct NoAllocSlot {
  unsigned long long ctx_id = 0;  // unique id of the context the address belongs to
  int32_t* ptr = nullptr;
};
NoAllocSlot g_noalloc[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <class Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<Fn>(p);
  return nullptr;
}

// Process-unique id of the calling thread's current context (0: none bound yet).
cudaError_t current_ctx_id(unsigned long long* id) {
  static const CtxGetCurrentFn get = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get || !get_id) return cudaErrorInitializationError;
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return cudaErrorInitializationError;
  *id = 0;
  if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorInitializationError;
  return cudaSuccess;
}
}  // namespace

// Device address of g_noalloc_scratch in the current device's context.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with the device
// current (cudaGetSymbolAddress) and cached per device together with the id of the context
// it was found in (ids are never reused within a process); a new context on that device,
// after cudaDeviceReset or a primary context released and created again (the module is
// then loaded again, possibly elsewhere), is looked up afresh.
static cudaError_t noalloc_scratch(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  unsigned long long id = 0;
  if ((e = current_ctx_id(&id)) != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocSlot& slot = g_noalloc[dev];
  if (!slot.ptr || id == 0 || slot.ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // binds the primary context if needed
    if (e != cudaSuccess) return e;
    if ((e = current_ctx_id(&id)) != cudaSuccess) return e;
    if (id == 0) return cudaErrorInitializationError;
    slot.ptr = static_cast<int32_t*>(p);
    slot.ctx_id = id;
  }
  *out = slot.ptr;
  return cudaSuccess;
}

cudaError_t launch_route_permute(const float* logits, int64_t T, int E, int k, int ns, int score,
                                 int renorm, int32_t* ids, float* w, int32_t* counts,
                                 int32_t* offsets, int32_t* row2assign, int32_t* assign2row,
                                 int32_t* scratch, unsigned* gbar, int* status,
                                 uint64_t limit_ns, cudaStream_t stream, int* launches) {
  if (T == 0) return permute_empty(E + ns, counts, offsets, stream, launches);
  ++*launches;
  const int need = (E + 31) / 32;
#define MOE_FUSED(V)                                                                           \
  return launch_fused<V>(logits, T, E, k, ns, score, renorm, ids, w, counts, offsets,          \
                         row2assign, assign2row, scratch, gbar, status, limit_ns, stream)
  if (need <= 1) MOE_FUSED(1);
  if (need <= 2) MOE_FUSED(2);
  if (need <= 4) MOE_FUSED(4);
  if (need <= 8) MOE_FUSED(8);
  if (need <= 16) MOE_FUSED(16);
  MOE_FUSED(32);
#undef MOE_FUSED
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
