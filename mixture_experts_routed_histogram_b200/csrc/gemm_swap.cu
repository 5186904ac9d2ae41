// gemm_swap.cu -- decode-sized grouped GEMMs with the operands swapped: the expert's
// weight rows are the MMA's M=128 side and the few routed token rows are its N side.
//
// Source: GC-MoE (arXiv 2611.16219, abstract) on decode: with few tokens per expert the
// path is bound by streaming the weights, and its MMA swaps A and B so the weights fill the
// large MMA dimension while the activations take the small one.  FlashInfer PR #6465 tunes
// small token tiles (N16 / N64) for the same reason.  The operations are those of
// gemm_bf16.cu (TileScale PR #70 "Design" kernels 1 and 2).
//
// Per task: 128 weight rows x NT token rows, K streamed through a STAGES-deep ring of
// (16 KB weight box + NT*128 B token box) stages -- almost all of shared memory holds
// weights, so each SM keeps ~170 KB of weight bytes in flight.
//   GEMM1: the 128 weight rows are 64 gate rows and the 64 matching up rows; the epilogue
//          passes the gate half through shared memory to the warps that hold the up half,
//          which write act = silu(g)*u for the tile's 64 features of each token row.  With
//          K split (slice count set on the host), it writes fp32 gate|up partial sums and
//          swiglu_parts_kernel finishes act.
//   GEMM2: 128 output features; with partial sums (the forward's decode path) it runs
//          stream-K: the (tile, K block) units of the busy tiles, counted on the device, are
//          cut into one contiguous range per SM, so that even one token (two experts)
//          streams its weights on every SM.  A range's piece of a tile writes fp32 partial
//          sums to slot j = its index among the tile's pieces (the last piece zero-fills the
//          slots after it); the slot count goes to a workspace word and the split-aware
//          combine adds the slots in order.  (The same split for GEMM1 measured no faster:
//          with the weights streaming from HBM, SMs that finish early do not matter while
//          the others still saturate it.)
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "kernels.h"
#include "launch.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int BMW = 128;  // weight rows per task (MMA M)
constexpr int BK = 64;

struct SwapArgs {
  const int32_t* offsets;
  const int32_t* row2assign;  // GEMM1
  const uint16_t* x;          // GEMM1: token rows [T][K]
  uint16_t* out;              // GEMM1 (S == 1): act [R][I]; GEMM2 (S == 1): y [R][H]
  float* part;                // S > 1: partial sums, GEMM1 [S][R][2I] (gate | up), GEMM2 [S][R][H]
  int* status;
  int E, k_top;
  int n_out;                  // I (GEMM1) or H (GEMM2)
  int K;
  int ftiles;                 // feature tiles per expert: I/64 (GEMM1) or H/128 (GEMM2)
  int splits;                 // K slices (GEMM1); GEMM2: the most slices it may choose
  int* splits_used;           // GEMM2 with splits > 1: the slice count it chose (for the combine)
  int b_rows;                 // weight rows per expert: 2I or H
  int64_t R;
  int inject_stall;
  uint64_t wait_limit_ns;
};

template <bool GEMM1, int NT, int STAGES>
struct SwapCfg {
  static constexpr int THREADS = GEMM1 ? 32 * 7 : 32 * 6;
  static constexpr int A_BYTES = BMW * BK * 2;   // weights
  static constexpr int B_BYTES = NT * BK * 2;    // token rows
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int GBUF_OFF = STAGES * STAGE;                // GEMM1: gate values
  static constexpr int GBUF_BYTES = GEMM1 ? 2 * 64 * NT * 4 : 0;  // one per accumulator
  static constexpr int BAR_OFF = GBUF_OFF + GBUF_BYTES;
  static constexpr int NBAR = 2 * STAGES + 5;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int OFFS_OFF = MISC_OFF + 16;
  static constexpr int TILE_OFF = OFFS_OFF + 4 * (kMaxExperts + 1);
  static constexpr int TOTAL = TILE_OFF + 4 * (kMaxExperts + 1);
  static constexpr int ALLOC = TOTAL + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * NT < 32 ? 32 : 2 * NT;
  static constexpr uint32_t FULL_COUNT = GEMM1 ? 1 + 32 : 1;
  static_assert(STAGE % 1024 == 0, "stage alignment");
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 128, "token tile");
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

// task -> (expert, token tile, feature tile, K slice); tasks of expert e occupy
// [tile_start[e] * ftiles * S, tile_start[e+1] * ftiles * S).
__device__ __forceinline__ void decode_swap(int task, const int* s_tile, int E, int per_tile,
                                            int splits, int& e, int& tt, int& ft, int& sp) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tile[mid] * per_tile <= task) lo = mid; else hi = mid;
  }
  e = lo;
  const int local = task - s_tile[e] * per_tile;
  tt = local / per_tile;
  const int rest = local - tt * per_tile;
  ft = rest / splits;
  sp = rest - ft * splits;
}

__device__ __forceinline__ int64_t i64min(int64_t a, int64_t b) { return a < b ? a : b; }
__device__ __forceinline__ int64_t i64max(int64_t a, int64_t b) { return a > b ? a : b; }

// The work of one CTA.  Round robin: tasks c, c + P, ... of the (expert, token tile,
// feature tile, K slice) queue.  Stream-K (the decode GEMM2 with partial sums): the
// (tile, K block) units of all tiles, U of them, are dealt to the first P' CTAs as equal
// contiguous ranges [c U / P', (c+1) U / P'), cut at tile boundaries into segments; the
// segment of tile t that CTA c holds writes partial-sum slot c - (first CTA of t), and the
// CTA holding a tile's last K block also clears its higher slots up to the slot count the
// combine sums, so every slot it reads is defined and the sum keeps a fixed order.
struct SwapWork {
  int e, tt, ft;        // expert, token tile, feature tile
  int kb0, kb1;         // K blocks [kb0, kb1)
  int slot;             // partial-sum slot
  bool last;            // this segment ends the tile (stream-K: clear the higher slots)
};

struct SwapIter {
  const int* s_tile;
  int E, ftiles, splits, kb_all;
  bool sk;
  int64_t u, u_hi, U;   // stream-K range of this CTA
  int P;                // stream-K CTAs
  int task, total, step;  // round robin
  __device__ __forceinline__ int owner(int64_t unit) const {   // CTA holding a unit
    return static_cast<int>(((unit + 1) * P - 1) / U);
  }
  __device__ __forceinline__ bool next(SwapWork& w) {
    int sp = 0;
    if (sk) {
      if (u >= u_hi) return false;
      const int tile = static_cast<int>(u / kb_all);
      w.kb0 = static_cast<int>(u - static_cast<int64_t>(tile) * kb_all);
      w.kb1 = static_cast<int>(i64min(kb_all, w.kb0 + (u_hi - u)));
      w.slot = owner(u) - owner(static_cast<int64_t>(tile) * kb_all);
      w.last = w.kb1 == kb_all;
      u += w.kb1 - w.kb0;
      decode_swap(tile, s_tile, E, ftiles, 1, w.e, w.tt, w.ft, sp);
      return true;
    }
    if (task >= total) return false;
    decode_swap(task, s_tile, E, ftiles * splits, splits, w.e, w.tt, w.ft, sp);
    const int kb_per = kb_all / splits;
    w.kb0 = sp * kb_per;
    w.kb1 = w.kb0 + kb_per;
    w.slot = sp;
    w.last = false;
    task += step;
    return true;
  }
};

// CTAs that share the stream-K work: all of them, unless that leaves fewer than 24 K
// blocks per CTA (a task switch costs about 16 K blocks of streaming) or lets one tile of
// kb blocks span more than kMaxSplits CTAs (each CTA's range is >= ceil(kb / 15) units).
__device__ __forceinline__ int64_t stream_k_ctas(int64_t units, int64_t kb, int grid) {
  const int64_t min_len = i64max(24, (kb + kMaxSplits - 2) / (kMaxSplits - 1));
  return i64max(1, i64min(grid, units / min_len));
}

// Partial-sum slots a tile of kb blocks can span when U units are dealt to P CTAs.
__device__ __forceinline__ int stream_k_slots(int64_t U, int64_t kb, int64_t P) {
  const int64_t len = i64max(1, U / P);   // the shortest CTA range
  return static_cast<int>(i64min(kMaxSplits, (kb + len - 1) / len + 1));
}

__device__ __forceinline__ float silu_mul_s(float g, float u) {
  return g / (1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int NT>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NT]) {
  static_assert(NT % 16 == 0, "NT");
#pragma unroll
  for (int c = 0; c < NT; c += 32) {
    if constexpr (NT >= 32) {
      uint32_t t[32];
      tmem_ld_32x32b_x32(taddr + c, t);
#pragma unroll
      for (int i = 0; i < 32; ++i) r[c + i] = t[i];
    }
  }
  if constexpr (NT == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  }
}

template <bool GEMM1, int NT, int STAGES>
__global__ void __launch_bounds__(SwapCfg<GEMM1, NT, STAGES>::THREADS, 1)
    swap_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmW,
                          const __grid_constant__ CUtensorMap tmT, const SwapArgs args) {
  using C = SwapCfg<GEMM1, NT, STAGES>;
  constexpr uint32_t IDESC = idesc_bf16_f32<BMW, NT>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  volatile int* s_never = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 8);
  int* s_splits = reinterpret_cast<int*>(smem + C::MISC_OFF + 12);
  int* s_off = reinterpret_cast<int*>(smem + C::OFFS_OFF);
  int* s_tile = reinterpret_cast<int*>(smem + C::TILE_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int E = args.E;
  const uint64_t lim = args.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], C::FULL_COUNT);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    *s_never = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    if constexpr (!GEMM1) tma_prefetch_desc(&tmT);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  // GEMM1 reads the token rows, row2assign and the offsets in several roles: every thread
  // waits for the kernels before it.  GEMM2's weights and expert offsets are final before
  // the kernel just ahead of it could start (the offsets come from the front end, which had
  // completed by then), so only its producer waits -- after issuing the weight boxes of its
  // first ring of stages -- and the token rows (act, from GEMM1) are loaded after the wait;
  // the weights stream while GEMM1 finishes.  The offsets are read through L2 (__ldcg).
  if constexpr (GEMM1) pdl_wait();
  pdl_launch_dependents();  // the next kernel's CTAs may take SMs as this grid's CTAs exit
  for (int i = threadIdx.x; i <= E; i += C::THREADS) s_off[i] = __ldcg(args.offsets + i);
  __syncthreads();
  if (warp == 0) {  // token tiles of NT rows per expert
    const int per = (E + 31) / 32;
    const int e0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) local += (s_off[e + 1] - s_off[e] + NT - 1) / NT;
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int run = incl - local;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) {
        s_tile[e] = run;
        run += (s_off[e + 1] - s_off[e] + NT - 1) / NT;
      }
    }
    if (lane == 31) {
      s_tile[E] = incl;
      // args.splits > 1 selects the partial-sum output.  GEMM2 then runs stream-K; the
      // number of partial-sum slots a tile can span (what the combine sums) is stored
      if (!GEMM1 && args.splits > 1) {
        const int64_t kb = args.K / BK;
        const int64_t U = static_cast<int64_t>(incl) * args.ftiles * kb;
        *s_splits = stream_k_slots(U, kb, stream_k_ctas(U, kb, gridDim.x));
      } else {
        *s_splits = args.splits;
      }
      if (!GEMM1 && args.splits_used && blockIdx.x == 0) *args.splits_used = *s_splits;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int kb_all = args.K / BK;
  const bool stream_k = !GEMM1 && args.splits > 1;
  const int splits = stream_k ? 1 : *s_splits;   // round robin: K slices per tile
  const int nslots = *s_splits;                   // stream-K: partial-sum slots
  const int per_tile = args.ftiles * splits;
  const int total = s_tile[E] * per_tile;
  const int kb_per = kb_all / splits;
  auto make_iter = [&]() {
    SwapIter it{};
    it.s_tile = s_tile;
    it.E = E;
    it.ftiles = args.ftiles;
    it.splits = splits;
    it.kb_all = kb_all;
    it.sk = stream_k;
    if (stream_k) {
      it.U = static_cast<int64_t>(s_tile[E]) * args.ftiles * kb_all;
      it.P = static_cast<int>(stream_k_ctas(it.U, kb_all, gridDim.x));
      const int c = static_cast<int>(blockIdx.x);
      it.u = c < it.P ? static_cast<int64_t>(c) * it.U / it.P : it.U;
      it.u_hi = c < it.P ? static_cast<int64_t>(c + 1) * it.U / it.P : it.U;
    } else {
      it.task = blockIdx.x;
      it.total = total;
      it.step = gridDim.x;
    }
    return it;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t fill = 0;
    int skipped = -1;
    bool ok = true;
    // GEMM2: token-row loads of the fills issued before the wait for the kernel ahead
    bool waited = GEMM1;
    int npend = 0;
    uint32_t pend_fill[STAGES];
    int pend_row[STAGES], pend_kb[STAGES];
    auto flush = [&]() {
      pdl_wait();
      waited = true;
      if (lane == 0)
        for (int i = 0; i < npend; ++i) {
          const int ps = static_cast<int>(pend_fill[i] % STAGES);
          tma_load_2d(smem + ps * C::STAGE + C::A_BYTES, &tmT, &full[ps], pend_kb[i] * BK,
                      pend_row[i]);
        }
      __syncwarp();
    };
    SwapIter it = make_iter();
    SwapWork wk;
    while (ok && it.next(wk)) {
      const int e = wk.e, tt = wk.tt, ft = wk.ft;
      const int row0 = s_off[e] + tt * NT;
      const int wrow = GEMM1 ? e * args.b_rows + ft * 64 : e * args.b_rows + ft * BMW;
      for (int kb = wk.kb0; kb < wk.kb1; ++kb, ++fill) {
        const int s = fill % STAGES;
        const uint32_t ph = (fill / STAGES) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, s_abort, lim))) {
          ok = false;
          break;
        }
        if (args.inject_stall && blockIdx.x == 0 && fill == 0) {
          skipped = 0;
          continue;
        }
        uint8_t* w_dst = smem + s * C::STAGE;
        uint8_t* t_dst = w_dst + C::A_BYTES;
        if (lane == 0) {
          if constexpr (GEMM1) {
            mbar_arrive_expect_tx(&full[s], C::A_BYTES);
            tma_load_2d(w_dst, &tmW, &full[s], kb * BK, wrow);                  // 64 gate rows
            tma_load_2d(w_dst + 64 * 128, &tmW, &full[s], kb * BK, wrow + args.n_out);  // up
          } else {
            mbar_arrive_expect_tx(&full[s], C::STAGE);
            tma_load_2d(w_dst, &tmW, &full[s], kb * BK, wrow);
            if (waited) tma_load_2d(t_dst, &tmT, &full[s], kb * BK, row0);
          }
        }
        if (!waited) {   // (GEMM2 only) the token rows of this fill wait for the flush
          pend_fill[npend] = fill;
          pend_row[npend] = row0;
          pend_kb[npend] = kb;
          if (++npend == STAGES) flush();   // before the ring is reused
        }
        __syncwarp();
      }
    }
    if (!waited) flush();   // fewer fills than stages, or the loop gave up
    if (!ok && lane == 0) {
      *s_abort = 1;
      set_status(args.status, kStatusTimeout);
    }
    for (uint32_t f = fill > static_cast<uint32_t>(STAGES) ? fill - STAGES : 0; f < fill; ++f) {
      if (static_cast<int>(f) == skipped) continue;
      mbar_wait(&full[f % STAGES], (f / STAGES) & 1u, s_never, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t fill = 0, tc = 0;
      bool ok = true;
      SwapIter it = make_iter();
      SwapWork wk;
      while (ok && it.next(wk)) {
        const int acc = tc & 1;
        const uint32_t aph = (tc >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, s_abort, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * NT);
        for (int kb = 0; kb < wk.kb1 - wk.kb0; ++kb, ++fill) {
          const int s = fill % STAGES;
          const uint32_t ph = (fill / STAGES) & 1u;
          if (!mbar_wait(&full[s], ph, s_abort, lim)) {
            ok = false;
            break;
          }
          if constexpr (GEMM1) fence_async_smem();
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + s * C::STAGE));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + s * C::STAGE + C::A_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, IDESC, (kb | kk) != 0 ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        ++tc;
      }
      if (!ok) {
        *s_abort = 1;
        set_status(args.status, kStatusTimeout);
      }
      if (fill > 0) {
        mma_commit(drain);
        mbar_wait(drain, 0, s_never, lim);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------------------ token-row gather (GEMM1)
    if constexpr (GEMM1) {
      constexpr int PER = NT * 8 / 32;  // 16-byte copies per lane per stage
      uint32_t fill = 0;
      bool ok = true;
      for (int task = blockIdx.x; task < total && ok; task += gridDim.x) {
        int e, tt, ft, sp;
        decode_swap(task, s_tile, E, per_tile, splits, e, tt, ft, sp);
        const int row0 = s_off[e] + tt * NT;
        const int rows = min(NT, s_off[e + 1] - row0);
        const uint16_t* src[PER];
        int dst_off[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int idx = lane + 32 * i;   // (row, chunk) = (idx / 8, idx % 8)
          const int r = idx >> 3, chunk = idx & 7;
          const int tok = __ldg(args.row2assign + row0 + (r < rows ? r : 0)) / args.k_top;
          src[i] = args.x + static_cast<int64_t>(tok) * args.K + chunk * 8;
          dst_off[i] = r * 128 + ((chunk ^ (r & 7)) << 4);
        }
        for (int kb = 0; kb < kb_per; ++kb, ++fill) {
          const int s = fill % STAGES;
          const uint32_t ph = (fill / STAGES) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, s_abort, lim))) {
            ok = false;
            break;
          }
          const uint32_t t_base = smem_u32(smem + s * C::STAGE + C::A_BYTES);
          const int kk = (sp * kb_per + kb) * BK;
#pragma unroll
          for (int i = 0; i < PER; ++i) cp_async_16(t_base + dst_off[i], src[i] + kk);
          cp_async_mbar_arrive_noinc(&full[s]);
        }
      }
      if (!ok && lane == 0) {
        *s_abort = 1;
        set_status(args.status, kStatusTimeout);
      }
      cp_async_wait_all();
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int q = warp & 3;          // TMEM lanes 32q..32q+31 = weight rows of the tile
    uint32_t tc = 0;
    bool ok = true;
    SwapIter it = make_iter();
    SwapWork wk;
    while (it.next(wk)) {
      const int e = wk.e, tt = wk.tt, ft = wk.ft, sp = wk.slot;
      const int row0 = s_off[e] + tt * NT;
      const int rows = min(NT, s_off[e + 1] - row0);
      const int acc = tc & 1;
      const uint32_t aph = (tc >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, s_abort, lim))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc * NT);
      uint32_t v[NT];
      tmem_ld_cols<NT>(tb, v);
      tmem_ld_wait();
      if (GEMM1 && args.splits > 1) {
        // K slice of gate (rows 0-63) and up (rows 64-127) sums; SwiGLU runs after the slices
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        const int j = (q & 1) * 32 + lane;
        const int col = (q < 2 ? 0 : args.n_out) + ft * 64 + j;
        float* dst = args.part + static_cast<int64_t>(sp) * args.R * (2 * args.n_out);
#pragma unroll
        for (int c = 0; c < NT; ++c)
          if (c < rows) dst[static_cast<int64_t>(row0 + c) * (2 * args.n_out) + col] = __uint_as_float(v[c]);
      } else if constexpr (GEMM1) {
        // rows 0-63 of the tile are gate features, 64-127 the matching up features
        float* gbuf = reinterpret_cast<float*>(smem + C::GBUF_OFF) + acc * 64 * NT;
        const int j = (q & 1) * 32 + lane;     // feature within the tile's 64
        if (q < 2) {
#pragma unroll
          for (int c = 0; c < NT; ++c) gbuf[c * 64 + j] = __uint_as_float(v[c]);
        }
        tc_fence_before();
        named_bar_sync(1, 128);
        if (lane == 0) mbar_arrive(&tempty[acc]);
        if (q >= 2) {
          const int col = ft * 64 + j;
#pragma unroll
          for (int c = 0; c < NT; ++c) {
            if (c < rows) {
              const float a = silu_mul_s(gbuf[c * 64 + j], __uint_as_float(v[c]));
              args.out[static_cast<int64_t>(row0 + c) * args.n_out + col] =
                  static_cast<uint16_t>(pack_bf16x2(a, 0.0f) & 0xFFFFu);
            }
          }
        }
        named_bar_sync(1, 128);   // gbuf[acc] may be rewritten two tiles later
      } else {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        const int o = ft * BMW + q * 32 + lane;
        if (args.splits > 1) {
          float* dst = args.part + static_cast<int64_t>(sp) * args.R * args.n_out;
#pragma unroll
          for (int c = 0; c < NT; ++c)
            if (c < rows) dst[static_cast<int64_t>(row0 + c) * args.n_out + o] = __uint_as_float(v[c]);
          if (wk.last)   // stream-K: the tile's unused higher slots read as zeros
            for (int z = sp + 1; z < nslots; ++z) {
              float* zd = args.part + static_cast<int64_t>(z) * args.R * args.n_out;
              for (int c = 0; c < rows; ++c)
                zd[static_cast<int64_t>(row0 + c) * args.n_out + o] = 0.0f;
            }
        } else {
#pragma unroll
          for (int c = 0; c < NT; ++c)
            if (c < rows)
              args.out[static_cast<int64_t>(row0 + c) * args.n_out + o] =
                  static_cast<uint16_t>(pack_bf16x2(__uint_as_float(v[c]), 0.0f) & 0xFFFFu);
        }
      }
      ++tc;
    }
    if (!ok && lane == 0) {
      *s_abort = 1;
      set_status(args.status, kStatusTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// act[r][i] = silu(sum_s g) * (sum_s u) from the K-sliced GEMM1 partial sums (slice order)
__global__ void swiglu_parts_kernel(const float* __restrict__ part, int splits, int64_t R, int I,
                                    uint16_t* __restrict__ act) {
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
  pdl_wait();
  pdl_launch_dependents();
  if (i >= R * I) return;
  const int64_t r = i / I;
  const int c = static_cast<int>(i - r * I);
  const int64_t slice = R * 2 * I;
  // every slice's loads are issued before the first add (the sum stays in slice order)
  float2 g[kMaxSplits], u[kMaxSplits];
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) {
    if (s < splits) {
      const float* p = part + s * slice + r * 2 * I;
      g[s] = *reinterpret_cast<const float2*>(p + c);
      u[s] = *reinterpret_cast<const float2*>(p + I + c);
    }
  }
  float g0 = 0.f, g1 = 0.f, u0 = 0.f, u1 = 0.f;
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) {
    if (s < splits) {
      g0 += g[s].x; g1 += g[s].y; u0 += u[s].x; u1 += u[s].y;
    }
  }
  *reinterpret_cast<uint32_t*>(act + r * I + c) = pack_bf16x2(silu_mul_s(g0, u0), silu_mul_s(g1, u1));
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_swap() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool tmap_bf16_swap(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                    uint32_t box_outer) {
  auto fn = encode_fn_swap();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {BK, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool GEMM1, int NT>
cudaError_t run_swap(const CUtensorMap& w, const CUtensorMap& t, const SwapArgs& args,
                     cudaStream_t stream) {
  // fill shared memory with stages after the gate buffer and the bookkeeping (two barriers
  // per stage, five more, the expert offsets and tile starts, 1 KB of alignment slack)
  using C1 = SwapCfg<GEMM1, NT, 1>;
  constexpr int FIXED = C1::GBUF_BYTES + 5 * 8 + 16 + 8 * (kMaxExperts + 1) + 1024;
  constexpr int STAGES = (227 * 1024 - FIXED) / (C1::STAGE + 16);
  using Cf = SwapCfg<GEMM1, NT, STAGES>;
  auto kern = swap_gemm_bf16_kernel<GEMM1, NT, STAGES>;
  static cudaError_t attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::ALLOC);
  if (attr != cudaSuccess) return attr;
  return launch_k(kern, dim3(num_sms()), dim3(Cf::THREADS), Cf::ALLOC, stream, w, t, args);
}

template <bool GEMM1>
cudaError_t run_swap_nt(int nt, const CUtensorMap& w, const CUtensorMap& t, const SwapArgs& a,
                        cudaStream_t stream) {
  switch (nt) {
    case 16: return run_swap<GEMM1, 16>(w, t, a, stream);
    case 32: return run_swap<GEMM1, 32>(w, t, a, stream);
    default: return run_swap<GEMM1, 64>(w, t, a, stream);
  }
}

}  // namespace

int swap_token_tile(int64_t T) {
  return T <= 16 ? 16 : (T <= 32 ? 32 : 64);
}

bool use_swap_gemm(int64_t T) { return T <= 64; }

// K slices for GEMM1: enough (expert, feature tile, slice) tasks that the last, partial
// wave over the SMs costs little (>= 6 waves), counting at most min(E, R) busy experts;
// slices divide the K blocks and keep >= 8 blocks each.
static int splits_for(int64_t busy_tiles, int kb, int waves) {
  int best = 1;
  for (int s = 1; s <= std::min(kb, kMaxSplits); ++s) {
    if (kb % s != 0 || kb / s < 8) continue;
    best = s;
    if (busy_tiles * s >= static_cast<int64_t>(waves) * num_sms()) break;
  }
  return best;
}

// GEMM2: the most K slices its kernel may choose (it picks the count on the device from
// the busy tiles): the largest divisor of the K blocks that keeps >= 24 blocks per slice.
int swap_splits(const GemmProblem& p) {
  const int kb = p.I / BK;
  int best = 1;
  for (int s = 2; s <= std::min(kb, kMaxSplits); ++s)
    if (kb % s == 0 && kb / s >= 24) best = s;
  return best;
}

int swap_splits_gemm1(const GemmProblem& p) {
  return splits_for(std::min<int64_t>(p.E, p.R) * (p.I / 64), p.H / BK, 6);
}

cudaError_t launch_gemm1_swap(const GemmProblem& p, const uint16_t* x, const int32_t* row2assign,
                              const int32_t* offsets, const uint16_t* w13, uint16_t* act,
                              float* part, int splits, int* status, cudaStream_t stream,
                              int* launches) {
  if (p.R == 0) return cudaSuccess;
  const int nt = swap_token_tile(p.T);
  CUtensorMap tw, tt{};
  if (!tmap_bf16_swap(&tw, w13, p.H, static_cast<uint64_t>(p.E) * 2 * p.I, 64))
    return cudaErrorInvalidValue;
  SwapArgs a{};
  a.offsets = offsets;
  a.row2assign = row2assign;
  a.x = x;
  a.out = act;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.I;
  a.K = p.H;
  a.ftiles = p.I / 64;
  a.splits = splits;
  a.part = part;
  a.b_rows = 2 * p.I;
  a.R = p.R;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  cudaError_t e = run_swap_nt<true>(nt, tw, tt, a, stream);
  if (e != cudaSuccess || splits <= 1) return e;
  ++*launches;
  const int64_t pairs = p.R * p.I / 2;
  return launch_k(swiglu_parts_kernel, dim3(static_cast<unsigned>((pairs + 255) / 256)), dim3(256),
                  0, stream, static_cast<const float*>(part), splits, p.R, p.I, act);
}

cudaError_t launch_gemm2_swap(const GemmProblem& p, const uint16_t* act, const int32_t* offsets,
                              const uint16_t* w2, uint16_t* y, float* part, int splits,
                              int* splits_used, int* status, cudaStream_t stream,
                              int* launches) {
  if (p.R == 0) return cudaSuccess;
  const int nt = swap_token_tile(p.T);
  CUtensorMap tw, tt;
  if (!tmap_bf16_swap(&tw, w2, p.I, static_cast<uint64_t>(p.E) * p.H, BMW) ||
      !tmap_bf16_swap(&tt, act, p.I, p.R, nt))
    return cudaErrorInvalidValue;
  SwapArgs a{};
  a.offsets = offsets;
  a.out = y;
  a.part = part;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.H;
  a.K = p.I;
  a.ftiles = p.H / BMW;
  a.splits = splits;
  a.splits_used = splits_used;
  a.b_rows = p.H;
  a.R = p.R;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  return run_swap_nt<false>(nt, tw, tt, a, stream);
}

}  // namespace moe
