// gemm_bf16_2sm.cu -- the BF16 grouped GEMMs on SM pairs (tcgen05 cta_group::2).
//
// Same operations as gemm_bf16.cu (GEMM1 + SwiGLU over gathered token rows, GEMM2 over the
// expert-sorted act rows; TileScale PR #70 "Design" kernels 1 and 2, flat task queue;
// FlashInfer PR #5129 sorted I/O), but each task is a 256-row tile computed by a cluster of
// two CTAs on two SMs: every CTA stages its own 128 A rows and half of the 256 B rows, the
// leader CTA issues one M=256, N=256 MMA per K=16 step, and each CTA's TMEM receives its own
// 128 rows of the accumulator.  Per SM this halves the B bytes per MMA (32 KB stages, six
// of them in shared memory instead of four 48 KB ones), which is what keeps the tensor
// pipe fed on the large-T workloads.
//
// Pair protocol (all waits bounded):
//   full[s]  (leader)  GEMM2: one expect-tx arrival by the leader for both CTAs' TMA bytes.
//                      GEMM1: the same for the B halves, plus one arrival per CTA from its
//                      relay warp once that CTA's cp.async rows of the stage have landed
//                      (counted on the local afull[s], then forwarded to the leader after a
//                      proxy fence, with a CTA-scope remote arrive: a cluster-scope release
//                      there costs a fence per stage and halved the kernel's speed).
//   empty[s] (both)    one multicast commit from the leader's MMA thread.
//   tfull[a] (both)    one multicast commit when a tile's MMAs are done.
//   tempty[a](leader)  one arrival per epilogue warp of either CTA (8).
#include <cudaTypedefs.h>
#include <stdlib.h>

#include <mutex>
#include <string>

#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int BM = 128;   // rows per CTA (256 per pair)
constexpr int BK = 64;
constexpr int BN = 256;   // MMA N (per pair); each CTA stages BN/2 B rows
constexpr int kLoaderWarps = 4;
constexpr int kRelayWarp = 6 + kLoaderWarps;  // GEMM1: forwards landed A stages to the leader

struct PairArgs {
  const int32_t* offsets;
  const int32_t* row2assign;   // GEMM1
  const uint16_t* a_rows;      // GEMM1: x [T][K]
  uint16_t* out;               // act [R][I] or y [R][H]
  int* status;
  int E, k_top, n_out, K, n_tiles, b_rows;
  int inject_stall;
  uint64_t wait_limit_ns;
};

template <bool GEMM1, int STAGES>
struct PairCfg {
  static constexpr int THREADS = GEMM1 ? 32 * (7 + kLoaderWarps) : 192;
  static constexpr int A_BYTES = BM * BK * 2;         // 16 KB
  static constexpr int B_BYTES = (BN / 2) * BK * 2;   // 16 KB: this CTA's half of B
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int BAR_OFF = STAGES * STAGE;
  static constexpr int NBAR = 3 * STAGES + 5;   // full, empty, afull (GEMM1), acc, drain
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int OFFS_OFF = MISC_OFF + 16;
  static constexpr int TILE_OFF = OFFS_OFF + 4 * (kMaxExperts + 1);
  static constexpr int EPI_OFF = (TILE_OFF + 4 * (kMaxExperts + 1) + 1023) / 1024 * 1024;
  static constexpr int TOTAL = EPI_OFF + kEpiBytes;  // + the epilogue's staging buffers
  static constexpr int ALLOC = TOTAL + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static constexpr uint32_t FULL_COUNT = GEMM1 ? 1 + 2 : 1;  // + one relay per CTA
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void decode_pair(int task, const int* s_tile, int E, int n_tiles,
                                            int& e, int& pt, int& nt) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tile[mid] * n_tiles <= task) lo = mid; else hi = mid;
  }
  e = lo;
  const int local = task - s_tile[e] * n_tiles;
  const int ptiles = s_tile[e + 1] - s_tile[e];
  nt = local / ptiles;
  pt = local - nt * ptiles;
}

// silu(g)*u with the approximate divide (the quotient is 0 once the denominator overflows)
__device__ __forceinline__ float silu_mul2(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

template <bool GEMM1, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<GEMM1, STAGES>::THREADS, 1)
    pair_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA,
                          const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmC, const PairArgs args) {
  using C = PairCfg<GEMM1, STAGES>;
  constexpr uint32_t IDESC = idesc_bf16_f32<2 * BM, BN>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* afull = drain + 1;   // GEMM1: this CTA's A rows of a stage have landed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  volatile int* s_never = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 8);
  int* s_off = reinterpret_cast<int*>(smem + C::OFFS_OFF);
  int* s_tile = reinterpret_cast<int*>(smem + C::TILE_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();   // 0 = leader
  const int E = args.E;
  const uint64_t lim = args.wait_limit_ns;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], C::FULL_COUNT);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(drain, 1);
    if constexpr (GEMM1)
      for (int s = 0; s < STAGES; ++s) mbar_init(&afull[s], 32 * kLoaderWarps);
    *s_abort = 0;
    *s_never = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if constexpr (!GEMM1) tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_2sm(s_tmem, C::TMEM_COLS);
    tmem_relinquish_2sm();
  }
  pdl_wait();  // the offsets (and every other input) come from earlier kernels
  pdl_launch_dependents();  // the next kernel's CTAs may take SMs as this grid's CTAs exit
  for (int i = threadIdx.x; i <= E; i += C::THREADS) s_off[i] = __ldg(args.offsets + i);
  __syncthreads();
  if (warp == 0) {  // pair-tile prefix over experts (256 rows per pair tile)
    const int per = (E + 31) / 32;
    const int e0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) local += (s_off[e + 1] - s_off[e] + 2 * BM - 1) / (2 * BM);
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
        run += (s_off[e + 1] - s_off[e] + 2 * BM - 1) / (2 * BM);
      }
    }
    if (lane == 31) s_tile[E] = incl;
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = s_tile[E] * args.n_tiles;
  const int kblocks = args.K / BK;
  const uint32_t full_leader0 = mapa_shared(smem_u32(full), 0);      // leader's full[0]
  const uint32_t tempty_leader0 = mapa_shared(smem_u32(tempty), 0);  // leader's tempty[0]

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    uint32_t fill = 0;
    int skipped = -1;
    bool ok = true;
    for (int task = pair; task < total && ok; task += npairs) {
      int e, pt, nt;
      decode_pair(task, s_tile, E, args.n_tiles, e, pt, nt);
      const int row0 = s_off[e] + pt * 2 * BM + static_cast<int>(rank) * BM;
      // GEMM1: CTA 0 stages the 128 gate rows, CTA 1 the matching 128 up rows.
      // GEMM2: CTA r stages output columns [nt*256 + r*128, +128).
      const int brow = GEMM1 ? e * args.b_rows + nt * (BN / 2) + static_cast<int>(rank) * args.n_out
                             : e * args.b_rows + nt * BN + static_cast<int>(rank) * (BN / 2);
      for (int kb = 0; kb < kblocks; ++kb, ++fill) {
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
        uint8_t* a_dst = smem + s * C::STAGE;
        uint8_t* b_dst = a_dst + C::A_BYTES;
        const uint32_t fb = full_leader0 + 8u * static_cast<uint32_t>(s);
        if (lane == 0) {
          if (rank == 0)
            mbar_arrive_expect_tx(&full[s], GEMM1 ? 2 * C::B_BYTES : 2 * C::STAGE);
          if constexpr (!GEMM1) tma_load_2d_2sm(a_dst, &tmA, fb, kb * BK, row0);
          tma_load_2d_2sm(b_dst, &tmB, fb, kb * BK, brow);
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {
      *s_abort = 1;
      set_status(args.status, kStatusTimeout);
    }
    // the last fills' copies have landed once the MMA released them (empty) -- wait for
    // that, bounded, so no copy targets this CTA after it exits
    for (uint32_t f = fill > static_cast<uint32_t>(STAGES) ? fill - STAGES : 0; f < fill; ++f) {
      if (static_cast<int>(f) == skipped) continue;
      mbar_wait(&empty[f % STAGES], ((f / STAGES) & 1u), s_never, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (rank == 0 && lane == 0) {
      uint32_t fill = 0, tc = 0;
      bool ok = true;
      for (int task = pair; task < total && ok; task += npairs) {
        const int acc = tc & 1;
        const uint32_t aph = (tc >> 1) & 1u;
        if (!mbar_wait_cluster(&tempty[acc], aph ^ 1u, s_abort, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++fill) {
          const int s = fill % STAGES;
          const uint32_t ph = (fill / STAGES) & 1u;
          if (!mbar_wait_cluster(&full[s], ph, s_abort, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + s * C::STAGE));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + s * C::STAGE + C::A_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ss_2sm(d_tmem, ad + 2 * kk, bd + 2 * kk, IDESC, (kb | kk) != 0 ? 1u : 0u);
          mma_commit_2sm(&empty[s]);
        }
        if (!ok) break;
        mma_commit_2sm(&tfull[acc]);
        ++tc;
      }
      if (!ok) {
        *s_abort = 1;
        set_status(args.status, kStatusTimeout);
      }
      if (fill > 0) {  // every pair MMA issued above has completed once this arrives
        mma_commit_2sm(drain);
        mbar_wait(drain, 0, s_never, lim);
      }
    }
    __syncwarp();
  } else if (warp == kRelayWarp) {
    // ------------------------------------------------------------ relay (GEMM1, both CTAs)
    if constexpr (GEMM1) {
      if (lane == 0) {
        uint32_t fill = 0;
        bool ok = true;
        for (int task = pair; task < total && ok; task += npairs) {
          for (int kb = 0; kb < kblocks; ++kb, ++fill) {
            const int s = fill % STAGES;
            if (!mbar_wait(&afull[s], (fill / STAGES) & 1u, s_abort, lim)) {
              ok = false;
              break;
            }
            fence_async_smem();  // cp.async rows (generic proxy) -> the leader's MMA reads
            mbar_arrive_remote(full_leader0 + 8u * static_cast<uint32_t>(s));
          }
        }
        if (!ok) {
          *s_abort = 1;
          set_status(args.status, kStatusTimeout);
        }
      }
      __syncwarp();
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------ A gather (GEMM1, both CTAs)
    if constexpr (GEMM1) {
      const int lw = warp - 6;
      const int sub = lane >> 3;
      const int chunk = lane & 7;
      uint32_t fill = 0;
      bool ok = true;
      for (int task = pair; task < total && ok; task += npairs) {
        int e, pt, nt;
        decode_pair(task, s_tile, E, args.n_tiles, e, pt, nt);
        const int row0 = s_off[e] + pt * 2 * BM + static_cast<int>(rank) * BM;
        const int rows = s_off[e + 1] - row0;  // may be <= 0 for the upper half of a last tile
        const int rfirst = s_off[e];           // a valid row of this expert
        const uint16_t* src[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = lw * 32 + i * 4 + sub;
          const int rr = r < rows ? row0 + r : rfirst;
          const int tok = __ldg(args.row2assign + rr) / args.k_top;
          src[i] = args.a_rows + static_cast<int64_t>(tok) * args.K + chunk * 8;
        }
        for (int kb = 0; kb < kblocks; ++kb, ++fill) {
          const int s = fill % STAGES;
          const uint32_t ph = (fill / STAGES) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, s_abort, lim))) {
            ok = false;
            break;
          }
          const uint32_t a_base = smem_u32(smem + s * C::STAGE);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = lw * 32 + i * 4 + sub;
            cp_async_16(a_base + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * BK);
          }
          cp_async_mbar_arrive_noinc(&afull[s]);
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
    const int q = warp & 3;
    const int r_in = q * 32 + lane;
    EpiStager st{smem_u32(smem + C::EPI_OFF + q * kEpiWarpBytes), 0u};
    uint32_t tc = 0;
    bool ok = true;
    for (int task = pair; task < total; task += npairs) {
      int e, pt, nt;
      decode_pair(task, s_tile, E, args.n_tiles, e, pt, nt);
      const int row0 = s_off[e] + pt * 2 * BM + static_cast<int>(rank) * BM;
      const int rows = s_off[e + 1] - row0;
      const int acc = tc & 1;
      const uint32_t aph = (tc >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, s_abort, lim))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc * BN);
      const bool valid = r_in < rows;
      const bool whole = rows - q * 32 >= 32;  // all 32 rows of this warp are the expert's
      const int64_t row = row0 + r_in;
      if constexpr (GEMM1) {
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(tb + c, g);
          tmem_ld_32x32b_x32(tb + BN / 2 + c, u);
          tmem_ld_wait();
          const int col = nt * (BN / 2) + c;
          if (col < args.n_out) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(silu_mul2(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                  silu_mul2(__uint_as_float(g[2 * i + 1]),
                                            __uint_as_float(u[2 * i + 1])));
            if (whole)
              epi_store_chunk(st, &tmC, pk, col, row0 + q * 32, lane);
            else if (valid)
              epi_store_row(args.out + row * args.n_out + col, pk);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v32[32];
          tmem_ld_32x32b_x32(tb + c, v32);
          tmem_ld_wait();
          const int col = nt * BN + c;
          if (col < args.n_out) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(v32[2 * i]), __uint_as_float(v32[2 * i + 1]));
            if (whole)
              epi_store_chunk(st, &tmC, pk, col, row0 + q * 32, lane);
            else if (valid)
              epi_store_row(args.out + row * args.n_out + col, pk);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8u * static_cast<uint32_t>(acc));
      ++tc;
    }
    if (!ok && lane == 0) {
      *s_abort = 1;
      set_status(args.status, kStatusTimeout);
    }
    epi_drain(lane);
  }

  tc_fence_before();
  cluster_sync();  // neither CTA leaves while the pair's MMAs or signals may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem_base, C::TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_2sm() {
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

bool tmap_bf16_2sm(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                   uint32_t box_outer) {
  auto fn = encode_fn_2sm();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {BK, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool GEMM1, int STAGES>
cudaError_t run_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                     const PairArgs& args, cudaStream_t stream) {
  using Cf = PairCfg<GEMM1, STAGES>;
  auto kern = pair_gemm_bf16_kernel<GEMM1, STAGES>;
  static cudaError_t attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::ALLOC);
  if (attr != cudaSuccess) return attr;
  const int grid = num_sms() & ~1;
  return launch_k(kern, dim3(grid), dim3(Cf::THREADS), Cf::ALLOC, stream, a, b, c, args);
}

}  // namespace

// Which grouped GEMMs run on SM pairs.  The pair kernels run their padded work about 10 %
// faster than the single-SM ones (half the B bytes per SM), but their 256-row tiles pad
// more rows: at ~500 rows per expert 20 % against 11 %.  So GEMM2 (contiguous A by TMA)
// pairs once an expert averages >= 768 rows, or >= 384 when its K is short (<= 1024: the
// deeper ring of the pair kernel then pays; measured at 512 rows per expert: K = 768
// 203 -> 198 us, K = 8192 587 -> 603 us), and GEMM1 (whose gathered A reaches the leader
// through a relay warp) stays on single SMs (measured slower on pairs at 512-4096 rows
// per expert).  MOE_PAIR_GEMM=0/1 forces the choice for both (a tuning and test switch).
int pair_gemm_override() {
  static const int force = [] {
    const char* e = getenv("MOE_PAIR_GEMM");
    return e ? atoi(e) : -1;
  }();
  return force;
}

bool use_pair_gemm(int64_t R, int E, int K) {
  if (pair_gemm_override() >= 0) return pair_gemm_override() != 0;
  const int64_t per_expert = R / E;
  return per_expert >= 768 || (K <= 1024 && per_expert >= 384);
}

bool use_pair_gemm1(int64_t R, int E) {
  (void)R; (void)E;
  return pair_gemm_override() == 1;
}

cudaError_t launch_gemm1_bf16_2sm(const GemmProblem& p, const uint16_t* x,
                                  const int32_t* row2assign, const int32_t* offsets,
                                  const uint16_t* w13, uint16_t* act, int* status,
                                  cudaStream_t stream, int* launches) {
  if (p.R == 0) return cudaSuccess;
  if (p.I % 128 != 0) return cudaErrorInvalidValue;
  CUtensorMap ta{}, tb, tc;
  if (!tmap_bf16_2sm(&tb, w13, p.H, static_cast<uint64_t>(p.E) * 2 * p.I, BN / 2) ||
      !make_tmap_epi(encode_fn_2sm(), &tc, act, p.I, p.R))
    return cudaErrorInvalidValue;
  PairArgs a{};
  a.offsets = offsets;
  a.row2assign = row2assign;
  a.a_rows = x;
  a.out = act;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.I;
  a.K = p.H;
  a.n_tiles = p.I / (BN / 2);
  a.b_rows = 2 * p.I;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  return run_pair<true, 6>(ta, tb, tc, a, stream);
}

cudaError_t launch_gemm2_bf16_2sm(const GemmProblem& p, const uint16_t* act,
                                  const int32_t* offsets, const uint16_t* w2, uint16_t* y,
                                  int* status, cudaStream_t stream, int* launches) {
  if (p.R == 0) return cudaSuccess;
  CUtensorMap ta, tb, tc;
  if (!tmap_bf16_2sm(&ta, act, p.I, p.R, BM) ||
      !tmap_bf16_2sm(&tb, w2, p.I, static_cast<uint64_t>(p.E) * p.H, BN / 2) ||
      !make_tmap_epi(encode_fn_2sm(), &tc, y, p.H, p.R))
    return cudaErrorInvalidValue;
  PairArgs a{};
  a.offsets = offsets;
  a.out = y;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.H;
  a.K = p.I;
  a.n_tiles = (p.H + BN - 1) / BN;
  a.b_rows = p.H;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  return run_pair<false, 6>(ta, tb, tc, a, stream);
}

}  // namespace moe
