// gemm_bf16.cu -- grouped GEMMs over the expert-sorted row space on sm_100a tensor cores.
//
//   GEMM1 + SwiGLU: act[r][i] = silu(x[tok(r)] . W13[e][i]) * (x[tok(r)] . W13[e][I+i])
//   GEMM1 + ReLU2:  act[r][i] = max(x[tok(r)] . W1[e][i], 0)^2
//   GEMM2:          y[r][o]   = act[r] . W2[e][o]
//
// Sources: TileScale PR #70 (distributed FP8 MegaMoE), "Design" -- kernel 1 is GEMM1 with
// the SwiGLU fused into its epilogue, kernel 2 is GEMM2; its first listed change replaces
// a per-tile expert rescan by a flat m-task queue, and another lets the MMA overwrite the
// accumulator on the first k-step instead of clearing it.  FlashInfer PR #5129 (cuTile
// BF16 fused MoE), "sorted I/O": GEMM1 gathers token rows for A and writes expert-sorted
// rows, which GEMM2 reads as a contiguous A operand.
//
// B200 design (one persistent CTA per SM; 6 warps, plus 4 loader warps for GEMM1):
//   warp 0      producer: TMA loads into a STAGES-deep shared-memory ring guarded by
//               full/empty mbarriers.  B is a 2-D tile load (GEMM1 SwiGLU: the 128 gate
//               rows and the matching 128 up rows of one expert, stacked; ReLU2: 256
//               consecutive W1 rows); GEMM2's A is a 2-D tile of the sorted act rows.
//   warps 6-9   GEMM1 only: gather the tile's token rows of x with 16-byte cp.async into
//               the 128-byte-swizzled layout (tile::gather4 by the producer instead is a
//               tuning switch, MOE_GEMM1_GATHER=tma4, measured slower).
//   warp 1      TMEM owner + MMA issuer: one thread issues tcgen05.mma (M=128, N=BN,
//               K=16, bf16 -> fp32) into one of two TMEM accumulators, commits each stage
//               back to its empty barrier and each finished tile to the epilogue.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (each warp owns its 32-lane TMEM
//               quadrant = 32 rows), SwiGLU or ReLU2 (GEMM1) or plain conversion (GEMM2)
//               to bf16, each 32x32 chunk staged in shared memory and stored by TMA
//               (epilogue.cuh); then frees the accumulator for the next tile.
// Tasks are a flat (expert, n-tile, m-tile) queue built in shared memory from the
// expert offsets: CTA c takes tasks c, c + gridDim, ...  Consecutive tasks share the
// same weight tile (n-tile) of one expert, so the SMs working at the same time read each
// weight tile from HBM about once and hit L2 for the rest.  Empty experts contribute
// no task, and every role walks the same task sequence, so pipeline phases stay in step.
// Every mbarrier wait is bounded; on expiry the CTA records MOE_ERR_DEVICE_TIMEOUT,
// unwinds all roles, drains in-flight copies and MMAs and frees its TMEM.
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

constexpr int BM = 128;        // rows per tile (MMA M)
constexpr int BK = 64;         // bf16 elements per 128-byte swizzled row

// How the A operand reaches shared memory.
enum AMode : int {
  kATile = 0,     // contiguous rows: one 2-D TMA box per stage (GEMM2)
  kAGather4 = 1,  // token rows: 32 TMA tile::gather4 loads per stage (GEMM1 alternative)
  kACpAsync = 2,  // token rows: 4 loader warps, 16-byte cp.async into the swizzled layout
};
constexpr int kLoaderWarps = 4;
__host__ __device__ constexpr int threads_for(int amode) {
  return amode == kACpAsync ? 32 * (6 + kLoaderWarps) : 192;
}

struct KArgs {
  const int32_t* offsets;      // [E+1]
  const int32_t* row2assign;   // GEMM1 only
  const uint16_t* a_rows;      // GEMM1 cp.async mode: x [T][K]
  uint16_t* out;               // act [R][I] (GEMM1) or y [R][H] (GEMM2)
  int* status;
  int E, k_top;
  int n_out;                   // output columns: I (GEMM1) or H (GEMM2)
  int K;                       // reduction length: H (GEMM1) or I (GEMM2)
  int n_tiles;                 // output column tiles per expert
  int b_rows;                  // weight rows per expert: 2I (GEMM1) or H (GEMM2)
  int inject_stall;            // test hook: CTA 0 skips its first stage fill
  uint64_t wait_limit_ns;
};

template <int BN, int STAGES>
struct Layout {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int BAR_OFF = STAGES * STAGE;
  static constexpr int NBAR = 2 * STAGES + 5;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int OFFS_OFF = MISC_OFF + 16;
  static constexpr int TILE_OFF = OFFS_OFF + 4 * (kMaxExperts + 1);
  static constexpr int EPI_OFF = (TILE_OFF + 4 * (kMaxExperts + 1) + 1023) / 1024 * 1024;
  static constexpr int TOTAL = EPI_OFF + kEpiBytes;  // + the epilogue's staging buffers
  static constexpr int ALLOC = TOTAL + 1024;  // slack for the 1024-byte alignment
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

// task -> (expert, m-tile, n-tile): tasks of expert e occupy
// [tile_start[e] * n_tiles, tile_start[e+1] * n_tiles), n-tile major.
__device__ __forceinline__ void decode_task(int task, const int* s_tile, int E, int n_tiles,
                                            int& e, int& mt, int& nt) {
  int lo = 0, hi = E;  // s_tile[lo] * n_tiles <= task < s_tile[hi] * n_tiles
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tile[mid] * n_tiles <= task) lo = mid; else hi = mid;
  }
  e = lo;
  const int local = task - s_tile[e] * n_tiles;
  const int mtiles = s_tile[e + 1] - s_tile[e];
  nt = local / mtiles;
  mt = local - nt * mtiles;
}

// silu(g)*u with the approximate divide: for g -> -inf the denominator overflows to +inf and
// the quotient is 0, the limit of silu
__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ float relu2(float g) { return g > 0.0f ? g * g : 0.0f; }

// ACT (GEMM1): 0 = SwiGLU, the tile's B rows are BN/2 gate rows and the matching BN/2 up
// rows and it outputs BN/2 columns; 1 = ReLU2, BN consecutive W1 rows, BN output columns.
template <bool GEMM1, int AMODE, int BN, int STAGES, int ACT = 0>
__global__ void __launch_bounds__(threads_for(AMODE), 1)
    grouped_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmC, const KArgs args) {
  using L = Layout<BN, STAGES>;
  constexpr int kThreads = threads_for(AMODE);
  static_assert(GEMM1 || AMODE == kATile, "GEMM2 reads contiguous rows");
  constexpr int BN_OUT = GEMM1 && ACT == 0 ? BN / 2 : BN;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  constexpr uint32_t IDESC = idesc_bf16_f32<BM, BN>();
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM columns");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  volatile int* s_never = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);
  int* s_off = reinterpret_cast<int*>(smem + L::OFFS_OFF);
  int* s_tile = reinterpret_cast<int*>(smem + L::TILE_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int E = args.E;
  const uint64_t lim = args.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // cp.async mode: the B producer's expect-tx arrival + one per loader thread
      mbar_init(&full[s], AMODE == kACpAsync ? 1 + 32 * kLoaderWarps : 1);
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
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();  // the offsets (and every other input) come from earlier kernels
  pdl_launch_dependents();  // the next kernel's CTAs may take SMs as this grid's CTAs exit
  for (int i = threadIdx.x; i <= E; i += kThreads) s_off[i] = __ldg(args.offsets + i);
  __syncthreads();
  if (warp == 0) {  // m-tile prefix over experts; lane l owns a contiguous expert range
    const int per = (E + 31) / 32;
    const int e0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) local += (s_off[e + 1] - s_off[e] + BM - 1) / BM;
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
        run += (s_off[e + 1] - s_off[e] + BM - 1) / BM;
      }
    }
    if (lane == 31) s_tile[E] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = s_tile[E] * args.n_tiles;
  const int kblocks = args.K / BK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t fill = 0;
    int skipped = -1;
    bool ok = true;
    for (int task = blockIdx.x; task < total && ok; task += gridDim.x) {
      int e, mt, nt;
      decode_task(task, s_tile, E, args.n_tiles, e, mt, nt);
      const int row0 = s_off[e] + mt * BM;
      const int rows = min(BM, s_off[e + 1] - row0);
      int tk0 = 0, tk1 = 0, tk2 = 0, tk3 = 0;
      if constexpr (AMODE == kAGather4) {
        const int r = lane * 4;
        tk0 = __ldg(args.row2assign + row0 + (r + 0 < rows ? r + 0 : 0)) / args.k_top;
        tk1 = __ldg(args.row2assign + row0 + (r + 1 < rows ? r + 1 : 0)) / args.k_top;
        tk2 = __ldg(args.row2assign + row0 + (r + 2 < rows ? r + 2 : 0)) / args.k_top;
        tk3 = __ldg(args.row2assign + row0 + (r + 3 < rows ? r + 3 : 0)) / args.k_top;
      }
      const int brow = e * args.b_rows + nt * BN_OUT;
      for (int kb = 0; kb < kblocks; ++kb, ++fill) {
        const int s = fill % STAGES;
        const uint32_t ph = (fill / STAGES) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, s_abort, lim))) {
          ok = false;
          break;
        }
        if (args.inject_stall && blockIdx.x == 0 && fill == 0) {
          skipped = 0;  // test hook: leave this stage unfilled so the consumer times out
          continue;
        }
        uint8_t* a_dst = smem + s * L::STAGE;
        uint8_t* b_dst = a_dst + L::A_BYTES;
        if (lane == 0)
          mbar_arrive_expect_tx(&full[s], AMODE == kACpAsync ? L::B_BYTES : L::STAGE);
        __syncwarp();
        if constexpr (GEMM1) {
          if constexpr (AMODE == kAGather4)
            tma_gather4(a_dst + lane * 4 * 128, &tmA, &full[s], kb * BK, tk0, tk1, tk2, tk3);
          if (lane == 0) {
            tma_load_2d(b_dst, &tmB, &full[s], kb * BK, brow);
            tma_load_2d(b_dst + (BN / 2) * 128, &tmB, &full[s], kb * BK,
                        brow + (ACT == 0 ? args.n_out : BN / 2));
          }
        } else {
          if (lane == 0) {
            tma_load_2d(a_dst, &tmA, &full[s], kb * BK, row0);
            tma_load_2d(b_dst, &tmB, &full[s], kb * BK, brow);
          }
        }
      }
    }
    if (!ok && lane == 0) {
      *s_abort = 1;
      set_status(args.status, kStatusTimeout);
    }
    // no copy may still be writing shared memory when the CTA exits
    for (uint32_t f = fill > static_cast<uint32_t>(STAGES) ? fill - STAGES : 0; f < fill; ++f) {
      if (static_cast<int>(f) == skipped) continue;
      mbar_wait(&full[f % STAGES], (f / STAGES) & 1u, s_never, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t fill = 0, tc = 0;
      bool ok = true;
      for (int task = blockIdx.x; task < total && ok; task += gridDim.x) {
        const int acc = tc & 1;
        const uint32_t aph = (tc >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, s_abort, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++fill) {
          const int s = fill % STAGES;
          const uint32_t ph = (fill / STAGES) & 1u;
          if (!mbar_wait(&full[s], ph, s_abort, lim)) {
            ok = false;
            break;
          }
          if constexpr (AMODE == kACpAsync) fence_async_smem();  // cp.async data -> MMA reads
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + s * L::STAGE));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + s * L::STAGE + L::A_BYTES));
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
      if (fill > 0) {       // every MMA issued above has completed once this arrives
        mma_commit(drain);
        mbar_wait(drain, 0, s_never, lim);
      }
    }
    __syncwarp();
  } else if (warp >= 6) {
    // ------------------------------------------------------------ A gather (cp.async)
    if constexpr (AMODE == kACpAsync) {
      const int lw = warp - 6;
      const int sub = lane >> 3;    // row within a group of 4
      const int chunk = lane & 7;   // 16-byte chunk within the 128-byte row
      uint32_t fill = 0;
      bool ok = true;
      for (int task = blockIdx.x; task < total && ok; task += gridDim.x) {
        int e, mt, nt;
        decode_task(task, s_tile, E, args.n_tiles, e, mt, nt);
        const int row0 = s_off[e] + mt * BM;
        const int rows = min(BM, s_off[e + 1] - row0);
        const uint16_t* src[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = lw * 32 + i * 4 + sub;
          const int tok = __ldg(args.row2assign + row0 + (r < rows ? r : 0)) / args.k_top;
          src[i] = args.a_rows + static_cast<int64_t>(tok) * args.K + chunk * 8;
        }
        for (int kb = 0; kb < kblocks; ++kb, ++fill) {
          const int s = fill % STAGES;
          const uint32_t ph = (fill / STAGES) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, s_abort, lim))) {
            ok = false;
            break;
          }
          const uint32_t a_base = smem_u32(smem + s * L::STAGE);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = lw * 32 + i * 4 + sub;
            cp_async_16(a_base + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * BK);
          }
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
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp can access
    const int r_in = q * 32 + lane;
    EpiStager st{smem_u32(smem + L::EPI_OFF + q * kEpiWarpBytes), 0u};
    uint32_t tc = 0;
    bool ok = true;
    for (int task = blockIdx.x; task < total; task += gridDim.x) {
      int e, mt, nt;
      decode_task(task, s_tile, E, args.n_tiles, e, mt, nt);
      const int row0 = s_off[e] + mt * BM;
      const int rows = min(BM, s_off[e + 1] - row0);
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
      if constexpr (GEMM1 && ACT == 1) {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v32[32];
          tmem_ld_32x32b_x32(tb + c, v32);
          tmem_ld_wait();
          const int col = nt * BN_OUT + c;
          if (col < args.n_out) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(relu2(__uint_as_float(v32[2 * i])),
                                  relu2(__uint_as_float(v32[2 * i + 1])));
            if (whole)
              epi_store_chunk(st, &tmC, pk, col, row0 + q * 32, lane);
            else if (valid)
              epi_store_row(args.out + row * args.n_out + col, pk);
          }
        }
      } else if constexpr (GEMM1) {
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(tb + c, g);
          tmem_ld_32x32b_x32(tb + BN / 2 + c, u);
          tmem_ld_wait();
          const int col = nt * BN_OUT + c;
          if (col < args.n_out) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                  silu_mul(__uint_as_float(g[2 * i + 1]),
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
          const int col = nt * BN_OUT + c;
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
      if (lane == 0) mbar_arrive(&tempty[acc]);
      ++tc;
    }
    if (!ok && lane == 0) {
      *s_abort = 1;
      set_status(args.status, kStatusTimeout);
    }
    epi_drain(lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// bf16 matrix [outer][inner] (row stride `inner` elements), box {box_inner, box_outer},
// 128-byte swizzle.
bool make_tmap_bf16(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                    uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool GEMM1, int AMODE, int BN, int STAGES, int ACT = 0>
cudaError_t run(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                const KArgs& args, cudaStream_t stream) {
  using L = Layout<BN, STAGES>;
  auto kern = grouped_gemm_bf16_kernel<GEMM1, AMODE, BN, STAGES, ACT>;
  static cudaError_t attr = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (attr != cudaSuccess) return attr;
  return launch_k(kern, dim3(num_sms()), dim3(threads_for(AMODE)), L::ALLOC, stream, a, b, c, args);
}

// GEMM1 A-operand path: cp.async gather (default) or TMA gather4 (MOE_GEMM1_GATHER=tma4,
// a tuning switch).
bool use_gather4() {
  static const bool v = [] {
    const char* e = getenv("MOE_GEMM1_GATHER");
    return e && std::string(e) == "tma4";
  }();
  return v;
}

}  // namespace

int num_sms() {
  static int n = [] {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v > 0 ? v : 148;
  }();
  return n;
}

int g_inject_stall = 0;  // test hook set through moe_debug_inject_stall

cudaError_t launch_gemm1_bf16(const GemmProblem& p, const uint16_t* x, const int32_t* row2assign,
                              const int32_t* offsets, const uint16_t* w13, uint16_t* act,
                              int* status, cudaStream_t stream, int* launches) {
  if (p.R == 0) return cudaSuccess;
  const bool relu2 = p.act == 1;
  if (!relu2 && use_swap_gemm(p.T))
    return launch_gemm1_swap(p, x, row2assign, offsets, w13, act, nullptr, 1, status, stream,
                             launches);
  if (use_pair_swap(p))
    return launch_gemm1_pair_swap(p, x, row2assign, offsets, w13, act, status, stream, launches);
  if (!relu2 && p.I % 128 == 0 && !use_gather4() && use_pair_gemm1(p.R, p.E))
    return launch_gemm1_bf16_2sm(p, x, row2assign, offsets, w13, act, status, stream, launches);
  // SwiGLU: 128 gate + 128 up rows per tile when I % 128 == 0, else 64 + 64;
  // ReLU2: 256 consecutive W1 rows per tile (the last tile's columns past I are dropped)
  const bool wide = relu2 || (p.I % 128) == 0;
  const int bn = wide ? 256 : 128;
  const int bn_out = relu2 ? bn : bn / 2;
  CUtensorMap ta, tb;
  CUtensorMap tc;
  if (!make_tmap_bf16(&ta, x, p.H, p.T, BK, 1) ||
      !make_tmap_bf16(&tb, w13, p.H, static_cast<uint64_t>(p.E) * (relu2 ? 1 : 2) * p.I, BK,
                      bn / 2) ||
      !make_tmap_epi(encode_fn(), &tc, act, p.I, p.R))
    return cudaErrorInvalidValue;
  KArgs a{};
  a.offsets = offsets;
  a.row2assign = row2assign;
  a.a_rows = x;
  a.out = act;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.I;
  a.K = p.H;
  a.n_tiles = (p.I + bn_out - 1) / bn_out;
  a.b_rows = (relu2 ? 1 : 2) * p.I;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  if (relu2) return run<true, kACpAsync, 256, 4, 1>(ta, tb, tc, a, stream);
  if (use_gather4())
    return wide ? run<true, kAGather4, 256, 4>(ta, tb, tc, a, stream)
                : run<true, kAGather4, 128, 6>(ta, tb, tc, a, stream);
  return wide ? run<true, kACpAsync, 256, 4>(ta, tb, tc, a, stream)
              : run<true, kACpAsync, 128, 6>(ta, tb, tc, a, stream);
}

cudaError_t launch_gemm2_bf16(const GemmProblem& p, const uint16_t* act, const int32_t* offsets,
                              const uint16_t* w2, uint16_t* y, int* status, cudaStream_t stream,
                              int* launches) {
  if (p.R == 0) return cudaSuccess;
  if (use_swap_gemm(p.T) && p.H % 128 == 0)
    return launch_gemm2_swap(p, act, offsets, w2, y, nullptr, 1, nullptr, status, stream,
                             launches);
  if (use_pair_swap(p))
    return launch_gemm2_pair_swap(p, act, offsets, w2, y, status, stream, launches);
  if (use_pair_gemm(p.R, p.E, p.I))
    return launch_gemm2_bf16_2sm(p, act, offsets, w2, y, status, stream, launches);
  constexpr int bn = 256;
  CUtensorMap ta, tb;
  CUtensorMap tc;
  if (!make_tmap_bf16(&ta, act, p.I, p.R, BK, BM) ||
      !make_tmap_bf16(&tb, w2, p.I, static_cast<uint64_t>(p.E) * p.H, BK, bn) ||
      !make_tmap_epi(encode_fn(), &tc, y, p.H, p.R))
    return cudaErrorInvalidValue;
  KArgs a{};
  a.offsets = offsets;
  a.out = y;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.H;
  a.K = p.I;
  a.n_tiles = (p.H + bn - 1) / bn;
  a.b_rows = p.H;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  return run<false, kATile, bn, 4>(ta, tb, tc, a, stream);
}

}  // namespace moe
