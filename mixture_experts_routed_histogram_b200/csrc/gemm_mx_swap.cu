// gemm_mx_swap.cu -- block-scaled grouped GEMMs for few tokens per expert, with the
// operands swapped: MXFP4 weight rows are the MMA's M=128 side (e2m1 A, K32 UE8M0 scales)
// and the e4m3 token rows its N side (1x128 scales).
//
// Sources: the FP8 x MXFP4 workload of FlashInfer PR #6465 (E=512, top-k 10: a few rows
// per expert until T is in the thousands; its tactic pool uses N16 / N64 tiles there) and
// GC-MoE (arXiv 2611.16219, abstract): FP4 weights as the A operand and FP8 activations as
// B in a block-scaled MMA for decode.  Operations as in gemm_mx.cu (TileScale PR #70
// "Design": GEMM1 + SwiGLU + 1x128 requantisation, GEMM2).
//
//   GEMM1: a task is 128 act features x NT token rows: its stages hold the 128 gate rows
//          and the 128 matching up rows of the weights (two MMAs per K step into two
//          accumulators), so each TMEM lane holds the gate and up sums of one feature for
//          all NT tokens; the per-token 1x128 requantisation reduces |act| over the 128
//          lanes (4 warps) through shared memory.
//   GEMM2: a task is 128 output features x NT token rows (act rows by TMA).
// Scale factors of each stage are gathered with 4-byte cp.async into 512-byte atoms and
// copied to TMEM with tcgen05.cp, as in gemm_mx.cu.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"
#include "launch.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int BMW = 128;  // weight rows per MMA (M)
constexpr int BK = 128;   // K elements per stage

struct MxSwapArgs {
  const int32_t* offsets;
  const int32_t* row2assign;  // GEMM1
  const uint8_t* xq;          // GEMM1: token rows e4m3 [T][K]
  const uint32_t* t_sfw;      // UE8M0 words of the token rows: [rows][K/128]
  const uint8_t* w_sf;        // UE8M0 bytes of the weights: [E * w_rows][K/32]
  void* out;                  // GEMM1: act e4m3 [R][I]; GEMM2: y bf16 [R][H]
  float* out_sf;              // GEMM1: act scales fp32 [R][I/128] (nullable)
  uint32_t* out_sfw;          // GEMM1: act scale words [R][I/128]
  int* status;
  int E, k_top;
  int n_out;                  // I (GEMM1) or H (GEMM2)
  int K;
  int ftiles;                 // 128-feature tiles per expert
  int w_rows;                 // weight rows per expert: 2I or H
  int64_t R;
  int inject_stall;
  uint64_t wait_limit_ns;
};

template <bool GEMM1, int NT, int STAGES, int NW2 = 1>
struct MxSwapCfg {
  static constexpr int THREADS = 32 * 7;                 // TMA, MMA, 4 epilogue, loader
  // weight tiles (MMAs) per stage: GEMM1 the gate and up tiles; GEMM2 one or two
  // consecutive 128-feature tiles
  static constexpr int NW = GEMM1 ? 2 : NW2;
  static constexpr int W_BYTES = NW * BMW * BK;          // smem (codes unpacked to bytes)
  static constexpr int W_TX = NW * BMW * BK / 2;         // bytes TMA moves
  static constexpr int T_BYTES = NT * BK;                // e4m3 token rows
  static constexpr int STAGE = W_BYTES + T_BYTES;
  static constexpr int SF_BYTES = (NW + 1) * 512;        // SFA per weight tile + SFB
  static constexpr int SF_OFF = STAGES * STAGE;
  static constexpr int RED_OFF = SF_OFF + STAGES * SF_BYTES;  // GEMM1: per-warp amax [4][NT]
  static constexpr int RED_BYTES = GEMM1 ? 4 * NT * 4 : 0;
  static constexpr int BAR_OFF = RED_OFF + RED_BYTES;
  static constexpr int NBAR = 2 * STAGES + 5;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int OFFS_OFF = MISC_OFF + 16;
  static constexpr int TILE_OFF = OFFS_OFF + 4 * (kMaxExperts + 1);
  static constexpr int TOTAL = TILE_OFF + 4 * (kMaxExperts + 1);
  static constexpr int ALLOC = TOTAL + 1024;
  static constexpr int ACC_COLS = NW * NT;               // one accumulator set
  static constexpr int SF_COLS = 4 * (NW + 1);
  static constexpr int SF_TMEM = 2 * ACC_COLS;
  static constexpr uint32_t TMEM_COLS = SF_TMEM + STAGES * SF_COLS <= 256 ? 256 : 512;
  static constexpr uint32_t FULL_COUNT = 1 + 32;
  static_assert(STAGE % 1024 == 0, "stage alignment");
  static_assert(SF_TMEM + STAGES * SF_COLS <= 512, "TMEM budget");
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void decode_mxs(int task, const int* s_tile, int E, int ftiles,
                                           int& e, int& tt, int& ft) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tile[mid] * ftiles <= task) lo = mid; else hi = mid;
  }
  e = lo;
  const int local = task - s_tile[e] * ftiles;
  tt = local / ftiles;
  ft = local - tt * ftiles;
}

__device__ __forceinline__ float silu_mul_mxs(float g, float u) {
  return g / (1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ int atom_off(int r) { return 16 * (r & 31) + 4 * (r >> 5); }

__device__ __forceinline__ void named_bar_sync_mxs(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int NT>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t (&r)[NT]) {
  if constexpr (NT == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
#pragma unroll
    for (int c = 0; c < NT; c += 32) {
      uint32_t t[32];
      tmem_ld_32x32b_x32(taddr + c, t);
#pragma unroll
      for (int i = 0; i < 32; ++i) r[c + i] = t[i];
    }
  }
}

template <bool GEMM1, int NT, int STAGES, int NW2>
__global__ void __launch_bounds__(MxSwapCfg<GEMM1, NT, STAGES, NW2>::THREADS, 1)
    mx_swap_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmT, const MxSwapArgs args) {
  using C = MxSwapCfg<GEMM1, NT, STAGES, NW2>;
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
  pdl_wait();
  pdl_launch_dependents();  // the next kernel's CTAs may take SMs as this grid's CTAs exit
  for (int i = threadIdx.x; i <= E; i += C::THREADS) s_off[i] = __ldg(args.offsets + i);
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
    if (lane == 31) s_tile[E] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = s_tile[E] * args.ftiles;
  const int kblocks = args.K / BK;
  const int G = args.K / 128;              // token scale words per row
  const int wsf_row = args.K / 32;         // weight scale bytes per row

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t fill = 0;
    int skipped = -1;
    bool ok = true;
    for (int task = blockIdx.x; task < total && ok; task += gridDim.x) {
      int e, tt, ft;
      decode_mxs(task, s_tile, E, args.ftiles, e, tt, ft);
      const int row0 = s_off[e] + tt * NT;
      const int wrow = e * args.w_rows + ft * BMW * (GEMM1 ? 1 : C::NW);
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
        uint8_t* w_dst = smem + s * C::STAGE;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], C::W_TX + (GEMM1 ? 0 : C::T_BYTES));
          tma_load_2d(w_dst, &tmW, &full[s], kb * BK, wrow);
          if constexpr (GEMM1) {
            tma_load_2d(w_dst + BMW * BK, &tmW, &full[s], kb * BK, wrow + args.n_out);  // up
          } else {
#pragma unroll
            for (int w = 1; w < C::NW; ++w)
              tma_load_2d(w_dst + w * BMW * BK, &tmW, &full[s], kb * BK, wrow + w * BMW);
            tma_load_2d(w_dst + C::W_BYTES, &tmT, &full[s], kb * BK, row0);
          }
        }
        __syncwarp();
      }
    }
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
      for (int task = blockIdx.x; task < total && ok; task += gridDim.x) {
        const int acc = tc & 1;
        const uint32_t aph = (tc >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, s_abort, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(acc * C::ACC_COLS);
        for (int kb = 0; kb < kblocks; ++kb, ++fill) {
          const int s = fill % STAGES;
          const uint32_t ph = (fill / STAGES) & 1u;
          if (!mbar_wait(&full[s], ph, s_abort, lim)) {
            ok = false;
            break;
          }
          fence_async_smem();
          tc_fence_after();
          const uint32_t sfc = tmem_base + static_cast<uint32_t>(C::SF_TMEM + s * C::SF_COLS);
          const uint32_t sfs = smem_u32(smem + C::SF_OFF + s * C::SF_BYTES);
#pragma unroll
          for (int b = 0; b < C::NW + 1; ++b)
            tmem_cp_32x128b_warpx4(sfc + 4 * b, rows16_desc(sfs + 512 * b));
          const uint32_t tsfb = sfc + 4 * C::NW;  // token scales follow the weight scales
          const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + s * C::STAGE + C::W_BYTES));
#pragma unroll
          for (int w = 0; w < C::NW; ++w) {
            const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + s * C::STAGE + w * BMW * BK));
#pragma unroll
            for (int ks = 0; ks < BK / 32; ++ks) {
              // A = e2m1 weights (format 5), B = e4m3 tokens (format 0), UE8M0 scales
              const uint32_t idesc = (static_cast<uint32_t>(ks) << 4) | (5u << 7) | (0u << 10) |
                                     (static_cast<uint32_t>(NT >> 3) << 17) | (1u << 23) |
                                     (static_cast<uint32_t>(BMW >> 4) << 24) |
                                     (static_cast<uint32_t>(ks) << 29);
              mma_mxf8f6f4_ss(d0 + static_cast<uint32_t>(w * NT), ad + 2 * ks, bd + 2 * ks, idesc,
                              (sfc + 4 * w) | (static_cast<uint32_t>(ks) << 30),
                              tsfb | (static_cast<uint32_t>(ks) << 30), (kb | ks) != 0 ? 1u : 0u);
            }
          }
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
    // ------------------------------------------------------------ cp.async loader
    // GEMM1: NT token rows (e4m3), the weight-scale atoms of the gate and up tiles and the
    // token-scale atom; GEMM2: the weight-scale atom and the token-scale atom.
    uint32_t fill = 0;
    bool ok = true;
    constexpr int ROWC = GEMM1 ? NT * 8 / 32 : 1;  // 16-byte token-row copies per lane
    for (int task = blockIdx.x; task < total && ok; task += gridDim.x) {
      int e, tt, ft;
      decode_mxs(task, s_tile, E, args.ftiles, e, tt, ft);
      const int row0 = s_off[e] + tt * NT;
      const int rows = min(NT, s_off[e + 1] - row0);
      const int64_t wrow = static_cast<int64_t>(e) * args.w_rows + ft * BMW * (GEMM1 ? 1 : C::NW);
      const uint8_t* trow[ROWC];
      int tdst[ROWC];
      if constexpr (GEMM1) {
#pragma unroll
        for (int i = 0; i < ROWC; ++i) {
          const int idx = lane + 32 * i;
          const int r = idx >> 3, chunk = idx & 7;
          const int tok = __ldg(args.row2assign + row0 + (r < rows ? r : 0)) / args.k_top;
          trow[i] = args.xq + static_cast<int64_t>(tok) * args.K + chunk * 16;
          tdst[i] = r * 128 + ((chunk ^ (r & 7)) << 4);
        }
      }
      for (int kb = 0; kb < kblocks; ++kb, ++fill) {
        const int s = fill % STAGES;
        const uint32_t ph = (fill / STAGES) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, s_abort, lim))) {
          ok = false;
          break;
        }
        const uint32_t sfs = smem_u32(smem + C::SF_OFF + s * C::SF_BYTES);
        if constexpr (GEMM1) {
          const uint32_t tb = smem_u32(smem + s * C::STAGE + C::W_BYTES);
#pragma unroll
          for (int i = 0; i < ROWC; ++i) cp_async_16(tb + tdst[i], trow[i] + kb * BK);
        }
        // weight scales: rows lane + 32 j of each weight tile
#pragma unroll
        for (int w = 0; w < C::NW; ++w)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int r = lane + 32 * j;
            const int64_t woff = GEMM1 ? (w ? args.n_out : 0) : w * BMW;
            const uint8_t* src = args.w_sf + (wrow + woff + r) * wsf_row + kb * 4;
            cp_async_4(sfs + 512 * w + atom_off(r), src);
          }
        // token scales: the NT rows of the tile (rows past the end reuse a valid row)
#pragma unroll
        for (int j = 0; j < (NT + 31) / 32; ++j) {
          const int r = lane + 32 * j;
          if (r < NT) {
            int64_t tr;
            if constexpr (GEMM1) {
              tr = __ldg(args.row2assign + row0 + (r < rows ? r : 0)) / args.k_top;
            } else {
              tr = min(static_cast<int64_t>(row0 + r), args.R - 1);
            }
            cp_async_4(sfs + 512 * C::NW + atom_off(r), args.t_sfw + tr * G + kb);
          }
        }
        cp_async_mbar_arrive_noinc(&full[s]);
      }
    }
    if (!ok && lane == 0) {
      *s_abort = 1;
      set_status(args.status, kStatusTimeout);
    }
    cp_async_wait_all();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int q = warp & 3;
    const int j = q * 32 + lane;  // feature (weight row) of the tile this thread holds
    float* red = reinterpret_cast<float*>(smem + C::RED_OFF);
    uint32_t tc = 0;
    bool ok = true;
    for (int task = blockIdx.x; task < total; task += gridDim.x) {
      int e, tt, ft;
      decode_mxs(task, s_tile, E, args.ftiles, e, tt, ft);
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
                          static_cast<uint32_t>(acc * C::ACC_COLS);
      if constexpr (GEMM1) {
        uint32_t g[NT], u[NT];
        tmem_ld_n<NT>(tb, g);
        tmem_ld_n<NT>(tb + NT, u);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        float a[NT];
#pragma unroll
        for (int c = 0; c < NT; ++c) {
          a[c] = silu_mul_mxs(__uint_as_float(g[c]), __uint_as_float(u[c]));
          float m = fabsf(a[c]);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
          if (lane == 0) red[q * NT + c] = m;
        }
        named_bar_sync_mxs(1, 128);
        uint8_t* act = static_cast<uint8_t*>(args.out);
#pragma unroll
        for (int c = 0; c < NT; ++c) {
          const float amax = fmaxf(fmaxf(red[c], red[NT + c]), fmaxf(red[2 * NT + c], red[3 * NT + c]));
          const int se = fp8_scale_exponent(amax);
          if (c < rows) {
            const int64_t row = row0 + c;
            act[row * args.n_out + ft * 128 + j] =
                static_cast<uint8_t>(cvt_e4m3x2(a[c] * pow2f(-se), 0.0f) & 0xFFu);
            if (j == 0) {
              const int64_t gi = row * (args.n_out / 128) + ft;
              if (args.out_sf) args.out_sf[gi] = pow2f(se);
              args.out_sfw[gi] = static_cast<uint32_t>(se + 127) * 0x01010101u;
            }
          }
        }
        named_bar_sync_mxs(1, 128);  // red[] is rewritten by the next task
      } else {
        uint32_t v[C::NW][NT];
#pragma unroll
        for (int w = 0; w < C::NW; ++w) tmem_ld_n<NT>(tb + w * NT, v[w]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        uint16_t* y = static_cast<uint16_t*>(args.out);
#pragma unroll
        for (int w = 0; w < C::NW; ++w) {
          const int o = (ft * C::NW + w) * BMW + j;
#pragma unroll
          for (int c = 0; c < NT; ++c)
            if (c < rows)
              y[static_cast<int64_t>(row0 + c) * args.n_out + o] =
                  static_cast<uint16_t>(pack_bf16x2(__uint_as_float(v[w][c]), 0.0f) & 0xFFFFu);
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

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_mxs() {
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

bool tmap_mxs(CUtensorMap* m, const void* ptr, bool fp4, uint64_t inner, uint64_t outer,
              uint32_t box_outer) {
  auto fn = encode_fn_mxs();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {fp4 ? inner / 2 : inner};
  cuuint32_t box[2] = {128, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, fp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
            const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool GEMM1, int NT, int NW2>
cudaError_t run_mxs(const CUtensorMap& w, const CUtensorMap& t, const MxSwapArgs& a,
                    cudaStream_t stream) {
  // as many stages as shared memory holds beside the reduction buffer and the bookkeeping
  // (two barriers per stage, five more, the expert offsets and tile starts, 1 KB of
  // alignment slack): the FP4 weight tiles take twice their HBM bytes once unpacked, so the
  // ring depth is what keeps enough HBM data in flight per SM
  using C1 = MxSwapCfg<GEMM1, NT, 1, NW2>;
  constexpr int FIXED = C1::RED_BYTES + 5 * 8 + 16 + 8 * (kMaxExperts + 1) + 1024;
  constexpr int STAGES0 = (227 * 1024 - FIXED) / (C1::STAGE + C1::SF_BYTES + 16);
  constexpr int STAGES = STAGES0 > 8 ? 8 : STAGES0;
  using Cf = MxSwapCfg<GEMM1, NT, STAGES, NW2>;
  auto kern = mx_swap_gemm_kernel<GEMM1, NT, STAGES, NW2>;
  static cudaError_t attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::ALLOC);
  if (attr != cudaSuccess) return attr;
  return launch_k(kern, dim3(num_sms()), dim3(Cf::THREADS), Cf::ALLOC, stream, w, t, a);
}

template <bool GEMM1, int NW2>
cudaError_t run_mxs_nt(int nt, const CUtensorMap& w, const CUtensorMap& t, const MxSwapArgs& a,
                       cudaStream_t stream) {
  switch (nt) {
    case 16: return run_mxs<GEMM1, 16, NW2>(w, t, a, stream);
    case 32: return run_mxs<GEMM1, 32, NW2>(w, t, a, stream);
    default: return run_mxs<GEMM1, 64, NW2>(w, t, a, stream);
  }
}

}  // namespace

// Few rows per expert (<= 48 on average): weights on the MMA's M side.
bool use_mx_swap(int64_t R, int E) { return R <= static_cast<int64_t>(E) * 48; }

static int mx_token_tile(int64_t R, int E) {
  const int64_t avg = (R + E - 1) / E;
  return avg <= 12 ? 16 : (avg <= 28 ? 32 : 64);
}

cudaError_t launch_gemm1_mx_swap(const GemmProblem& p, const uint8_t* xq, const uint32_t* sxw,
                                 const int32_t* row2assign, const int32_t* offsets,
                                 const uint8_t* w13p, const uint8_t* w13sf, uint8_t* act,
                                 float* act_sf, uint32_t* act_sfw, int* status,
                                 cudaStream_t stream, int* launches) {
  if (p.R == 0) return cudaSuccess;
  CUtensorMap tw, tt{};
  if (!tmap_mxs(&tw, w13p, true, p.H, static_cast<uint64_t>(p.E) * 2 * p.I, BMW))
    return cudaErrorInvalidValue;
  MxSwapArgs a{};
  a.offsets = offsets;
  a.row2assign = row2assign;
  a.xq = xq;
  a.t_sfw = sxw;
  a.w_sf = w13sf;
  a.out = act;
  a.out_sf = act_sf;
  a.out_sfw = act_sfw;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.I;
  a.K = p.H;
  a.ftiles = p.I / 128;
  a.w_rows = 2 * p.I;
  a.R = p.R;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  return run_mxs_nt<true, 1>(mx_token_tile(p.R, p.E), tw, tt, a, stream);
}

cudaError_t launch_gemm2_mx_swap(const GemmProblem& p, const uint8_t* act, const uint32_t* act_sfw,
                                 const int32_t* offsets, const uint8_t* w2p, const uint8_t* w2sf,
                                 uint16_t* y, int* status, cudaStream_t stream, int* launches) {
  if (p.R == 0) return cudaSuccess;
  const int nt = mx_token_tile(p.R, p.E);
  CUtensorMap tw, tt;
  if (!tmap_mxs(&tw, w2p, true, p.I, static_cast<uint64_t>(p.E) * p.H, BMW) ||
      !tmap_mxs(&tt, act, false, p.I, p.R, nt))
    return cudaErrorInvalidValue;
  MxSwapArgs a{};
  a.offsets = offsets;
  a.t_sfw = act_sfw;
  a.w_sf = w2sf;
  a.out = y;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.H;
  a.K = p.I;
  // two 128-feature weight tiles per task when H allows: twice the weight bytes per stage
  const bool pair = p.H % (2 * BMW) == 0 && nt <= 32;  // (64-row token tiles: registers)
  a.ftiles = p.H / (pair ? 2 * BMW : BMW);
  a.w_rows = p.H;
  a.R = p.R;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  if (pair) return nt == 16 ? run_mxs<false, 16, 2>(tw, tt, a, stream)
                            : run_mxs<false, 32, 2>(tw, tt, a, stream);
  return run_mxs_nt<false, 1>(nt, tw, tt, a, stream);
}

}  // namespace moe
