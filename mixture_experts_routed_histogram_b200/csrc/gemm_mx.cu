// gemm_mx.cu -- block-scaled grouped GEMMs: FP8 e4m3 activations with one power-of-two
// scale per 1x128 group x MXFP4 e2m1 weights with one UE8M0 scale per 32 K, on the
// sm_100a tensor cores (tcgen05.mma kind::mxf8f6f4.block_scale), fp32 accumulation.
//
//   GEMM1 + SwiGLU + requant: act = e4m3(silu(g)*u / s) with s the 1x128 power-of-two scale
//   GEMM2:                    y   = (act * s_act) . (W2 * s_w)^T, bf16 out
//
// Sources: TileScale PR #70 (distributed FP8 MegaMoE), "Design": FP8 E4M3 activations with
// fp32 per-128-element scales, kernel 1 = GEMM1 + SwiGLU quantising straight into its
// staging tile, kernel 2 = GEMM2; its description of keeping one TMA stage per scale group
// and issuing the scale loads at the top of the k-step.  FlashInfer PR #6465 (Hopper
// MXFP4 x FP8 MegaMoE), benchmark setup: MXFP4 weights with K32 scaling, FP8 activations,
// BF16 input/output, H=2560, E=512, top-k 10, I=640.
//
// Design (same persistent, warp-specialised skeleton as the BF16 kernels):
//   * a stage is K=128 (one 128-byte swizzled row of e4m3 per A row, and 128 e2m1 codes
//     per B row, which TMA unpacks to 128 bytes: 16 codes + an 8-byte gap per 16 bytes);
//   * the activation scale of a stage is one 1x128 group, i.e. the same UE8M0 byte for all
//     four K32 blocks; weight scales are K32 bytes as prepared;
//   * the scale factors of a stage sit in 512-byte atoms laid out as the MMA expects (row
//     r at byte 16*(r%32) + 4*(r/32), one byte per K32 block) and are copied into a
//     per-stage TMEM slot with tcgen05.cp before the stage's four MMAs.  GEMM1's loader
//     threads read their rows' scale words four stages ahead with plain 16-byte loads and
//     store them into the atoms; GEMM2's scale warp gathers them with 4-byte cp.async;
//   * GEMM1 tiles are 128 rows x (128 gate + 128 up) columns so that the SwiGLU output of a
//     tile is exactly one 1x128 requantisation group per row; its accumulator (256 TMEM
//     columns) is single-buffered to leave room for the scale slots, and the epilogue
//     hands it back as soon as it has read it.  GEMM2 tiles are 128 x 256 the same way
//     (H % 256 == 0), else 128 x 128 with a double-buffered accumulator.
#include <cudaTypedefs.h>

#include <mutex>

#include "epilogue.cuh"
#include "kernels.h"
#include "launch.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 128;  // elements per stage (one 128-byte swizzle row of 8-bit data)
constexpr int kLoaderWarps = 4;

struct MxArgs {
  const int32_t* offsets;    // [E+1]
  const int32_t* row2assign; // GEMM1
  const uint8_t* a_rows;     // GEMM1: xq [T][K] e4m3
  const uint32_t* a_sfw;     // UE8M0 words (byte x4) of A: [rows of A][K/128]
  const uint8_t* b_sf;       // UE8M0 bytes of B: [E * b_rows][K/32]
  void* out;                 // GEMM1: act e4m3 [R][I]; GEMM2: y bf16 [R][H]
  float* out_sf;             // GEMM1: act scales fp32 [R][I/128] (may be null)
  uint32_t* out_sfw;         // GEMM1: act scale words [R][I/128]
  int* status;
  int E, k_top;
  int n_out;                 // I (GEMM1) or H (GEMM2)
  int K;                     // H (GEMM1) or I (GEMM2)
  int n_tiles;
  int b_rows;                // 2I (GEMM1) or H (GEMM2)
  int64_t R;
  int inject_stall;
  uint64_t wait_limit_ns;
};

// GEMM2 runs with BN2 = 256 (one accumulator, handed back right after the epilogue has
// read it) when H % 256 == 0, else with BN2 = 128 (two accumulators).
template <bool GEMM1, int BN2, int STAGES>
struct MxCfg {
  static constexpr int BN = GEMM1 ? 256 : BN2;       // MMA N
  static constexpr int BN_OUT = GEMM1 ? 128 : BN2;   // output columns per tile
  static constexpr int NACC = BN == 256 ? 1 : 2;     // TMEM accumulators
  static constexpr int THREADS = GEMM1 ? 32 * (6 + kLoaderWarps) : 32 * 7;
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = BN * BK;            // shared-memory footprint
  static constexpr int B_TX = BN * BK / 2;           // bytes TMA moves for the codes
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int SF_BYTES = 512 + (BN / 128) * 512;
  static constexpr int SF_OFF = STAGES * STAGE;
  static constexpr int BAR_OFF = SF_OFF + STAGES * SF_BYTES;
  static constexpr int NBAR = 2 * STAGES + 5;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int OFFS_OFF = MISC_OFF + 16;
  static constexpr int TILE_OFF = OFFS_OFF + 4 * (kMaxExperts + 1);
  // GEMM2 stages its bf16 output through per-warp buffers for TMA stores
  static constexpr int EPI_OFF = (TILE_OFF + 4 * (kMaxExperts + 1) + 1023) / 1024 * 1024;
  static constexpr int TOTAL = EPI_OFF + (GEMM1 ? 0 : kEpiBytes);
  static constexpr int ALLOC = TOTAL + 1024;
  static constexpr int SF_COLS = 4 + BN / 32;        // TMEM columns per stage: SFA + SFB
  static constexpr int SF_TMEM = NACC * BN;
  static constexpr uint32_t TMEM_COLS = 512;
  // expect-tx arrival + per loader thread: GEMM1 a cp.async arrival and a store arrival,
  // GEMM2 (one scale warp) a cp.async arrival
  static constexpr uint32_t FULL_COUNT = 1 + (GEMM1 ? 2 * 32 * kLoaderWarps : 32);
  static_assert(STAGE % 1024 == 0, "stage alignment");
  static_assert(SF_TMEM + STAGES * SF_COLS <= static_cast<int>(TMEM_COLS), "TMEM budget");
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void decode_task_mx(int task, const int* s_tile, int E, int n_tiles,
                                               int& e, int& mt, int& nt) {
  int lo = 0, hi = E;
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
__device__ __forceinline__ float silu_mul_mx(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// byte offset of row r (0..127) in a 512-byte scale atom
__device__ __forceinline__ int sf_atom_off(int r) { return 16 * (r & 31) + 4 * (r >> 5); }

template <bool GEMM1, int BN2, int STAGES>
__global__ void __launch_bounds__(MxCfg<GEMM1, BN2, STAGES>::THREADS, 1)
    mx_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmC, const MxArgs args) {
  using C = MxCfg<GEMM1, BN2, STAGES>;
  constexpr int BN = C::BN;
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
    if constexpr (!GEMM1) tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();  // the offsets (and every other input) come from earlier kernels
  pdl_launch_dependents();  // the next kernel's CTAs may take SMs as this grid's CTAs exit
  for (int i = threadIdx.x; i <= E; i += C::THREADS) s_off[i] = __ldg(args.offsets + i);
  __syncthreads();
  if (warp == 0) {
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
  // Round r gives this CTA task r * P + (c + r) % P: an expert's m-tiles are neighbours in
  // the task order, and the rotation gives them CTAs of alternating parity round by round.
  // Without it the CTAs holding an expert's short last m-tile (always the odd ones at an
  // even grid) ran ahead of their partners, whose reads of the same weight tile then missed
  // L2: GEMM1 read 1.25-1.33x its algorithmic bytes from DRAM at T = 8192, 1.03x with it.
  auto task_of = [&](int r) {
    return r * static_cast<int>(gridDim.x) +
           static_cast<int>((blockIdx.x + static_cast<unsigned>(r)) % gridDim.x);
  };
  const int kblocks = args.K / BK;
  const int sf_row_bytes = args.K / 32;   // bytes of B scales per weight row

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    uint32_t fill = 0;
    int skipped = -1;
    bool ok = true;
    for (int round = 0, task = task_of(0); task < total && ok; task = task_of(++round)) {
      int e, mt, nt;
      decode_task_mx(task, s_tile, E, args.n_tiles, e, mt, nt);
      const int row0 = s_off[e] + mt * BM;
      const int brow = e * args.b_rows + nt * C::BN_OUT;
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
        if (lane == 0) {
          if constexpr (GEMM1) {
            mbar_arrive_expect_tx(&full[s], C::B_TX);
            tma_load_2d(b_dst, &tmB, &full[s], kb * BK, brow);
            tma_load_2d(b_dst + 128 * BK, &tmB, &full[s], kb * BK, brow + args.n_out);
          } else {
            mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_TX);
            tma_load_2d(a_dst, &tmA, &full[s], kb * BK, row0);
#pragma unroll
            for (int b = 0; b < BN / 128; ++b)
              tma_load_2d(b_dst + b * 128 * BK, &tmB, &full[s], kb * BK, brow + 128 * b);
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
      for (int round = 0, task = task_of(0); task < total && ok; task = task_of(++round)) {
        const int acc = C::NACC == 2 ? static_cast<int>(tc & 1) : 0;
        const uint32_t aph = C::NACC == 2 ? (tc >> 1) & 1u : tc & 1u;
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
          fence_async_smem();  // cp.async-written scales and rows -> tcgen05 reads
          tc_fence_after();
          const uint32_t sf_col = tmem_base + static_cast<uint32_t>(C::SF_TMEM + s * C::SF_COLS);
          const uint32_t sf_smem = smem_u32(smem + C::SF_OFF + s * C::SF_BYTES);
          tmem_cp_32x128b_warpx4(sf_col, rows16_desc(sf_smem));
#pragma unroll
          for (int b = 0; b < BN / 128; ++b)
            tmem_cp_32x128b_warpx4(sf_col + 4 + 4 * b, rows16_desc(sf_smem + 512 + 512 * b));
          const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + s * C::STAGE));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + s * C::STAGE + C::A_BYTES));
#pragma unroll
          for (int ks = 0; ks < BK / 32; ++ks)
            mma_mxf8f6f4_ss(d_tmem, ad + 2 * ks, bd + 2 * ks,
                            idesc_mx_e4m3_e2m1<BM, BN>(static_cast<uint32_t>(ks)),
                            sf_col | (static_cast<uint32_t>(ks) << 30),
                            (sf_col + 4) | (static_cast<uint32_t>(ks) << 30),
                            (kb | ks) != 0 ? 1u : 0u);
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
  } else if (warp >= 6) {
    // ------------------------------------------------------------ cp.async loaders
    uint32_t fill = 0;
    bool ok = true;
    if constexpr (GEMM1) {
      // A rows (e4m3) + the stage's scale atoms: 128 threads, thread t owns scale row t.
      // The rows go by 16-byte cp.async (tracked by the no-increment arrival); the scale
      // words of the thread's three rows (token row of A, gate and up rows of B) are read
      // with plain loads one group of 4 stages ahead, written into the stage's atoms with
      // st.shared and published by a second, regular arrival after a proxy fence.
      const int lw = warp - 6;
      const int sub = lane >> 3;
      const int chunk = lane & 7;
      const int t = lw * 32 + lane;
      const int G = args.K / 128;          // scale words per row (one per K=128 stage)
      // rows start on 16 bytes (4 words per load) when G % 4 == 0 and both bases are aligned
      const bool vec = (G & 3) == 0 && ((reinterpret_cast<uintptr_t>(args.a_sfw) |
                                         reinterpret_cast<uintptr_t>(args.b_sf)) & 15u) == 0;
      for (int round = 0, task = task_of(0); task < total && ok; task = task_of(++round)) {
        int e, mt, nt;
        decode_task_mx(task, s_tile, E, args.n_tiles, e, mt, nt);
        const int row0 = s_off[e] + mt * BM;
        const int rows = min(BM, s_off[e + 1] - row0);
        const uint8_t* src[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = lw * 32 + i * 4 + sub;
          const int tok = __ldg(args.row2assign + row0 + (r < rows ? r : 0)) / args.k_top;
          src[i] = args.a_rows + static_cast<int64_t>(tok) * args.K + chunk * 16;
        }
        const int tok_t = __ldg(args.row2assign + row0 + (t < rows ? t : 0)) / args.k_top;
        const int64_t brow = static_cast<int64_t>(e) * args.b_rows + nt * C::BN_OUT;
        const uint32_t* wrow[3] = {
            args.a_sfw + static_cast<int64_t>(tok_t) * G,
            reinterpret_cast<const uint32_t*>(args.b_sf + (brow + t) * sf_row_bytes),
            reinterpret_cast<const uint32_t*>(args.b_sf + (brow + args.n_out + t) * sf_row_bytes)};
        uint32_t cw[3][4], nw[3][4];
        auto load_group = [&](int g0, uint32_t (&w)[3][4]) {
#pragma unroll
          for (int r = 0; r < 3; ++r) {
            if (vec) {
              const uint4 v = __ldg(reinterpret_cast<const uint4*>(wrow[r] + g0));
              w[r][0] = v.x; w[r][1] = v.y; w[r][2] = v.z; w[r][3] = v.w;
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j) w[r][j] = g0 + j < G ? __ldg(wrow[r] + g0 + j) : 0u;
            }
          }
        };
        load_group(0, cw);
        const int sfo = sf_atom_off(t);
        for (int kb = 0; kb < kblocks; ++kb, ++fill) {
          const int gi = kb & 3;
          if (gi == 0 && kb + 4 < kblocks) load_group(kb + 4, nw);
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
          const uint32_t sf_base = smem_u32(smem + C::SF_OFF + s * C::SF_BYTES);
#pragma unroll
          for (int r = 0; r < 3; ++r) {
            const uint32_t v = gi == 0 ? cw[r][0] : gi == 1 ? cw[r][1] : gi == 2 ? cw[r][2] : cw[r][3];
            st_shared_b32(sf_base + 512 * r + sfo, v);
          }
          fence_async_smem();  // the atom words (generic proxy) -> tcgen05.cp (async proxy)
          cp_async_mbar_arrive_noinc(&full[s]);
          mbar_arrive(&full[s]);
          if (gi == 3) {
#pragma unroll
            for (int r = 0; r < 3; ++r)
#pragma unroll
              for (int j = 0; j < 4; ++j) cw[r][j] = nw[r][j];
          }
        }
      }
    } else {
      // one warp: the stage's scale atoms (128 A rows, BN B rows) -- 4 + BN/32 words per lane
      const int G = args.K / 128;
      for (int round = 0, task = task_of(0); task < total && ok; task = task_of(++round)) {
        int e, mt, nt;
        decode_task_mx(task, s_tile, E, args.n_tiles, e, mt, nt);
        const int64_t row0 = s_off[e] + mt * BM;
        const int64_t brow = static_cast<int64_t>(e) * args.b_rows + nt * C::BN_OUT;
        const uint32_t* sfa_src[4];
        const uint8_t* sfb_src[BN / 32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = lane + 32 * j;
          const int64_t ra = min(row0 + r, args.R - 1);  // rows past the end: any valid row
          sfa_src[j] = args.a_sfw + ra * G;
        }
#pragma unroll
        for (int j = 0; j < BN / 32; ++j)
          sfb_src[j] = args.b_sf + (brow + lane + 32 * j) * sf_row_bytes;
        for (int kb = 0; kb < kblocks; ++kb, ++fill) {
          const int s = fill % STAGES;
          const uint32_t ph = (fill / STAGES) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, s_abort, lim))) {
            ok = false;
            break;
          }
          const uint32_t sf_base = smem_u32(smem + C::SF_OFF + s * C::SF_BYTES);
#pragma unroll
          for (int j = 0; j < 4; ++j)  // row lane + 32 j of the atom
            cp_async_4(sf_base + 16 * lane + 4 * j, sfa_src[j] + kb);
#pragma unroll
          for (int j = 0; j < BN / 32; ++j)  // B row lane + 32 j: atom j / 4, slot j % 4
            cp_async_4(sf_base + 512 + 512 * (j >> 2) + 16 * lane + 4 * (j & 3),
                       sfb_src[j] + kb * 4);
          cp_async_mbar_arrive_noinc(&full[s]);
        }
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
    const int r_in = q * 32 + lane;
    EpiStager st{smem_u32(smem + C::EPI_OFF + q * kEpiWarpBytes), 0u};
    uint32_t tc = 0;
    bool ok = true;
    for (int round = 0, task = task_of(0); task < total; task = task_of(++round)) {
      int e, mt, nt;
      decode_task_mx(task, s_tile, E, args.n_tiles, e, mt, nt);
      const int row0 = s_off[e] + mt * BM;
      const int rows = min(BM, s_off[e + 1] - row0);
      const int acc = C::NACC == 2 ? static_cast<int>(tc & 1) : 0;
      const uint32_t aph = C::NACC == 2 ? (tc >> 1) & 1u : tc & 1u;
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
        // one pass over the accumulator: the row's 128 SwiGLU outputs stay in registers and
        // the accumulator goes back to the MMA warp before the requantisation and the stores
        // (it is single-buffered, so the next tile's MMAs wait for exactly this much)
        float a[128];
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < 128; c += 16) {
          uint32_t g[16], u[16];
          tmem_ld_32x32b_x16(tb + c, g);
          tmem_ld_32x32b_x16(tb + 128 + c, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            a[c + i] = silu_mul_mx(__uint_as_float(g[i]), __uint_as_float(u[i]));
            amax = fmaxf(amax, fabsf(a[c + i]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        const int se = fp8_scale_exponent(amax);
        const float inv = pow2f(-se);
        if (valid) {
          // e4m3 codes of act / 2^se: the row's 128 bytes as eight 16-byte stores
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) +
                                                row * args.n_out + nt * 128);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float* p = a + 16 * v + 4 * i;
              w[i] = static_cast<uint32_t>(cvt_e4m3x2(p[0] * inv, p[1] * inv)) |
                     (static_cast<uint32_t>(cvt_e4m3x2(p[2] * inv, p[3] * inv)) << 16);
            }
            dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          const int64_t gi = row * (args.n_out / 128) + nt;
          if (args.out_sf) args.out_sf[gi] = pow2f(se);
          args.out_sfw[gi] = static_cast<uint32_t>(se + 127) * 0x01010101u;
        }
      } else if constexpr (C::NACC == 1) {
        // single accumulator: read all BN columns as packed bf16 pairs, hand the
        // accumulator back to the MMA warp, then stage and store
        uint16_t* y = static_cast<uint16_t*>(args.out);
        uint32_t pk[BN / 32][16];
#pragma unroll
        for (int c = 0; c < BN / 32; c += 2) {
          uint32_t v0[32], v1[32];
          tmem_ld_32x32b_x32(tb + 32 * c, v0);
          tmem_ld_32x32b_x32(tb + 32 * c + 32, v1);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            pk[c][i] = pack_bf16x2(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]));
            pk[c + 1][i] = pack_bf16x2(__uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          const int col = nt * C::BN_OUT + 32 * c;
          if (col < args.n_out) {
            if (whole)
              epi_store_chunk(st, &tmC, pk[c], col, row0 + q * 32, lane);
            else if (valid)
              epi_store_row(y + row * args.n_out + col, pk[c]);
          }
        }
      } else {
        uint16_t* y = static_cast<uint16_t*>(args.out);
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v32[32];
          tmem_ld_32x32b_x32(tb + c, v32);
          tmem_ld_wait();
          const int col = nt * C::BN_OUT + c;
          if (col < args.n_out) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(v32[2 * i]), __uint_as_float(v32[2 * i + 1]));
            if (whole)
              epi_store_chunk(st, &tmC, pk, col, row0 + q * 32, lane);
            else if (valid)
              epi_store_row(y + row * args.n_out + col, pk);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
      }
      ++tc;
    }
    if (!ok && lane == 0) {
      *s_abort = 1;
      set_status(args.status, kStatusTimeout);
    }
    if constexpr (!GEMM1) epi_drain(lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// fp32 power-of-two scales -> UE8M0 words (the byte repeated for the four K32 blocks)
__global__ void scale_words_kernel(const float* __restrict__ s, uint32_t* __restrict__ w,
                                   int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  if (i >= n) return;
  int e;
  frexpf(__ldg(s + i), &e);  // 2^p = 0.5 * 2^(p+1)
  int b = e + 126;
  b = b < 0 ? 0 : (b > 254 ? 254 : b);
  w[i] = static_cast<uint32_t>(b) * 0x01010101u;
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_mx() {
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

// 8-bit [outer][inner] matrix (e4m3 codes), box {128, box_outer}, 128-byte swizzle.
bool make_tmap_u8(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                  uint32_t box_outer) {
  auto fn = encode_fn_mx();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {128, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed e2m1 [outer][inner] (inner counted in 4-bit codes, 2 per byte), unpacked by TMA
// into 16-byte groups of 16 codes + 8 bytes of gap; box {128 codes, box_outer}.
bool make_tmap_fp4(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                   uint32_t box_outer) {
  auto fn = encode_fn_mx();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner / 2};
  cuuint32_t box[2] = {128, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(ptr), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool GEMM1, int BN2, int STAGES>
cudaError_t run_mx(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                   const MxArgs& args, cudaStream_t stream) {
  using Cf = MxCfg<GEMM1, BN2, STAGES>;
  auto kern = mx_grouped_gemm_kernel<GEMM1, BN2, STAGES>;
  static cudaError_t attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::ALLOC);
  if (attr != cudaSuccess) return attr;
  return launch_k(kern, dim3(num_sms()), dim3(Cf::THREADS), Cf::ALLOC, stream, a, b, c, args);
}

}  // namespace

cudaError_t launch_scale_words(const float* s, uint32_t* w, int64_t n, cudaStream_t stream,
                               int* launches) {
  if (n == 0) return cudaSuccess;
  ++*launches;
  return launch_k(scale_words_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0,
                  stream, s, w, n);
}

cudaError_t launch_gemm1_mx(const GemmProblem& p, const uint8_t* xq, const uint32_t* sxw,
                            const int32_t* row2assign, const int32_t* offsets,
                            const uint8_t* w13p, const uint8_t* w13sf, uint8_t* act,
                            float* act_sf, uint32_t* act_sfw, int* status, cudaStream_t stream,
                            int* launches) {
  if (p.R == 0) return cudaSuccess;
  if (use_mx_swap(p.R, p.E))
    return launch_gemm1_mx_swap(p, xq, sxw, row2assign, offsets, w13p, w13sf, act, act_sf,
                                act_sfw, status, stream, launches);
  CUtensorMap ta{}, tb, tc{};
  if (!make_tmap_fp4(&tb, w13p, p.H, static_cast<uint64_t>(p.E) * 2 * p.I, 128))
    return cudaErrorInvalidValue;
  MxArgs a{};
  a.offsets = offsets;
  a.row2assign = row2assign;
  a.a_rows = xq;
  a.a_sfw = sxw;
  a.b_sf = w13sf;
  a.out = act;
  a.out_sf = act_sf;
  a.out_sfw = act_sfw;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.I;
  a.K = p.H;
  a.n_tiles = p.I / 128;
  a.b_rows = 2 * p.I;
  a.R = p.R;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  return run_mx<true, 256, 4>(ta, tb, tc, a, stream);
}

cudaError_t launch_gemm2_mx(const GemmProblem& p, const uint8_t* act, const uint32_t* act_sfw,
                            const int32_t* offsets, const uint8_t* w2p, const uint8_t* w2sf,
                            uint16_t* y, int* status, cudaStream_t stream, int* launches) {
  if (p.R == 0) return cudaSuccess;
  if (use_mx_swap(p.R, p.E))
    return launch_gemm2_mx_swap(p, act, act_sfw, offsets, w2p, w2sf, y, status, stream, launches);
  CUtensorMap ta, tb, tc;
  if (!make_tmap_u8(&ta, act, p.I, p.R, BM) ||
      !make_tmap_fp4(&tb, w2p, p.I, static_cast<uint64_t>(p.E) * p.H, 128) ||
      !make_tmap_epi(encode_fn_mx(), &tc, y, p.H, p.R))
    return cudaErrorInvalidValue;
  MxArgs a{};
  a.offsets = offsets;
  a.a_sfw = act_sfw;
  a.b_sf = w2sf;
  a.out = y;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.H;
  a.K = p.I;
  const bool wide = p.H % 256 == 0;
  a.n_tiles = p.H / (wide ? 256 : 128);
  a.b_rows = p.H;
  a.R = p.R;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  return wide ? run_mx<false, 256, 4>(ta, tb, tc, a, stream)
              : run_mx<false, 128, 6>(ta, tb, tc, a, stream);
}

}  // namespace moe
