// gemm_pair_swap.cu -- the BF16 grouped GEMMs of large batches on SM pairs with the
// operands swapped: the expert's weight rows are the MMA's M = 256 side (128 per CTA of
// the pair) and the expert's routed token rows are its N side, in chunks of up to 256.
//
//   GEMM1 + SwiGLU: act[r][i] = silu(x[tok(r)] . W13[e][i]) * (x[tok(r)] . W13[e][I+i])
//   GEMM1 + ReLU2:  act[r][i] = max(x[tok(r)] . W1[e][i], 0)^2
//   GEMM2:          y[r][o]   = act[r] . W2[e][o]
//
// Sources: TileScale PR #70 (distributed FP8 MegaMoE), "Design" -- kernel 1 is GEMM1 with
// SwiGLU fused into its epilogue, kernel 2 is GEMM2, tasks come from a flat queue built
// from the expert offsets (its first listed change), and the MMA overwrites the
// accumulator on the first k-step.  FlashInfer PR #5129 (cuTile BF16 fused MoE), "sorted
// I/O": GEMM1 gathers token rows and writes expert-sorted rows, which GEMM2 reads
// contiguously.  GC-MoE (abstract) and FlashInfer PR #6465 put the weights on the large
// MMA dimension and the tokens on the small one; here that is done for every batch size.
//
// Why this shape on B200.  A tcgen05 pair MMA (cta_group::2, M = 256) reads the N-side
// operand half from each CTA, so per SM and per K = 64 step the ring moves 16 KB of weights
// plus at most 16 KB of token rows for a 128 x 256 x 64 block of MMA work -- a third less
// than the 48 KB of a single-SM 128 x 256 tile.  Filling shared memory and the MMA's
// operand reads set the pace of both, not the tensor pipe: timing-only copies of this
// kernel took 0.65x the time with no MMAs and reached ~1.58 PFLOP/s on the tensor pipe with
// every MMA issued twice, while one 256-token MMA set per 32 KB stage runs at ~716 SM clocks
// against 512 of MMA work.  And because N may be any multiple of 16 up to 256, an expert's
// last chunk is padded to 16 rows, not to a 128- or 256-row tile.
//
// Tasks: (expert e, feature tile ft, token chunk c), chunk-fastest, so the pairs running at
// the same time share each weight tile through L2.  Chunk c covers sorted rows
// [offsets[e] + 256c, +256) of the expert (the last one fewer); N = that count rounded up
// to 16; CTA r of the pair stages token rows [r * N/2, (r+1) * N/2) of the chunk.
//   SwiGLU: feature tile = 128 act columns; CTA r holds 128 weight rows for act columns
//           [128 ft + 64 r, +64), loaded through a 5-D view of W13 as four blocks of (16
//           gate rows, the 16 matching up rows), so TMEM lanes 32q..32q+15 hold gate sums
//           and lanes 32q+16..32q+31 the up sums of the same 16 features.
//   ReLU2 / GEMM2: feature tile = 256 W1 / W2 rows; CTA r holds rows [256 ft + 128 r, +128).
// Weight rows past the expert's own (a ragged last feature tile) read the next expert's
// rows or the tensor map's zero fill; their outputs are never stored.
//
// Roles per CTA: warp 0 TMA producer (weights; GEMM2 also the token rows, one 128-row box
// per stage), warp 1 TMEM owner and, in the leader CTA, the MMA issuer,
// warps 2-5 epilogue, and for GEMM1 warps 6-9 gather the token rows of x with 16-byte
// cp.async and warp 10 relays "this CTA's rows of the stage have landed" to the leader.
// Pair protocol: full[s] lives in the leader and counts both CTAs'
// TMA bytes (one expect-tx arrival by the leader) plus, for GEMM1, one relay arrival per
// CTA; the leader's commits multicast to both CTAs' empty[s] and tfull[acc]; tempty[acc]
// in the leader takes one arrival per epilogue warp of either CTA.  Every wait is bounded;
// a CTA that gives up also raises its partner's abort flag, so the pair unwinds together.
//
// Epilogue: the accumulator holds [feature (lane)][token (column)], the transpose of the
// row-major output.  A warp reads 32-token blocks of its lane quadrant with tcgen05.ld
// 16x256b (the m16n8 accumulator fragment), applies SwiGLU / ReLU2, packs token pairs into
// bf16x2 and writes token rows with stmatrix .trans into a swizzled staging buffer, which
// one TMA tensor store writes out when all 32 rows belong to the chunk (else row by row, so
// the next expert's rows are never touched).
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"
#include "launch.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int BK = 64;           // bf16 elements per 128-byte swizzled row
constexpr int kChunk = 256;      // token rows per task at most (MMA N)
constexpr int kHalf = kChunk / 2;
constexpr int WROWS = 128;       // weight rows per CTA (MMA M = 256 per pair)
constexpr int kLoaderWarps = 4;
constexpr int kRelayWarp = 6 + kLoaderWarps;

enum Mode : int { kSwiGLU = 0, kReLU2 = 1, kGemm2 = 2 };

struct PsArgs {
  const int32_t* offsets;      // [E+1]
  const int32_t* row2assign;   // GEMM1
  const uint16_t* x;           // GEMM1: token rows [T][K]
  uint16_t* out;               // act [R][I] (GEMM1) or y [R][H] (GEMM2)
  int* status;
  int E, k_top;
  int n_out;                   // output columns: I (GEMM1) or H (GEMM2)
  int K;                       // reduction length: H (GEMM1) or I (GEMM2)
  int ftiles;                  // feature tiles per expert
  int b_rows;                  // weight rows per expert: 2I, I (ReLU2) or H
  int inject_stall;
  uint64_t wait_limit_ns;
};

template <int MODE, int STAGES>
struct PsCfg {
  static constexpr bool GATHER = MODE != kGemm2;
  static constexpr int THREADS = GATHER ? 32 * (7 + kLoaderWarps) : 192;
  static constexpr int A_BYTES = WROWS * BK * 2;    // 16 KB of weight rows
  static constexpr int B_BYTES = kHalf * BK * 2;    // up to 16 KB of token rows
  static constexpr int STAGE = A_BYTES + B_BYTES;
  // epilogue staging: 32 token rows of the warp's features (SwiGLU 16, else 32) per store
  static constexpr int ROW_BYTES = MODE == kSwiGLU ? 32 : 64;
  static constexpr int STG_BYTES = 32 * ROW_BYTES;
  static constexpr int EPI_OFF = STAGES * STAGE;
  static constexpr int EPI_BYTES = 4 * 2 * STG_BYTES;         // 4 warps, double-buffered
  static constexpr int BAR_OFF = EPI_OFF + EPI_BYTES;
  // full, empty, afull per stage; tfull x2, tempty x2, drain
  static constexpr int NBAR = 3 * STAGES + 5;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int OFFS_OFF = MISC_OFF + 16;
  static constexpr int TILE_OFF = OFFS_OFF + 4 * (kMaxExperts + 1);
  static constexpr int TOTAL = TILE_OFF + 4 * (kMaxExperts + 1);
  static constexpr int ALLOC = TOTAL + 1024;   // slack for the 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 2 * kChunk;
  static constexpr uint32_t FULL_COUNT = GATHER ? 1 + 2 : 1;
  static_assert(STAGE % 1024 == 0 && EPI_OFF % 1024 == 0, "alignment");
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

// task -> (expert, feature tile, chunk): tasks of expert e occupy
// [s_tile[e] * ftiles, s_tile[e+1] * ftiles), chunk-fastest.
__device__ __forceinline__ void decode_ps(int task, const int* s_tile, int E, int ftiles, int& e,
                                          int& ft, int& ch) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tile[mid] * ftiles <= task) lo = mid; else hi = mid;
  }
  e = lo;
  const int local = task - s_tile[e] * ftiles;
  const int nck = s_tile[e + 1] - s_tile[e];
  ft = local / nck;
  ch = local - ft * nck;
}

// A chunk's rows: the first sorted row, the rows that belong to the expert, the MMA's N.
struct Chunk {
  int row0, nvalid, n;
};
__device__ __forceinline__ Chunk chunk_of(const int* s_off, int e, int ch) {
  Chunk c;
  c.row0 = s_off[e] + ch * kChunk;
  c.nvalid = min(kChunk, s_off[e + 1] - c.row0);
  c.n = (c.nvalid + 15) & ~15;
  return c;
}

__device__ __forceinline__ float silu_mul_ps(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;  // 0 once the denominator overflows
}

__device__ __forceinline__ float relu2_ps(float g) { return g > 0.0f ? g * g : 0.0f; }

// One warp's output staging: 32 token rows of ROW_BYTES (the warp's features, bf16) in the
// TMA swizzle of that row width (ROW_BYTES 64: 16-byte unit u of row r at u ^ ((r >> 1) & 3);
// 32: at u ^ ((r >> 2) & 1)), double-buffered.  Every block commits one bulk async-group
// (empty when its rows were stored directly), so before a buffer is written again its store
// from two blocks earlier has read it once at most one newer group is pending.
template <int ROW_BYTES>
struct Stager {
  uint32_t base;  // this warp's two buffers
  uint32_t n;     // blocks staged so far
  static __device__ __forceinline__ uint32_t unit_addr(uint32_t buf, int row, int unit) {
    const uint32_t sw = ROW_BYTES == 64 ? (static_cast<uint32_t>(row >> 1) & 3u)
                                        : (static_cast<uint32_t>(row >> 2) & 1u);
    return buf + static_cast<uint32_t>(row * ROW_BYTES) +
           ((static_cast<uint32_t>(unit) ^ sw) << 4);
  }
  __device__ __forceinline__ uint32_t next(int lane) {
    const uint32_t buf = base + (n & 1u) * static_cast<uint32_t>(32 * ROW_BYTES);
    if (n >= 2 && lane == 0) bulk_wait_group_read<1>();
    __syncwarp();
    ++n;
    return buf;
  }
  // Store the staged rows (this warp's features at column `col`) at sorted rows row0..:
  // one TMA box of 32 rows when all of them are the chunk's (`rows` >= 32), else row by
  // row (lane j copies row j), so the next expert's rows are never touched.
  __device__ __forceinline__ void store(uint32_t buf, const CUtensorMap* tm, uint16_t* out,
                                        int n_out, int col, int row0, int rows, int lane) {
    fence_async_smem();   // generic-proxy writes -> the TMA engine's reads
    __syncwarp();
    if (rows >= 32) {
      if (lane == 0) tma_store_2d(tm, buf, col, row0);
    } else if (lane < rows) {
      uint4* d = reinterpret_cast<uint4*>(out + static_cast<int64_t>(row0 + lane) * n_out + col);
#pragma unroll
      for (int u = 0; u < ROW_BYTES / 16; ++u) d[u] = ld_shared_v4(unit_addr(buf, lane, u));
    }
    if (lane == 0) bulk_commit_group();
  }
};

// One 32-token block (columns cb.. of the accumulator) of an epilogue warp, through the
// m16n8 fragment layout: tcgen05.ld 16x256b gives thread t the values of features t/4 and
// t/4 + 8 (of a 16-lane group) for token pairs 2(t%4), 2(t%4)+1 of every 8-token chunk; a
// pair packs into one bf16x2 register, i.e. one row of an 8x8 (feature x token) matrix, and
// stmatrix .trans writes its columns -- token rows of 8 features, 16 bytes -- into the
// staging buffer.  NB = 32, or 16 for a chunk's last half block.
//   SwiGLU: lanes 0-15 of the warp's quadrant hold gate sums, lanes 16-31 the up sums of
//           the same 16 features: act = silu(g) * u, 16 features per token row.
//   else:   lanes 0-15 and 16-31 are 32 consecutive features (ReLU2 applies max(.,0)^2).
template <int MODE, int NB>
__device__ __forceinline__ void epi_block(uint32_t tq, uint32_t buf, int lane) {
  constexpr int CH = NB / 8;   // 8-token chunks
  uint32_t a[16], b[16];
  if constexpr (NB == 32) {
    tmem_ld_16x256b_x4(tq, a);
    tmem_ld_16x256b_x4(tq + (16u << 16), b);
  } else {
    tmem_ld_16x256b_x2(tq, a);
    tmem_ld_16x256b_x2(tq + (16u << 16), b);
  }
  tmem_ld_wait();
  const int i = lane >> 3, j = lane & 7;   // this lane addresses row j of matrix i
  if constexpr (MODE == kSwiGLU) {
    uint32_t p[8];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      p[2 * c] = pack_bf16x2(silu_mul_ps(__uint_as_float(a[4 * c]), __uint_as_float(b[4 * c])),
                             silu_mul_ps(__uint_as_float(a[4 * c + 1]),
                                         __uint_as_float(b[4 * c + 1])));
      p[2 * c + 1] = pack_bf16x2(
          silu_mul_ps(__uint_as_float(a[4 * c + 2]), __uint_as_float(b[4 * c + 2])),
          silu_mul_ps(__uint_as_float(a[4 * c + 3]), __uint_as_float(b[4 * c + 3])));
    }
    // matrices (features 0-7 | 8-15) x (chunk 2m | 2m+1): token row 8(2m + i/2) + j, unit i%2
#pragma unroll
    for (int m = 0; m < CH / 2; ++m)
      stmatrix_x4_trans(Stager<32>::unit_addr(buf, 8 * (2 * m + (i >> 1)) + j, i & 1), p[4 * m],
                        p[4 * m + 1], p[4 * m + 2], p[4 * m + 3]);
  } else {
    auto f = [](uint32_t v) {
      const float x = __uint_as_float(v);
      return MODE == kReLU2 ? relu2_ps(x) : x;
    };
    // chunk c: matrices of features 0-7, 8-15 (a) and 16-23, 24-31 (b) -> units 0..3
#pragma unroll
    for (int c = 0; c < CH; ++c)
      stmatrix_x4_trans(Stager<64>::unit_addr(buf, 8 * c + j, i),
                        pack_bf16x2(f(a[4 * c]), f(a[4 * c + 1])),
                        pack_bf16x2(f(a[4 * c + 2]), f(a[4 * c + 3])),
                        pack_bf16x2(f(b[4 * c]), f(b[4 * c + 1])),
                        pack_bf16x2(f(b[4 * c + 2]), f(b[4 * c + 3])));
  }
}

template <int MODE, int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PsCfg<MODE, STAGES>::THREADS, 1)
    pair_swap_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                          const __grid_constant__ CUtensorMap tmT,
                          const __grid_constant__ CUtensorMap tmO, const PsArgs args) {
  using C = PsCfg<MODE, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* afull = empty + STAGES;   // GEMM1: this CTA's gathered rows of a stage landed
  uint64_t* tfull = afull + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
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
      mbar_init(&afull[s], 32 * kLoaderWarps);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    *s_never = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    if constexpr (MODE == kGemm2) tma_prefetch_desc(&tmT);
  }
  if (warp == 1) {
    tmem_alloc_2sm(s_tmem, C::TMEM_COLS);
    tmem_relinquish_2sm();
  }
  pdl_wait();  // the offsets (and every other input) come from earlier kernels
  pdl_launch_dependents();
  for (int i = threadIdx.x; i <= E; i += C::THREADS) s_off[i] = __ldg(args.offsets + i);
  __syncthreads();
  if (warp == 0) {  // chunk prefix over experts (256 token rows per chunk)
    const int per = (E + 31) / 32;
    const int e0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) local += (s_off[e + 1] - s_off[e] + kChunk - 1) / kChunk;
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
        run += (s_off[e + 1] - s_off[e] + kChunk - 1) / kChunk;
      }
    }
    if (lane == 31) s_tile[E] = incl;
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = s_tile[E] * args.ftiles;
  const int kblocks = args.K / BK;
  const uint32_t full_leader0 = mapa_shared(smem_u32(full), 0);
  const uint32_t tempty_leader0 = mapa_shared(smem_u32(tempty), 0);
  const uint32_t peer_abort = mapa_shared(smem_u32(const_cast<int*>(s_abort)), rank ^ 1u);
  auto give_up = [&]() {   // this CTA and its partner unwind; the status records why
    *s_abort = 1;
    st_cluster_u32(peer_abort, 1u);
    set_status(args.status, kStatusTimeout);
  };
  // this CTA's weight rows in feature tile ft of expert e: SwiGLU the 16-row block index
  // (in units of 16 features) of its first 64 act features; else the first W1/W2 row
  auto weight_row = [&](int e, int ft) {
    return MODE == kSwiGLU ? (ft * 128 + static_cast<int>(rank) * 64) / 16
                           : e * args.b_rows + ft * 256 + static_cast<int>(rank) * WROWS;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    uint32_t fill = 0;
    int skipped = -1;
    bool ok = true;
    for (int task = pair; task < total && ok; task += npairs) {
      int e, ft, ch;
      decode_ps(task, s_tile, E, args.ftiles, e, ft, ch);
      const Chunk c = chunk_of(s_off, e, ch);
      const int half = c.n >> 1;
      const int trow = c.row0 + static_cast<int>(rank) * half;   // this CTA's token rows
      const int wrow = weight_row(e, ft);
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
        uint8_t* a_dst = smem + s * C::STAGE;
        uint8_t* b_dst = a_dst + C::A_BYTES;
        const uint32_t fb = full_leader0 + 8u * static_cast<uint32_t>(s);
        if (lane == 0) {
          if (rank == 0)
            mbar_arrive_expect_tx(&full[s], MODE == kGemm2 ? 2 * C::STAGE : 2 * C::A_BYTES);
          if constexpr (MODE == kSwiGLU) {
            // four blocks of (16 gate rows, the 16 matching up rows): [block][gate|up][16]
            tma_load_5d_2sm(a_dst, &tmW, fb, kb * BK, 0, 0, wrow, e);
          } else {
            tma_load_2d_2sm(a_dst, &tmW, fb, kb * BK, wrow);
          }
          // GEMM2: always a whole 128-row box of token rows, whatever the chunk's N (rows
          // past the expert's are the next expert's or the zero fill; the MMA reads N/2 of
          // them).  Boxes sized to the chunk -- up to five per stage for a short last chunk
          // -- measured far slower: Qwen3-30B-A3B-shaped GEMM2 255 against 205 us.
          if constexpr (MODE == kGemm2) tma_load_2d_2sm(b_dst, &tmT, fb, kb * BK, trow);
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) give_up();
    // no copy may still be writing shared memory when the CTA exits: the last fills have
    // landed once the MMA released them (empty); on the abort path these waits end within
    // one limit in total
    const uint64_t deadline = globaltimer_ns() + lim;
    for (uint32_t f = fill > static_cast<uint32_t>(STAGES) ? fill - STAGES : 0; f < fill; ++f) {
      if (static_cast<int>(f) == skipped) continue;
      if (!mbar_wait_until(&empty[f % STAGES], (f / STAGES) & 1u, deadline)) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (rank == 0 && lane == 0) {
      uint32_t fill = 0, tc = 0;
      bool ok = true;
      for (int task = pair; task < total && ok; task += npairs) {
        int e, ft, ch;
        decode_ps(task, s_tile, E, args.ftiles, e, ft, ch);
        const Chunk c = chunk_of(s_off, e, ch);
        const uint32_t idesc = idesc_bf16_f32_rt(2 * WROWS, c.n);
        const int acc = tc & 1;
        const uint32_t aph = (tc >> 1) & 1u;
        if (!mbar_wait_cluster(&tempty[acc], aph ^ 1u, s_abort, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kChunk);
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
            mma_bf16_ss_2sm(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit_2sm(&empty[s]);
        }
        if (!ok) break;
        mma_commit_2sm(&tfull[acc]);
        ++tc;
      }
      if (!ok) give_up();
      if (fill > 0) {  // every pair MMA issued above has completed once this arrives
        mma_commit_2sm(drain);
        mbar_wait(drain, 0, s_never, lim);
      }
    }
    __syncwarp();
  } else if (warp == kRelayWarp) {
    // ------------------------------------------------------------ relay (GEMM1, both CTAs)
    if constexpr (C::GATHER) {
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
        if (!ok) give_up();
      }
      __syncwarp();
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------ token-row gather (GEMM1)
    if constexpr (C::GATHER) {
      const int lw = warp - 6;
      const int sub = lane >> 3;    // row within a group of 4
      const int chunk = lane & 7;   // 16-byte chunk within the 128-byte row
      uint32_t fill = 0;
      bool ok = true;
      for (int task = pair; task < total && ok; task += npairs) {
        int e, ft, ch;
        decode_ps(task, s_tile, E, args.ftiles, e, ft, ch);
        const Chunk c = chunk_of(s_off, e, ch);
        const int half = c.n >> 1;
        const int first = static_cast<int>(rank) * half;   // chunk position of row 0 here
        const uint16_t* src[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = lw * 32 + i * 4 + sub;
          // padding rows (past the expert's rows) copy the chunk's first row; unused
          const int rr = first + r < c.nvalid ? c.row0 + first + r : c.row0;
          const int tok = __ldg(args.row2assign + rr) / args.k_top;
          src[i] = args.x + static_cast<int64_t>(tok) * args.K + chunk * 8;
        }
        for (int kb = 0; kb < kblocks; ++kb, ++fill) {
          const int s = fill % STAGES;
          const uint32_t ph = (fill / STAGES) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, s_abort, lim))) {
            ok = false;
            break;
          }
          const uint32_t b_base = smem_u32(smem + s * C::STAGE + C::A_BYTES);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = lw * 32 + i * 4 + sub;
            if (r < half) cp_async_16(b_base + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * BK);
          }
          cp_async_mbar_arrive_noinc(&afull[s]);
        }
      }
      if (!ok && lane == 0) give_up();
      cp_async_wait_all();
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int q = warp & 3;          // TMEM lanes 32q..32q+31 = weight rows of this CTA
    Stager<C::ROW_BYTES> st{smem_u32(smem + C::EPI_OFF + q * 2 * C::STG_BYTES), 0u};
    uint32_t tc = 0;
    bool ok = true;
    for (int task = pair; task < total; task += npairs) {
      int e, ft, ch;
      decode_ps(task, s_tile, E, args.ftiles, e, ft, ch);
      const Chunk c = chunk_of(s_off, e, ch);
      const int acc = tc & 1;
      const uint32_t aph = (tc >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, s_abort, lim))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc * kChunk);
      // output columns of this warp: SwiGLU 16 act features (lanes 32q.. are features
      // 16q.. of the CTA's 64), else 32 W1/W2 rows
      const int col = MODE == kSwiGLU ? ft * 128 + static_cast<int>(rank) * 64 + q * 16
                                      : ft * 256 + static_cast<int>(rank) * WROWS + q * 32;
      if (col < args.n_out) {   // whole warp: n_out is a multiple of 64
        for (int cb = 0; cb < c.n; cb += 32) {
          const uint32_t buf = st.next(lane);
          if (c.n - cb >= 32) epi_block<MODE, 32>(tq + cb, buf, lane);
          else epi_block<MODE, 16>(tq + cb, buf, lane);
          st.store(buf, &tmO, args.out, args.n_out, col, c.row0 + cb,
                   min(min(32, c.n - cb), c.nvalid - cb), lane);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8u * static_cast<uint32_t>(acc));
      ++tc;
    }
    if (!ok && lane == 0) give_up();
    if (lane == 0) bulk_wait_group_all();   // every store has completed before the exit
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();  // neither CTA leaves while the pair's MMAs or signals may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_ps() {
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

// bf16 [outer][inner] (row stride `inner`), box {box_inner, box_outer}, given swizzle.
bool tmap_ps(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
             uint32_t box_outer, CUtensorMapSwizzle swz, CUtensorMapL2promotion l2) {
  auto fn = encode_fn_ps();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool tmap_operand(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t rows) {
  return tmap_ps(m, ptr, inner, outer, BK, rows, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// Output bf16 [rows][cols] for the epilogue's stores: boxes of 32 rows x `box_cols` columns
// (32 -> 64-byte rows, 64-byte swizzle; 16 -> 32-byte rows, 32-byte swizzle).
bool tmap_out(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_cols) {
  return tmap_ps(m, ptr, cols, rows, box_cols, 32,
                 box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B,
                 CU_TENSOR_MAP_L2_PROMOTION_NONE);
}

// W13 bf16 [E][2I][H] viewed as 5-D (H, 16 rows, gate|up, I/16 blocks, E) -- strides H,
// I*H, 16*H and 2I*H elements -- so that one box {64, 16, 2, 4, 1} lands in shared memory
// as [block][gate|up][16 rows][64 K]: each 16 gate rows followed by the matching 16 up
// rows (128-byte swizzle, like the 2-D operand tiles).
bool tmap_w13_interleaved(CUtensorMap* m, const void* ptr, int H, int I, int E) {
  auto fn = encode_fn_ps();
  if (!fn) return false;
  const cuuint64_t h = static_cast<cuuint64_t>(H), i = static_cast<cuuint64_t>(I);
  cuuint64_t dims[5] = {h, 16, 2, i / 16, static_cast<cuuint64_t>(E)};
  cuuint64_t strides[4] = {h * 2, i * h * 2, 16 * h * 2, 2 * i * h * 2};
  cuuint32_t box[5] = {BK, 16, 2, 4, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

constexpr int kStages = 6;

template <int MODE>
cudaError_t run_ps(const CUtensorMap& w, const CUtensorMap& t, const CUtensorMap& o, const PsArgs& a,
                   cudaStream_t stream) {
  using Cf = PsCfg<MODE, kStages>;
  auto kern = pair_swap_gemm_kernel<MODE, kStages>;
  static cudaError_t attr =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::ALLOC);
  if (attr != cudaSuccess) return attr;
  const int grid = num_sms() & ~1;
  return launch_k(kern, dim3(grid), dim3(Cf::THREADS), Cf::ALLOC, stream, w, t, o, a);
}

}  // namespace

cudaError_t launch_gemm1_pair_swap(const GemmProblem& p, const uint16_t* x,
                                   const int32_t* row2assign, const int32_t* offsets,
                                   const uint16_t* w13, uint16_t* act, int* status,
                                   cudaStream_t stream, int* launches) {
  if (p.R == 0) return cudaSuccess;
  const bool relu2 = p.act == 1;
  CUtensorMap tw, to, tt{};
  const bool maps = relu2 ? tmap_operand(&tw, w13, p.H, static_cast<uint64_t>(p.E) * p.I, WROWS)
                         : tmap_w13_interleaved(&tw, w13, p.H, p.I, p.E);
  if (!maps || !tmap_out(&to, act, p.I, p.R, relu2 ? 32 : 16)) return cudaErrorInvalidValue;
  PsArgs a{};
  a.offsets = offsets;
  a.row2assign = row2assign;
  a.x = x;
  a.out = act;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.I;
  a.K = p.H;
  a.ftiles = relu2 ? (p.I + 255) / 256 : (p.I + 127) / 128;
  a.b_rows = (relu2 ? 1 : 2) * p.I;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  return relu2 ? run_ps<kReLU2>(tw, tt, to, a, stream) : run_ps<kSwiGLU>(tw, tt, to, a, stream);
}

cudaError_t launch_gemm2_pair_swap(const GemmProblem& p, const uint16_t* act,
                                   const int32_t* offsets, const uint16_t* w2, uint16_t* y,
                                   int* status, cudaStream_t stream, int* launches) {
  if (p.R == 0) return cudaSuccess;
  CUtensorMap tw, to, tt;
  if (!tmap_operand(&tw, w2, p.I, static_cast<uint64_t>(p.E) * p.H, WROWS) ||
      !tmap_operand(&tt, act, p.I, p.R, kHalf) || !tmap_out(&to, y, p.H, p.R, 32))
    return cudaErrorInvalidValue;
  PsArgs a{};
  a.offsets = offsets;
  a.out = y;
  a.status = status;
  a.E = p.E;
  a.k_top = p.k;
  a.n_out = p.H;
  a.K = p.I;
  a.ftiles = (p.H + 255) / 256;
  a.b_rows = p.H;
  a.inject_stall = g_inject_stall;
  a.wait_limit_ns = p.wait_limit_ns;
  ++*launches;
  return run_ps<kGemm2>(tw, tt, to, a, stream);
}

}  // namespace moe
