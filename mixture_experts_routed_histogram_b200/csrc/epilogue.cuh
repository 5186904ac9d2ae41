// epilogue.cuh -- bf16 output stores of the GEMM epilogues through shared memory and TMA.
//
// An epilogue warp owns 32 output rows of a tile (its TMEM lane quadrant).  Writing them
// straight from registers makes every 16-byte store instruction touch 32 different rows,
// i.e. 32 cache lines, which keeps the load/store unit busy for the whole tile.  Instead
// each 32-column chunk goes registers -> a 2 KB staging buffer (32 rows x 64 bytes, laid out
// with the 64-byte swizzle so that the row-per-lane writes are free of bank conflicts) ->
// one TMA tensor store, issued and tracked by lane 0 in its bulk async-group.  Every warp
// has two buffers; a buffer is written again two chunks later, once the store issued from
// it has finished reading shared memory.
//
// A TMA store writes whole boxes, so it is used only when all 32 rows of the warp belong to
// the tile's expert: rows past the expert's end are the next expert's rows in the
// expert-sorted output and must not be overwritten.  Those warps store their valid rows
// directly.  Columns past the tensor's end are clipped by TMA.
#pragma once

#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace moe {

constexpr int kEpiBufBytes = 2048;                // 32 rows x 32 bf16
constexpr int kEpiWarpBytes = 2 * kEpiBufBytes;   // double-buffered
constexpr int kEpiWarps = 4;
constexpr int kEpiBytes = kEpiWarps * kEpiWarpBytes;

struct EpiStager {
  uint32_t base;  // shared address of this warp's two buffers (512-byte aligned)
  uint32_t n;     // chunks stored so far
};

// Stage one 32-row x 32-column bf16 chunk (pk: this lane's row, 16 packed pairs) and store
// it at (col, row) of the output tensor map.  All 32 lanes call this.
__device__ __forceinline__ void epi_store_chunk(EpiStager& st, const CUtensorMap* tm,
                                                const uint32_t (&pk)[16], int col, int row,
                                                int lane) {
  const uint32_t buf = st.base + (st.n & 1u) * kEpiBufBytes;
  if (st.n >= 2) {
    if (lane == 0) bulk_wait_group_read<1>();  // the store issued from buf has read it
    __syncwarp();
  }
  // 64-byte swizzle: 16-byte unit u of row r sits at unit u ^ ((r >> 1) & 3)
  const uint32_t rp = buf + static_cast<uint32_t>(lane) * 64u;
  const uint32_t sw = static_cast<uint32_t>(lane >> 1) & 3u;
#pragma unroll
  for (int u = 0; u < 4; ++u)
    st_shared_v4(rp + ((static_cast<uint32_t>(u) ^ sw) << 4), pk[4 * u], pk[4 * u + 1],
                 pk[4 * u + 2], pk[4 * u + 3]);
  fence_async_smem();  // generic-proxy writes -> the TMA engine's reads
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tm, buf, col, row);
    bulk_commit_group();
  }
  ++st.n;
}

// The direct path for warps with rows past the expert's end: lane = row, 64 bytes.
__device__ __forceinline__ void epi_store_row(uint16_t* dst, const uint32_t (&pk)[16]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int v = 0; v < 4; ++v) d[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
}

// Before the CTA exits: every store of this warp has completed.
__device__ __forceinline__ void epi_drain(int lane) {
  if (lane == 0) bulk_wait_group_all();
  __syncwarp();
}

// Host: tensor map of a bf16 [rows][cols] output for epi_store_chunk (box 32 x 32, 64-byte
// swizzle).  `fn` is the driver's cuTensorMapEncodeTiled.
inline bool make_tmap_epi(PFN_cuTensorMapEncodeTiled_v12000 fn, CUtensorMap* m, const void* ptr,
                          uint64_t cols, uint64_t rows) {
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace moe
