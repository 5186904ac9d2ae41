// gemm_bf16.cu -- which kernel runs the BF16 grouped GEMMs of a problem.
//
//   GEMM1 + SwiGLU: act[r][i] = silu(x[tok(r)] . W13[e][i]) * (x[tok(r)] . W13[e][I+i])
//   GEMM1 + ReLU2:  act[r][i] = max(x[tok(r)] . W1[e][i], 0)^2
//   GEMM2:          y[r][o]   = act[r] . W2[e][o]
//
// TileScale PR #70 (distributed FP8 MegaMoE), "Design": kernel 1 is GEMM1 with SwiGLU
// fused into its epilogue, kernel 2 is GEMM2.  Decode-sized batches (T <= 64; SwiGLU for
// GEMM1) run on single SMs with the weights on the MMA's M = 128 side and K split into
// slices (gemm_swap.cu); every other batch runs on SM pairs with the weights on the
// M = 256 side and chunks of up to 256 token rows on the N side (gemm_pair_swap.cu).
// The pair kernels replaced single-SM 128 x 256 tiles and 256-row SM-pair tiles; measured
// against them (same build otherwise, alternating runs on one B200) the forward pass was
// faster on every large-batch workload: Qwen3-30B-A3B-shaped 644.6 against 661.7 us,
// Llama-4-Scout-shaped 1761 against 1905 us, the D=4096 E=64 k=8 grid point 5774
// against 6239 us, the ReLU2 Nemotron shape 1049 against 1104 us.
#include <cuda_runtime.h>

#include "kernels.h"

namespace moe {

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
  if (p.act != 1 && use_swap_gemm(p.T))
    return launch_gemm1_swap(p, x, row2assign, offsets, w13, act, nullptr, 1, status, stream,
                             launches);
  return launch_gemm1_pair_swap(p, x, row2assign, offsets, w13, act, status, stream, launches);
}

cudaError_t launch_gemm2_bf16(const GemmProblem& p, const uint16_t* act, const int32_t* offsets,
                              const uint16_t* w2, uint16_t* y, int* status, cudaStream_t stream,
                              int* launches) {
  if (p.R == 0) return cudaSuccess;
  if (use_swap_gemm(p.T) && p.H % 128 == 0)
    return launch_gemm2_swap(p, act, offsets, w2, y, nullptr, 1, nullptr, status, stream,
                             launches);
  return launch_gemm2_pair_swap(p, act, offsets, w2, y, status, stream, launches);
}

}  // namespace moe
