// kernels.h -- host-side launchers of the CUDA kernels (internal C++ interface used by
// the C ABI in api.cu).  Every launcher only enqueues work on `stream` and returns the
// launch error; argument validation is done by the caller.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;

// Routing: ids/w [T][k + ns] from logits [T][E]: the top-k, then the ns shared experts
// E .. E+ns-1 with weight 1.
cudaError_t launch_route(const float* logits, int32_t* ids, float* w, int64_t T, int E, int k,
                         int ns, int score, int renorm, cudaStream_t stream, int* launches);

// Histogram / prefix sum / stable scatter of the T*k assignments (chunks of 64 tokens,
// fewer and larger chunks beyond 128 of them).  `scratch` holds the per-chunk histograms
// and their scans.
size_t permute_scratch_bytes(int64_t T, int E);
cudaError_t launch_permute(const int32_t* ids, int64_t T, int k, int E, int32_t* counts,
                           int32_t* offsets, int32_t* row2assign, int32_t* assign2row,
                           int32_t* scratch, int* status, cudaStream_t stream, int* launches);

// The same permutation with its scratch in a static device array (no workspace); fits()
// tells whether the problem's scratch stays within that array.
bool permute_noalloc_fits(int64_t T, int E);
cudaError_t launch_permute_noalloc(const int32_t* ids, int64_t T, int k, int E, int32_t* counts,
                                   int32_t* offsets, int32_t* row2assign, int32_t* assign2row,
                                   cudaStream_t stream, int* launches);

// Routing + histogram + prefix sum + stable scatter in one single-CTA launch, for
// decode-sized batches (use_route_permute_small).  Same outputs as launch_route followed
// by launch_permute.
// (E, k: routed experts and top-k; ns shared experts are appended as in launch_route.)
bool use_route_permute_small(int64_t T, int E_all, int k_all);
cudaError_t launch_route_permute_small(const float* logits, int64_t T, int E, int k, int ns,
                                       int score, int renorm, int32_t* ids, float* w,
                                       int32_t* counts, int32_t* offsets, int32_t* row2assign,
                                       int32_t* assign2row, cudaStream_t stream, int* launches);

// Routing + histogram + prefix sum + stable scatter for larger batches in one cooperative
// launch (one CTA per chunk of launch_permute, a grid-wide barrier between the histograms
// and the scatter).  Same outputs as launch_route followed by launch_permute.  `scratch`
// holds the per-block histograms and their scans (route_permute_scratch_bytes); `gbar` two
// zero-initialised words of the barrier (left zeroed by each call); a barrier wait beyond
// limit_ns sets `status`.
size_t route_permute_scratch_bytes(int64_t T, int E);
cudaError_t launch_route_permute(const float* logits, int64_t T, int E, int k, int ns, int score,
                                 int renorm, int32_t* ids, float* w, int32_t* counts,
                                 int32_t* offsets, int32_t* row2assign, int32_t* assign2row,
                                 int32_t* scratch, unsigned* gbar, int* status,
                                 uint64_t limit_ns, cudaStream_t stream, int* launches);

// Weighted top-k combine.
cudaError_t launch_combine(const uint16_t* y, const float* w, const int32_t* assign2row,
                           uint16_t* out, int64_t T, int H, int k, cudaStream_t stream,
                           int* launches);

// 1x128 e4m3 activation quantiser; sxw (nullable) also receives the UE8M0 word of each
// scale (its byte repeated four times), the form the block-scaled GEMMs read.
cudaError_t launch_quant_x(const uint16_t* x, uint8_t* xq, float* sx, uint32_t* sxw, int64_t T,
                           int H, cudaStream_t stream, int* launches);

// fp32 power-of-two scales -> UE8M0 words.
cudaError_t launch_scale_words(const float* s, uint32_t* w, int64_t n, cudaStream_t stream,
                               int* launches);

// MXFP4 weight preparation (K32 UE8M0 scales).
cudaError_t launch_quant_w_mxfp4(const uint16_t* w, uint8_t* packed, uint8_t* sf, int64_t rows,
                                 int K, cudaStream_t stream, int* launches);

struct GemmProblem {
  int64_t T;      // tokens (GEMM1 A rows)
  int64_t R;      // routed rows
  int H, I, E, k;
  int act;        // GEMM1 activation: 0 SwiGLU (W13 [E][2I][H]), 1 ReLU2 (W1 [E][I][H])
  uint64_t wait_limit_ns;
};

// Grouped GEMM1 + SwiGLU (or ReLU2), BF16 (x gathered by row2assign, act expert-sorted):
// the decode-sized kernels for T <= 64 (SwiGLU), else the SM-pair kernels.
cudaError_t launch_gemm1_bf16(const GemmProblem& p, const uint16_t* x, const int32_t* row2assign,
                              const int32_t* offsets, const uint16_t* w13, uint16_t* act,
                              int* status, cudaStream_t stream, int* launches);

// Grouped GEMM2, BF16 (act expert-sorted, y expert-sorted).
cudaError_t launch_gemm2_bf16(const GemmProblem& p, const uint16_t* act, const int32_t* offsets,
                              const uint16_t* w2, uint16_t* y, int* status, cudaStream_t stream,
                              int* launches);

// Large-batch BF16 GEMMs on SM pairs with the weights on the MMA's M = 256 side and
// chunks of up to 256 token rows on its N side (gemm_pair_swap.cu).
cudaError_t launch_gemm1_pair_swap(const GemmProblem& p, const uint16_t* x,
                                   const int32_t* row2assign, const int32_t* offsets,
                                   const uint16_t* w13, uint16_t* act, int* status,
                                   cudaStream_t stream, int* launches);
cudaError_t launch_gemm2_pair_swap(const GemmProblem& p, const uint16_t* act,
                                   const int32_t* offsets, const uint16_t* w2, uint16_t* y,
                                   int* status, cudaStream_t stream, int* launches);

// Decode-sized GEMMs with weights on the MMA's M side and token rows on its N side.
constexpr int kMaxSplits = 16;
bool use_swap_gemm(int64_t T);
int swap_splits(const GemmProblem& p);        // the most K slices GEMM2 may choose
int swap_splits_gemm1(const GemmProblem& p);  // K slices of GEMM1
// splits == 1 fuses SwiGLU; splits > 1 writes fp32 gate|up partial sums part[splits][R][2I]
// and a second kernel finishes act = silu(g)*u.
cudaError_t launch_gemm1_swap(const GemmProblem& p, const uint16_t* x, const int32_t* row2assign,
                              const int32_t* offsets, const uint16_t* w13, uint16_t* act,
                              float* part, int splits, int* status, cudaStream_t stream,
                              int* launches);
// splits == 1 writes y (bf16); splits > 1 writes fp32 partial sums part[S][R][H] for the
// S <= splits slices the kernel chooses from the busy tiles, and stores S in *splits_used.
cudaError_t launch_gemm2_swap(const GemmProblem& p, const uint16_t* act, const int32_t* offsets,
                              const uint16_t* w2, uint16_t* y, float* part, int splits,
                              int* splits_used, int* status, cudaStream_t stream,
                              int* launches);
// Combine from K-split partial sums: out[t] = sum_j w[t,j] * sum_s part[s][assign2row[t,j]],
// with the slice count S read from *splits (written by the GEMM2 before it).
cudaError_t launch_combine_parts(const float* part, const int* splits, int64_t R, const float* w,
                                 const int32_t* assign2row, uint16_t* out, int64_t T, int H,
                                 int k, cudaStream_t stream, int* launches);

// Block-scaled grouped GEMM1 + SwiGLU + 1x128 requantisation (e4m3 x MXFP4).
cudaError_t launch_gemm1_mx(const GemmProblem& p, const uint8_t* xq, const uint32_t* sxw,
                            const int32_t* row2assign, const int32_t* offsets,
                            const uint8_t* w13p, const uint8_t* w13sf, uint8_t* act,
                            float* act_sf, uint32_t* act_sfw, int* status, cudaStream_t stream,
                            int* launches);

// Block-scaled grouped GEMM2 (e4m3 act x MXFP4 W2, bf16 y).
cudaError_t launch_gemm2_mx(const GemmProblem& p, const uint8_t* act, const uint32_t* act_sfw,
                            const int32_t* offsets, const uint8_t* w2p, const uint8_t* w2sf,
                            uint16_t* y, int* status, cudaStream_t stream, int* launches);

// The block-scaled GEMMs with weights on the MMA's M side, for few rows per expert
// (use_mx_swap); same inputs and outputs as launch_gemm1_mx / launch_gemm2_mx.
bool use_mx_swap(int64_t R, int E);
cudaError_t launch_gemm1_mx_swap(const GemmProblem& p, const uint8_t* xq, const uint32_t* sxw,
                                 const int32_t* row2assign, const int32_t* offsets,
                                 const uint8_t* w13p, const uint8_t* w13sf, uint8_t* act,
                                 float* act_sf, uint32_t* act_sfw, int* status,
                                 cudaStream_t stream, int* launches);
cudaError_t launch_gemm2_mx_swap(const GemmProblem& p, const uint8_t* act, const uint32_t* act_sfw,
                                 const int32_t* offsets, const uint8_t* w2p, const uint8_t* w2sf,
                                 uint16_t* y, int* status, cudaStream_t stream, int* launches);

int num_sms();

// Test hook: when non-zero, CTA 0 of each grouped-GEMM launch skips its first stage fill.
extern int g_inject_stall;

}  // namespace moe
