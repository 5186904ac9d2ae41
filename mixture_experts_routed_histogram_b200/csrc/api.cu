// api.cu -- the C ABI declared in include/moe.h: host-side argument checks, workspace
// carving and the ordering of the kernels on the caller's stream.  No allocation, no
// synchronisation (except moe_get_device_status and moe_debug_stage_times, which exist to
// synchronise; the optional per-stage timing creates its CUDA events once per thread).
#include <stdint.h>
#include <stdlib.h>

#include <algorithm>

#include "kernels.h"
#include "moe.h"

namespace {

thread_local int g_last_launches = 0;

// Per-stage timing of moe_forward (moe_debug_time_stages): an event before the first launch
// and one after each stage, on the forward's stream.
constexpr int kMaxTimedStages = 8;
struct StageTimer {
  bool on = false;
  cudaEvent_t ev[kMaxTimedStages + 1] = {};
  const char* name[kMaxTimedStages] = {};
  int n = -1;  // stages recorded by the last forward (-1: none)
  void begin(cudaStream_t st) {
    n = -1;
    if (!on) return;
    for (cudaEvent_t& e : ev)
      if (!e && cudaEventCreate(&e) != cudaSuccess) return;
    if (cudaEventRecord(ev[0], st) == cudaSuccess) n = 0;
  }
  void mark(cudaStream_t st, const char* what) {
    if (n < 0 || n >= kMaxTimedStages) return;
    if (cudaEventRecord(ev[n + 1], st) != cudaSuccess) {
      n = -1;
      return;
    }
    name[n++] = what;
  }
};
thread_local StageTimer g_timer;
uint64_t g_wait_limit_ns = 4000000000ull;  // 4 s per bounded device wait

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;

size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// Shared experts are folded in as experts E .. E+n_shared-1 and slots k .. k+n_shared-1:
// every stage after routing works on e_all experts and k_all slots per token.
int e_all(const moe_shape_t& s) { return s.E + s.n_shared; }
int k_all(const moe_shape_t& s) { return s.k + s.n_shared; }

// Workspace regions (byte offsets from the workspace base).
struct WsLayout {
  size_t status, ids, w, counts, offsets, r2a, a2r, scratch, xq, sx, sxw, act, act_sf, act_sfw,
      y, part, total;
};

WsLayout layout(const moe_shape_t& s) {
  const size_t T = static_cast<size_t>(s.T), R = T * k_all(s), H = s.H, I = s.I, E = e_all(s);
  const bool fp8 = s.dtype == MOE_DTYPE_FP8_MXFP4;
  WsLayout L{};
  size_t o = 0;
  L.status = o; o += kStatusBytes;
  L.ids = o; o = up(o + 4 * R);
  L.w = o; o = up(o + 4 * R);
  L.counts = o; o = up(o + 4 * E);
  L.offsets = o; o = up(o + 4 * (E + 1));
  L.r2a = o; o = up(o + 4 * R);
  L.a2r = o; o = up(o + 4 * R);
  L.scratch = o;
  o = up(o + std::max(moe::permute_scratch_bytes(static_cast<int64_t>(T), e_all(s)),
                      moe::route_permute_scratch_bytes(static_cast<int64_t>(T), e_all(s))));
  L.xq = o; o = up(o + (fp8 ? T * H : 0));
  L.sx = o; o = up(o + (fp8 ? 4 * T * (H / 128) : 0));
  L.sxw = o; o = up(o + (fp8 ? 4 * T * (H / 128) : 0));
  L.act = o; o = up(o + (fp8 ? R * I : 2 * R * I));
  L.act_sf = o; o = up(o + (fp8 ? 4 * R * (I / 128) : 0));
  L.act_sfw = o; o = up(o + (fp8 ? 4 * R * (I / 128) : 0));
  L.y = o; o = up(o + 2 * R * H);
  // decode-sized BF16 forward: fp32 partial sums of the K-split GEMM2
  const bool swap = !fp8 && moe::use_swap_gemm(s.T) && H % 128 == 0;
  L.part = o;
  o = up(o + (swap ? 4 * static_cast<size_t>(moe::kMaxSplits) * R * std::max(H, 2 * I) : 0));
  L.total = o;
  return L;
}

moe_status_t check_shape(const moe_shape_t* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->H <= 0 || s->I <= 0 || s->E <= 0 || s->k <= 0) return MOE_ERR_INVALID_ARG;
  if ((s->score != MOE_SCORE_SOFTMAX && s->score != MOE_SCORE_SIGMOID) ||
      (s->dtype != MOE_DTYPE_BF16 && s->dtype != MOE_DTYPE_FP8_MXFP4) ||
      (s->renormalize != 0 && s->renormalize != 1) ||
      (s->activation != MOE_ACT_SWIGLU && s->activation != MOE_ACT_RELU2))
    return MOE_ERR_INVALID_ARG;
  if (s->activation == MOE_ACT_RELU2 && s->dtype != MOE_DTYPE_BF16)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->k > s->E || s->n_shared < 0) return MOE_ERR_INVALID_ARG;
  if (k_all(*s) > moe::kMaxTopK || e_all(*s) > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->T * static_cast<int64_t>(k_all(*s)) >= (static_cast<int64_t>(1) << 31))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  const int q = s->dtype == MOE_DTYPE_BF16 ? 64 : 128;
  if (s->H % q != 0 || s->I % q != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                    \
  do {                                   \
    moe_status_t st_ = (expr);           \
    if (st_ != MOE_OK) return st_;       \
  } while (0)

moe_status_t need_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  }
  return MOE_OK;
}

moe::GemmProblem problem(const moe_shape_t& s) {
  moe::GemmProblem p{};
  p.T = s.T;
  p.R = s.T * k_all(s);
  p.H = s.H;
  p.I = s.I;
  p.E = e_all(s);
  p.k = k_all(s);
  p.act = s.activation;
  p.wait_limit_ns = g_wait_limit_ns;
  return p;
}

int* status_word(void* ws) { return reinterpret_cast<int*>(ws); }
// K slices the decode-sized GEMM2 chose, for the combine after it (in the status region)
int* splits_word(void* ws) { return reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + 64); }
// arrival count and generation of the front end's grid-wide barrier (in the status region)
unsigned* grid_barrier_words(void* ws) {
  return reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) + 128);
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

}  // namespace

extern "C" {

size_t moe_workspace_size(const moe_shape_t* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return layout(*shape).total;
}

moe_status_t moe_workspace_region(const moe_shape_t* shape, int32_t region, size_t* offset,
                                  size_t* bytes) {
  if (!offset || !bytes || check_shape(shape) != MOE_OK) return MOE_ERR_INVALID_ARG;
  const WsLayout L = layout(*shape);
  const size_t R = static_cast<size_t>(shape->T) * k_all(*shape), E = e_all(*shape);
  switch (region) {
    case MOE_WS_IDS: *offset = L.ids; *bytes = 4 * R; break;
    case MOE_WS_W: *offset = L.w; *bytes = 4 * R; break;
    case MOE_WS_COUNTS: *offset = L.counts; *bytes = 4 * E; break;
    case MOE_WS_OFFSETS: *offset = L.offsets; *bytes = 4 * (E + 1); break;
    case MOE_WS_ROW2ASSIGN: *offset = L.r2a; *bytes = 4 * R; break;
    case MOE_WS_ASSIGN2ROW: *offset = L.a2r; *bytes = 4 * R; break;
    default: return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream) {
  g_last_launches = 0;
  if (!ws) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return MOE_ERR_MISALIGNED;
  if (ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  g_last_launches = 1;
  return cuda_status(cudaMemsetAsync(ws, 0, kStatusBytes, stream));
}

moe_status_t moe_route(const moe_shape_t* shape, const float* logits, int32_t* ids, float* w,
                       cudaStream_t stream) {
  g_last_launches = 0;
  MOE_TRY(check_shape(shape));
  if (shape->T == 0) return MOE_OK;
  MOE_TRY(need_ptrs({logits, ids, w}));
  int n = 0;
  cudaError_t e = moe::launch_route(logits, ids, w, shape->T, shape->E, shape->k,
                                    shape->n_shared, shape->score,
                                    shape->renormalize, stream, &n);
  g_last_launches = n;
  return cuda_status(e);
}

moe_status_t moe_permute(const moe_shape_t* shape, const int32_t* ids, int32_t* counts,
                         int32_t* offsets, int32_t* row2assign, int32_t* assign2row, void* ws,
                         size_t ws_bytes, cudaStream_t stream) {
  g_last_launches = 0;
  MOE_TRY(check_shape(shape));
  MOE_TRY(need_ptrs({counts, offsets, ws}));
  const int64_t R = shape->T * k_all(*shape);
  if (R > 0) MOE_TRY(need_ptrs({ids, row2assign, assign2row}));
  const WsLayout L = layout(*shape);
  if (ws_bytes < L.scratch + moe::permute_scratch_bytes(shape->T, e_all(*shape)))
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  int n = 0;
  cudaError_t e = moe::launch_permute(ids, shape->T, k_all(*shape), e_all(*shape), counts, offsets,
                                      row2assign, assign2row, at<int32_t>(ws, L.scratch),
                                      status_word(ws), stream, &n);
  g_last_launches = n;
  return cuda_status(e);
}

moe_status_t moe_permute_noalloc(const moe_shape_t* shape, const int32_t* ids, int32_t* counts,
                                 int32_t* offsets, int32_t* row2assign, int32_t* assign2row,
                                 cudaStream_t stream) {
  g_last_launches = 0;
  MOE_TRY(check_shape(shape));
  MOE_TRY(need_ptrs({counts, offsets}));
  const int64_t R = shape->T * k_all(*shape);
  if (R > 0) MOE_TRY(need_ptrs({ids, row2assign, assign2row}));
  if (!moe::permute_noalloc_fits(shape->T, e_all(*shape))) return MOE_ERR_UNSUPPORTED_SHAPE;
  int n = 0;
  cudaError_t e = moe::launch_permute_noalloc(ids, shape->T, k_all(*shape), e_all(*shape), counts, offsets,
                                              row2assign, assign2row, stream, &n);
  g_last_launches = n;
  return cuda_status(e);
}

moe_status_t moe_quantize_x(const moe_shape_t* shape, const uint16_t* x, uint8_t* xq, float* sx,
                            cudaStream_t stream) {
  g_last_launches = 0;
  MOE_TRY(check_shape(shape));
  if (shape->H % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (shape->T == 0) return MOE_OK;
  MOE_TRY(need_ptrs({x, xq, sx}));
  int n = 0;
  cudaError_t e = moe::launch_quant_x(x, xq, sx, nullptr, shape->T, shape->H, stream, &n);
  g_last_launches = n;
  return cuda_status(e);
}

moe_status_t moe_quantize_weights_mxfp4(int64_t rows, int32_t K, const uint16_t* w,
                                        uint8_t* packed, uint8_t* sf, cudaStream_t stream) {
  g_last_launches = 0;
  if (rows < 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (K % 32 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!w || !packed || !sf) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(packed)) return MOE_ERR_MISALIGNED;
  int n = 0;
  cudaError_t e = moe::launch_quant_w_mxfp4(w, packed, sf, rows, K, stream, &n);
  g_last_launches = n;
  return cuda_status(e);
}

moe_status_t moe_grouped_gemm1_swiglu(const moe_shape_t* shape, const void* a, const float* sa,
                                      const int32_t* row2assign, const int32_t* offsets,
                                      const void* w13, const uint8_t* w13_sf, void* act,
                                      float* act_sf, void* ws, size_t ws_bytes,
                                      cudaStream_t stream) {
  g_last_launches = 0;
  MOE_TRY(check_shape(shape));
  MOE_TRY(need_ptrs({offsets, ws}));
  if (ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (shape->T == 0) return MOE_OK;
  MOE_TRY(need_ptrs({a, row2assign, w13, act}));
  int n = 0;
  if (shape->dtype == MOE_DTYPE_FP8_MXFP4) {
    MOE_TRY(need_ptrs({sa, w13_sf, act_sf}));
    if (!aligned32(w13)) return MOE_ERR_MISALIGNED;
    const WsLayout L = layout(*shape);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    uint32_t* sxw = at<uint32_t>(ws, L.sxw);
    cudaError_t e = moe::launch_scale_words(sa, sxw, shape->T * (shape->H / 128), stream, &n);
    if (e == cudaSuccess)
      e = moe::launch_gemm1_mx(problem(*shape), static_cast<const uint8_t*>(a), sxw, row2assign,
                               offsets, static_cast<const uint8_t*>(w13), w13_sf,
                               static_cast<uint8_t*>(act), act_sf, at<uint32_t>(ws, L.act_sfw),
                               status_word(ws), stream, &n);
    g_last_launches = n;
    return cuda_status(e);
  }
  cudaError_t e = moe::launch_gemm1_bf16(problem(*shape), static_cast<const uint16_t*>(a),
                                         row2assign, offsets, static_cast<const uint16_t*>(w13),
                                         static_cast<uint16_t*>(act), status_word(ws), stream, &n);
  g_last_launches = n;
  return cuda_status(e);
}

moe_status_t moe_grouped_gemm2(const moe_shape_t* shape, const void* act, const float* act_sf,
                               const int32_t* offsets, const void* w2, const uint8_t* w2_sf,
                               uint16_t* y, void* ws, size_t ws_bytes, cudaStream_t stream) {
  g_last_launches = 0;
  MOE_TRY(check_shape(shape));
  MOE_TRY(need_ptrs({offsets, ws}));
  if (ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (shape->T == 0) return MOE_OK;
  MOE_TRY(need_ptrs({act, w2, y}));
  int n = 0;
  if (shape->dtype == MOE_DTYPE_FP8_MXFP4) {
    MOE_TRY(need_ptrs({act_sf, w2_sf}));
    if (!aligned32(w2)) return MOE_ERR_MISALIGNED;
    const WsLayout L = layout(*shape);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    uint32_t* asw = at<uint32_t>(ws, L.act_sfw);
    const int64_t R = shape->T * k_all(*shape);
    cudaError_t e = moe::launch_scale_words(act_sf, asw, R * (shape->I / 128), stream, &n);
    if (e == cudaSuccess)
      e = moe::launch_gemm2_mx(problem(*shape), static_cast<const uint8_t*>(act), asw, offsets,
                               static_cast<const uint8_t*>(w2), w2_sf, y, status_word(ws), stream,
                               &n);
    g_last_launches = n;
    return cuda_status(e);
  }
  cudaError_t e = moe::launch_gemm2_bf16(problem(*shape), static_cast<const uint16_t*>(act),
                                         offsets, static_cast<const uint16_t*>(w2), y,
                                         status_word(ws), stream, &n);
  g_last_launches = n;
  return cuda_status(e);
}

moe_status_t moe_combine(const moe_shape_t* shape, const uint16_t* y, const float* w,
                         const int32_t* assign2row, uint16_t* out, cudaStream_t stream) {
  g_last_launches = 0;
  MOE_TRY(check_shape(shape));
  if (shape->T == 0) return MOE_OK;
  MOE_TRY(need_ptrs({y, w, assign2row, out}));
  int n = 0;
  cudaError_t e = moe::launch_combine(y, w, assign2row, out, shape->T, shape->H, k_all(*shape), stream,
                                      &n);
  g_last_launches = n;
  return cuda_status(e);
}

moe_status_t moe_forward(const moe_shape_t* shape, const uint16_t* x, const float* logits,
                         const void* w13, const uint8_t* w13_sf, const void* w2,
                         const uint8_t* w2_sf, uint16_t* out, int32_t* ids_out, void* ws,
                         size_t ws_bytes, cudaStream_t stream) {
  g_last_launches = 0;
  g_timer.n = -1;
  MOE_TRY(check_shape(shape));
  if (!ws) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return MOE_ERR_MISALIGNED;
  const WsLayout L = layout(*shape);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (shape->T == 0) return MOE_OK;
  MOE_TRY(need_ptrs({x, logits, w13, w2, out}));
  if (ids_out && !aligned16(ids_out)) return MOE_ERR_MISALIGNED;
  const bool fp8 = shape->dtype == MOE_DTYPE_FP8_MXFP4;
  if (fp8) {
    MOE_TRY(need_ptrs({w13_sf, w2_sf}));
    if (!aligned32(w13) || !aligned32(w2)) return MOE_ERR_MISALIGNED;
  }

  const int64_t T = shape->T, R = T * k_all(*shape);
  int32_t* ids = ids_out ? ids_out : at<int32_t>(ws, L.ids);
  float* w = at<float>(ws, L.w);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* r2a = at<int32_t>(ws, L.r2a);
  int32_t* a2r = at<int32_t>(ws, L.a2r);
  uint16_t* act = at<uint16_t>(ws, L.act);
  uint16_t* y = at<uint16_t>(ws, L.y);
  int* status = status_word(ws);
  const moe::GemmProblem p = problem(*shape);
  int n = 0;
  cudaError_t e;
  g_timer.begin(stream);
  if (moe::use_route_permute_small(T, e_all(*shape), k_all(*shape))) {
    if ((e = moe::launch_route_permute_small(logits, T, shape->E, shape->k, shape->n_shared,
                                             shape->score,
                                             shape->renormalize, ids, w, counts, offsets, r2a,
                                             a2r, stream, &n)) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_timer.mark(stream, "route_permute");
  } else {
    if ((e = moe::launch_route_permute(logits, T, shape->E, shape->k, shape->n_shared,
                                       shape->score, shape->renormalize, ids, w, counts,
                                       offsets, r2a, a2r, at<int32_t>(ws, L.scratch),
                                       grid_barrier_words(ws), status, g_wait_limit_ns, stream,
                                       &n)) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_timer.mark(stream, "route_permute");
  }
  if (fp8) {
    uint8_t* xq = at<uint8_t>(ws, L.xq);
    uint32_t* sxw = at<uint32_t>(ws, L.sxw);
    uint8_t* aq = at<uint8_t>(ws, L.act);
    uint32_t* asw = at<uint32_t>(ws, L.act_sfw);
    if ((e = moe::launch_quant_x(x, xq, at<float>(ws, L.sx), sxw, T, shape->H, stream, &n)) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    g_timer.mark(stream, "quantize_x");
    if ((e = moe::launch_gemm1_mx(p, xq, sxw, r2a, offsets, static_cast<const uint8_t*>(w13),
                                  w13_sf, aq, nullptr, asw, status, stream, &n)) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_timer.mark(stream, "gemm1_swiglu");
    if ((e = moe::launch_gemm2_mx(p, aq, asw, offsets, static_cast<const uint8_t*>(w2), w2_sf, y,
                                  status, stream, &n)) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_timer.mark(stream, "gemm2");
  } else if (moe::use_swap_gemm(T) && shape->H % 128 == 0) {
    // decode-sized: weights on the MMA's M side; GEMM2 splits K and the combine adds the
    // partial sums.  (GEMM1 with ReLU2 runs on the SM-pair kernel at every batch size.)
    const int splits = moe::swap_splits(p);
    float* part = at<float>(ws, L.part);  // GEMM1's partials are consumed before GEMM2's
    if (p.act == MOE_ACT_RELU2)
      e = moe::launch_gemm1_bf16(p, x, r2a, offsets, static_cast<const uint16_t*>(w13), act,
                                 status, stream, &n);
    else
      e = moe::launch_gemm1_swap(p, x, r2a, offsets, static_cast<const uint16_t*>(w13), act,
                                 part, moe::swap_splits_gemm1(p), status, stream, &n);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    g_timer.mark(stream, "gemm1_swiglu");
    int* splits_used = splits_word(ws);
    if ((e = moe::launch_gemm2_swap(p, act, offsets, static_cast<const uint16_t*>(w2), y, part,
                                    splits, splits_used, status, stream, &n)) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_timer.mark(stream, "gemm2");
    if (splits > 1) {
      if ((e = moe::launch_combine_parts(part, splits_used, R, w, a2r, out, T, shape->H,
                                         k_all(*shape), stream, &n)) != cudaSuccess)
        return MOE_ERR_CUDA;
      g_timer.mark(stream, "combine");
      g_last_launches = n;
      return MOE_OK;
    }
  } else {
    if ((e = moe::launch_gemm1_bf16(p, x, r2a, offsets, static_cast<const uint16_t*>(w13), act,
                                    status, stream, &n)) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_timer.mark(stream, "gemm1_swiglu");
    if ((e = moe::launch_gemm2_bf16(p, act, offsets, static_cast<const uint16_t*>(w2), y, status,
                                    stream, &n)) != cudaSuccess)
      return MOE_ERR_CUDA;
    g_timer.mark(stream, "gemm2");
  }
  if ((e = moe::launch_combine(y, w, a2r, out, T, shape->H, k_all(*shape), stream, &n)) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  g_timer.mark(stream, "combine");
  g_last_launches = n;
  return MOE_OK;
}

moe_status_t moe_get_device_status(void* ws, cudaStream_t stream) {
  g_last_launches = 0;
  if (!ws) return MOE_ERR_INVALID_ARG;
  int host = 0;
  if (cudaMemcpyAsync(&host, ws, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  // after a device-side failure the whole status block (with the grid barrier's words,
  // which a wait that gave up may leave mid-count) starts again from zero
  if (host != 0 && cudaMemsetAsync(ws, 0, kStatusBytes, stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status_t>(host);
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_MISALIGNED: return "misaligned pointer";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_BAD_INDEX: return "expert id out of range";
  }
  return "unknown status";
}

int moe_last_launch_count(void) { return g_last_launches; }

void moe_debug_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns ? ns : 4000000000ull; }

void moe_debug_inject_stall(int on) { moe::g_inject_stall = on ? 1 : 0; }

void moe_debug_time_stages(int on) {
  g_timer.on = on != 0;
  g_timer.n = -1;
}

int moe_debug_stage_times(const char** names, float* ms, int max) {
  const int n = g_timer.n;
  if (n <= 0) return 0;
  if (cudaEventSynchronize(g_timer.ev[n]) != cudaSuccess) return -1;
  for (int i = 0; i < n && i < max; ++i) {
    if (cudaEventElapsedTime(&ms[i], g_timer.ev[i], g_timer.ev[i + 1]) != cudaSuccess) return -1;
    names[i] = g_timer.name[i];
  }
  return n;
}

}  // extern "C"
