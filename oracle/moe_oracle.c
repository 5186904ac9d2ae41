/*
 * moe_oracle.c -- plain fp64 CPU oracle for the routed-expert MoE MLP forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file: only the tests, the package smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes is the plain definition of a routed mixture-of-experts MLP, written
 * one token and one selected expert at a time, in double precision:
 *
 *   routing      top-k experts per token by descending router logit, with weights
 *                (softmax renormalised over the selected k, or the sigmoid of the
 *                selected logit).  The pages (TileScale PR #70, "Design"; FlashInfer
 *                PR #6465, the MXFP4 x FP8 workload with top-k 10) name routing and
 *                top-k but fix neither the score function nor the tie rule; the
 *                readings used here are: ties go to the lower expert index, slot j is
 *                the j-th largest, renormalisation as the workload states.
 *   histogram    per-expert counts of the T*k (token, slot) assignments, exclusive
 *                prefix sum, and a stable scatter into an expert-sorted row space
 *                (FlashInfer PR #5129, "sorted I/O": expert-sorted intermediate rows).
 *   expert MLP   g = h.Wgate^T, u = h.Wup^T, a = silu(g)*u, y = a.Wdown^T
 *                (TileScale PR #70, "Design": kernel 1 is GEMM1 + SwiGLU, kernel 2 is
 *                GEMM2).  Gate rows come first in the fused [2I, H] matrix (reading).
 *                The ReLU2 variant (FlashInfer PR #5129, the Nemotron-3.5-Lightning
 *                shape measured with ReLU2): g = h.W1^T with W1 [I, H], a = max(g, 0)^2
 *                -- read as the non-gated squared ReLU, the pages name only "ReLU2".
 *   combine      out[t] = sum over slots j (ascending) of w[t,j] * y_j, rounded once to
 *                bf16 (TileScale PR #70, the top-k slot reduction of kernel 2).
 *   shared       n_shared always-on experts (index E + s) as extra slots of weight 1 after
 *                the k routed ones (the pages fold shared experts into the compute; the
 *                slot reading is this file's).
 *   block-scaled activations: FP8 e4m3 with one power-of-two fp32 scale per 1x128 group
 *                (TileScale PR #70, "Design": FP8 E4M3 with fp32 per-128-element
 *                scales); weights: MXFP4 e2m1 with one UE8M0 scale per 32 consecutive
 *                K elements (FlashInfer PR #6465, the MXFP4 K32 workload).  The scale
 *                rule for activations (smallest power of two that keeps amax within
 *                448) and the weight rule (OCP MX: 2^(floor(log2 amax) - 2)) are the
 *                readings; the pages only name the formats.
 *
 * Number formats are decoded from their bit fields and encoded by rounding the real
 * value to the format's grid (round to nearest, ties to even) and then looking the
 * rounded value up in the decode table, so the encoder can be checked against the
 * decoder by eye.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------------------ */
/* number formats                                                                       */
/* ------------------------------------------------------------------------------------ */

double orc_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round |a| (a >= 0, finite) to a binary grid with p significant bits whose smallest
 * normal value is 2^emin (values below it are subnormal with a fixed quantum).
 * Ties go to the even neighbour (rint in the default rounding mode). */
static double round_to_grid(double a, int p, int emin) {
  if (a == 0.0) return 0.0;
  int e;
  frexp(a, &e);        /* a = m * 2^e, m in [0.5, 1)  =>  floor(log2 a) = e - 1 */
  int exp2 = e - 1;
  if (exp2 < emin) exp2 = emin;
  double q = ldexp(1.0, exp2 - (p - 1));
  return rint(a / q) * q;
}

uint16_t orc_f64_to_bf16_rne(double v) {
  if (isnan(v)) return 0x7fc0;
  double a = fabs(v);
  double r = round_to_grid(a, 8, -126);
  double maxf = ldexp(2.0 - ldexp(1.0, -7), 127);
  float f;
  if (r > maxf) f = INFINITY; else f = (float)r; /* r is on the bf16 grid: exact in float */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  uint16_t bits = (uint16_t)(u >> 16);
  if (signbit(v)) bits |= 0x8000;
  return bits;
}

/* FP8 e4m3 "fn": sign, 4 exponent bits (bias 7), 3 mantissa bits, no infinities,
 * S.1111.111 is NaN, largest finite 448. */
double orc_e4m3_decode(uint8_t c) {
  int s = c >> 7, E = (c >> 3) & 15, M = c & 7;
  double v;
  if (E == 15 && M == 7) return NAN;
  if (E == 0) v = ldexp((double)M, -9);                 /* M/8 * 2^(1-7) */
  else        v = ldexp(1.0 + M / 8.0, E - 7);
  return s ? -v : v;
}

uint8_t orc_e4m3_encode_rne_satfinite(double v) {
  if (isnan(v)) return 0x7f;
  double r = round_to_grid(fabs(v), 4, -6);
  if (r > 448.0) r = 448.0;
  for (int c = 0; c < 128; ++c)
    if (orc_e4m3_decode((uint8_t)c) == r) return (uint8_t)(c | (signbit(v) ? 0x80 : 0));
  return 0x7f; /* unreachable for finite v */
}

/* FP4 e2m1: sign, 2 exponent bits (bias 1), 1 mantissa bit; values 0, .5, 1, 1.5, 2,
 * 3, 4, 6.  Only the low nibble of c is read. */
double orc_e2m1_decode(uint8_t c) {
  int s = (c >> 3) & 1, E = (c >> 1) & 3, M = c & 1;
  double v = (E == 0) ? 0.5 * M : ldexp(1.0 + M / 2.0, E - 1);
  return s ? -v : v;
}

uint8_t orc_e2m1_encode_rne_satfinite(double v) {
  double r = round_to_grid(fabs(v), 2, 0);
  if (r > 6.0) r = 6.0;
  for (int c = 0; c < 8; ++c)
    if (orc_e2m1_decode((uint8_t)c) == r) return (uint8_t)(c | (signbit(v) ? 0x8 : 0));
  return 0x7; /* unreachable */
}

/* UE8M0: an unsigned biased exponent, value 2^(b-127); 255 is NaN. */
double orc_ue8m0_decode(uint8_t b) {
  if (b == 255) return NAN;
  return ldexp(1.0, (int)b - 127);
}

/* ------------------------------------------------------------------------------------ */
/* routing                                                                              */
/* ------------------------------------------------------------------------------------ */

/* score: 0 = softmax, 1 = sigmoid.  renorm: renormalise the k selected weights to sum 1.
 * Returns 0, or -1 on bad arguments. */
int orc_route(int64_t T, int E, int k, int score, int renorm, const float *logits,
              int32_t *ids, double *w) {
  if (T < 0 || E < 1 || k < 1 || k > E) return -1;
  char *sel = (char *)malloc((size_t)E);
  if (!sel) return -1;
  for (int64_t t = 0; t < T; ++t) {
    const float *l = logits + t * (int64_t)E;
    memset(sel, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (sel[e]) continue;
        if (best < 0 || (double)l[e] > (double)l[best]) best = e; /* strict: lower index wins ties */
      }
      sel[best] = 1;
      ids[t * k + j] = best;
    }
    if (score == 0) {
      double m = -INFINITY;
      for (int e = 0; e < E; ++e) if ((double)l[e] > m) m = (double)l[e];
      double den = 0.0;
      if (renorm) for (int j = 0; j < k; ++j) den += exp((double)l[ids[t * k + j]] - m);
      else        for (int e = 0; e < E; ++e) den += exp((double)l[e] - m);
      for (int j = 0; j < k; ++j) w[t * k + j] = exp((double)l[ids[t * k + j]] - m) / den;
    } else {
      double sum = 0.0;
      for (int j = 0; j < k; ++j) {
        w[t * k + j] = 1.0 / (1.0 + exp(-(double)l[ids[t * k + j]]));
        sum += w[t * k + j];
      }
      if (renorm) for (int j = 0; j < k; ++j) w[t * k + j] /= sum;
    }
  }
  free(sel);
  return 0;
}

/* Shared experts folded into the routed computation (GC-MoE "shared experts folded into
 * the compute role"; DeepGEMM's "fused shared-expert execution" as the TileScale PR
 * mentions it): experts E .. E+n_shared-1 run on every token with weight 1, read as
 * extra slots k .. k+n_shared-1 appended after the k routed ones.  ids/w are
 * [T][k + n_shared]. */
int orc_route_shared(int64_t T, int E, int k, int n_shared, int score, int renorm,
                     const float *logits, int32_t *ids, double *w) {
  if (n_shared < 0) return -1;
  const int ks = k + n_shared;
  int32_t *rid = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T * k + 1));
  double *rw = (double *)malloc(sizeof(double) * (size_t)(T * k + 1));
  if (!rid || !rw) { free(rid); free(rw); return -1; }
  int rc = orc_route(T, E, k, score, renorm, logits, rid, rw);
  if (rc == 0) {
    for (int64_t t = 0; t < T; ++t) {
      for (int j = 0; j < k; ++j) {
        ids[t * ks + j] = rid[t * k + j];
        w[t * ks + j] = rw[t * k + j];
      }
      for (int s = 0; s < n_shared; ++s) {
        ids[t * ks + k + s] = E + s;
        w[t * ks + k + s] = 1.0;
      }
    }
  }
  free(rid); free(rw);
  return rc;
}

/* ------------------------------------------------------------------------------------ */
/* histogram, exclusive prefix sum, stable permutation                                  */
/* ------------------------------------------------------------------------------------ */

int orc_permute(int64_t T, int E, int k, const int32_t *ids, int32_t *counts,
                int32_t *offsets, int32_t *row2assign, int32_t *assign2row) {
  int64_t R = T * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t a = 0; a < R; ++a) {
    if (ids[a] < 0 || ids[a] >= E) return -1;
    counts[ids[a]] += 1;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
  if (!fill) return -1;
  for (int e = 0; e < E; ++e) fill[e] = offsets[e];
  for (int64_t a = 0; a < R; ++a) {      /* ascending a: stable within each expert */
    int32_t r = fill[ids[a]]++;
    row2assign[r] = (int32_t)a;
    assign2row[a] = r;
  }
  free(fill);
  return 0;
}

/* ------------------------------------------------------------------------------------ */
/* block-scaled quantisers                                                              */
/* ------------------------------------------------------------------------------------ */

/* Power-of-two scale exponent for one 1x128 group: the smallest integer s with
 * amax <= 448 * 2^s, clamped to [-127, 127] so that 2^s is also a UE8M0 value;
 * amax == 0 gives s = 0. */
static int fp8_group_exponent(double amax) {
  if (amax == 0.0) return 0;
  int s = -127;
  while (s < 127 && amax > ldexp(448.0, s)) ++s;
  return s;
}

/* Quantise rows of `cols` values (cols % 128 == 0) to e4m3 codes with one fp32
 * power-of-two scale per 128 consecutive columns. */
void orc_quant_fp8_rows(int64_t rows, int cols, const double *v, uint8_t *codes,
                        float *scales) {
  int G = cols / 128;
  for (int64_t r = 0; r < rows; ++r) {
    for (int g = 0; g < G; ++g) {
      const double *p = v + r * cols + g * 128;
      double amax = 0.0;
      for (int i = 0; i < 128; ++i) if (fabs(p[i]) > amax) amax = fabs(p[i]);
      int s = fp8_group_exponent(amax);
      scales[r * G + g] = (float)ldexp(1.0, s);
      for (int i = 0; i < 128; ++i)
        codes[r * cols + g * 128 + i] = orc_e4m3_encode_rne_satfinite(ldexp(p[i], -s));
    }
  }
}

/* The same for bf16 input rows (the activation quantiser of the block-scaled path). */
void orc_quant_fp8_bf16_rows(int64_t rows, int cols, const uint16_t *x, uint8_t *codes,
                             float *scales) {
  double *tmp = (double *)malloc(sizeof(double) * (size_t)cols);
  for (int64_t r = 0; r < rows; ++r) {
    for (int c = 0; c < cols; ++c) tmp[c] = orc_bf16_to_f64(x[r * cols + c]);
    orc_quant_fp8_rows(1, cols, tmp, codes + r * cols, scales + r * (cols / 128));
  }
  free(tmp);
}

/* MXFP4 weights (OCP MX rule): per row and per 32 consecutive K, X = floor(log2 amax)-2,
 * UE8M0 byte = clamp(X + 127, 0, 254) (amax == 0 gives byte 0), codes = e2m1 of
 * w / 2^(byte-127).  packed[r][k/2] holds element k in its low nibble when k is even. */
void orc_quant_mxfp4(int64_t rows, int K, const uint16_t *w, uint8_t *packed, uint8_t *sf) {
  int G = K / 32;
  for (int64_t r = 0; r < rows; ++r) {
    for (int g = 0; g < G; ++g) {
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) {
        double a = fabs(orc_bf16_to_f64(w[r * K + g * 32 + i]));
        if (a > amax) amax = a;
      }
      int byte = 0;
      if (amax > 0.0) {
        int e;
        frexp(amax, &e);
        int X = (e - 1) - 2;
        byte = X + 127;
        if (byte < 0) byte = 0;
        if (byte > 254) byte = 254;
      }
      sf[r * G + g] = (uint8_t)byte;
      for (int i = 0; i < 32; ++i) {
        int kk = g * 32 + i;
        double q = ldexp(orc_bf16_to_f64(w[r * K + kk]), -(byte - 127));
        uint8_t c = orc_e2m1_encode_rne_satfinite(q);
        uint8_t *dst = packed + r * (K / 2) + kk / 2;
        if (kk % 2 == 0) *dst = (uint8_t)((*dst & 0xf0) | c);
        else             *dst = (uint8_t)((*dst & 0x0f) | (c << 4));
      }
    }
  }
}

static double mxfp4_value(const uint8_t *packed, const uint8_t *sf, int K, int64_t r, int kk) {
  uint8_t byte = packed[r * (K / 2) + kk / 2];
  uint8_t c = (kk % 2 == 0) ? (byte & 0xf) : (byte >> 4);
  return orc_e2m1_decode(c) * orc_ue8m0_decode(sf[r * (K / 32) + kk / 32]);
}

/* ------------------------------------------------------------------------------------ */
/* one expert's MLP on one token row                                                    */
/* ------------------------------------------------------------------------------------ */

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* act[i] = silu(h . W13[i]) * (h . W13[I+i]); W13 is this expert's [2I, H] bf16 block. */
static void expert_act_bf16(int H, int I, const double *h, const uint16_t *w13e, double *act) {
  for (int i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    const uint16_t *wg = w13e + (int64_t)i * H;
    const uint16_t *wu = w13e + (int64_t)(I + i) * H;
    for (int c = 0; c < H; ++c) g += h[c] * orc_bf16_to_f64(wg[c]);
    for (int c = 0; c < H; ++c) u += h[c] * orc_bf16_to_f64(wu[c]);
    act[i] = silu(g) * u;
  }
}

/* act[i] = max(h . W1[i], 0)^2; W1 is this expert's [I, H] bf16 block (ReLU2). */
static void expert_act_relu2_bf16(int H, int I, const double *h, const uint16_t *w1e,
                                  double *act) {
  for (int i = 0; i < I; ++i) {
    double g = 0.0;
    const uint16_t *wr = w1e + (int64_t)i * H;
    for (int c = 0; c < H; ++c) g += h[c] * orc_bf16_to_f64(wr[c]);
    act[i] = g > 0.0 ? g * g : 0.0;
  }
}

/* The activation of GEMM1: kind 0 = SwiGLU (W13 block [2I, H]), 1 = ReLU2 (W1 [I, H]). */
static void expert_act_kind_bf16(int kind, int H, int I, const double *h,
                                 const uint16_t *w13, int e, double *act) {
  if (kind == 1)
    expert_act_relu2_bf16(H, I, h, w13 + (int64_t)e * I * H, act);
  else
    expert_act_bf16(H, I, h, w13 + (int64_t)e * 2 * I * H, act);
}

/* y[o] = act . W2[o]; W2 is this expert's [H, I] bf16 block. */
static void expert_down_bf16(int H, int I, const double *act, const uint16_t *w2e, double *y) {
  for (int o = 0; o < H; ++o) {
    double s = 0.0;
    const uint16_t *wr = w2e + (int64_t)o * I;
    for (int i = 0; i < I; ++i) s += act[i] * orc_bf16_to_f64(wr[i]);
    y[o] = s;
  }
}

/* Block-scaled variants: the weights are the MXFP4 codes of expert e, dequantised
 * element by element as e2m1 * 2^(byte-127). */
static void expert_act_mx(int H, int I, const double *h, const uint8_t *w13p,
                          const uint8_t *w13sf, int e, double *act) {
  int64_t base = (int64_t)e * 2 * I;
  for (int i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    for (int c = 0; c < H; ++c) g += h[c] * mxfp4_value(w13p, w13sf, H, base + i, c);
    for (int c = 0; c < H; ++c) u += h[c] * mxfp4_value(w13p, w13sf, H, base + I + i, c);
    act[i] = silu(g) * u;
  }
}

static void expert_down_mx(int H, int I, const double *act, const uint8_t *w2p,
                           const uint8_t *w2sf, int e, double *y) {
  int64_t base = (int64_t)e * H;
  for (int o = 0; o < H; ++o) {
    double s = 0.0;
    for (int i = 0; i < I; ++i) s += act[i] * mxfp4_value(w2p, w2sf, I, base + o, i);
    y[o] = s;
  }
}

/* Requantise an fp64 activation row with the 1x128 e4m3 rule and return the
 * dequantised values in place (the block-scaled path's GEMM1 -> GEMM2 hand-off). */
static void requant_row_inplace(int I, double *act, uint8_t *codes, float *scales) {
  orc_quant_fp8_rows(1, I, act, codes, scales);
  for (int i = 0; i < I; ++i) act[i] = orc_e4m3_decode(codes[i]) * (double)scales[i / 128];
}

/* ------------------------------------------------------------------------------------ */
/* whole forward pass on a list of tokens                                               */
/* ------------------------------------------------------------------------------------ */

/* BF16 path.  ids/w come from orc_route.  For each listed token t:
 *   out[n][:] = sum_j w[t,j] * expert_mlp(ids[t,j], x[t]),  fp64, and its bf16 rounding. */
void orc_forward_bf16_act(int64_t T, int H, int I, int E, int k, int kind,
                          const uint16_t *x, const int32_t *ids, const double *w,
                          const uint16_t *w13, const uint16_t *w2, int64_t n_tok,
                          const int64_t *tok, double *out, uint16_t *out_bf16) {
  (void)T; (void)E;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t n = 0; n < n_tok; ++n) {
    int64_t t = tok[n];
    double *h = (double *)malloc(sizeof(double) * (size_t)H);
    double *act = (double *)malloc(sizeof(double) * (size_t)I);
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    double *acc = out + n * H;
    for (int c = 0; c < H; ++c) { h[c] = orc_bf16_to_f64(x[t * H + c]); acc[c] = 0.0; }
    for (int j = 0; j < k; ++j) {
      int e = ids[t * k + j];
      expert_act_kind_bf16(kind, H, I, h, w13, e, act);
      expert_down_bf16(H, I, act, w2 + (int64_t)e * H * I, y);
      for (int c = 0; c < H; ++c) acc[c] += w[t * k + j] * y[c];
    }
    for (int c = 0; c < H; ++c) out_bf16[n * H + c] = orc_f64_to_bf16_rne(acc[c]);
    free(h); free(act); free(y);
  }
}

void orc_forward_bf16(int64_t T, int H, int I, int E, int k, const uint16_t *x,
                      const int32_t *ids, const double *w, const uint16_t *w13,
                      const uint16_t *w2, int64_t n_tok, const int64_t *tok, double *out,
                      uint16_t *out_bf16) {
  orc_forward_bf16_act(T, H, I, E, k, 0, x, ids, w, w13, w2, n_tok, tok, out, out_bf16);
}

/* Block-scaled path: x is quantised per token (1x128 e4m3 + pow2 scale) and
 * dequantised; GEMM1 runs on the MXFP4 weights; the activation is requantised with the
 * same 1x128 rule when requant_act != 0; GEMM2 runs on the MXFP4 weights. */
void orc_forward_fp8_mxfp4(int64_t T, int H, int I, int E, int k, const uint16_t *x,
                           const int32_t *ids, const double *w, const uint8_t *w13p,
                           const uint8_t *w13sf, const uint8_t *w2p, const uint8_t *w2sf,
                           int requant_act, int64_t n_tok, const int64_t *tok, double *out,
                           uint16_t *out_bf16) {
  (void)T; (void)E;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t n = 0; n < n_tok; ++n) {
    int64_t t = tok[n];
    double *h = (double *)malloc(sizeof(double) * (size_t)H);
    double *act = (double *)malloc(sizeof(double) * (size_t)I);
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    uint8_t *xc = (uint8_t *)malloc((size_t)H);
    float *xs = (float *)malloc(sizeof(float) * (size_t)(H / 128));
    uint8_t *ac = (uint8_t *)malloc((size_t)I);
    float *as = (float *)malloc(sizeof(float) * (size_t)(I / 128));
    double *acc = out + n * H;
    orc_quant_fp8_bf16_rows(1, H, x + t * H, xc, xs);
    for (int c = 0; c < H; ++c) { h[c] = orc_e4m3_decode(xc[c]) * (double)xs[c / 128]; acc[c] = 0.0; }
    for (int j = 0; j < k; ++j) {
      int e = ids[t * k + j];
      expert_act_mx(H, I, h, w13p, w13sf, e, act);
      if (requant_act) requant_row_inplace(I, act, ac, as);
      expert_down_mx(H, I, act, w2p, w2sf, e, y);
      for (int c = 0; c < H; ++c) acc[c] += w[t * k + j] * y[c];
    }
    for (int c = 0; c < H; ++c) out_bf16[n * H + c] = orc_f64_to_bf16_rne(acc[c]);
    free(h); free(act); free(y); free(xc); free(xs); free(ac); free(as);
  }
}

/* ------------------------------------------------------------------------------------ */
/* single stages on listed rows of the expert-sorted row space                          */
/* ------------------------------------------------------------------------------------ */

/* GEMM1 + activation for listed rows: row n uses token tok[n] of x and expert exp_[n]. */
void orc_gemm1_bf16_rows_act(int kind, int H, int I, const uint16_t *x, const uint16_t *w13,
                             int64_t n_rows, const int64_t *tok, const int32_t *exp_,
                             double *act) {
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t n = 0; n < n_rows; ++n) {
    double *h = (double *)malloc(sizeof(double) * (size_t)H);
    for (int c = 0; c < H; ++c) h[c] = orc_bf16_to_f64(x[tok[n] * H + c]);
    expert_act_kind_bf16(kind, H, I, h, w13, exp_[n], act + n * I);
    free(h);
  }
}

void orc_gemm1_bf16_rows(int H, int I, const uint16_t *x, const uint16_t *w13, int64_t n_rows,
                         const int64_t *tok, const int32_t *exp_, double *act) {
  orc_gemm1_bf16_rows_act(0, H, I, x, w13, n_rows, tok, exp_, act);
}

/* GEMM2 for listed rows: y[n] = a[row[n]] . W2[exp_[n]]^T with a given as bf16 rows. */
void orc_gemm2_bf16_rows(int H, int I, const uint16_t *a, const uint16_t *w2, int64_t n_rows,
                         const int64_t *row, const int32_t *exp_, double *y) {
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t n = 0; n < n_rows; ++n) {
    double *act = (double *)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < I; ++i) act[i] = orc_bf16_to_f64(a[row[n] * I + i]);
    expert_down_bf16(H, I, act, w2 + (int64_t)exp_[n] * H * I, y + n * H);
    free(act);
  }
}

/* Block-scaled GEMM1 + SwiGLU (+ requant) for listed rows; x is given as e4m3 codes
 * with 1x128 scales.  act receives the dequantised result (after requant when on). */
void orc_gemm1_fp8_rows(int H, int I, const uint8_t *xq, const float *sx, const uint8_t *w13p,
                        const uint8_t *w13sf, int requant_act, int64_t n_rows,
                        const int64_t *tok, const int32_t *exp_, double *act) {
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t n = 0; n < n_rows; ++n) {
    double *h = (double *)malloc(sizeof(double) * (size_t)H);
    uint8_t *ac = (uint8_t *)malloc((size_t)I);
    float *as = (float *)malloc(sizeof(float) * (size_t)(I / 128));
    for (int c = 0; c < H; ++c)
      h[c] = orc_e4m3_decode(xq[tok[n] * H + c]) * (double)sx[tok[n] * (H / 128) + c / 128];
    expert_act_mx(H, I, h, w13p, w13sf, exp_[n], act + n * I);
    if (requant_act) requant_row_inplace(I, act + n * I, ac, as);
    free(h); free(ac); free(as);
  }
}

/* Block-scaled GEMM2 for listed rows; a is given as e4m3 codes with 1x128 scales. */
void orc_gemm2_fp8_rows(int H, int I, const uint8_t *aq, const float *sa, const uint8_t *w2p,
                        const uint8_t *w2sf, int64_t n_rows, const int64_t *row,
                        const int32_t *exp_, double *y) {
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t n = 0; n < n_rows; ++n) {
    double *act = (double *)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < I; ++i)
      act[i] = orc_e4m3_decode(aq[row[n] * I + i]) * (double)sa[row[n] * (I / 128) + i / 128];
    expert_down_mx(H, I, act, w2p, w2sf, exp_[n], y + n * H);
    free(act);
  }
}

/* Combine for listed tokens: out[n] = sum_j w[t,j] * y[assign2row[t*k+j]] (y as bf16
 * rows), fp64, ascending j, then one bf16 rounding. */
void orc_combine(int H, int k, const uint16_t *y, const float *w, const int32_t *assign2row,
                 int64_t n_tok, const int64_t *tok, double *out, uint16_t *out_bf16) {
  for (int64_t n = 0; n < n_tok; ++n) {
    int64_t t = tok[n];
    for (int c = 0; c < H; ++c) {
      double s = 0.0;
      for (int j = 0; j < k; ++j)
        s += (double)w[t * k + j] * orc_bf16_to_f64(y[(int64_t)assign2row[t * k + j] * H + c]);
      out[n * H + c] = s;
      out_bf16[n * H + c] = orc_f64_to_bf16_rne(s);
    }
  }
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
