// MoE-layer oracle: a plain, slow CPU statement of what the GPU path computes.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call
// this file; only the test suite, the smoke check and the benchmark's CPU
// baseline leg use it. It shares no code, header or table with the CUDA
// library: every definition below is written out again from its source.
//
// What it follows (the pages):
//  * The MoE layer has three stages per layer, token dispatch, grouped expert
//    GEMMs and a combine (GC-MoE feed item, "Key points"; GC-MoE explainer,
//    "Why Expert Parallelism Is Inefficient in MoE Decoding").
//  * Tokens go to experts according to the gating/routing result (GC-MoE
//    explainer, same section). The routing rule itself, softmax over the router
//    logits then top-k with optional renormalisation, is not printed on the
//    pages; it is the reading taken here (softmax is monotone, so the k
//    largest logits are the k largest probabilities).
//  * The expert FFN is a gated (SwiGLU) FFN with a requantisation fused after
//    the activation (GC-MoE feed item, "Full text"; explainer, "Two MMA
//    Implementations in the Compute Partition"). SwiGLU is read as
//    h = silu(x W_gate^T) * (x W_up^T), y = h W_down^T.
//  * FP8 operands carry block scale factors (explainer, tcgen05 paragraph of
//    "Two MMA Implementations"). The pages print a 32-element block; the layer
//    here uses 128-element blocks with power-of-two fp32 scales, which the same
//    block-scaled MMA consumes exactly.
//  * 4-bit weights are the microscaling (MX) form the same paragraph names:
//    every 32 consecutive elements share one exponent scale, and the weights
//    shrink to 4 bits. Read as the OCP MX formats: FP4 E2M1 elements with one
//    UE8M0 scale (2^(byte - 127)) per 32 elements along K.
//  * Combine weights each expert output by its routing weight and sums back in
//    token order (NVLinkOneSided abstract; Ascend report abstract: combine
//    reads expert outputs straight out of the expert windows).
//
// Precision: every sum and product is formed in double. A value is rounded
// only where the GPU path stores it (x to e4m3, h to fp32 then bf16/e4m3,
// y and out to fp32 then bf16); where the rounding decides an integer code
// the decision is taken from the fp32 value, the precision the kernels decide
// in.
//
// Parity pins live in tests/test_oracle_pins.py.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>
#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// dtype codes used by this oracle's own entry points
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_E4M3 = 2, ORC_E2M1 = 3 };

enum {
  ORC_OK = 0,
  ORC_BAD_ARG = 1,
  ORC_NONFINITE = 6,
};

typedef struct oracle_problem {
  int64_t T, H, E, k, I;
  int32_t x_dtype;    // ORC_F32 or ORC_BF16 (raw 16-bit patterns)
  int32_t xq_dtype;   // how tokens are stored for the experts
  int32_t w_dtype;    // expert weight dtype
  int32_t h_dtype;    // dtype of the SwiGLU output h
  int32_t y_dtype;    // ORC_F32 or ORC_BF16: expert output rows
  int32_t out_dtype;  // ORC_F32 or ORC_BF16: layer output
  int32_t renorm;     // 1: weights renormalised over the k selected experts
  int32_t identity;   // 1: every expert is the identity map on its input
  int32_t shared;     // 1: expert E is a shared expert every token also goes
                      //    through, added with weight 1 after the k routed ones
  // One pointer per expert (E + shared entries each). Expert e's matrices are
  // row-major: gate/up [I, H], down [H, I]; e4m3 scales fp32 [I/128, H/128]
  // and [H/128, I/128]. e2m1 weights hold two elements per byte (element 2i
  // in the low nibble of byte i of its row) with UE8M0 scale bytes
  // [I, H/32] and [H, I/32]. A NULL entry marks an expert whose weights were
  // not provided; using it is an error.
  const void* const* w_gate;
  const void* const* w_up;
  const void* const* w_down;
  const void* const* s_gate;  // e4m3 and e2m1 weights only
  const void* const* s_up;
  const void* const* s_down;
} oracle_problem;

// ---------------------------------------------------------------- formats --

// OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits with
// bias 7, 3 mantissa bits; exponent field 0 holds subnormals m * 2^-9; the
// all-ones pattern S.1111.111 is NaN and there is no infinity, so the largest
// finite magnitude is 1.75 * 2^8 = 448.
static double e4m3_value(uint8_t code) {
  const int sign = code >> 7;
  const int ef = (code >> 3) & 15;
  const int mf = code & 7;
  double mag;
  if (ef == 15 && mf == 7) return std::nan("");
  if (ef == 0) mag = std::ldexp((double)mf, -9);
  else mag = std::ldexp(1.0 + mf / 8.0, ef - 7);
  return sign ? -mag : mag;
}

// Round to the nearest E4M3 value, ties to an even mantissa, clamping
// magnitudes beyond 448 to 448 ("satfinite"). The sign of the input is kept,
// also when the magnitude rounds to zero.
static uint8_t e4m3_code(double v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  double a = std::fabs(v);
  if (a >= 448.0) return sign | 0x7E;
  const double min_normal = std::ldexp(1.0, -6);
  if (a < min_normal) {
    // subnormal grid, step 2^-9; n = 8 is the smallest normal, code 0x08
    double n = std::nearbyint(a / std::ldexp(1.0, -9));
    return sign | (uint8_t)n;
  }
  int e;
  double fr = std::frexp(a, &e);  // a = fr * 2^e, fr in [0.5, 1)
  int exp2 = e - 1;               // a = (2 fr) * 2^exp2, 2 fr in [1, 2)
  double mant = std::nearbyint((2.0 * fr - 1.0) * 8.0);
  if (mant == 8.0) { mant = 0.0; exp2 += 1; }
  int code = ((exp2 + 7) << 3) | (int)mant;
  if (code > 0x7E) code = 0x7E;
  return sign | (uint8_t)code;
}

// OCP MX FP4, E2M1: 1 sign bit (bit 3), 2 exponent bits with bias 1, 1
// mantissa bit; exponent field 0 holds the subnormal m * 2^-1. No infinity
// or NaN: the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6.
static double e2m1_value(uint8_t code) {
  const int sign = (code >> 3) & 1;
  const int ef = (code >> 1) & 3;
  const int mf = code & 1;
  const double mag = ef == 0 ? 0.5 * mf : std::ldexp(1.0 + 0.5 * mf, ef - 1);
  return sign ? -mag : mag;
}

// OCP MX UE8M0 scale: 2^(byte - 127); the byte 255 is NaN.
static double ue8m0_value(uint8_t b) {
  if (b == 255) return std::nan("");
  return std::ldexp(1.0, (int)b - 127);
}

// bfloat16: the upper 16 bits of an IEEE binary32.
static double bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// Round a binary32 value to bfloat16, nearest, ties to even; returned as the
// binary32 value it represents.
static float bf16_round_f32(float f) {
  if (std::isnan(f)) return f;
  if (f == 0.0f || std::isinf(f)) return f;
  double v = (double)f;
  int e;
  std::frexp(std::fabs(v), &e);
  int exp2 = e - 1;                      // |v| in [2^exp2, 2^(exp2+1))
  int q = exp2 < -126 ? -133 : exp2 - 7; // bf16 quantum: 8 significant bits
  double r = std::nearbyint(std::ldexp(v, -q));
  double out = std::ldexp(r, q);
  const double bf16_max = std::ldexp(255.0, 120);  // (2 - 2^-7) * 2^127
  if (std::fabs(out) > bf16_max) out = std::copysign(INFINITY, v);
  return (float)out;
}

static uint16_t bf16_bits_of(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

// Power-of-two block scale: the smallest 2^p with amax <= 448 * 2^p, p clamped
// to [-126, 127]; 1 for an all-zero block. Dividing by it is exact and never
// saturates.
static double pow2_scale(double amax) {
  if (!(amax > 0.0)) return 1.0;
  // every comparison below is exact: 448 * 2^p is a double for these p
  int p = std::ilogb(amax) - 8;
  if (p < -126) p = -126;
  if (p > 127) p = 127;
  while (p < 127 && std::ldexp(448.0, p) < amax) ++p;
  while (p > -126 && std::ldexp(448.0, p - 1) >= amax) --p;
  return std::ldexp(1.0, p);
}

// ----------------------------------------------------------- small helpers --

int oracle_e4m3_encode(const double* v, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_code(v[i]);
  return ORC_OK;
}

int oracle_e4m3_decode(const uint8_t* q, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(q[i]);
  return ORC_OK;
}

// 4-bit E2M1 codes (one per byte, low nibble) and UE8M0 scale bytes to doubles
int oracle_e2m1_decode(const uint8_t* q, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = e2m1_value(q[i] & 15);
  return ORC_OK;
}

int oracle_ue8m0_decode(const uint8_t* b, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = ue8m0_value(b[i]);
  return ORC_OK;
}

int oracle_bf16_round(const float* v, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_bits_of(bf16_round_f32(v[i]));
  return ORC_OK;
}

int oracle_pow2_scale(const double* amax, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = pow2_scale(amax[i]);
  return ORC_OK;
}

// ------------------------------------------------------------------ route --

// Per token: the k largest logits (equal logits: the lower expert index
// first), in descending order; weights are the softmax probabilities of the
// selected experts, either as they are (denominator over all E experts) or
// renormalised over the k selected ones.
int oracle_route(int64_t T, int64_t E, int64_t k, int32_t renorm,
                 const float* logits, int32_t* idx, float* w) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return ORC_BAD_ARG;
  for (int64_t i = 0; i < T * E; ++i)
    if (!std::isfinite(logits[i])) return ORC_NONFINITE;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    const float* s = logits + t * E;
    std::vector<std::pair<float, int32_t>> order(E);
    for (int64_t e = 0; e < E; ++e) order[e] = {-s[e], (int32_t)e};
    std::sort(order.begin(), order.end());  // ascending (-logit, index)
    const double m = (double)s[order[0].second];
    double denom = 0.0;
    if (renorm) {
      for (int64_t j = 0; j < k; ++j) denom += std::exp((double)s[order[j].second] - m);
    } else {
      for (int64_t e = 0; e < E; ++e) denom += std::exp((double)s[e] - m);
    }
    for (int64_t j = 0; j < k; ++j) {
      idx[t * k + j] = order[j].second;
      w[t * k + j] = (float)(std::exp((double)s[order[j].second] - m) / denom);
    }
  }
  return ORC_OK;
}

// Tokens per expert implied by a routing result.
int oracle_counts(int64_t T, int64_t E, int64_t k, const int32_t* idx, int32_t* counts) {
  for (int64_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t i = 0; i < T * k; ++i) {
    if (idx[i] < 0 || idx[i] >= E) return ORC_BAD_ARG;
    counts[idx[i]] += 1;
  }
  return ORC_OK;
}

// --------------------------------------------------------------- quantise --

// One row of n values (n a multiple of 128) to e4m3 codes with one
// power-of-two scale per 128 consecutive values; v is the binary32 row.
static void quantize_row(const float* v, int64_t n, uint8_t* q, float* s) {
  for (int64_t b = 0; b < n / 128; ++b) {
    double amax = 0.0;
    for (int64_t i = 0; i < 128; ++i) amax = std::max(amax, std::fabs((double)v[b * 128 + i]));
    const double sc = pow2_scale(amax);
    s[b] = (float)sc;
    for (int64_t i = 0; i < 128; ++i) q[b * 128 + i] = e4m3_code((double)v[b * 128 + i] / sc);
  }
}

// rows x H binary32 values -> e4m3 codes + per-128 scales
int oracle_quantize_rows(int64_t rows, int64_t H, const float* x, uint8_t* q, float* s) {
  if (H % 128) return ORC_BAD_ARG;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) quantize_row(x + r * H, H, q + r * H, s + r * (H / 128));
  return ORC_OK;
}

// ------------------------------------------------------------- expert FFN --

static double load_act(const void* p, int32_t dt, int64_t i) {
  if (dt == ORC_F32) return (double)((const float*)p)[i];
  return bf16_value(((const uint16_t*)p)[i]);
}

// element [r, c] of one expert's weight matrix of shape [rows, cols]
static inline double weight_at(const void* w, const void* s, int32_t dt,
                               int64_t cols, int64_t r, int64_t c) {
  const int64_t off = r * cols + c;
  if (dt == ORC_F32) return (double)((const float*)w)[off];
  if (dt == ORC_BF16) return bf16_value(((const uint16_t*)w)[off]);
  if (dt == ORC_E2M1) {
    const uint8_t byte = ((const uint8_t*)w)[r * (cols / 2) + c / 2];
    const uint8_t code = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
    return e2m1_value(code) * ue8m0_value(((const uint8_t*)s)[r * (cols / 32) + c / 32]);
  }
  const double sc = (double)((const float*)s)[(r / 128) * (cols / 128) + c / 128];
  return e4m3_value(((const uint8_t*)w)[off]) * sc;
}

static bool scaled_weights(int32_t dt) { return dt == ORC_E4M3 || dt == ORC_E2M1; }

static bool have_expert(const oracle_problem* p, int64_t e) {
  if (e < 0 || e >= p->E + (p->shared ? 1 : 0)) return false;
  if (!p->w_gate[e] || !p->w_up[e] || !p->w_down[e]) return false;
  if (scaled_weights(p->w_dtype) && (!p->s_gate[e] || !p->s_up[e] || !p->s_down[e])) return false;
  return true;
}

static double silu(double g) { return g / (1.0 + std::exp(-g)); }

// Expert e applied to one input row xh[H] (already in the precision the
// experts see). Writes the stored h (raw, h_dtype; hs for e4m3) and the stored
// y row (raw, y_dtype); yd receives the stored y as doubles.
static void expert_row(const oracle_problem* p, int64_t e, const double* xh,
                       void* h_raw, float* hs, void* y_raw, double* yd) {
  const int64_t H = p->H, I = p->I;
  const bool scaled = scaled_weights(p->w_dtype);
  const void* wg = p->w_gate[e];
  const void* wu = p->w_up[e];
  const void* wd = p->w_down[e];
  const void* sg = scaled ? p->s_gate[e] : nullptr;
  const void* su = scaled ? p->s_up[e] : nullptr;
  const void* sd = scaled ? p->s_down[e] : nullptr;
  std::vector<float> h32(I);
  std::vector<double> hh(I);
  for (int64_t i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    for (int64_t c = 0; c < H; ++c) {
      g += xh[c] * weight_at(wg, sg, p->w_dtype, H, i, c);
      u += xh[c] * weight_at(wu, su, p->w_dtype, H, i, c);
    }
    h32[i] = (float)(silu(g) * u);
  }
  if (p->h_dtype == ORC_F32) {
    for (int64_t i = 0; i < I; ++i) hh[i] = h32[i];
    if (h_raw) std::memcpy(h_raw, h32.data(), I * 4);
  } else if (p->h_dtype == ORC_BF16) {
    for (int64_t i = 0; i < I; ++i) {
      float r = bf16_round_f32(h32[i]);
      hh[i] = r;
      if (h_raw) ((uint16_t*)h_raw)[i] = bf16_bits_of(r);
    }
  } else {
    std::vector<uint8_t> q(I);
    std::vector<float> sc(I / 128);
    quantize_row(h32.data(), I, q.data(), sc.data());
    for (int64_t i = 0; i < I; ++i) hh[i] = e4m3_value(q[i]) * (double)sc[i / 128];
    if (h_raw) std::memcpy(h_raw, q.data(), I);
    if (hs) std::memcpy(hs, sc.data(), (I / 128) * 4);
  }
  for (int64_t c = 0; c < H; ++c) {
    double acc = 0.0;
    for (int64_t i = 0; i < I; ++i)
      acc += hh[i] * weight_at(wd, sd, p->w_dtype, I, c, i);
    float a32 = (float)acc;
    if (p->y_dtype == ORC_F32) {
      yd[c] = a32;
      if (y_raw) ((float*)y_raw)[c] = a32;
    } else {
      float r = bf16_round_f32(a32);
      yd[c] = r;
      if (y_raw) ((uint16_t*)y_raw)[c] = bf16_bits_of(r);
    }
  }
}

// The input row as the experts see it: x stored as xq_dtype (and, for e4m3,
// dequantised with its block scales). Raw codes go to xq_raw / xs if given.
static void token_input(const oracle_problem* p, const void* x, int64_t t, double* xh,
                        void* xq_raw, float* xs) {
  const int64_t H = p->H;
  std::vector<float> x32(H);
  for (int64_t c = 0; c < H; ++c) x32[c] = (float)load_act(x, p->x_dtype, t * H + c);
  if (p->xq_dtype == ORC_F32) {
    for (int64_t c = 0; c < H; ++c) xh[c] = x32[c];
    if (xq_raw) std::memcpy(xq_raw, x32.data(), H * 4);
  } else if (p->xq_dtype == ORC_BF16) {
    for (int64_t c = 0; c < H; ++c) {
      float r = bf16_round_f32(x32[c]);
      xh[c] = r;
      if (xq_raw) ((uint16_t*)xq_raw)[c] = bf16_bits_of(r);
    }
  } else {
    std::vector<uint8_t> q(H);
    std::vector<float> sc(H / 128);
    quantize_row(x32.data(), H, q.data(), sc.data());
    for (int64_t c = 0; c < H; ++c) xh[c] = e4m3_value(q[c]) * (double)sc[c / 128];
    if (xq_raw) std::memcpy(xq_raw, q.data(), H);
    if (xs) std::memcpy(xs, sc.data(), (H / 128) * 4);
  }
}

static int64_t dtype_bytes(int32_t dt) { return dt == ORC_F32 ? 4 : dt == ORC_BF16 ? 2 : 1; }

static int check_problem(const oracle_problem* p) {
  if (!p || p->T < 0 || p->H <= 0 || p->E <= 0 || p->k <= 0 || p->k > p->E || p->I <= 0)
    return ORC_BAD_ARG;
  if (p->shared != 0 && p->shared != 1) return ORC_BAD_ARG;
  if (p->xq_dtype == ORC_E4M3 && p->H % 128) return ORC_BAD_ARG;
  if (p->h_dtype == ORC_E4M3 && p->I % 128) return ORC_BAD_ARG;
  if (p->w_dtype == ORC_E4M3 && (p->H % 128 || p->I % 128)) return ORC_BAD_ARG;
  if (p->w_dtype == ORC_E2M1 && (p->H % 32 || p->I % 32)) return ORC_BAD_ARG;
  return ORC_OK;
}

// Experts applied to given rows: row r holds an input already in xq_dtype
// (codes + scales for e4m3) and goes to expert expert[r]. Outputs per row: h
// (h_dtype raw, hs for e4m3) and y (y_dtype raw). This checks the grouped FFN
// step on its own, fed with exactly the bytes the GPU dispatch wrote.
int oracle_expert_rows(const oracle_problem* p, int64_t rows, const int32_t* expert,
                       const void* xq, const float* xs, void* h_out, float* hs_out,
                       void* y_out) {
  int rc = check_problem(p);
  if (rc) return rc;
  const int64_t H = p->H, I = p->I;
  const int64_t hb = dtype_bytes(p->h_dtype), yb = dtype_bytes(p->y_dtype);
  for (int64_t r = 0; r < rows; ++r)
    if (!have_expert(p, expert[r])) return ORC_BAD_ARG;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < rows; ++r) {
    std::vector<double> xh(H), yd(H);
    for (int64_t c = 0; c < H; ++c) {
      if (p->xq_dtype == ORC_F32) xh[c] = ((const float*)xq)[r * H + c];
      else if (p->xq_dtype == ORC_BF16) xh[c] = bf16_value(((const uint16_t*)xq)[r * H + c]);
      else xh[c] = e4m3_value(((const uint8_t*)xq)[r * H + c]) * (double)xs[r * (H / 128) + c / 128];
    }
    expert_row(p, expert[r], xh.data(),
               h_out ? (char*)h_out + r * I * hb : nullptr,
               hs_out ? hs_out + r * (I / 128) : nullptr,
               y_out ? (char*)y_out + r * H * yb : nullptr, yd.data());
  }
  return ORC_OK;
}

// Weighted combine: out[t] = sum_j w[t,j] * y[t*k + j], summed in slot order,
// rounded once to out_dtype. y holds one row per (token, slot) pair in y_dtype.
int oracle_combine(int64_t T, int64_t k, int64_t H, int32_t y_dtype, const void* y,
                   const float* w, int32_t out_dtype, void* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int64_t j = 0; j < k; ++j)
        acc += (double)w[t * k + j] * load_act(y, y_dtype, (t * k + j) * H + c);
      float a32 = (float)acc;
      if (out_dtype == ORC_F32) ((float*)out)[t * H + c] = a32;
      else ((uint16_t*)out)[t * H + c] = bf16_bits_of(bf16_round_f32(a32));
    }
  }
  return ORC_OK;
}

// The whole layer for tokens [t0, t1): route (all T tokens, so idx/w are
// [T, k]), quantise, experts, combine. out is [t1-t0, H] in out_dtype.
// Optional per-token / per-pair intermediates (may be NULL):
//   xq_tok [t1-t0, H] xq_dtype raw, xs_tok [t1-t0, H/128],
//   y_pair [(t1-t0)*k, H] y_dtype raw.
int oracle_moe_layer(const oracle_problem* p, const void* x, const float* logits,
                     int64_t t0, int64_t t1, int32_t* idx, float* w, void* out,
                     void* xq_tok, float* xs_tok, void* y_pair) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (t0 < 0 || t1 > p->T || t0 > t1) return ORC_BAD_ARG;
  rc = oracle_route(p->T, p->E, p->k, p->renorm, logits, idx, w);
  if (rc) return rc;
  const int64_t H = p->H, k = p->k;
  // slots per token: the k routed experts, then the shared expert E (weight 1)
  const int64_t ks = k + (p->shared ? 1 : 0);
  const int64_t qb = dtype_bytes(p->xq_dtype), yb = dtype_bytes(p->y_dtype);
  if (!p->identity) {
    for (int64_t t = t0; t < t1; ++t)
      for (int64_t j = 0; j < k; ++j)
        if (!have_expert(p, idx[t * k + j])) return ORC_BAD_ARG;
    if (p->shared && !have_expert(p, p->E)) return ORC_BAD_ARG;
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = t0; t < t1; ++t) {
    const int64_t lt = t - t0;
    std::vector<double> xh(H), yd(H), acc(H, 0.0);
    token_input(p, x, t, xh.data(), xq_tok ? (char*)xq_tok + lt * H * qb : nullptr,
                xs_tok ? xs_tok + lt * (H / 128) : nullptr);
    for (int64_t j = 0; j < ks; ++j) {
      const int64_t e = j < k ? idx[t * k + j] : p->E;
      const double wj = j < k ? (double)w[t * k + j] : 1.0;
      void* yrow = y_pair ? (char*)y_pair + (lt * ks + j) * H * yb : nullptr;
      if (p->identity) {
        for (int64_t c = 0; c < H; ++c) yd[c] = xh[c];
      } else {
        expert_row(p, e, xh.data(), nullptr, nullptr, yrow, yd.data());
      }
      for (int64_t c = 0; c < H; ++c) acc[c] += wj * yd[c];
    }
    for (int64_t c = 0; c < H; ++c) {
      float a32 = (float)acc[c];
      if (p->out_dtype == ORC_F32) ((float*)out)[lt * H + c] = a32;
      else ((uint16_t*)out)[lt * H + c] = bf16_bits_of(bf16_round_f32(a32));
    }
  }
  return ORC_OK;
}

// Threads the OpenMP loops use from now on (n >= 1); returns the count in
// force. Timing aid only: the results do not depend on it.
int oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

}  // extern "C"
