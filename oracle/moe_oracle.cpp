// Plain CPU oracle of the routed, block-scaled-quantised MoE expert FFN layer.
//
// TEST INFRASTRUCTURE ONLY.  This file is the independent reference that the
// CUDA path is checked against.  Only the test suite, the smoke check and the
// benchmark's CPU-baseline leg load it.  It shares no code, header, table or
// constant generator with the CUDA library, and the library never calls it.
//
// What it computes and where that comes from:
//  * The layer itself (router logits -> softmax/top-k/renormalise -> expert
//    histogram and stable permutation -> grouped SwiGLU FFN over quantised
//    expert weights -> weighted un-permute combine) is the routed
//    Mixture-of-Experts forward pass of the FreeToken engine ("FreeToken"
//    upstream README, "About": an MoE serving engine over MXFP4 / NVFP4 / FP8 /
//    BF16 checkpoints).  The pages do not write the layer out as equations;
//    every step below is the plain textbook definition, with the readings of
//    the open points listed where they are used.
//  * FP8 W8A8 with one per-tensor scale per part of a fused projection, and a
//    dynamic activation scale: FreeToken commit 58f4b9ec0e (message on the
//    per-tensor FP8 fused projection path).
//  * Merged gate|up projection and a separate down projection
//    ("ffn_down_exps"): atomicmilkshake/FreeToken fork README, "What else
//    changed" and "Known limits".
//  * Code formats (not on the pages, which only name them): e2m1 and e8m0 from
//    the OCP Microscaling Formats (MX) v1.0 specification, e4m3 ("E4M3FN")
//    from the OCP 8-bit Floating Point specification; NVFP4 = e2m1 elements,
//    one e4m3 scale per 16 elements, one fp32 global scale per tensor; bf16
//    (the BF16 checkpoints of the upstream README, "About") = the upper half
//    of the fp32 encoding: 1 sign, 8 exponent, 7 mantissa bits, no scales.
//
// Precision: every sum, product and transcendental is evaluated in double.
// Where floating point decides an integer (a quantised code), the decision is
// taken in fp32, the precision of the kernels, with the exact fp32 operation
// sequence stated at each quantiser.  Parity pinned: see the oracle tests.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>
#include <limits>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

enum { FMT_NVFP4 = 1, FMT_MXFP4 = 2, FMT_FP8 = 3, FMT_BF16 = 4 };
enum { ACT_BF16 = 0, ACT_MATCH = 1 };

inline double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// Round a non-negative double that is an integer plus a fraction to the
// nearest integer, ties to even.
inline double round_half_even(double v) {
  double fl = std::floor(v);
  double diff = v - fl;
  if (diff > 0.5) return fl + 1.0;
  if (diff < 0.5) return fl;
  return (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// Code formats
// ---------------------------------------------------------------------------

// e2m1 (OCP MX v1.0, FP4 E2M1): bit 3 sign, bits 2..1 exponent (bias 1),
// bit 0 mantissa.  Exponent field 0 is subnormal: value = m * 0.5.
double orc_e2m1_decode(int code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

// e4m3 (OCP FP8 E4M3FN): bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0
// mantissa.  Exponent 0 is subnormal (m * 2^-9).  S.1111.111 is NaN; there is
// no infinity, the largest finite magnitude is 448.
double orc_e4m3_decode(int code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
  double mag = (e == 0) ? std::ldexp((double)m, -9) : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

// e8m0 (OCP MX v1.0 scale format): value 2^(c-127); 0xFF is NaN.
double orc_e8m0_decode(int code) {
  if ((code & 255) == 255) return std::numeric_limits<double>::quiet_NaN();
  return std::ldexp(1.0, (code & 255) - 127);
}

// fp32 -> e2m1, round to nearest with ties to even, saturating to +-6.  The
// sign of the input is kept, also when the magnitude rounds to zero.
// Implemented through the rounding thresholds of the e2m1 grid
// {0, .5, 1, 1.5, 2, 3, 4, 6}: a midpoint goes to the neighbour whose
// mantissa bit is 0.
int orc_e2m1_encode(float v) {
  int sign = std::signbit(v) ? 8 : 0;
  double a = std::fabs((double)v);
  int mag;
  if (a <= 0.25) mag = 0;        // 0.25 ties to 0 (m=0)
  else if (a < 0.75) mag = 1;    // 0.5
  else if (a <= 1.25) mag = 2;   // 1.0 (0.75 and 1.25 tie to 1.0)
  else if (a < 1.75) mag = 3;    // 1.5
  else if (a <= 2.5) mag = 4;    // 2.0 (1.75 and 2.5 tie to 2.0)
  else if (a < 3.5) mag = 5;     // 3.0
  else if (a <= 5.0) mag = 6;    // 4.0 (3.5 and 5 tie to 4.0)
  else mag = 7;                  // 6.0, saturated above
  return sign | mag;
}

// fp32 -> e4m3, round to nearest with ties to even, saturating to +-448
// (never producing the NaN code).  One rounding of the exact input value.
int orc_e4m3_encode(float v) {
  int sign = std::signbit(v) ? 0x80 : 0;
  double a = std::fabs((double)v);
  if (a == 0.0) return sign;
  int ex;
  std::frexp(a, &ex);            // a = f * 2^ex, f in [0.5, 1)
  int e = ex - 1;                // floor(log2 a)
  int code;
  if (e < -6) {                  // subnormal range, quantum 2^-9
    double m = round_half_even(std::ldexp(a, 9));
    code = (int)m;               // m == 8 is the smallest normal, code 0x08
  } else {
    double m = round_half_even(std::ldexp(a, 3 - e));  // in [8, 16]
    if (m == 16.0) { m = 8.0; e += 1; }
    if (e > 8) return sign | 0x7E;
    code = ((e + 7) << 3) | ((int)m - 8);
  }
  if (code > 0x7E) code = 0x7E;
  return sign | code;
}

// ---------------------------------------------------------------------------
// Quantisers (decisions in fp32; every fp32 operation rounds to nearest even)
// ---------------------------------------------------------------------------

float orc_amax(const float* x, int64_t n) {
  float m = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    float a = std::fabs(x[i]);
    if (a > m) m = a;
  }
  return m;
}

// NVFP4 per-tensor global scale from the tensor's amax: the largest block
// scale (448) times the largest element (6) spans the amax.
float orc_nvfp4_global_scale(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  return amax / 2688.0f;
}

// Per-tensor FP8 scale from the tensor's amax (amax maps to 448).
float orc_fp8_scale(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  return amax / 448.0f;
}

// NVFP4: rows x K (K % 16 == 0), blocks of 16 consecutive elements along K.
//   bmax = max |x| in the block
//   sc   = e4m3(bmax / (6 * g))                (fp32: t = 6*g; s = bmax / t)
//   r    = 1 / (dec(sc) * g)                   (fp32: p = dec*g; r = 1/p)
//   q_i  = e2m1(x_i * r)                       (fp32 product)
// An all-zero scale code gives an all-zero block.  Codes are packed two per
// byte, element 2i in the low nibble.  sf is [rows][K/16].
void orc_quant_nvfp4(const float* x, int64_t rows, int64_t K, float g, uint8_t* codes, uint8_t* sf) {
  const float six_g = 6.0f * g;
  for (int64_t r = 0; r < rows; ++r) {
    const float* xr = x + r * K;
    for (int64_t b = 0; b < K / 16; ++b) {
      float bmax = 0.0f;
      for (int i = 0; i < 16; ++i) bmax = std::max(bmax, std::fabs(xr[b * 16 + i]));
      float s = bmax / six_g;
      int sc = orc_e4m3_encode(s);
      sf[r * (K / 16) + b] = (uint8_t)sc;
      float dec = (float)orc_e4m3_decode(sc);
      float recip = 0.0f;
      if (dec != 0.0f) {
        float p = dec * g;
        recip = 1.0f / p;
      }
      for (int i = 0; i < 16; i += 2) {
        int q0 = 0, q1 = 0;
        if (dec != 0.0f) {
          q0 = orc_e2m1_encode(xr[b * 16 + i] * recip);
          q1 = orc_e2m1_encode(xr[b * 16 + i + 1] * recip);
        }
        codes[r * (K / 2) + (b * 16 + i) / 2] = (uint8_t)(q0 | (q1 << 4));
      }
    }
  }
}

// MXFP4 (OCP MX v1.0, conversion of a block of 32 to MX format): shared
// exponent X = floor(log2(bmax)) - emax_elem with emax_elem = 2 for e2m1,
// stored as the e8m0 code c = X + 127 clamped to [0, 254]; c = 0 for an
// all-zero (or subnormal-max) block.  q_i = e2m1(x_i * 2^(127-c)) in fp32,
// values above 6 saturate.  sf is [rows][K/32].
void orc_quant_mxfp4(const float* x, int64_t rows, int64_t K, uint8_t* codes, uint8_t* sf) {
  for (int64_t r = 0; r < rows; ++r) {
    const float* xr = x + r * K;
    for (int64_t b = 0; b < K / 32; ++b) {
      float bmax = 0.0f;
      for (int i = 0; i < 32; ++i) bmax = std::max(bmax, std::fabs(xr[b * 32 + i]));
      int c = 0;
      if (bmax >= std::ldexp(1.0f, -126)) {   // normal: floor(log2) is the exponent
        int ex;
        std::frexp((double)bmax, &ex);
        c = (ex - 1) - 2 + 127;
        if (c < 0) c = 0;
        if (c > 254) c = 254;
      }
      sf[r * (K / 32) + b] = (uint8_t)c;
      float inv = (float)std::ldexp(1.0, 127 - c);   // exact power of two
      for (int i = 0; i < 32; i += 2) {
        int q0 = orc_e2m1_encode(xr[b * 32 + i] * inv);
        int q1 = orc_e2m1_encode(xr[b * 32 + i + 1] * inv);
        codes[r * (K / 2) + (b * 32 + i) / 2] = (uint8_t)(q0 | (q1 << 4));
      }
    }
  }
}

// Per-tensor FP8 with scale s: inv = 1/s (fp32), q_i = e4m3(x_i * inv).
void orc_quant_fp8(const float* x, int64_t n, float s, uint8_t* codes) {
  float inv = 1.0f / s;
  for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)orc_e4m3_encode(x[i] * inv);
}

// fp32 -> bf16: keep the upper 16 bits of the fp32 encoding after rounding
// the lower 16 to nearest, ties to even (a carry may run into the exponent,
// up to infinity).  NaN stays a quiet NaN.
int orc_bf16_encode(float v) {
  uint32_t u;
  std::memcpy(&u, &v, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (int)((u >> 16) | 0x40u);
  const uint32_t low = u & 0xFFFFu, high = u >> 16;
  if (low > 0x8000u || (low == 0x8000u && (high & 1u))) return (int)((high + 1u) & 0xFFFFu);
  return (int)high;
}

// BF16 codes: one bf16 per element, little-endian uint16 in the code bytes.
void orc_quant_bf16(const float* x, int64_t n, uint8_t* codes) {
  for (int64_t i = 0; i < n; ++i) {
    const int b = orc_bf16_encode(x[i]);
    codes[2 * i] = (uint8_t)(b & 0xFF);
    codes[2 * i + 1] = (uint8_t)(b >> 8);
  }
}

// ---------------------------------------------------------------------------
// Dequantisation (exact in double)
// ---------------------------------------------------------------------------

// Decoded values of every code, filled once from the decoders above.
struct DecodeTables {
  double e2m1[16], e4m3[256], e8m0[256];
  DecodeTables() {
    for (int c = 0; c < 16; ++c) e2m1[c] = orc_e2m1_decode(c);
    for (int c = 0; c < 256; ++c) { e4m3[c] = orc_e4m3_decode(c); e8m0[c] = orc_e8m0_decode(c); }
  }
};
static const DecodeTables& tables() {
  static const DecodeTables t;
  return t;
}

// Element k of a quantised row.  NVFP4: e2m1 * e4m3 * g.  MXFP4: e2m1 * e8m0.
// FP8: e4m3 * s.
static inline double dq_elem(int fmt, const uint8_t* crow, const uint8_t* sfrow, double gs, int64_t k) {
  const DecodeTables& tb = tables();
  if (fmt == FMT_FP8) return tb.e4m3[crow[k]] * gs;
  if (fmt == FMT_BF16) return bf16_to_double((uint16_t)(crow[2 * k] | (crow[2 * k + 1] << 8)));
  int nib = (crow[k >> 1] >> ((k & 1) * 4)) & 15;
  double v = tb.e2m1[nib];
  if (fmt == FMT_NVFP4) return v * tb.e4m3[sfrow[k / 16]] * gs;
  return v * tb.e8m0[sfrow[k / 32]];
}

static inline int64_t row_bytes(int fmt, int64_t K) { return fmt == FMT_FP8 ? K : (fmt == FMT_BF16 ? 2 * K : K / 2); }
static inline int64_t sf_per_row(int fmt, int64_t K) {
  return fmt == FMT_NVFP4 ? K / 16 : (fmt == FMT_MXFP4 ? K / 32 : 0);
}

// Dequantise rows x K into double.
void orc_dequant(int fmt, const uint8_t* codes, const uint8_t* sf, double gs, int64_t rows, int64_t K,
                 double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k)
      out[r * K + k] = dq_elem(fmt, codes + r * row_bytes(fmt, K), sf ? sf + r * sf_per_row(fmt, K) : nullptr,
                               gs, k);
}

// ---------------------------------------------------------------------------
// Router: logits, top-k with renormalisation
// ---------------------------------------------------------------------------

// L[t,e] = sum_h x[t,h] * Wr[e,h] (+ b[e]); bf16 inputs, double arithmetic.
void orc_router_logits(const uint16_t* x, int64_t T, int32_t H, const uint16_t* wr, int32_t E,
                       const float* bias, double* logits) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int32_t e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int32_t h = 0; h < H; ++h) acc += bf16_to_double(x[t * H + h]) * bf16_to_double(wr[(int64_t)e * H + h]);
      if (bias) acc += (double)bias[e];
      logits[t * E + e] = acc;
    }
}

// The same logits in fp32, in the fixed summation orders of the library's
// CUDA-core router kernels, so that a routing decision taken on them can be
// compared bit for bit.  Near ties at the k-th pick are real: the
// atomicmilkshake/FreeToken fork README ("Known limits") reports a
// first-token argmax that flips between two plausible experts.  A product of
// two bf16 values is exact in fp32, so every step below is one fp32 rounding
// of a sum (std::fma on floats).
//  order 1 (small batches): 256 partial sums.  Partial p takes the 8
//    consecutive columns from 8p, then the 8 from 8p + 2048, from 8p + 4096,
//    and so on, adding one column at a time.  Each group of 32 partials
//    (p = 32g .. 32g + 31) is combined by exchange: for d = 16, 8, 4, 2, 1 in
//    turn, every partial q becomes its value plus the value of partial q xor d
//    (both from before the step); the group's sum is then partial 32g.  The
//    8 group sums are added in order g = 0 .. 7 onto 0, and the bias (or 0)
//    last.  Needs H % 8 == 0.
//  order 2 (sequential): one sum over h = 0 .. H-1 in turn, then the bias (or 0).
// Returns -1 for an unknown order or H % 8 != 0 with order 1.
int orc_router_logits_ordered(const uint16_t* x, int64_t T, int32_t H, const uint16_t* wr, int32_t E,
                              const float* bias, int32_t order, float* logits) {
  if (order != 1 && order != 2) return -1;
  if (order == 1 && H % 8 != 0) return -1;
  auto f32 = [](uint16_t b) { return (float)bf16_to_double(b); };
  for (int64_t t = 0; t < T; ++t)
    for (int32_t e = 0; e < E; ++e) {
      const uint16_t* xr = x + t * H;
      const uint16_t* wrow = wr + (int64_t)e * H;
      float sum = 0.0f;
      if (order == 2) {
        for (int32_t h = 0; h < H; ++h) sum = std::fma(f32(xr[h]), f32(wrow[h]), sum);
      } else {
        float part[256];
        for (int p = 0; p < 256; ++p) {
          float acc = 0.0f;
          for (int32_t h0 = 8 * p; h0 < H; h0 += 2048)
            for (int c = 0; c < 8; ++c) acc = std::fma(f32(xr[h0 + c]), f32(wrow[h0 + c]), acc);
          part[p] = acc;
        }
        for (int g = 0; g < 8; ++g) {
          float* v = part + 32 * g;
          for (int d = 16; d >= 1; d /= 2) {
            float nv[32];
            for (int q = 0; q < 32; ++q) nv[q] = v[q] + v[q ^ d];
            for (int q = 0; q < 32; ++q) v[q] = nv[q];
          }
        }
        for (int g = 0; g < 8; ++g) sum = sum + part[32 * g];
      }
      logits[t * E + e] = sum + (bias ? bias[e] : 0.0f);
    }
  return 0;
}

// Top-k: the k largest logits in descending order, ties to the lower expert
// index.  Softmax is monotone, so selecting on logits selects on
// probabilities.  Weights: softmax over E renormalised over the selected k,
// which equals exp(L_j - L_0) / sum_i exp(L_i - L_0) over the selected set.
// Returns 0, or -1 when a row holds a NaN or has no finite logit.
int orc_topk(const double* logits, int64_t T, int32_t E, int32_t k, int32_t* idx, double* w) {
  std::vector<int32_t> order(E);
  int status = 0;
  for (int64_t t = 0; t < T; ++t) {
    const double* L = logits + t * E;
    bool bad = false;
    for (int32_t e = 0; e < E; ++e) if (std::isnan(L[e])) bad = true;
    for (int32_t e = 0; e < E; ++e) order[e] = e;
    std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
      if (L[a] != L[b]) return L[a] > L[b];
      return a < b;
    });
    if (!bad && !(L[order[0]] > -std::numeric_limits<double>::infinity())) bad = true;
    if (bad) status = -1;
    double top = L[order[0]], denom = 0.0;
    for (int32_t j = 0; j < k; ++j) denom += std::exp(L[order[j]] - top);
    for (int32_t j = 0; j < k; ++j) {
      idx[t * k + j] = order[j];
      w[t * k + j] = std::exp(L[order[j]] - top) / denom;
    }
  }
  return status;
}

// ---------------------------------------------------------------------------
// Histogram, offsets and stable permutation
// ---------------------------------------------------------------------------

// counts[e] = #{i : idx[i] = e} over the S = T*k flat slots i = t*k + j;
// offsets = exclusive prefix sum (offsets[E] = S); slot i goes to position
// p = offsets[e] + (number of earlier slots with the same expert), so the
// permutation is stable in the flat index.  perm_token[p] = i / k,
// inv_perm[i] = p.  Returns -1 on an expert index outside [0, E).
int orc_permute(const int32_t* idx, int64_t T, int32_t k, int32_t E, int32_t* offsets, int32_t* perm_token,
                int32_t* inv_perm) {
  int64_t S = T * k;
  std::vector<int64_t> counts(E, 0);
  for (int64_t i = 0; i < S; ++i) {
    if (idx[i] < 0 || idx[i] >= E) return -1;
    counts[idx[i]]++;
  }
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) offsets[e + 1] = (int32_t)(offsets[e] + counts[e]);
  std::vector<int64_t> fill(E, 0);
  for (int64_t i = 0; i < S; ++i) {
    int32_t e = idx[i];
    int64_t p = offsets[e] + fill[e]++;
    perm_token[p] = (int32_t)(i / k);
    inv_perm[i] = (int32_t)p;
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Expert FFN and combine
// ---------------------------------------------------------------------------

// Quantised expert weights in the canonical layout.
//   w13   [E][2I][H/2 | H]   rows 0..I-1 gate, I..2I-1 up (merged projection)
//   w13_sf[E][2I][H/16 | H/32]  (NULL for FP8)
//   w13_gs[E][2]   NVFP4 global scale / FP8 per-tensor scale, per part
//   w2    [E][H][I/2 | I], w2_sf [E][H][I/16 | I/32], w2_gs [E]
typedef struct {
  int32_t fmt, E, H, I;
  const uint8_t* w13;
  const uint8_t* w13_sf;
  const float* w13_gs;
  const uint8_t* w2;
  const uint8_t* w2_sf;
  const float* w2_gs;
} orc_weights;

static double w13_elem(const orc_weights* W, int32_t e, int32_t row, int32_t h) {
  const int64_t rb = row_bytes(W->fmt, W->H), nsf = sf_per_row(W->fmt, W->H);
  const int64_t r = (int64_t)e * 2 * W->I + row;
  double gs = (W->fmt == FMT_MXFP4 || W->fmt == FMT_BF16) ? 1.0 : (double)W->w13_gs[e * 2 + (row >= W->I ? 1 : 0)];
  return dq_elem(W->fmt, W->w13 + r * rb, W->w13_sf ? W->w13_sf + r * nsf : nullptr, gs, h);
}

static double w2_elem(const orc_weights* W, int32_t e, int32_t o, int32_t i) {
  const int64_t rb = row_bytes(W->fmt, W->I), nsf = sf_per_row(W->fmt, W->I);
  const int64_t r = (int64_t)e * W->H + o;
  double gs = (W->fmt == FMT_MXFP4 || W->fmt == FMT_BF16) ? 1.0 : (double)W->w2_gs[e];
  return dq_elem(W->fmt, W->w2 + r * rb, W->w2_sf ? W->w2_sf + r * nsf : nullptr, gs, i);
}

// Activation of x for the layer: A16 keeps the bf16 values; MATCH quantises
// the whole [T,H] tensor in the weights' format and dequantises it.  The
// global/per-tensor scale is `static_scale` when > 0, otherwise derived from
// the tensor's amax (NVFP4: amax/2688, FP8: amax/448).  Writes the scale used.
static void activation_rows(int fmt, int act, const std::vector<float>& xf, int64_t rows, int32_t K,
                            float static_scale, std::vector<double>& out, float* scale_used) {
  out.assign((size_t)rows * K, 0.0);
  if (act == ACT_BF16) {
    for (size_t i = 0; i < out.size(); ++i) out[i] = (double)xf[i];
    if (scale_used) *scale_used = 1.0f;
    return;
  }
  std::vector<uint8_t> codes((size_t)rows * row_bytes(fmt, K));
  std::vector<uint8_t> sf((size_t)rows * std::max<int64_t>(1, sf_per_row(fmt, K)));
  float s = 1.0f;
  if (fmt == FMT_NVFP4) {
    s = static_scale > 0 ? static_scale : orc_nvfp4_global_scale(orc_amax(xf.data(), rows * K));
    orc_quant_nvfp4(xf.data(), rows, K, s, codes.data(), sf.data());
  } else if (fmt == FMT_MXFP4) {
    orc_quant_mxfp4(xf.data(), rows, K, codes.data(), sf.data());
  } else if (fmt == FMT_BF16) {
    // MATCH with bf16 weights: the activations are rounded to bf16
    orc_quant_bf16(xf.data(), rows * K, codes.data());
  } else {
    s = static_scale > 0 ? static_scale : orc_fp8_scale(orc_amax(xf.data(), rows * K));
    orc_quant_fp8(xf.data(), rows * K, s, codes.data());
  }
  if (scale_used) *scale_used = s;
  orc_dequant(fmt, codes.data(), (fmt == FMT_FP8 || fmt == FMT_BF16) ? nullptr : sf.data(), (double)s, rows, K,
              out.data());
}

// y for a list of slots (token row, expert): the SwiGLU expert FFN.
//   [g | u] = a_t . W13_e^T           (gate rows 0..I-1, up rows I..2I-1)
//   h       = g / (1 + exp(-g)) * u   (SiLU(g) * u)
//   y       = act(h) . W2_e^T
// act(h) is h itself in A16 mode; in MATCH mode h is rounded to fp32 and
// quantised like x, the per-tensor amax taken over all the slots' h.
// a_rows holds the (already activated) token rows, indexed by slot_row.
static void ffn_slots(const orc_weights* W, int act, const std::vector<double>& a_rows, int64_t n_slots,
                      const int32_t* slot_row, const int32_t* slot_expert, float a2_static, double* y,
                      int nthreads, float* a2_used) {
  const int32_t H = W->H, I = W->I;
  std::vector<double> hbuf((size_t)n_slots * I);
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
  for (int64_t p = 0; p < n_slots; ++p) {
    const double* a = a_rows.data() + (size_t)slot_row[p] * H;
    const int32_t e = slot_expert[p];
    for (int32_t i = 0; i < I; ++i) {
      double g = 0.0, u = 0.0;
      for (int32_t h = 0; h < H; ++h) {
        g += a[h] * w13_elem(W, e, i, h);
        u += a[h] * w13_elem(W, e, I + i, h);
      }
      hbuf[(size_t)p * I + i] = g / (1.0 + std::exp(-g)) * u;
    }
  }
  std::vector<double> hact;
  if (act == ACT_MATCH) {
    std::vector<float> hf(hbuf.size());
    for (size_t i = 0; i < hf.size(); ++i) hf[i] = (float)hbuf[i];
    activation_rows(W->fmt, act, hf, n_slots, I, a2_static, hact, a2_used);
  } else {
    hact.swap(hbuf);
    if (a2_used) *a2_used = 1.0f;
  }
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
  for (int64_t p = 0; p < n_slots; ++p) {
    const double* hv = hact.data() + (size_t)p * I;
    const int32_t e = slot_expert[p];
    for (int32_t o = 0; o < H; ++o) {
      double acc = 0.0;
      for (int32_t i = 0; i < I; ++i) acc += hv[i] * w2_elem(W, e, o, i);
      y[(size_t)p * H + o] = acc;
    }
  }
}

static void bf16_rows_to_float(const uint16_t* x, int64_t rows, int32_t H, std::vector<float>& out) {
  out.resize((size_t)rows * H);
  for (size_t i = 0; i < out.size(); ++i) out[i] = (float)bf16_to_double(x[i]);
}

// Grouped expert FFN over a permuted slot list: y_perm[p] = FFN_e(x[perm_token[p]])
// for p in [offsets[e], offsets[e+1]).  In MATCH mode x is quantised over the
// whole [T,H] tensor and h over all S slots.  a13_static / a2_static <= 0
// select the dynamic (amax-derived) scales.  Returns -1 on bad arguments.
int orc_grouped_ffn(const uint16_t* x, int64_t T, const int32_t* perm_token, const int32_t* offsets,
                    const orc_weights* W, int32_t act, float a13_static, float a2_static, double* y_perm,
                    int32_t nthreads, float* scales_used /* [2]: x scale, h scale; nullable */) {
  const int32_t E = W->E;
  const int64_t S = offsets[E];
  std::vector<int32_t> slot_expert(S), slot_row(S);
  for (int32_t e = 0; e < E; ++e)
    for (int64_t p = offsets[e]; p < offsets[e + 1]; ++p) slot_expert[p] = e;
  for (int64_t p = 0; p < S; ++p) {
    if (perm_token[p] < 0 || perm_token[p] >= T) return -1;
    slot_row[p] = perm_token[p];
  }
  std::vector<float> xf;
  bf16_rows_to_float(x, T, W->H, xf);
  std::vector<double> a;
  float s1 = 1.0f, s2 = 1.0f;
  activation_rows(W->fmt, act, xf, T, W->H, a13_static, a, &s1);
  ffn_slots(W, act, a, S, slot_row.data(), slot_expert.data(), a2_static, y_perm, nthreads, &s2);
  if (scales_used) { scales_used[0] = s1; scales_used[1] = s2; }
  return 0;
}

// out[t] = sum_{j<k} w[t,j] * y_perm[inv_perm[t*k+j]] (+ shared[t]), in double,
// accumulated in order j = 0..k-1.
void orc_combine(const double* y_perm, const int32_t* inv_perm, const double* w, int64_t T, int32_t k, int32_t H,
                 const double* shared_y, double* out) {
  for (int64_t t = 0; t < T; ++t)
    for (int32_t h = 0; h < H; ++h) {
      double acc = 0.0;
      for (int32_t j = 0; j < k; ++j) acc += w[t * k + j] * y_perm[(size_t)inv_perm[t * k + j] * H + h];
      if (shared_y) acc += shared_y[(size_t)t * H + h];
      out[(size_t)t * H + h] = acc;
    }
}

// The whole layer for a subset of tokens (all tokens when `tokens` is NULL),
// written per token from the definition: out[t] = sum_j w[t,j] * FFN_{idx[t,j]}(x_t)
// + FFN_shared(x_t).  The permutation is pure data movement and does not enter
// the values; orc_permute defines it separately.
//   act: 0 = A16 (bf16 activations, weight-only quantisation), 1 = MATCH.
//   a13_static, a2_static, sh_a2_static: static activation scales (> 0) or
//   dynamic (<= 0).  In MATCH mode the shared expert reads the same quantised
//   x as the routed experts and quantises its own h.
// Dynamic h scales need every slot's h, so with a subset and a dynamic h scale
// all tokens are evaluated.  router_order 0 takes the logits in double (the
// definition); 1 or 2 takes them in fp32 in one of the fixed orders of
// orc_router_logits_ordered, so that the routing decisions are the ones a
// router summing in that order takes.  Returns 0, or -1 on invalid input (NaN logits,
// out-of-range sizes).
int orc_moe_forward(const uint16_t* x, int64_t T, int32_t H, const uint16_t* wr, const float* bias, int32_t E,
                    int32_t k, const orc_weights* routed, const orc_weights* shared, int32_t act,
                    float a13_static, float a2_static, float sh_a2_static, const int32_t* tokens,
                    int64_t n_tokens, double* out, double* logits_out, int32_t* idx_out, double* w_out,
                    int32_t nthreads, int32_t router_order) {
  if (k < 1 || k > E || routed->E != E || routed->H != H) return -1;
  if (shared && (shared->H != H || shared->fmt != routed->fmt)) return -1;
  std::vector<int32_t> all;
  if (!tokens) {
    all.resize(T);
    for (int64_t t = 0; t < T; ++t) all[t] = (int32_t)t;
    tokens = all.data();
    n_tokens = T;
  }
  // MXFP4 and bf16 activations have no per-tensor scale
  const bool scaled = routed->fmt == FMT_NVFP4 || routed->fmt == FMT_FP8;
  const bool dyn_h = (act == ACT_MATCH && scaled && !(a2_static > 0));
  const bool dyn_sh = (shared && act == ACT_MATCH && scaled && !(sh_a2_static > 0));
  // Tokens whose FFN is evaluated: the subset, or all of them when a dynamic
  // h scale couples every slot.
  std::vector<int32_t> eval_tok;
  if (dyn_h || dyn_sh) {
    eval_tok.resize(T);
    for (int64_t t = 0; t < T; ++t) eval_tok[t] = (int32_t)t;
  } else {
    eval_tok.assign(tokens, tokens + n_tokens);
  }
  const int64_t NE = (int64_t)eval_tok.size();
  // Router for the evaluated tokens.
  std::vector<uint16_t> xe((size_t)NE * H);
  for (int64_t r = 0; r < NE; ++r) std::memcpy(&xe[(size_t)r * H], x + (size_t)eval_tok[r] * H, 2 * (size_t)H);
  std::vector<double> logits((size_t)NE * E), w((size_t)NE * k);
  std::vector<int32_t> idx((size_t)NE * k);
  if (router_order == 0) {
    orc_router_logits(xe.data(), NE, H, wr, E, bias, logits.data());
  } else {
    std::vector<float> lf((size_t)NE * E);
    if (orc_router_logits_ordered(xe.data(), NE, H, wr, E, bias, router_order, lf.data()) != 0) return -1;
    for (size_t i = 0; i < lf.size(); ++i) logits[i] = (double)lf[i];
  }
  int st = orc_topk(logits.data(), NE, E, k, idx.data(), w.data());
  // Activation of x: quantised over the whole tensor (all T tokens).
  std::vector<float> xf;
  bf16_rows_to_float(x, T, H, xf);
  std::vector<double> a_all;
  activation_rows(routed->fmt, act, xf, T, H, a13_static, a_all, nullptr);
  // Routed slots of the evaluated tokens.
  std::vector<int32_t> slot_row((size_t)NE * k), slot_exp((size_t)NE * k);
  for (int64_t r = 0; r < NE; ++r)
    for (int32_t j = 0; j < k; ++j) {
      slot_row[r * k + j] = eval_tok[r];
      slot_exp[r * k + j] = idx[r * k + j];
    }
  std::vector<double> y((size_t)NE * k * H);
  ffn_slots(routed, act, a_all, NE * k, slot_row.data(), slot_exp.data(), a2_static, y.data(), nthreads, nullptr);
  std::vector<double> ysh;
  if (shared) {
    std::vector<int32_t> zero((size_t)NE, 0);
    ysh.resize((size_t)NE * H);
    ffn_slots(shared, act, a_all, NE, eval_tok.data(), zero.data(), sh_a2_static, ysh.data(), nthreads, nullptr);
  }
  // Position of each requested token among the evaluated ones.
  std::vector<int64_t> pos(n_tokens);
  if (dyn_h || dyn_sh) {
    for (int64_t i = 0; i < n_tokens; ++i) pos[i] = tokens[i];
  } else {
    for (int64_t i = 0; i < n_tokens; ++i) pos[i] = i;
  }
  for (int64_t i = 0; i < n_tokens; ++i) {
    const int64_t r = pos[i];
    for (int32_t h = 0; h < H; ++h) {
      double acc = 0.0;
      for (int32_t j = 0; j < k; ++j) acc += w[r * k + j] * y[((size_t)r * k + j) * H + h];
      if (shared) acc += ysh[(size_t)r * H + h];
      out[(size_t)i * H + h] = acc;
    }
    if (logits_out) std::memcpy(logits_out + (size_t)i * E, &logits[(size_t)r * E], sizeof(double) * E);
    if (idx_out) std::memcpy(idx_out + (size_t)i * k, &idx[(size_t)r * k], sizeof(int32_t) * k);
    if (w_out) std::memcpy(w_out + (size_t)i * k, &w[(size_t)r * k], sizeof(double) * k);
  }
  return st;
}

int orc_num_threads_available(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
