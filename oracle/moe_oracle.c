/*
 * moe_oracle.c -- plain, slow CPU reference ("oracle") for the forward pass of a
 * quantized Mixture-of-Experts SwiGLU FFN layer and for its weight packing.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library; it is written from the
 * definitions below, in double precision wherever the method leaves the
 * precision open, and in fp32 exactly where a float decides an integer code.
 *
 * Sources (web pages the method is taken from):
 *  [R] "quantized MoE LLM inference" (cloud.baidu.com article 9434801), the
 *      expert-routing section: logits = router(x); idx = top_k(logits, k);
 *      w = softmax(logits[idx]); y = sum_i w_i * expert_i(x).
 *  [G] "MoE混合精度量化实战：门控保精度+专家激进压缩" (MoE mixed-precision
 *      quantization in practice), sec. 2.1: the gate/router is never quantized;
 *      expert-input activations use per-token dynamic scales; sec. 2.3 / 3.5:
 *      experts are packed in 128-column blocks, each block quantized on its own
 *      and concatenated into one stream; sec. 3.3: 4-bit code range [-8, 7].
 *  [A] AlphaQ single-GPU MoE quantization stack (mhpn.cn news 995352),
 *      sec. 2.2 / 4.2: per-expert, per-projection bit widths (gate 3-bit,
 *      middle 2-bit, output 4-bit) and group sizes of 32.
 *  [X] "Expert-aware quantisation: near-Q4 quality at near-Q2 size?": hot
 *      experts at 4-bit, cold experts at 2-bit.
 *
 * Readings taken where the pages are silent (each also stated at its function):
 *  - integer codes are symmetric: q in [-qmax, qmax], qmax = 2^(b-1)-1, the
 *    most negative code of [G] sec. 3.3 is left unused;
 *  - the sub-2-bit cold tier ([X], closing section: cold experts below 2 bits,
 *    precision falling with hotness) is a 1-bit sign code: q = +1 for w >= 0,
 *    else -1, with the group scale s = fp16_rne(sum|w| / 32) (fp32 sum in
 *    input order), the least-squares scale of a sign quantizer;
 *  - the scale of a group of 32 consecutive inputs of one output row is the
 *    fp16 round-to-nearest-even of the fp32 quotient amax/qmax (saturated to
 *    the largest finite fp16), and codes are taken against the rounded scale;
 *  - NVFP4: e2m1 codes, an e4m3 block scale per 16 inputs and one fp32 tensor
 *    scale per (expert, projection) equal to amax/(448*6);
 *  - top-k ties go to the lower expert index; the softmax runs over the k
 *    chosen logits only ([R]);
 *  - rows of one expert are ordered by ascending token (stable permutation);
 *  - NVFP4 layers quantize both the expert input x and the SwiGLU output h
 *    per row to e4m3 with scale amax/448 ([G] sec. 2.1).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------- */
/* Small binary floating-point formats, from their definitions.              */
/* A format has `mbits` explicit mantissa bits, an exponent bias `bias` and a  */
/* minimum normal exponent emin = 1 - bias; exponent field 0 is subnormal.    */
/* ------------------------------------------------------------------------- */

/* Round a >= 0 to the format's grid, ties to even mantissa, no upper bound. */
static double rne_grid(double a, int mbits, int emin) {
  if (a == 0.0) return 0.0;
  int ex;
  frexp(a, &ex);           /* a = f * 2^ex, 0.5 <= f < 1 */
  int e = ex - 1;          /* floor(log2(a)) */
  if (e < emin) e = emin;  /* subnormals share the smallest binade's spacing */
  double quantum = ldexp(1.0, e - mbits);
  double n = nearbyint(a / quantum); /* round-half-even (default mode) */
  return n * quantum;
}

/* Bit pattern (without sign) of a value a >= 0 that lies on the grid. */
static uint32_t grid_bits(double a, int mbits, int bias) {
  if (a == 0.0) return 0;
  int emin = 1 - bias;
  int ex;
  frexp(a, &ex);
  int e = ex - 1;
  if (e < emin) return (uint32_t)(a / ldexp(1.0, emin - mbits)); /* subnormal */
  uint32_t m = (uint32_t)(a / ldexp(1.0, e - mbits)) - (1u << mbits);
  return ((uint32_t)(e + bias) << mbits) | m;
}

static double bits_value(uint32_t bits, int ebits, int mbits, int bias) {
  uint32_t m = bits & ((1u << mbits) - 1u);
  uint32_t e = (bits >> mbits) & ((1u << ebits) - 1u);
  if (e == 0) return ldexp((double)m, 1 - bias - mbits);
  return ldexp((double)((1u << mbits) | m), (int)e - bias - mbits);
}

/* IEEE binary16, round-to-nearest-even, overflow to infinity. */
ORC_EXPORT uint16_t orc_f64_to_f16(double v) {
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  double a = fabs(v);
  if (isnan(v)) return 0x7E00u;
  double r = rne_grid(a, 10, -14);
  if (isinf(a) || r > 65504.0) return sign | 0x7C00u;
  return sign | (uint16_t)grid_bits(r, 10, 15);
}
ORC_EXPORT double orc_f16_to_f64(uint16_t h) {
  double s = (h & 0x8000u) ? -1.0 : 1.0;
  uint32_t e = (h >> 10) & 31u;
  if (e == 31u) return (h & 0x3FFu) ? NAN : s * INFINITY;
  return s * bits_value(h & 0x7FFFu, 5, 10, 15);
}

/* bfloat16 (8 exponent bits, 7 mantissa bits), round-to-nearest-even. */
ORC_EXPORT uint16_t orc_f64_to_bf16(double v) {
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  double a = fabs(v);
  if (isnan(v)) return 0x7FC0u;
  double r = rne_grid(a, 7, -126);
  if (isinf(a) || r > ldexp(255.0, 120)) return sign | 0x7F80u; /* max 0x7F7F = 255*2^120 */
  return sign | (uint16_t)grid_bits(r, 7, 127);
}
ORC_EXPORT double orc_bf16_to_f64(uint16_t b) {
  double s = (b & 0x8000u) ? -1.0 : 1.0;
  uint32_t e = (b >> 7) & 255u;
  if (e == 255u) return (b & 0x7Fu) ? NAN : s * INFINITY;
  return s * bits_value(b & 0x7FFFu, 8, 7, 127);
}

/* OCP FP8 E4M3 ("fn": no infinities, S.1111.111 is NaN, max 448):
   round-to-nearest-even, then saturate to +-448. */
ORC_EXPORT uint8_t orc_f64_to_e4m3_sat(double v) {
  uint8_t sign = signbit(v) ? 0x80u : 0u;
  if (isnan(v)) return 0x7Fu;
  double r = rne_grid(fabs(v), 3, -6);
  if (r > 448.0) r = 448.0;
  return sign | (uint8_t)grid_bits(r, 3, 7);
}
ORC_EXPORT double orc_e4m3_to_f64(uint8_t c) {
  if ((c & 0x7Fu) == 0x7Fu) return NAN;
  double s = (c & 0x80u) ? -1.0 : 1.0;
  return s * bits_value(c & 0x7Fu, 4, 3, 7);
}

/* OCP FP4 E2M1 (values 0, .5, 1, 1.5, 2, 3, 4, 6): round-to-nearest-even,
   saturate to +-6.  Code = sign<<3 | exponent<<1 | mantissa. */
ORC_EXPORT uint8_t orc_f64_to_e2m1_sat(double v) {
  uint8_t sign = signbit(v) ? 0x8u : 0u;
  double r = rne_grid(fabs(v), 1, 0);
  if (r > 6.0) r = 6.0;
  return sign | (uint8_t)grid_bits(r, 1, 1);
}
ORC_EXPORT double orc_e2m1_to_f64(uint8_t c) {
  double s = (c & 0x8u) ? -1.0 : 1.0;
  return s * bits_value(c & 0x7u, 2, 1, 1);
}

/* ------------------------------------------------------------------------- */
/* Weight formats.                                                           */
/* ------------------------------------------------------------------------- */
enum { ORC_INT1 = 1, ORC_INT2 = 2, ORC_INT3 = 3, ORC_INT4 = 4, ORC_NVFP4 = 16 };

static int fmt_ok(int f) {
  return f == ORC_INT1 || f == ORC_INT2 || f == ORC_INT3 || f == ORC_INT4 || f == ORC_NVFP4;
}

/* Integer group quantization of one row-major [N x K] fp32 matrix ([G] 3.3,
   [A] 4.2 with group 32).  Per (row n, group g of 32 consecutive k):
     amax = max |w|;  s = fp16_rne(amax / qmax) (fp32 division; saturated to
     65504);  q = clamp(rint(w / float(s)), -qmax, qmax) with fp32 division and
     round-half-even; s == 0 gives all-zero codes.
   bits = 1 (sign code, [X] closing section): s = fp16_rne(sum|w| / 32) (fp32
     sum in input order; saturated to 65504), q = +1 if w >= 0 else -1.  This s
     minimizes sum (w - s*q)^2 over s for the signs q.
   q[N*K] are the signed codes, s16[N*(K/32)] the fp16 scale bit patterns. */
ORC_EXPORT void orc_quant_int(const float* W, int N, int K, int bits, int8_t* q, uint16_t* s16) {
  const int qmax = (1 << (bits - 1)) - 1;
  const int G = K / 32;
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < G; ++g) {
      const float* w = W + (size_t)n * K + (size_t)g * 32;
      if (bits == 1) {
        float sum = 0.0f;
        for (int i = 0; i < 32; ++i) sum += fabsf(w[i]);
        uint16_t sb = orc_f64_to_f16((double)(sum / 32.0f));
        if ((sb & 0x7FFFu) == 0x7C00u) sb = 0x7BFFu;
        s16[(size_t)n * G + g] = sb;
        for (int i = 0; i < 32; ++i) q[(size_t)n * K + (size_t)g * 32 + i] = (int8_t)(w[i] >= 0.0f ? 1 : -1);
        continue;
      }
      float amax = 0.0f;
      for (int i = 0; i < 32; ++i) {
        float a = fabsf(w[i]);
        if (a > amax) amax = a;
      }
      float ratio = amax / (float)qmax;
      uint16_t sb = orc_f64_to_f16((double)ratio);
      if ((sb & 0x7FFFu) == 0x7C00u) sb = 0x7BFFu; /* saturate the scale */
      s16[(size_t)n * G + g] = sb;
      float sf = (float)orc_f16_to_f64(sb);
      for (int i = 0; i < 32; ++i) {
        int8_t c = 0;
        if (sf != 0.0f) {
          float r = rintf(w[i] / sf);
          if (r > (float)qmax) r = (float)qmax;
          if (r < (float)-qmax) r = (float)-qmax;
          c = (int8_t)r;
        }
        q[(size_t)n * K + (size_t)g * 32 + i] = c;
      }
    }
  }
}

/* NVFP4 quantization of one [N x K] matrix (reading of the NVFP4 format named
   on [R]; e2m1 values, e4m3 scale per 16 inputs, fp32 tensor scale):
     sT = amax(W) / (448*6) (fp32; 1 if amax == 0)
     per block of 16 k: sb = e4m3_rne_sat(amax_blk / (6*sT))   [fp32 ops]
                        v  = e2m1_rne_sat(w / (float(sb)*sT))  [fp32 product, fp32 division]
     sb == 0 gives all-zero codes.
   v[N*K] receives 4-bit codes, sb[N*(K/16)] e4m3 codes, *sT the tensor scale. */
ORC_EXPORT void orc_quant_nvfp4(const float* W, int N, int K, uint8_t* v, uint8_t* sb, float* sT_out) {
  float amax = 0.0f;
  for (size_t i = 0; i < (size_t)N * K; ++i) {
    float a = fabsf(W[i]);
    if (a > amax) amax = a;
  }
  float sT = (amax == 0.0f) ? 1.0f : amax / (448.0f * 6.0f);
  *sT_out = sT;
  const int B = K / 16;
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    for (int b = 0; b < B; ++b) {
      const float* w = W + (size_t)n * K + (size_t)b * 16;
      float bmax = 0.0f;
      for (int i = 0; i < 16; ++i) {
        float a = fabsf(w[i]);
        if (a > bmax) bmax = a;
      }
      float ratio = bmax / (6.0f * sT);
      uint8_t sc = orc_f64_to_e4m3_sat((double)ratio);
      sb[(size_t)n * B + b] = sc;
      float denom = (float)orc_e4m3_to_f64(sc) * sT;
      for (int i = 0; i < 16; ++i) {
        uint8_t c = 0;
        if (sc != 0) c = orc_f64_to_e2m1_sat((double)(w[i] / denom));
        v[(size_t)n * K + (size_t)b * 16 + i] = c;
      }
    }
  }
}

/* ------------------------------------------------------------------------- */
/* Packed layout ([G] 2.3: 128-column blocks quantized on their own and      */
/* concatenated).  Reading: tiles of 128 output rows x 128 inputs, tile order */
/* n-block major, k-block minor.  Inside a tile, 32-bit little-endian words   */
/* in the order [kg 0..3][word 0..b-1][n 0..127], where kg is the group of 32 */
/* inputs inside the tile and b the word count of a group (1, 2, 3, 4; NVFP4 */
/* 4).  Stored code u = q + 2^(b-1) (offset binary); b = 1: u = (q + 1) / 2  */
/* (the sign bit, 1 for q = +1); NVFP4 stores the e2m1 code.                  */
/* Inside a word, the two codes of each consecutive pair (2j, 2j+1) sit 16    */
/* bits apart (code 2j in the low half-word, code 2j+1 in the high one):      */
/*   b = 4: codes 8w..8w+7 in word w; code 8w+2j at bits 4j..4j+3, code      */
/*          8w+2j+1 at bits 16+4j..16+4j+3 (j = 0..3);                       */
/*   b = 1: codes 0..31 in word 0; code 2j at bit j, code 2j+1 at bit 16+j    */
/*          (j = 0..15);                                                      */
/*   b = 2: codes 16w..16w+15 in word w; code 16w+2j at bits 2j..2j+1, code  */
/*          16w+2j+1 at bits 16+2j..17+2j (j = 0..7);                        */
/*   b = 3: words 0-1 hold the low two bits of u exactly as b = 2; word 2     */
/*          holds bit 2 of u: of pair m = 4c+j (c, j = 0..3), code 2m at bit  */
/*          P = 8*(c/2) + c%2 + 2j and code 2m+1 at bit 16+P, so the bits of  */
/*          each run of four pairs sit at every other position.               */
/*   NVFP4: codes 8w..8w+7 in word w, code 8w+i at bits 4i..4i+3.            */
/* Scales: fp16 (int) or e4m3 bytes (NVFP4) in [N/128][K/gs][128] order,      */
/* gs = 32 (int) or 16 (NVFP4).                                               */
/* ------------------------------------------------------------------------- */
static size_t word_index(int n, int k, int K, int wpg, int w) {
  size_t nb = (size_t)(n / 128), kb = (size_t)(k / 128);
  size_t kg = (size_t)((k % 128) / 32);
  return (((nb * (size_t)(K / 128) + kb) * 4 + kg) * (size_t)wpg + (size_t)w) * 128 + (size_t)(n % 128);
}

/* bit offset of code i (0..31 of its group) inside its word, integer formats */
static int pair_shift(int i, int width, int per_word) {
  int c = i % per_word; /* position inside the word's run of codes */
  return (c % 2) * 16 + (c / 2) * width;
}

/* bit of word 2 holding bit 2 of 3-bit code i (0..31 of its group) */
static int int3_high_shift(int i) {
  int m = i / 2, c = m / 4, j = m % 4;
  return (i % 2) * 16 + 8 * (c / 2) + c % 2 + 2 * j;
}

/* code (already offset / e2m1, 0..15) of element (n, k) is placed into words */
static void put_code(uint32_t* words, int n, int k, int K, int fmt, uint32_t u) {
  int i = k % 32;
  if (fmt == ORC_NVFP4) {
    words[word_index(n, k, K, 4, i / 8)] |= (u & 15u) << (4 * (i % 8));
  } else if (fmt == ORC_INT4) {
    words[word_index(n, k, K, 4, i / 8)] |= (u & 15u) << pair_shift(i, 4, 8);
  } else if (fmt == ORC_INT2) {
    words[word_index(n, k, K, 2, i / 16)] |= (u & 3u) << pair_shift(i, 2, 16);
  } else if (fmt == ORC_INT1) {
    words[word_index(n, k, K, 1, 0)] |= (u & 1u) << pair_shift(i, 1, 32);
  } else { /* INT3 */
    words[word_index(n, k, K, 3, i / 16)] |= (u & 3u) << pair_shift(i, 2, 16);
    words[word_index(n, k, K, 3, 2)] |= ((u >> 2) & 1u) << int3_high_shift(i);
  }
}

static uint32_t get_code(const uint32_t* words, int n, int k, int K, int fmt) {
  int i = k % 32;
  if (fmt == ORC_NVFP4) return (words[word_index(n, k, K, 4, i / 8)] >> (4 * (i % 8))) & 15u;
  if (fmt == ORC_INT4) return (words[word_index(n, k, K, 4, i / 8)] >> pair_shift(i, 4, 8)) & 15u;
  if (fmt == ORC_INT2) return (words[word_index(n, k, K, 2, i / 16)] >> pair_shift(i, 2, 16)) & 3u;
  if (fmt == ORC_INT1) return (words[word_index(n, k, K, 1, 0)] >> pair_shift(i, 1, 32)) & 1u;
  uint32_t lo = (words[word_index(n, k, K, 3, i / 16)] >> pair_shift(i, 2, 16)) & 3u;
  uint32_t hi = (words[word_index(n, k, K, 3, 2)] >> int3_high_shift(i)) & 1u;
  return lo | (hi << 2);
}

static size_t scale_index(int n, int g, int groups) {
  return ((size_t)(n / 128) * (size_t)groups + (size_t)g) * 128 + (size_t)(n % 128);
}

ORC_EXPORT uint64_t orc_code_bytes(int fmt, int N, int K) {
  return (uint64_t)N * (uint64_t)K * (uint64_t)(fmt == ORC_NVFP4 ? 4 : fmt) / 8u;
}
ORC_EXPORT uint64_t orc_scale_bytes(int fmt, int N, int K) {
  return fmt == ORC_NVFP4 ? (uint64_t)N * (uint64_t)(K / 16) : (uint64_t)N * (uint64_t)(K / 32) * 2u;
}

/* Pack integer codes q[N*K] (signed) and fp16 scales s16[N*K/32] into the layout. */
ORC_EXPORT void orc_pack_int(const int8_t* q, const uint16_t* s16, int N, int K, int bits,
                             uint8_t* codes, uint8_t* scales) {
  memset(codes, 0, orc_code_bytes(bits, N, K));
  uint32_t* words = (uint32_t*)codes;
  const int off = 1 << (bits - 1);
  /* rows own disjoint words, so rows can be packed in parallel */
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k)
      put_code(words, n, k, K, bits,
               bits == 1 ? (uint32_t)((q[(size_t)n * K + k] + 1) >> 1) : (uint32_t)(q[(size_t)n * K + k] + off));
  uint16_t* sc = (uint16_t*)scales;
  for (int n = 0; n < N; ++n)
    for (int g = 0; g < K / 32; ++g) sc[scale_index(n, g, K / 32)] = s16[(size_t)n * (K / 32) + g];
}

ORC_EXPORT void orc_unpack_int(const uint8_t* codes, const uint8_t* scales, int N, int K, int bits,
                               int8_t* q, uint16_t* s16) {
  const uint32_t* words = (const uint32_t*)codes;
  const int off = 1 << (bits - 1);
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) {
      const int u = (int)get_code(words, n, k, K, bits);
      q[(size_t)n * K + k] = (int8_t)(bits == 1 ? 2 * u - 1 : u - off);
    }
  const uint16_t* sc = (const uint16_t*)scales;
  for (int n = 0; n < N; ++n)
    for (int g = 0; g < K / 32; ++g) s16[(size_t)n * (K / 32) + g] = sc[scale_index(n, g, K / 32)];
}

ORC_EXPORT void orc_pack_nvfp4(const uint8_t* v, const uint8_t* sb, int N, int K, uint8_t* codes,
                               uint8_t* scales) {
  memset(codes, 0, orc_code_bytes(ORC_NVFP4, N, K));
  uint32_t* words = (uint32_t*)codes;
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) put_code(words, n, k, K, ORC_NVFP4, v[(size_t)n * K + k]);
  for (int n = 0; n < N; ++n)
    for (int b = 0; b < K / 16; ++b) scales[scale_index(n, b, K / 16)] = sb[(size_t)n * (K / 16) + b];
}

ORC_EXPORT void orc_unpack_nvfp4(const uint8_t* codes, const uint8_t* scales, int N, int K, uint8_t* v,
                                 uint8_t* sb) {
  const uint32_t* words = (const uint32_t*)codes;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) v[(size_t)n * K + k] = (uint8_t)get_code(words, n, k, K, ORC_NVFP4);
  for (int n = 0; n < N; ++n)
    for (int b = 0; b < K / 16; ++b) sb[(size_t)n * (K / 16) + b] = scales[scale_index(n, b, K / 16)];
}

/* Dequantize row n of a packed matrix into w[K] (double, exact):
   int: float(s) * q;  NVFP4: e2m1(v) * e4m3(sb) * sT. */
ORC_EXPORT void orc_decode_row(const uint8_t* codes, const uint8_t* scales, int fmt, int N, int K,
                               float sT, int n, double* w) {
  (void)N;
  const uint32_t* words = (const uint32_t*)codes;
  if (fmt == ORC_NVFP4) {
    for (int k = 0; k < K; ++k) {
      uint32_t c = get_code(words, n, k, K, fmt);
      double s = orc_e4m3_to_f64(scales[scale_index(n, k / 16, K / 16)]);
      w[k] = orc_e2m1_to_f64((uint8_t)c) * s * (double)sT;
    }
  } else {
    const uint16_t* sc = (const uint16_t*)scales;
    const int off = 1 << (fmt - 1);
    for (int k = 0; k < K; ++k) {
      const int u = (int)get_code(words, n, k, K, fmt);
      const int q = fmt == ORC_INT1 ? 2 * u - 1 : u - off;
      w[k] = orc_f16_to_f64(sc[scale_index(n, k / 32, K / 32)]) * (double)q;
    }
  }
}

/* ------------------------------------------------------------------------- */
/* Whole-layer buffer.  Header (16384 bytes, little-endian):                 */
/*   [0]  u32 magic 0x51454F4D   [4] u32 version 1                           */
/*   [8]  i32 E   [12] i32 H   [16] i32 F   [20..32) zero                    */
/*   [32] u8  fmt[768]        (E*3 used; order gate, up, down)              */
/*   [800]   u64 code_off[768]   [6944] u64 scale_off[768]                   */
/*   [13088] f32 tscale[768]  (NVFP4 tensor scales; 0 for integer entries)   */
/* Sections follow from byte 16384 in (expert, projection) order, codes then */
/* scales, each starting on a 256-byte boundary.  gate/up are [F x H],       */
/* down is [H x F] (N output rows by K inputs).                              */
/* ------------------------------------------------------------------------- */
#define ORC_HDR_BYTES 16384u
#define ORC_OFF_FMT 32u
#define ORC_OFF_CODE 800u
#define ORC_OFF_SCALE 6944u
#define ORC_OFF_TS 13088u

static uint64_t up256(uint64_t x) { return (x + 255u) & ~(uint64_t)255u; }

static void proj_shape(int p, int H, int F, int* N, int* K) {
  if (p < 2) { *N = F; *K = H; } else { *N = H; *K = F; }
}

/* Layout query: total bytes and per-(expert, projection) offsets; -1 on bad arguments. */
ORC_EXPORT int orc_layer_layout(int E, int H, int F, const uint8_t* fmt, uint64_t* code_off,
                                uint64_t* scale_off, uint64_t* total) {
  if (E < 1 || E > 256 || H < 128 || F < 128 || H % 128 || F % 128) return -1;
  uint64_t pos = ORC_HDR_BYTES;
  for (int e = 0; e < E; ++e)
    for (int p = 0; p < 3; ++p) {
      int f = fmt[e * 3 + p], N, K;
      if (!fmt_ok(f)) return -1;
      proj_shape(p, H, F, &N, &K);
      pos = up256(pos);
      code_off[e * 3 + p] = pos;
      pos += orc_code_bytes(f, N, K);
      pos = up256(pos);
      scale_off[e * 3 + p] = pos;
      pos += orc_scale_bytes(f, N, K);
    }
  *total = up256(pos);
  return 0;
}

/* Pack experts [e0, e0+ne) of a layer; W is fp32 [ne][3][N*K].  `out` is the
   full-layer buffer (size from orc_layer_layout); the header is (re)written and
   the tensor scales of the packed experts are filled in. */
ORC_EXPORT int orc_pack_layer(const float* W, int e0, int ne, int E, int H, int F, const uint8_t* fmt,
                              uint8_t* out) {
  uint64_t code_off[768], scale_off[768], total;
  if (orc_layer_layout(E, H, F, fmt, code_off, scale_off, &total)) return -1;
  if (e0 < 0 || ne < 0 || e0 + ne > E) return -1;
  uint32_t u32;
  int32_t i32;
  u32 = 0x51454F4Du; memcpy(out + 0, &u32, 4);
  u32 = 1u; memcpy(out + 4, &u32, 4);
  i32 = E; memcpy(out + 8, &i32, 4);
  i32 = H; memcpy(out + 12, &i32, 4);
  i32 = F; memcpy(out + 16, &i32, 4);
  memset(out + 20, 0, 12);
  memset(out + ORC_OFF_FMT, 0, 768);
  memcpy(out + ORC_OFF_FMT, fmt, (size_t)E * 3);
  memset(out + ORC_OFF_CODE, 0, 768 * 8);
  memcpy(out + ORC_OFF_CODE, code_off, (size_t)E * 3 * 8);
  memset(out + ORC_OFF_SCALE, 0, 768 * 8);
  memcpy(out + ORC_OFF_SCALE, scale_off, (size_t)E * 3 * 8);
  memset(out + ORC_OFF_TS + 3072, 0, ORC_HDR_BYTES - ORC_OFF_TS - 3072);
  /* tensor-scale slots past the layer's E*3 entries are zero */
  memset(out + ORC_OFF_TS + (size_t)E * 3 * 4, 0, (size_t)(768 - E * 3) * 4);
  float* ts = (float*)(out + ORC_OFF_TS);
  for (int i = 0; i < ne; ++i) {
    int e = e0 + i;
    for (int p = 0; p < 3; ++p) {
      int f = fmt[e * 3 + p], N, K;
      proj_shape(p, H, F, &N, &K);
      const float* w = W + ((size_t)i * 3 + p) * (size_t)H * F;
      uint8_t* codes = out + code_off[e * 3 + p];
      uint8_t* scales = out + scale_off[e * 3 + p];
      if (f == ORC_NVFP4) {
        uint8_t* v = (uint8_t*)malloc((size_t)N * K);
        uint8_t* sb = (uint8_t*)malloc((size_t)N * (K / 16));
        float sT;
        orc_quant_nvfp4(w, N, K, v, sb, &sT);
        orc_pack_nvfp4(v, sb, N, K, codes, scales);
        float tsv = sT;
        memcpy(&ts[e * 3 + p], &tsv, 4);
        free(v);
        free(sb);
      } else {
        int8_t* q = (int8_t*)malloc((size_t)N * K);
        uint16_t* s16 = (uint16_t*)malloc((size_t)N * (K / 32) * 2);
        orc_quant_int(w, N, K, f, q, s16);
        orc_pack_int(q, s16, N, K, f, codes, scales);
        float z = 0.0f;
        memcpy(&ts[e * 3 + p], &z, 4);
        free(q);
        free(s16);
      }
    }
  }
  return 0;
}

typedef struct {
  int E, H, F;
  const uint8_t* fmt;
  const uint64_t* code_off;
  const uint64_t* scale_off;
  const float* ts;
} layer_view;

static layer_view view_of(const uint8_t* layer) {
  layer_view v;
  memcpy(&v.E, layer + 8, 4);
  memcpy(&v.H, layer + 12, 4);
  memcpy(&v.F, layer + 16, 4);
  v.fmt = layer + ORC_OFF_FMT;
  v.code_off = (const uint64_t*)(layer + ORC_OFF_CODE);
  v.scale_off = (const uint64_t*)(layer + ORC_OFF_SCALE);
  v.ts = (const float*)(layer + ORC_OFF_TS);
  return v;
}

ORC_EXPORT void orc_layer_decode_row(const uint8_t* layer, int e, int p, int n, double* w) {
  layer_view L = view_of(layer);
  int N, K;
  proj_shape(p, L.H, L.F, &N, &K);
  int i = e * 3 + p;
  orc_decode_row(layer + L.code_off[i], layer + L.scale_off[i], L.fmt[i], N, K, L.ts[i], n, w);
}

/* ------------------------------------------------------------------------- */
/* Forward stages.                                                           */
/* ------------------------------------------------------------------------- */

/* Router ([G] 2.1: never quantized): logits[t,e] = sum_h x[t,h]*Wr[e,h] + b[e],
   accumulated in double, stored as fp32.  x is bf16 bit patterns [T,H]. */
ORC_EXPORT void orc_router(const uint16_t* x, int T, int H, const float* Wr, const float* b, int E,
                           float* logits) {
#pragma omp parallel
  {
    double* xr = (double*)malloc((size_t)H * sizeof(double));
#pragma omp for schedule(static)
    for (int t = 0; t < T; ++t) {
      for (int h = 0; h < H; ++h) xr[h] = orc_bf16_to_f64(x[(size_t)t * H + h]);
      for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int h = 0; h < H; ++h) acc += xr[h] * (double)Wr[(size_t)e * H + h];
        if (b) acc += (double)b[e];
        logits[(size_t)t * E + e] = (float)acc;
      }
    }
    free(xr);
  }
}

/* Top-k then softmax over the chosen k ([R]).  k passes; each pass scans the
   experts in ascending order with a strict '>' and skips the ones already
   chosen, so ties go to the lower index.  Weights in double, stored fp32, in
   selection order. */
ORC_EXPORT void orc_topk_softmax(const float* logits, int T, int E, int k, int32_t* idx, float* w) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    unsigned char chosen[256];
    memset(chosen, 0, sizeof(chosen));
    double lv[8];
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (chosen[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e;
      }
      chosen[best] = 1;
      idx[(size_t)t * k + j] = best;
      lv[j] = (double)l[best];
    }
    double den = 0.0;
    for (int j = 0; j < k; ++j) den += exp(lv[j] - lv[0]);
    for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = (float)(exp(lv[j] - lv[0]) / den);
  }
}

/* Permutation by expert: counts, exclusive offsets[E+1], and the rows of each
   expert in ascending (t, j) order: perm[row] = t*k + j, inv[t*k + j] = row. */
ORC_EXPORT void orc_permute(const int32_t* idx, int T, int k, int E, int32_t* counts, int32_t* offsets,
                            int32_t* perm, int32_t* inv) {
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int i = 0; i < T * k; ++i) counts[idx[i]]++;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int e = idx[t * k + j];
      int row = offsets[e] + fill[e]++;
      perm[row] = t * k + j;
      inv[t * k + j] = row;
    }
  free(fill);
}

/* Per-row dynamic FP8 quantization ([G] 2.1 per-token dynamic scales; e4m3,
   scale = amax/448): s = amax/448 in fp32 (1 if amax == 0);
   q = e4m3_rne_sat(a / s) with fp32 division. */
ORC_EXPORT void orc_act_quant_e4m3(const float* a, int R, int C, uint8_t* q, float* s) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < R; ++r) {
    const float* row = a + (size_t)r * C;
    float amax = 0.0f;
    for (int c = 0; c < C; ++c) {
      float v = fabsf(row[c]);
      if (v > amax) amax = v;
    }
    float sc = (amax == 0.0f) ? 1.0f : amax / 448.0f;
    s[r] = sc;
    for (int c = 0; c < C; ++c) q[(size_t)r * C + c] = orc_f64_to_e4m3_sat((double)(row[c] / sc));
  }
}

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* Gate/up stage of one expert for R activation rows a[R,H] (double) with row
   scales a_scale[R] (NULL = 1):  g = a_scale * W'g a,  u = a_scale * W'u a,
   h = silu(g) * u  (double, no intermediate rounding). */
ORC_EXPORT void orc_gateup(const uint8_t* layer, int e, const double* a, const double* a_scale, int R,
                           double* h) {
  layer_view L = view_of(layer);
  const int H = L.H, F = L.F;
#pragma omp parallel
  {
    double* wg = (double*)malloc((size_t)H * sizeof(double));
    double* wu = (double*)malloc((size_t)H * sizeof(double));
#pragma omp for schedule(static)
    for (int n = 0; n < F; ++n) {
      orc_layer_decode_row(layer, e, 0, n, wg);
      orc_layer_decode_row(layer, e, 1, n, wu);
      for (int r = 0; r < R; ++r) {
        const double* x = a + (size_t)r * H;
        double g = 0.0, u = 0.0;
        for (int k = 0; k < H; ++k) {
          g += wg[k] * x[k];
          u += wu[k] * x[k];
        }
        double sc = a_scale ? a_scale[r] : 1.0;
        g *= sc;
        u *= sc;
        h[(size_t)r * F + n] = silu(g) * u;
      }
    }
    free(wg);
    free(wu);
  }
}

/* Down stage of one expert: o[r,:] = h_scale[r] * W'd h[r,:]  (double). */
ORC_EXPORT void orc_down(const uint8_t* layer, int e, const double* hin, const double* h_scale, int R,
                         double* o) {
  layer_view L = view_of(layer);
  const int H = L.H, F = L.F;
#pragma omp parallel
  {
    double* wd = (double*)malloc((size_t)F * sizeof(double));
#pragma omp for schedule(static)
    for (int n = 0; n < H; ++n) {
      orc_layer_decode_row(layer, e, 2, n, wd);
      for (int r = 0; r < R; ++r) {
        const double* x = hin + (size_t)r * F;
        double acc = 0.0;
        for (int k = 0; k < F; ++k) acc += wd[k] * x[k];
        o[(size_t)r * H + n] = acc * (h_scale ? h_scale[r] : 1.0);
      }
    }
    free(wd);
  }
}

/* Weighted combine ([R]): y[t,n] = bf16_rne( sum_{j ascending} w[t,j] * o[inv[t*k+j], n] ),
   summed in double. */
ORC_EXPORT void orc_combine(const double* o, const float* w, const int32_t* inv, int T, int k, int H,
                            uint16_t* y) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t)
    for (int n = 0; n < H; ++n) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) acc += (double)w[t * k + j] * o[(size_t)inv[t * k + j] * H + n];
      y[(size_t)t * H + n] = orc_f64_to_bf16(acc);
    }
}

/* Whole layer.  layer: host copy of a packed layer buffer; x bf16 [T,H];
   Wr fp32 [E,H]; b fp32 [E] or NULL.  y bf16 [T,H].  Optional outputs (NULL to
   skip): idx[T*k], w[T*k], counts[E], perm[T*k], xq[T*H] and sx[T] (NVFP4),
   hq[T*k*F] and sh[T*k] (NVFP4, rows in expert-sorted order).
   Returns -1 for a layer that mixes NVFP4 with integer formats. */
ORC_EXPORT int orc_moe_forward(const uint8_t* layer, const uint16_t* x, int T, const float* Wr,
                               const float* b, int k, uint16_t* y, int32_t* idx_out, float* w_out,
                               int32_t* counts_out, int32_t* perm_out, uint8_t* xq_out, float* sx_out,
                               uint8_t* hq_out, float* sh_out) {
  layer_view L = view_of(layer);
  const int E = L.E, H = L.H, F = L.F;
  int n_fp4 = 0;
  for (int i = 0; i < E * 3; ++i) n_fp4 += (L.fmt[i] == ORC_NVFP4);
  if (n_fp4 != 0 && n_fp4 != E * 3) return -1;
  const int fp4 = (n_fp4 != 0);
  const int R = T * k;

  float* logits = (float*)malloc((size_t)T * E * sizeof(float));
  int32_t* idx = (int32_t*)malloc((size_t)R * sizeof(int32_t));
  float* w = (float*)malloc((size_t)R * sizeof(float));
  int32_t* counts = (int32_t*)malloc((size_t)E * sizeof(int32_t));
  int32_t* offsets = (int32_t*)malloc((size_t)(E + 1) * sizeof(int32_t));
  int32_t* perm = (int32_t*)malloc((size_t)R * sizeof(int32_t));
  int32_t* inv = (int32_t*)malloc((size_t)R * sizeof(int32_t));
  orc_router(x, T, H, Wr, b, E, logits);
  orc_topk_softmax(logits, T, E, k, idx, w);
  orc_permute(idx, T, k, E, counts, offsets, perm, inv);

  /* per-token activations (double) and scales */
  double* xa = (double*)malloc((size_t)T * H * sizeof(double));
  double* xs = (double*)malloc((size_t)T * sizeof(double));
  uint8_t* xq = NULL;
  float* sx = NULL;
  if (fp4) {
    float* xf = (float*)malloc((size_t)T * H * sizeof(float));
    for (size_t i = 0; i < (size_t)T * H; ++i) xf[i] = (float)orc_bf16_to_f64(x[i]);
    xq = (uint8_t*)malloc((size_t)T * H);
    sx = (float*)malloc((size_t)T * sizeof(float));
    orc_act_quant_e4m3(xf, T, H, xq, sx);
    for (size_t i = 0; i < (size_t)T * H; ++i) xa[i] = orc_e4m3_to_f64(xq[i]);
    for (int t = 0; t < T; ++t) xs[t] = (double)sx[t];
    free(xf);
  } else {
    for (size_t i = 0; i < (size_t)T * H; ++i) xa[i] = orc_bf16_to_f64(x[i]);
    for (int t = 0; t < T; ++t) xs[t] = 1.0;
  }

  double* o = (double*)malloc((size_t)R * H * sizeof(double));
  for (int e = 0; e < E; ++e) {
    const int r0 = offsets[e], ne = counts[e];
    if (ne == 0) continue;
    double* a = (double*)malloc((size_t)ne * H * sizeof(double));
    double* as = (double*)malloc((size_t)ne * sizeof(double));
    double* hh = (double*)malloc((size_t)ne * F * sizeof(double));
    double* hs = NULL;
    for (int r = 0; r < ne; ++r) {
      int t = perm[r0 + r] / k;
      memcpy(a + (size_t)r * H, xa + (size_t)t * H, (size_t)H * sizeof(double));
      as[r] = xs[t];
    }
    orc_gateup(layer, e, a, as, ne, hh);
    if (fp4) {
      float* hf = (float*)malloc((size_t)ne * F * sizeof(float));
      uint8_t* hq = (uint8_t*)malloc((size_t)ne * F);
      float* sh = (float*)malloc((size_t)ne * sizeof(float));
      hs = (double*)malloc((size_t)ne * sizeof(double));
      for (size_t i = 0; i < (size_t)ne * F; ++i) hf[i] = (float)hh[i];
      orc_act_quant_e4m3(hf, ne, F, hq, sh);
      for (size_t i = 0; i < (size_t)ne * F; ++i) hh[i] = orc_e4m3_to_f64(hq[i]);
      for (int r = 0; r < ne; ++r) hs[r] = (double)sh[r];
      if (hq_out) memcpy(hq_out + (size_t)r0 * F, hq, (size_t)ne * F);
      if (sh_out) memcpy(sh_out + r0, sh, (size_t)ne * sizeof(float));
      free(hf);
      free(hq);
      free(sh);
    }
    orc_down(layer, e, hh, hs, ne, o + (size_t)r0 * H);
    free(a);
    free(as);
    free(hh);
    free(hs);
  }
  orc_combine(o, w, inv, T, k, H, y);

  if (idx_out) memcpy(idx_out, idx, (size_t)R * sizeof(int32_t));
  if (w_out) memcpy(w_out, w, (size_t)R * sizeof(float));
  if (counts_out) memcpy(counts_out, counts, (size_t)E * sizeof(int32_t));
  if (perm_out) memcpy(perm_out, perm, (size_t)R * sizeof(int32_t));
  if (fp4 && xq_out) memcpy(xq_out, xq, (size_t)T * H);
  if (fp4 && sx_out) memcpy(sx_out, sx, (size_t)T * sizeof(float));
  free(logits); free(idx); free(w); free(counts); free(offsets); free(perm); free(inv);
  free(xa); free(xs); free(xq); free(sx); free(o);
  return 0;
}
