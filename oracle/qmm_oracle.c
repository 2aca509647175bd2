/*
 * qmm_oracle.c -- plain, slow CPU definition of the packed 4-bit weight
 * dequantise-and-multiply path.  TEST INFRASTRUCTURE ONLY: the test suite,
 * the smoke check and the benchmark's CPU-baseline leg are the only callers.
 * It shares no code, table or header with the CUDA library; every constant
 * and conversion below is written out here from the format definitions.
 *
 * Sources the definitions follow (page title, section):
 *   [MARK-Q]  "Mark-Experimental-V3-8B", section "Quantization": IQ4_NL is an
 *             18-byte block per 32 weights, a 2-byte FP16 scale d followed by
 *             16 bytes holding 32 four-bit indices into the printed 16-entry
 *             non-linear table.
 *   [MARK-M]  same page, section "Mixture-of-Experts (MoE)": 32 routed
 *             experts, top-4 per token; expert weights stored as contiguous
 *             3-D tensors ("Quantization", last bullet).
 *   [MAMBA-R] "Mamb2_8B_FP4_Recall_SQ3.25", section "Representation",
 *             paragraph "Weights": E2M1 FP4 codes with signed magnitudes
 *             0, 0.5, 1, 1.5, 2, 3, 4, 6, 16-element groups along the input
 *             axis, an E4M3FN block scale per group and an FP32 global scale
 *             per matrix; the weights are decoded to FP16.
 *   [MAMBA-S] same page, section "Storage and runtime memory": the decoded
 *             weights are held as resident FP16 tensors.
 *   [ZQ-MX]   "1bit.gg zyphra", section "What these numbers say": MXFP4
 *             experts are E2M1 codes, 32 per group, with one E8M0 scale byte
 *             per group (the OCP microscaling format).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - IQ4_NL block: scale first, little-endian; low nibble of qs[j] is weight
 *     j of the block, high nibble is weight j+16.
 *   - FP4 codes: row-major [n][k/2] bytes, low nibble = even k.  Scales are a
 *     separate row-major [n][k/16] array (fp16 or E4M3FN bytes).
 *   - The config-literal FP4-G16 variant uses one fp16 scale per group and
 *     no global scale.
 *   - Decoding rounds once to fp16 (round to nearest, ties to even, fp16
 *     subnormals kept): w = fp16(code * scale).  For the E4M3FN variant the
 *     product code * e4m3 * g is rounded to fp32 first (the FP32 global
 *     scale is an fp32 multiply) and then to fp16.
 *   - MXFP4: the codes are laid out as for FP4-G16; the scales are a
 *     separate row-major [n][k/32] array of E8M0 bytes; w = fp16(code *
 *     2^(e-127)), one rounding; e = 0xFF is NaN.
 *   - The matrix product is y[m][n] = sum_k w16[n][k] * x[m][k], evaluated
 *     here in double precision in ascending k.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_FMT_IQ4_NL 1
#define ORC_FMT_FP4G16_F16 2
#define ORC_FMT_FP4G16_E4M3 3
#define ORC_FMT_MXFP4 4

/* ---------------------------------------------------------------------- */
/* IEEE 754 binary16 (half precision): 1 sign, 5 exponent (bias 15),      */
/* 10 fraction bits; exponent field 0 = zero/subnormal, 31 = inf/NaN.     */
/* ---------------------------------------------------------------------- */

double orc_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int f = h & 0x3FF;
  double v;
  if (e == 0) {
    v = ldexp((double)f, -24); /* subnormal: f * 2^-14 / 2^10 */
  } else if (e == 31) {
    v = (f == 0) ? INFINITY : NAN;
  } else {
    v = ldexp(1024.0 + (double)f, e - 15 - 10);
  }
  return sign ? -v : v;
}

/* Round a non-negative double holding an integer-plus-fraction value to the
 * nearest integer, ties to even.  q must be below 2^52. */
static double orc_round_half_even(double q) {
  double fl = floor(q);
  double diff = q - fl; /* exact for q < 2^52 */
  if (diff > 0.5) return fl + 1.0;
  if (diff < 0.5) return fl;
  return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* Convert a double to the nearest binary16 value, ties to even, with
 * subnormals, overflow to infinity and NaN kept as NaN.  The input is assumed
 * to already be the exact value to round (one rounding step). */
uint16_t orc_f64_to_f16(double v) {
  uint16_t sign = signbit(v) ? 0x8000 : 0;
  if (isnan(v)) return (uint16_t)(sign | 0x7E00);
  double a = fabs(v);
  if (isinf(a)) return (uint16_t)(sign | 0x7C00);
  /* The largest finite value is 65504 = (2 - 2^-10) * 2^15; halfway to the
   * next binade step (65536) is 65520, which rounds to even = infinity. */
  if (a >= 65520.0) return (uint16_t)(sign | 0x7C00);
  if (a < ldexp(1.0, -14)) {
    /* subnormal range: values are multiples of 2^-24 */
    double q = ldexp(a, 24);
    double r = orc_round_half_even(q); /* may reach 1024 = smallest normal */
    return (uint16_t)(sign | (uint16_t)r);
  }
  int ex;
  double fr = frexp(a, &ex); /* a = fr * 2^ex, fr in [0.5, 1) */
  int E = ex - 1;            /* a in [2^E, 2^(E+1)) */
  double q = ldexp(a, 10 - E); /* in [1024, 2048) */
  double r = orc_round_half_even(q);
  (void)fr;
  if (r >= 2048.0) { r = 1024.0; E += 1; }
  if (E > 15) return (uint16_t)(sign | 0x7C00);
  return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)(r - 1024.0));
}

/* ---------------------------------------------------------------------- */
/* OCP 8-bit E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no     */
/* infinities; only S.1111.111 is NaN; exponent field 0 is subnormal.     */
/* ---------------------------------------------------------------------- */
double orc_e4m3_to_f64(uint8_t b) {
  int sign = (b >> 7) & 1;
  int e = (b >> 3) & 0xF;
  int m = b & 7;
  double v;
  if (e == 15 && m == 7) {
    v = NAN;
  } else if (e == 0) {
    v = ldexp((double)m, -9); /* m/8 * 2^(1-7) */
  } else {
    v = ldexp(8.0 + (double)m, e - 7 - 3);
  }
  return sign ? -v : v;
}

/* ---------------------------------------------------------------------- */
/* E2M1 (FP4): 1 sign, 2 exponent (bias 1), 1 mantissa bit.  Exponent     */
/* field 0 is subnormal (m * 0.5); otherwise 2^(e-1) * (1 + m/2).  This   */
/* gives the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 named in [MAMBA-R].    */
/* ---------------------------------------------------------------------- */
double orc_e2m1_to_f64(uint8_t nib) {
  int sign = (nib >> 3) & 1;
  int e = (nib >> 1) & 3;
  int m = nib & 1;
  double v;
  if (e == 0) {
    v = 0.5 * (double)m;
  } else {
    v = ldexp(1.0 + 0.5 * (double)m, e - 1);
  }
  return sign ? -v : v;
}

/* ---------------------------------------------------------------------- */
/* OCP MX E8M0 scale: an unsigned biased exponent, value 2^(e-127); no     */
/* sign, no zero; only 0xFF is NaN ([ZQ-MX] names the type).               */
/* ---------------------------------------------------------------------- */
double orc_e8m0_to_f64(uint8_t b) {
  if (b == 0xFF) return NAN;
  return ldexp(1.0, (int)b - 127);
}

/* The IQ4_NL non-linear table printed in [MARK-Q]. */
static const int orc_iq4nl_table[16] = {-127, -104, -83, -65, -49, -35, -22, -10,
                                        1,    13,   25,  38,  53,  69,  89,  113};

int orc_iq4nl_value(int idx) { return orc_iq4nl_table[idx & 15]; }

/* ---------------------------------------------------------------------- */
/* Sizes                                                                  */
/* ---------------------------------------------------------------------- */

/* Bytes of the packed code/block array of one [n][k] matrix. */
int64_t orc_data_bytes(int fmt, int64_t n, int64_t k) {
  if (fmt == ORC_FMT_IQ4_NL) return n * (k / 32) * 18; /* [MARK-Q]: 18 B per 32 */
  return n * (k / 2);                                  /* two 4-bit codes per byte */
}

/* Bytes of the separate scale array (0 for IQ4_NL, whose scale is inside
 * each block). */
int64_t orc_scale_bytes(int fmt, int64_t n, int64_t k) {
  if (fmt == ORC_FMT_FP4G16_F16) return n * (k / 16) * 2;
  if (fmt == ORC_FMT_FP4G16_E4M3) return n * (k / 16) * 1;
  if (fmt == ORC_FMT_MXFP4) return n * (k / 32) * 1; /* [ZQ-MX]: one byte per 32 */
  return 0;
}

/* ---------------------------------------------------------------------- */
/* Dequantisation: one row at a time                                      */
/* ---------------------------------------------------------------------- */

/* Decode row `row` of a packed matrix into fp16 bit patterns out[k]. */
void orc_dequant_row(int fmt, int64_t n, int64_t k, const uint8_t* data, const uint8_t* scales,
                     float global_scale, int64_t row, uint16_t* out) {
  (void)n;
  if (fmt == ORC_FMT_IQ4_NL) {
    int64_t nblk = k / 32;
    for (int64_t b = 0; b < nblk; b++) {
      const uint8_t* blk = data + (row * nblk + b) * 18;
      uint16_t dbits = (uint16_t)(blk[0] | (blk[1] << 8)); /* little-endian fp16 */
      double d = orc_f16_to_f64(dbits);
      const uint8_t* qs = blk + 2;
      for (int j = 0; j < 16; j++) {
        int lo = qs[j] & 0x0F;
        int hi = qs[j] >> 4;
        out[b * 32 + j] = orc_f64_to_f16(d * (double)orc_iq4nl_table[lo]);
        out[b * 32 + j + 16] = orc_f64_to_f16(d * (double)orc_iq4nl_table[hi]);
      }
    }
    return;
  }
  const uint8_t* codes = data + row * (k / 2);
  for (int64_t kk = 0; kk < k; kk++) {
    uint8_t byte = codes[kk / 2];
    uint8_t nib = (kk % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
    double c = orc_e2m1_to_f64(nib);
    int64_t g = kk / 16;
    if (fmt == ORC_FMT_FP4G16_F16) {
      const uint8_t* sp = scales + (row * (k / 16) + g) * 2;
      double s = orc_f16_to_f64((uint16_t)(sp[0] | (sp[1] << 8)));
      out[kk] = orc_f64_to_f16(c * s);
    } else if (fmt == ORC_FMT_MXFP4) {
      /* c has two significant bits and the scale is a power of two from
       * 2^-127 to 2^127, so the double product is exact. */
      double s = orc_e8m0_to_f64(scales[row * (k / 32) + kk / 32]);
      out[kk] = orc_f64_to_f16(c * s);
    } else {
      double e = orc_e4m3_to_f64(scales[row * (k / 16) + g]);
      /* c*e has at most 6 significant bits and global_scale 24, so the
       * double product is exact; (float) rounds it once to fp32 (round to
       * nearest even), and the fp16 conversion rounds the fp32 value. */
      float p32 = (float)(c * e * (double)global_scale);
      out[kk] = orc_f64_to_f16((double)p32);
    }
  }
}

/* Decode a whole [n][k] matrix into out[n][k] fp16 bit patterns. */
void orc_dequant(int fmt, int64_t n, int64_t k, const uint8_t* data, const uint8_t* scales,
                 float global_scale, uint16_t* out) {
  for (int64_t r = 0; r < n; r++) orc_dequant_row(fmt, n, k, data, scales, global_scale, r, out + r * k);
}

/* ---------------------------------------------------------------------- */
/* Encoders: fp16 weights -> packed bytes.  The pages fix the formats but   */
/* not the quantiser; the readings below take the plainest choice of scale */
/* and then the nearest representable weight ("parity unpinned" for the   */
/* scale choice; the nearest-value step is pinned by the tests).           */
/*   FP4-G16 (fp16 scale): s = fp16(amax / 6) per group of 16, amax = the  */
/*     largest |w| of the group (6 = the largest E2M1 magnitude).           */
/*   MXFP4: e = floor(log2(amax)) - 2 + 127 clamped to [0, 254] (the OCP MX */
/*     shared exponent; 2 = the E2M1 maximum's exponent), e = 0 for amax = 0,*/
/*     254 for an infinite amax.                                            */
/*   IQ4_NL: d = fp16(m / -127), m the first element of largest |w| of the  */
/*     block, so that it maps to the table's -127 entry.                    */
/* Then each weight takes the code whose decoded value (exactly as the      */
/* decoders define it) is nearest; on equal distance the lowest code (FP4:  */
/* 0..7 are +0, 0.5, .. 6, 8..15 their negatives; IQ4_NL: table order).     */
/* A NaN weight takes code 0.                                               */
/* ---------------------------------------------------------------------- */
static int orc_nearest_code(double w, const double* cand, int ncand) {
  int best = 0;
  double be = fabs(w - cand[0]);
  for (int i = 1; i < ncand; i++) {
    double e = fabs(w - cand[i]);
    if (e < be) { be = e; best = i; }
  }
  return best;
}

/* w [n][k] fp16 bits -> data (codes or blocks) and scales, in the layouts of
 * orc_dequant_row.  fmt: FP4G16_F16, MXFP4 or IQ4_NL (E4M3 is not encoded). */
void orc_quantize(int fmt, int64_t n, int64_t k, const uint16_t* w, uint8_t* data, uint8_t* scales) {
  double cand[16];
  for (int64_t r = 0; r < n; r++) {
    const uint16_t* wr = w + r * k;
    if (fmt == ORC_FMT_IQ4_NL) {
      for (int64_t b = 0; b < k / 32; b++) {
        double m = 0.0, am = 0.0;
        for (int j = 0; j < 32; j++) {
          double v = orc_f16_to_f64(wr[b * 32 + j]);
          if (fabs(v) > am) { am = fabs(v); m = v; }
        }
        uint16_t dbits = orc_f64_to_f16(m / -127.0);
        double d = orc_f16_to_f64(dbits);
        for (int i = 0; i < 16; i++) cand[i] = orc_f16_to_f64(orc_f64_to_f16(d * (double)orc_iq4nl_table[i]));
        uint8_t* blk = data + (r * (k / 32) + b) * 18;
        blk[0] = (uint8_t)(dbits & 0xFF);
        blk[1] = (uint8_t)(dbits >> 8);
        for (int j = 0; j < 16; j++) {
          int lo = orc_nearest_code(orc_f16_to_f64(wr[b * 32 + j]), cand, 16);
          int hi = orc_nearest_code(orc_f16_to_f64(wr[b * 32 + j + 16]), cand, 16);
          blk[2 + j] = (uint8_t)(lo | (hi << 4));
        }
      }
      continue;
    }
    const int g = (fmt == ORC_FMT_MXFP4) ? 32 : 16;
    for (int64_t q = 0; q < k / g; q++) {
      double am = 0.0;
      for (int j = 0; j < g; j++) {
        double v = fabs(orc_f16_to_f64(wr[q * g + j]));
        if (v > am) am = v;
      }
      double sc;
      if (fmt == ORC_FMT_MXFP4) {
        int e = 0;
        if (isinf(am)) {
          e = 254; /* an infinite weight: the largest scale */
        } else if (am > 0.0) {
          int ex;
          frexp(am, &ex); /* am = fr * 2^ex, fr in [0.5, 1): floor(log2(am)) = ex - 1 */
          e = ex - 1 - 2 + 127;
          if (e < 0) e = 0;
          if (e > 254) e = 254;
        }
        scales[r * (k / 32) + q] = (uint8_t)e;
        sc = orc_e8m0_to_f64((uint8_t)e);
      } else {
        uint16_t sbits = orc_f64_to_f16(am / 6.0);
        scales[(r * (k / 16) + q) * 2] = (uint8_t)(sbits & 0xFF);
        scales[(r * (k / 16) + q) * 2 + 1] = (uint8_t)(sbits >> 8);
        sc = orc_f16_to_f64(sbits);
      }
      for (int c = 0; c < 16; c++) cand[c] = orc_f16_to_f64(orc_f64_to_f16(orc_e2m1_to_f64((uint8_t)c) * sc));
      for (int j = 0; j < g; j += 2) {
        int c0 = orc_nearest_code(orc_f16_to_f64(wr[q * g + j]), cand, 16);
        int c1 = orc_nearest_code(orc_f16_to_f64(wr[q * g + j + 1]), cand, 16);
        data[r * (k / 2) + (q * g + j) / 2] = (uint8_t)(c0 | (c1 << 4));
      }
    }
  }
}

/* ---------------------------------------------------------------------- */
/* Matrix product on the decoded weights                                  */
/* ---------------------------------------------------------------------- */

/* y[i][r] = sum_k w16[r][k] * x[i][k] in double, ascending k, and
 * absy[i][r] = sum_k |w16[r][k] * x[i][k]| (the tolerance scale).
 * x is [m][k] fp16 bits; y and absy are [m][n] doubles (absy may be NULL).
 * This single definition serves the decode GEMV (small m) and the prefill
 * GEMM (m = window length): both compute the same sum. */
void orc_matmul(int fmt, int64_t n, int64_t k, const uint8_t* data, const uint8_t* scales,
                float global_scale, const uint16_t* x, int64_t m, double* y, double* absy) {
  uint16_t* w = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(k > 0 ? k : 1));
  double* wd = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
  double* xd = (double*)malloc(sizeof(double) * (size_t)((m * k) > 0 ? m * k : 1));
  for (int64_t i = 0; i < m * k; i++) xd[i] = orc_f16_to_f64(x[i]);
  for (int64_t r = 0; r < n; r++) {
    orc_dequant_row(fmt, n, k, data, scales, global_scale, r, w);
    for (int64_t kk = 0; kk < k; kk++) wd[kk] = orc_f16_to_f64(w[kk]);
    for (int64_t i = 0; i < m; i++) {
      double s = 0.0, sa = 0.0;
      const double* xr = xd + i * k;
      for (int64_t kk = 0; kk < k; kk++) {
        double p = wd[kk] * xr[kk];
        s += p;
        sa += fabs(p);
      }
      y[i * n + r] = s;
      if (absy) absy[i * n + r] = sa;
    }
  }
  free(w);
  free(wd);
  free(xd);
}

/* The same sum for a list of (i, r) output coordinates only: out[c] =
 * y[mi[c]][ri[c]], absout[c] = sum |w x|.  Used to check single outputs of
 * full-size products that would take too long to compute whole. */
void orc_matmul_sampled(int fmt, int64_t n, int64_t k, const uint8_t* data, const uint8_t* scales,
                        float global_scale, const uint16_t* x, int64_t m, const int64_t* mi,
                        const int64_t* ri, int64_t count, double* out, double* absout) {
  uint16_t* w = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(k > 0 ? k : 1));
  (void)m;
  for (int64_t c = 0; c < count; c++) {
    orc_dequant_row(fmt, n, k, data, scales, global_scale, ri[c], w);
    const uint16_t* xr = x + mi[c] * k;
    double s = 0.0, sa = 0.0;
    for (int64_t kk = 0; kk < k; kk++) {
      double p = orc_f16_to_f64(w[kk]) * orc_f16_to_f64(xr[kk]);
      s += p;
      sa += fabs(p);
    }
    out[c] = s;
    if (absout) absout[c] = sa;
  }
  free(w);
}

/* ---------------------------------------------------------------------- */
/* Routed experts [MARK-M]                                                */
/* ---------------------------------------------------------------------- */

/* Bucket the t*topk (token, slot) pairs by chosen expert: a counting sort.
 * offsets[e] .. offsets[e+1]-1 index perm[], which lists pair indices
 * p = token*topk + slot in ascending p within each expert (the stable
 * order).  Returns the number of ids outside [0, num_experts), which are
 * left out of every bucket. */
int64_t orc_route(const int32_t* ids, int64_t t, int64_t topk, int64_t num_experts, int32_t* offsets,
                  int32_t* perm) {
  int64_t bad = 0;
  for (int64_t e = 0; e <= num_experts; e++) offsets[e] = 0;
  for (int64_t p = 0; p < t * topk; p++) {
    int32_t e = ids[p];
    if (e < 0 || e >= num_experts) { bad++; continue; }
    offsets[e + 1] += 1;
  }
  for (int64_t e = 0; e < num_experts; e++) offsets[e + 1] += offsets[e];
  int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * (size_t)(num_experts > 0 ? num_experts : 1));
  for (int64_t e = 0; e < num_experts; e++) fill[e] = offsets[e];
  for (int64_t p = 0; p < t * topk; p++) {
    int32_t e = ids[p];
    if (e < 0 || e >= num_experts) continue;
    perm[fill[e]++] = (int32_t)p;
  }
  free(fill);
  return bad;
}

/* For every (token, slot): y[token][slot][:] = W_e x_token with
 * e = ids[token][slot], W_e the e-th [n][k] matrix of the expert stack
 * (expert e's data at data + e*data_stride bytes, scales at
 * scales + e*scale_stride bytes).  Pairs whose id is out of range are left
 * untouched.  Only the listed pairs are computed when pairs != NULL. */
void orc_grouped_gemv(int fmt, int64_t n, int64_t k, const uint8_t* data, int64_t data_stride,
                      const uint8_t* scales, int64_t scale_stride, float global_scale,
                      int64_t num_experts, const uint16_t* x, const int32_t* ids, int64_t t,
                      int64_t topk, double* y, double* absy) {
  double* yr = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double* ar = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  for (int64_t tok = 0; tok < t; tok++) {
    for (int64_t s = 0; s < topk; s++) {
      int32_t e = ids[tok * topk + s];
      if (e < 0 || e >= num_experts) continue;
      const uint8_t* de = data + (int64_t)e * data_stride;
      const uint8_t* se = scales ? scales + (int64_t)e * scale_stride : NULL;
      orc_matmul(fmt, n, k, de, se, global_scale, x + tok * k, 1, yr, ar);
      for (int64_t r = 0; r < n; r++) {
        y[(tok * topk + s) * n + r] = yr[r];
        if (absy) absy[(tok * topk + s) * n + r] = ar[r];
      }
    }
  }
  free(yr);
  free(ar);
}

/* ---------------------------------------------------------------------- */
/* Mixture-of-experts block around the grouped GEMV [MARK-M]:             */
/*   s_{t,e} = Softmax_e(x_t W_router^T + b_e), the top-k experts by s    */
/*   carry weights g_i = s_{t,i}; a routed expert is                       */
/*   F(x) = (SiLU(x W_gate) * (x W_up)) W_down; the routed part of the    */
/*   layer output is sum_i g_i F_i(x).                                     */
/* Readings: W_router is a dense fp16 [E][k] matrix and b an fp32 [E]       */
/* vector; g_i is the softmax score itself (no renormalisation over the    */
/* top-k); the top-k is decided on the logits rounded to fp32 (the         */
/* precision the GPU decides in), larger first, ties to the lower expert   */
/* index.                                                                  */
/* ---------------------------------------------------------------------- */

/* logits[t][e] = fp32(sum_k x[t][k] * w[e][k] (double) + b[e]);
 * ids[t][j], g[t][j] (double): the top-k experts and their softmax scores;
 * probs[t][e] (double, may be NULL): the full softmax. */
void orc_router_topk(const uint16_t* x, const uint16_t* w, const float* b, int64_t t, int64_t k, int64_t E,
                     int64_t topk, float* logits, int32_t* ids, double* g, double* probs) {
  double* p = (double*)malloc(sizeof(double) * (size_t)(E > 0 ? E : 1));
  char* taken = (char*)malloc((size_t)(E > 0 ? E : 1));
  for (int64_t i = 0; i < t; i++) {
    double mx = -INFINITY;
    for (int64_t e = 0; e < E; e++) {
      double s = 0.0;
      for (int64_t kk = 0; kk < k; kk++) s += orc_f16_to_f64(x[i * k + kk]) * orc_f16_to_f64(w[e * k + kk]);
      float z = (float)(s + (double)b[e]);
      logits[i * E + e] = z;
      if ((double)z > mx) mx = (double)z;
    }
    double den = 0.0;
    for (int64_t e = 0; e < E; e++) {
      p[e] = exp((double)logits[i * E + e] - mx);
      den += p[e];
    }
    for (int64_t e = 0; e < E; e++) {
      p[e] /= den;
      if (probs) probs[i * E + e] = p[e];
      taken[e] = 0;
    }
    for (int64_t j = 0; j < topk; j++) {
      int64_t best = -1;
      for (int64_t e = 0; e < E; e++) {
        if (taken[e]) continue;
        if (best < 0 || logits[i * E + e] > logits[i * E + best]) best = e;
      }
      taken[best] = 1;
      ids[i * topk + j] = (int32_t)best;
      g[i * topk + j] = p[best];
    }
  }
  free(p);
  free(taken);
}

/* SiLU(z) = z / (1 + exp(-z)). */
double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* h[p][j] = SiLU(gu[p][j]) * gu[p][f + j] for the gate+up product rows
 * gu[p] = [gate (f values) | up (f values)] of each (token, slot) pair. */
void orc_swiglu(const double* gu, int64_t pairs, int64_t f, double* h) {
  for (int64_t p = 0; p < pairs; p++)
    for (int64_t j = 0; j < f; j++) h[p * f + j] = orc_silu(gu[p * 2 * f + j]) * gu[p * 2 * f + f + j];
}

/* out[t][j] = sum_s g[t][s] * y[t][s][j]. */
void orc_combine(const double* y, const double* g, int64_t t, int64_t topk, int64_t n, double* out) {
  for (int64_t i = 0; i < t; i++)
    for (int64_t j = 0; j < n; j++) {
      double s = 0.0;
      for (int64_t q = 0; q < topk; q++) s += g[i * topk + q] * y[(i * topk + q) * n + j];
      out[i * n + j] = s;
    }
}
