// k_quant.cuh -- encoders: resident fp16 weights -> packed 4-bit blocks.
//
// The pages fix the formats ("Mamb2_8B_FP4_Recall_SQ3.25", section
// "Representation": E2M1 codes in 16-element groups along k; "1bit.gg
// zyphra", MXFP4 experts: 32 E2M1 codes and one E8M0 byte per group;
// "Mark-Experimental-V3-8B", section "Quantization": IQ4_NL blocks) but not
// the quantiser.  Reading: FP4-G16 s = fp16(amax / 6); MXFP4 e = floor(log2
// amax) - 2 + 127 in [0, 254] (0 for amax = 0, 254 for an infinite amax);
// IQ4_NL d = fp16(m / -127), m the first element of largest |w|.  Each
// weight then takes the code whose decoded value -- computed exactly as the
// decoders compute it -- is nearest, distances in double (exact for fp16
// operands), the lowest code on equal distance; a NaN weight takes code 0.
//
// One thread per group: 16 (FP4-G16) or 32 weights (MXFP4, IQ4_NL).  The
// scale divisions are correctly rounded in fp32 and then to fp16; amax / 6
// and m / 127 are never near an fp16 rounding tie unless exact, so the
// result equals the exact rational rounding.
#pragma once
#include "k_dequant.cuh"
#include "qmm_dev.cuh"

namespace qmm {

__device__ __forceinline__ int nearest_code(double w, const double (&cand)[16]) {
  int best = 0;
  double be = fabs(w - cand[0]);
#pragma unroll
  for (int i = 1; i < 16; i++) {
    const double e = fabs(w - cand[i]);
    if (e < be) {
      be = e;
      best = i;
    }
  }
  return best;
}

__device__ __forceinline__ double h2d(uint32_t h16) {
  return (double)__half2float(__ushort_as_half((unsigned short)(h16 & 0xFFFFu)));
}

// E2M1 code c as an fp16 bit pattern (exact).
__device__ __forceinline__ uint32_t e2m1_f16_bits(int c) { return e2m1x2_to_f16x2((uint32_t)c) & 0xFFFFu; }

template <int FMT>  // 2: FP4-G16 fp16 scale, 4: MXFP4
__global__ void __launch_bounds__(128) quantize_fp4_kernel(const uint16_t* __restrict__ w, uint8_t* __restrict__ codes,
                                                           uint8_t* __restrict__ scales, int64_t groups) {
  constexpr int G = (FMT == 4) ? 32 : 16;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < groups; i += (int64_t)gridDim.x * blockDim.x) {
    uint32_t wv[G / 2];
#pragma unroll
    for (int q = 0; q < G / 8; q++) {
      const uint4 v = *reinterpret_cast<const uint4*>(w + i * G + 8 * q);
      wv[4 * q] = v.x; wv[4 * q + 1] = v.y; wv[4 * q + 2] = v.z; wv[4 * q + 3] = v.w;
    }
    float am = 0.f;
#pragma unroll
    for (int j = 0; j < G / 2; j++) {
      const float2 f = f16x2_to_f32x2(wv[j]);
      if (fabsf(f.x) > am) am = fabsf(f.x);
      if (fabsf(f.y) > am) am = fabsf(f.y);
    }
    double cand[16];
    if (FMT == 4) {
      uint32_t e = 0u;
      if (isinf(am)) e = 254u;
      else if (am > 0.f) {
        const int e2 = (int)((__float_as_uint(am) >> 23) & 0xFFu) - 127 - 2 + 127;  // floor(log2 am) - 2 + 127
        e = (uint32_t)(e2 < 0 ? 0 : (e2 > 254 ? 254 : e2));
      }
      scales[i] = (uint8_t)e;
      const float sf = e8m0_to_f32(e);
#pragma unroll
      for (int c = 0; c < 16; c++) cand[c] = h2d(mx_scale_any(e2m1_f16_bits(c), sf));
    } else {
      const uint32_t s = __half_as_ushort(__float2half_rn(__fdiv_rn(am, 6.0f)));
      reinterpret_cast<uint16_t*>(scales)[i] = (uint16_t)s;
#pragma unroll
      for (int c = 0; c < 16; c++) cand[c] = h2d(hmul2(e2m1_f16_bits(c), s));
    }
    uint32_t out[G / 8];
#pragma unroll
    for (int q = 0; q < G / 8; q++) {
      uint32_t word = 0u;
#pragma unroll
      for (int j = 0; j < 4; j++) {  // byte j of the word: weights 8q + 2j, 8q + 2j + 1
        const uint32_t pair = wv[4 * q + j];
        const int c0 = nearest_code(h2d(pair), cand), c1 = nearest_code(h2d(pair >> 16), cand);
        word |= (uint32_t)(c0 | (c1 << 4)) << (8 * j);
      }
      out[q] = word;
    }
    if (G == 32) *reinterpret_cast<uint4*>(codes + i * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    else *reinterpret_cast<uint2*>(codes + i * 8) = make_uint2(out[0], out[1]);
  }
}

__global__ void __launch_bounds__(128) quantize_iq4nl_kernel(const uint16_t* __restrict__ w, uint8_t* __restrict__ blocks,
                                                             int64_t nblocks) {
  for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks; b += (int64_t)gridDim.x * blockDim.x) {
    uint32_t wv[16];
#pragma unroll
    for (int q = 0; q < 4; q++) {
      const uint4 v = *reinterpret_cast<const uint4*>(w + b * 32 + 8 * q);
      wv[4 * q] = v.x; wv[4 * q + 1] = v.y; wv[4 * q + 2] = v.z; wv[4 * q + 3] = v.w;
    }
    float am = 0.f, m = 0.f;  // first element of largest magnitude
#pragma unroll
    for (int j = 0; j < 16; j++) {
      const float2 f = f16x2_to_f32x2(wv[j]);
      if (fabsf(f.x) > am) { am = fabsf(f.x); m = f.x; }
      if (fabsf(f.y) > am) { am = fabsf(f.y); m = f.y; }
    }
    const uint32_t d = __half_as_ushort(__float2half_rn(__fdiv_rn(m, -127.0f)));
    double cand[16];
#pragma unroll
    for (int i = 0; i < 16; i++)
      cand[i] = h2d(hmul2((uint32_t)__half_as_ushort(__int2half_rn(c_iq4nl_kv[i])), d));
    uint16_t* o = reinterpret_cast<uint16_t*>(blocks + b * 18);  // 2-byte aligned
    o[0] = (uint16_t)d;
#pragma unroll
    for (int h = 0; h < 8; h++) {  // index bytes 2h, 2h+1: weights (2h, 2h+16), (2h+1, 2h+17)
      const uint32_t lo2 = wv[h], hi2 = wv[8 + h];
      const int a0 = nearest_code(h2d(lo2), cand), a1 = nearest_code(h2d(lo2 >> 16), cand);
      const int b0 = nearest_code(h2d(hi2), cand), b1 = nearest_code(h2d(hi2 >> 16), cand);
      o[1 + h] = (uint16_t)((a0 | (b0 << 4)) | ((a1 | (b1 << 4)) << 8));
    }
  }
}

}  // namespace qmm
