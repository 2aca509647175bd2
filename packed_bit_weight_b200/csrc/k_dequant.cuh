// k_dequant.cuh -- packed 4-bit weights -> resident fp16, bit-exact.
//
// The decode rule is the one the model cards imply for their FP16 runtime
// ("Mamb2_8B_FP4_Recall_SQ3.25", sections "Representation" and "Storage and
// runtime memory"; "Mark-Experimental-V3-8B", section "Quantization"): one
// rounding of code * scale to fp16 (nearest even, subnormals kept).  On the
// GPU the code value is exact in fp16 and a single f16x2 multiply performs
// exactly that rounding.  For E4M3 block scales the exact fp16 product
// code*e4m3 is widened to fp32, multiplied by the fp32 global scale (one fp32
// rounding) and narrowed to fp16 (second rounding), as specified.
//
// The kernels are bandwidth-bound streams (read 0.5625-0.625 B, write 2 B per
// weight): a grid-stride loop over groups with 16-byte stores.
#pragma once
#include "qmm_dev.cuh"

namespace qmm {

// IQ4_NL table as fp16-exact integers.
__constant__ int8_t c_iq4nl_kv[16] = {-127, -104, -83, -65, -49, -35, -22, -10, 1, 13, 25, 38, 53, 69, 89, 113};

// FP4-G16: one thread per 16-weight group (8 code bytes, one scale).
template <int FMT>
__global__ void __launch_bounds__(256) dequant_fp4_kernel(const uint8_t* __restrict__ codes,
                                                          const uint8_t* __restrict__ scales, float g,
                                                          uint16_t* __restrict__ out, int64_t groups) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < groups; i += (int64_t)gridDim.x * blockDim.x) {
    const uint2 q = *reinterpret_cast<const uint2*>(codes + i * 8);
    uint32_t w[8];
    e2m1x8_to_f16x2(q.x, *reinterpret_cast<uint32_t(*)[4]>(&w[0]));
    e2m1x8_to_f16x2(q.y, *reinterpret_cast<uint32_t(*)[4]>(&w[4]));
    if (FMT == 2) {  // fp16 group scale: fp16(code * s) in one multiply
      const uint32_t s = reinterpret_cast<const uint16_t*>(scales)[i];
      const uint32_t ss = s | (s << 16);
#pragma unroll
      for (int j = 0; j < 8; j++) w[j] = hmul2(w[j], ss);
    } else {  // E4M3 block scale and fp32 global scale
      const uint32_t e = e4m3x2_to_f16x2(scales[i]);  // low half = e (exact), high half = 0
      const uint32_t ee = bcast_lo(e);
#pragma unroll
      for (int j = 0; j < 8; j++) {
        const float2 ce = f16x2_to_f32x2(hmul2(w[j], ee));  // code*e exact in fp16
        w[j] = f32x2_to_f16x2(ce.x * g, ce.y * g);
      }
    }
    uint4* o = reinterpret_cast<uint4*>(out + i * 16);
    o[0] = make_uint4(w[0], w[1], w[2], w[3]);
    o[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

// MXFP4: one thread per 32-weight group (16 code bytes, one E8M0 byte);
// fp16(code * 2^(e-127)), one rounding ("1bit.gg zyphra", MXFP4 experts).
__global__ void __launch_bounds__(256) dequant_mxfp4_kernel(const uint8_t* __restrict__ codes,
                                                            const uint8_t* __restrict__ scales,
                                                            uint16_t* __restrict__ out, int64_t groups) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < groups; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 q = *reinterpret_cast<const uint4*>(codes + i * 16);
    const uint32_t b = scales[i];
    uint32_t w[16];
    e2m1x8_to_f16x2(q.x, *reinterpret_cast<uint32_t(*)[4]>(&w[0]));
    e2m1x8_to_f16x2(q.y, *reinterpret_cast<uint32_t(*)[4]>(&w[4]));
    e2m1x8_to_f16x2(q.z, *reinterpret_cast<uint32_t(*)[4]>(&w[8]));
    e2m1x8_to_f16x2(q.w, *reinterpret_cast<uint32_t(*)[4]>(&w[12]));
    if (e8m0_f16_ok(b)) {
      const uint32_t ss = e8m0_to_f16x2(b);
#pragma unroll
      for (int j = 0; j < 16; j++) w[j] = hmul2(w[j], ss);
    } else {
      const float sf = e8m0_to_f32(b);
#pragma unroll
      for (int j = 0; j < 16; j++) w[j] = mx_scale_any(w[j], sf);
    }
    uint4* o = reinterpret_cast<uint4*>(out + i * 32);
#pragma unroll
    for (int j = 0; j < 4; j++) o[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  }
}

// IQ4_NL: one thread per 18-byte block (2-byte aligned: read as 9 halves).
__global__ void __launch_bounds__(256) dequant_iq4nl_kernel(const uint8_t* __restrict__ blocks,
                                                            uint16_t* __restrict__ out, int64_t nblocks) {
  __shared__ uint32_t kvh[16];  // kv as fp16 bit patterns
  if (threadIdx.x < 16) kvh[threadIdx.x] = __half_as_ushort(__int2half_rn(c_iq4nl_kv[threadIdx.x]));
  __syncthreads();
  for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks; b += (int64_t)gridDim.x * blockDim.x) {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(blocks + b * 18);
    const uint32_t d = p[0];
    const uint32_t dd = d | (d << 16);
    uint32_t lo[8], hi[8];  // lo[j/2] = weights (j, j+1), hi[j/2] = weights (16+j, 17+j)
#pragma unroll
    for (int h = 0; h < 8; h++) {
      const uint32_t two = p[1 + h];  // qs[2h] (low byte), qs[2h+1]
      const uint32_t b0 = two & 0xFF, b1 = two >> 8;
      lo[h] = hmul2(kvh[b0 & 15] | (kvh[b1 & 15] << 16), dd);
      hi[h] = hmul2(kvh[b0 >> 4] | (kvh[b1 >> 4] << 16), dd);
    }
    uint4* o = reinterpret_cast<uint4*>(out + b * 32);
    o[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    o[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
    o[2] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    o[3] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
  }
}

// Copy n16 16-byte units from src (page-locked host memory through its device
// mapping) to dst, one unit per thread (the grid covers n16).  Launched with
// programmatic dependent launch: the read across the bus starts while the
// kernel before it on the stream (the previous call's GEMV, which may still
// read dst) runs; dst is written only after griddepcontrol.wait.  It lets the
// GEMV launched after it start at once (launch_dependents first): the GEMV
// streams its weights while this copy crosses the bus, and waits for it
// before it reads x.
__global__ void fetch16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t n16) {
  asm volatile("griddepcontrol.launch_dependents;" :::);
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint4 v = make_uint4(0, 0, 0, 0);
  if (i < n16) v = src[i];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (i < n16) dst[i] = v;
}

// y[i] = 0 for i < count (a product over an empty k axis).
__global__ void zero_fill_kernel(uint16_t* __restrict__ y, int64_t count) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x)
    y[i] = 0;
}

}  // namespace qmm
