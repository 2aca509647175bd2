// k_gemv.cuh -- fused dequantise-and-multiply for decode batches (m <= 16).
//
// y[m][n] = sum_k x[m][k] * W[n][k], W decoded from packed 4-bit blocks in
// registers, products on the legacy warp MMA (m16n8k16, f16 in, f32
// accumulate).  The MMA's M dimension is 16 weight rows and its N dimension
// 8 tokens, so one instruction consumes 256 decoded weights: at m <= 8 this
// replaces ~2 CUDA-core instructions per weight (convert + FMA) with
// 1/256 of an MMA, leaving the issue budget to the nibble decode, which is the
// ALU cost that has to keep up with HBM.
//
// Inside an MMA the order of the 16 k values is free as long as the A
// fragment (weights) and the B fragment (activations) agree.  The kernels use
// it to give every lane contiguous bytes: in a "segment" of 32 consecutive k a
// lane owns 16 code bytes of one row; MMA step i takes its bytes 2i (k 4i,
// 4i+1) and 2i+1 (k 4i+2, 4i+3), and the matching activations are the 8 bytes
// x[4i .. 4i+3] of the same segment.
#pragma once
#include "qmm_dev.cuh"

namespace qmm {

// ---------------------------------------------------------------------------
// Generic kernel: any k the format allows, any n, m <= 16, all formats.
// One warp per 16-row tile, the natural MMA fragment layout, byte loads.
// Used for small or odd shapes (and as the IQ4_NL decode path).
// ---------------------------------------------------------------------------
template <int FMT>
__device__ __forceinline__ uint32_t generic_pair(const uint8_t* __restrict__ data, const uint8_t* __restrict__ scales,
                                                 int64_t row, int64_t n, int64_t k, int64_t kk,
                                                 const uint32_t* kvh) {
  // decoded weights (row, kk) and (row, kk+1) as f16x2; kk is even.
  if (row >= n) return 0u;
  if (FMT == 1) {
    const int64_t b = kk >> 5;
    const int j = (int)(kk & 31);
    const uint8_t* blk = data + (row * (k >> 5) + b) * 18;
    const uint32_t d = (uint32_t)blk[0] | ((uint32_t)blk[1] << 8);
    const int jj = j & 15;
    const uint32_t q0 = blk[2 + jj], q1 = blk[3 + jj];
    const uint32_t i0 = (j < 16) ? (q0 & 15) : (q0 >> 4);
    const uint32_t i1 = (j < 16) ? (q1 & 15) : (q1 >> 4);
    return hmul2(kvh[i0] | (kvh[i1] << 16), d | (d << 16));
  } else {
    const uint32_t byte = data[row * (k >> 1) + (kk >> 1)];
    const uint32_t c = e2m1x2_to_f16x2(byte);
    if (FMT == 4) {  // MXFP4: one E8M0 byte per 32
      const uint32_t e = scales[row * (k >> 5) + (kk >> 5)];
      return e8m0_f16_ok(e) ? hmul2(c, e8m0_to_f16x2(e)) : mx_scale_any(c, e8m0_to_f32(e));
    }
    const int64_t gi = row * (k >> 4) + (kk >> 4);
    if (FMT == 2) {
      const uint32_t s = reinterpret_cast<const uint16_t*>(scales)[gi];
      return hmul2(c, s | (s << 16));
    } else {
      return hmul2(c, bcast_lo(e4m3x2_to_f16x2(scales[gi])));  // code*e exact; g applied to the sum
    }
  }
}

template <int FMT>
__global__ void __launch_bounds__(128) gemv_generic_kernel(const uint8_t* __restrict__ data,
                                                           const uint8_t* __restrict__ scales, float g,
                                                           const uint16_t* __restrict__ x, uint16_t* __restrict__ y,
                                                           int64_t n, int64_t k, int m) {
  __shared__ uint32_t kvh[16];
  if (threadIdx.x < 16) kvh[threadIdx.x] = __half_as_ushort(__int2half_rn(c_iq4nl_kv[threadIdx.x]));
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int grp = lane >> 2, tig = lane & 3;
  const int64_t tile = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int64_t r0 = tile * 16 + grp, r1 = r0 + 8;
  if (tile * 16 >= n) return;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  const int nt = (m > 8) ? 2 : 1;
  for (int64_t k0 = 0; k0 < k; k0 += 16) {
    const int64_t ka = k0 + 2 * tig, kb = ka + 8;
    const uint32_t a0 = generic_pair<FMT>(data, scales, r0, n, k, ka, kvh);
    const uint32_t a1 = generic_pair<FMT>(data, scales, r1, n, k, ka, kvh);
    const uint32_t a2 = generic_pair<FMT>(data, scales, r0, n, k, kb, kvh);
    const uint32_t a3 = generic_pair<FMT>(data, scales, r1, n, k, kb, kvh);
    for (int j = 0; j < nt; j++) {
      const int tok = grp + 8 * j;
      uint32_t b0 = 0, b1 = 0;
      if (tok < m) {
        b0 = *reinterpret_cast<const uint32_t*>(x + tok * k + ka);
        b1 = *reinterpret_cast<const uint32_t*>(x + tok * k + kb);
      }
      mma_16816(acc[j], a0, a1, a2, a3, b0, b1);
    }
  }
  const float gs = (FMT == 3) ? g : 1.0f;
  for (int j = 0; j < nt; j++) {
    const int t0 = 8 * j + 2 * tig, t1 = t0 + 1;
    if (r0 < n && t0 < m) y[t0 * n + r0] = f32_to_f16_bits(acc[j][0] * gs);
    if (r0 < n && t1 < m) y[t1 * n + r0] = f32_to_f16_bits(acc[j][1] * gs);
    if (r1 < n && t0 < m) y[t0 * n + r1] = f32_to_f16_bits(acc[j][2] * gs);
    if (r1 < n && t1 < m) y[t1 * n + r1] = f32_to_f16_bits(acc[j][3] * gs);
  }
}

// ---------------------------------------------------------------------------
// Streaming FP4-G16 kernel, register-direct (no shared-memory staging).
//
// One CTA = one tile of 16 weight rows over the whole k; its 8 warps split k
// into equal ranges of SPW segments of 128 (64 code bytes per row).  Each lane
// owns rows grp and grp+8 and, in every segment, the 16 code bytes at
// 16*tig (plus their two group scales): it issues all of its loads for the
// tile at once (16-byte ld.global.nc with an L2 256-byte prefetch hint, no L1
// allocation), so a warp has SPW*1.25 KB in flight and the several CTAs
// resident per SM keep HBM busy.  The bytes then go straight into MMA
// fragments (same k order as the TMA kernel).  The WPC partial tiles are
// summed in shared memory in a fixed order.  Launched with programmatic
// dependent launch: the weight loads are issued before griddepcontrol.wait, so
// a CTA that starts while the previous kernel drains already streams its
// weights; activations are read and y written only after the wait.
// ---------------------------------------------------------------------------
// The same streaming loads as volatile asm: kept after griddepcontrol.wait
// when they are written after it (a plain asm load may be hoisted above).
__device__ __forceinline__ uint4 ldg_stream128_after(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_stream32_after(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_stream16_after(const void* p) {
  unsigned short v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ldg_stream128(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_stream32(const void* p) {
  uint32_t v;
  asm("ld.global.nc.L1::no_allocate.L2::256B.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_stream8(const void* p) {
  unsigned short v;
  asm("ld.global.nc.L1::no_allocate.L2::256B.u8 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_stream16(const void* p) {
  unsigned short v;
  asm("ld.global.nc.L1::no_allocate.L2::256B.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
// 256-bit streaming loads (sm_100): 32 contiguous bytes per lane, so the
// four lanes of a weight row cover a whole 128-byte line per instruction.
// p must be 32-byte aligned.
__device__ __forceinline__ void ldg_stream256(const void* p, uint4& lo, uint4& hi) {
  asm("ld.global.nc.L1::no_allocate.L2::256B.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
      : "l"(p));
}
__device__ __forceinline__ uint2 ldg_stream64(const void* p) {
  uint2 v;
  asm("ld.global.nc.L1::no_allocate.L2::256B.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
// 256-bit activation load (L1-allocating; p 32-byte aligned).
__device__ __forceinline__ void ldg_x256(const void* p, uint4& lo, uint4& hi) {
  asm("ld.global.nc.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
      : "l"(p));
}
__device__ __forceinline__ uint4 ldg_x128(const void* p) {
  uint4 v;
  asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

constexpr int kLdgWarps = 8;

// Programmatic dependent launch: let the next kernel on the stream start
// launching now; wait until the previous kernel's writes are visible.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Decode and multiply a warp's SPW segments of one 16-row tile, held in
// registers (code bytes qa/qb of rows grp and grp+8, group-scale pairs sa/sb
// as f16x2), against tokens grp and grp+8 (when < m) read from global memory.
// Measured alternatives, both slower on the in_proj shape: loading a clamped
// token row in every lane instead of zero-filling the columns past m (27 %:
// 8x the L1 traffic), and zero-filling once before the segment loop (18 %:
// the compiler then keeps fewer of the tile's loads in flight).
// WIDE: the lane's bytes of two consecutive segments 2w, 2w+1 are the 32
// contiguous bytes at 32*tig of a 256-k span (one 256-bit load), so segment
// 2w+h holds k = 256w + 64*tig + 32h + [0, 32) instead of 128s + 32*tig.
// XW: the token row's 64 bytes per segment as two 256-bit loads (x rows
// 32-byte aligned).
// MX1 (MXFP4): every group of the warp's segments has f1 = 1 (its scale is
// an fp16 value), so one multiply by f2 gives the same bits as two.
template <int FMT, int NT, int SPW, bool WIDE = false, bool XW = false, bool MX1 = false>
__device__ __forceinline__ void ldg_tile_mma(float (&acc)[NT][4], const uint4 (&qa)[SPW], const uint4 (&qb)[SPW],
                                             const uint32_t (&sa)[SPW], const uint32_t (&sb)[SPW], int seg0, int grp,
                                             int tig, const uint16_t* __restrict__ x, int k, int m) {
#pragma unroll
  for (int i = 0; i < SPW; i++) {
    const int s = seg0 + i;
    const int kseg = WIDE ? (s >> 1) * 256 + tig * 64 + (s & 1) * 32 : s * 128 + tig * 32;
    uint32_t xb[NT][16];
#pragma unroll
    for (int j = 0; j < NT; j++) {
      const int tok = grp + 8 * j;
      if (tok < m) {
        const uint16_t* xp = x + (int64_t)tok * k + kseg;
        if (XW) {
#pragma unroll
          for (int q = 0; q < 2; q++) {
            uint4 lo, hi;
            ldg_x256(xp + 16 * q, lo, hi);
            xb[j][8 * q] = lo.x; xb[j][8 * q + 1] = lo.y; xb[j][8 * q + 2] = lo.z; xb[j][8 * q + 3] = lo.w;
            xb[j][8 * q + 4] = hi.x; xb[j][8 * q + 5] = hi.y; xb[j][8 * q + 6] = hi.z; xb[j][8 * q + 7] = hi.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 4; q++) {
            const uint4 v = ldg_x128(xp + 8 * q);
            xb[j][4 * q] = v.x; xb[j][4 * q + 1] = v.y; xb[j][4 * q + 2] = v.z; xb[j][4 * q + 3] = v.w;
          }
        }
      } else {
#pragma unroll
        for (int q = 0; q < 16; q++) xb[j][q] = 0u;
      }
    }
    // group scales as f16x2: two fp16 groups per lane (FP4-G16), or one
    // E8M0 group (MXFP4: a power of two, applied as two fp16 factors so that
    // scales outside the fp16 range round exactly once too)
    uint32_t sa0, sa1, sb0, sb1;
    // FP4-G16: the two groups' scales; MXFP4: the one group's two fp16
    // factors (the first is 1 when the scale is an fp16 value)
    sa0 = bcast_lo(sa[i]); sa1 = bcast_hi(sa[i]); sb0 = bcast_lo(sb[i]); sb1 = bcast_hi(sb[i]);
    uint32_t wa[16], wb[16];
    e2m1x8_to_f16x2(qa[i].x, *reinterpret_cast<uint32_t(*)[4]>(&wa[0]));
    e2m1x8_to_f16x2(qa[i].y, *reinterpret_cast<uint32_t(*)[4]>(&wa[4]));
    e2m1x8_to_f16x2(qa[i].z, *reinterpret_cast<uint32_t(*)[4]>(&wa[8]));
    e2m1x8_to_f16x2(qa[i].w, *reinterpret_cast<uint32_t(*)[4]>(&wa[12]));
    e2m1x8_to_f16x2(qb[i].x, *reinterpret_cast<uint32_t(*)[4]>(&wb[0]));
    e2m1x8_to_f16x2(qb[i].y, *reinterpret_cast<uint32_t(*)[4]>(&wb[4]));
    e2m1x8_to_f16x2(qb[i].z, *reinterpret_cast<uint32_t(*)[4]>(&wb[8]));
    e2m1x8_to_f16x2(qb[i].w, *reinterpret_cast<uint32_t(*)[4]>(&wb[12]));
#pragma unroll
    for (int st = 0; st < 8; st++) {
      uint32_t a0, a1, a2, a3;
      if (FMT == 4 && MX1) {  // f1 = 1: code * f2 rounds once
        a0 = hmul2(wa[2 * st], sa1); a2 = hmul2(wa[2 * st + 1], sa1);
        a1 = hmul2(wb[2 * st], sb1); a3 = hmul2(wb[2 * st + 1], sb1);
      } else if (FMT == 4) {  // the lane's one group: code * f1 exact, * f2 rounds once
        a0 = hmul2(hmul2(wa[2 * st], sa0), sa1); a2 = hmul2(hmul2(wa[2 * st + 1], sa0), sa1);
        a1 = hmul2(hmul2(wb[2 * st], sb0), sb1); a3 = hmul2(hmul2(wb[2 * st + 1], sb0), sb1);
      } else {  // group st/4 of the lane's two
        const uint32_t sA = (st < 4) ? sa0 : sa1, sB = (st < 4) ? sb0 : sb1;
        a0 = hmul2(wa[2 * st], sA); a2 = hmul2(wa[2 * st + 1], sA);
        a1 = hmul2(wb[2 * st], sB); a3 = hmul2(wb[2 * st + 1], sB);
      }
#pragma unroll
      for (int j = 0; j < NT; j++) mma_16816(acc[j], a0, a1, a2, a3, xb[j][2 * st], xb[j][2 * st + 1]);
    }
  }
}

// The WPC warps' partial sums of one tile meet in shared memory and are added
// in warp order (deterministic); rows n0.. of y are stored.  Ends with every
// thread past a __syncthreads, so `red` may be reused afterwards only after
// another one.
template <int FMT, int NT, int WPC>
__device__ __forceinline__ void ldg_tile_store(float (&red)[WPC][16][16], const float (&acc)[NT][4], int warp, int grp,
                                               int tig, int n0, int n, int m, float g, uint16_t* __restrict__ y) {
#pragma unroll
  for (int j = 0; j < NT; j++) {
    const int t0 = 8 * j + 2 * tig;
    red[warp][t0][grp] = acc[j][0];
    red[warp][t0 + 1][grp] = acc[j][1];
    red[warp][t0][grp + 8] = acc[j][2];
    red[warp][t0 + 1][grp + 8] = acc[j][3];
  }
  __syncthreads();
  const float gs = (FMT == 3) ? g : 1.0f;
  for (int idx = threadIdx.x; idx < 16 * m; idx += WPC * 32) {
    const int row = idx & 15, tok = idx >> 4;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < WPC; w++) v += red[w][tok][row];
    if (n0 + row < n) y[(int64_t)tok * n + n0 + row] = f32_to_f16_bits(v * gs);
  }
}

// Segments [I0, I1) of ldg_tile_load, FP4-G16 scales (fp16 or E4M3), with
// volatile loads (AFTER: issued after the dependency wait and kept there).
template <int FMT, int SPW, int I0, int I1, bool AFTER>
__device__ __forceinline__ void ldg_tile_load_part(uint4 (&qa)[SPW], uint4 (&qb)[SPW], uint32_t (&sa)[SPW],
                                                   uint32_t (&sb)[SPW], const uint8_t* __restrict__ codes,
                                                   const uint8_t* __restrict__ scales, int64_t ra, int64_t rb,
                                                   bool va, bool vb, int seg0, int tig, int64_t crow, int64_t srow) {
  static_assert(FMT == 2 || FMT == 3, "FP4-G16 scales");
#pragma unroll
  for (int i = I0; i < I1; i++) {
    const int seg = seg0 + i;
    const int64_t cb = (int64_t)seg * 64 + tig * 16;
    const int64_t gi = (int64_t)seg * 8 + tig * 2;
    if (AFTER) {
      qa[i] = va ? ldg_stream128_after(codes + ra * crow + cb) : make_uint4(0, 0, 0, 0);
      qb[i] = vb ? ldg_stream128_after(codes + rb * crow + cb) : make_uint4(0, 0, 0, 0);
      if (FMT == 2) {
        sa[i] = va ? ldg_stream32_after(scales + (ra * srow + gi) * 2) : 0u;
        sb[i] = vb ? ldg_stream32_after(scales + (rb * srow + gi) * 2) : 0u;
      } else {
        sa[i] = va ? e4m3x2_to_f16x2(ldg_stream16_after(scales + ra * srow + gi)) : 0u;
        sb[i] = vb ? e4m3x2_to_f16x2(ldg_stream16_after(scales + rb * srow + gi)) : 0u;
      }
    } else {
      qa[i] = va ? ldg_stream128(codes + ra * crow + cb) : make_uint4(0, 0, 0, 0);
      qb[i] = vb ? ldg_stream128(codes + rb * crow + cb) : make_uint4(0, 0, 0, 0);
      if (FMT == 2) {
        sa[i] = va ? ldg_stream32(scales + (ra * srow + gi) * 2) : 0u;
        sb[i] = vb ? ldg_stream32(scales + (rb * srow + gi) * 2) : 0u;
      } else {
        sa[i] = va ? e4m3x2_to_f16x2(ldg_stream16(scales + ra * srow + gi)) : 0u;
        sb[i] = vb ? e4m3x2_to_f16x2(ldg_stream16(scales + rb * srow + gi)) : 0u;
      }
    }
  }
}

// Loads of one lane's SPW segments (128-bit layout: 16 code bytes of rows ra
// and rb at 16*tig of each 64-byte segment, and the two group scales they
// use; rows past n read as zero codes, scale 1 for MXFP4).
template <int FMT, int SPW>
__device__ __forceinline__ void ldg_tile_load(uint4 (&qa)[SPW], uint4 (&qb)[SPW], uint32_t (&sa)[SPW],
                                              uint32_t (&sb)[SPW], const uint8_t* __restrict__ codes,
                                              const uint8_t* __restrict__ scales, int64_t ra, int64_t rb, bool va,
                                              bool vb, int seg0, int tig, int64_t crow, int64_t srow) {
#pragma unroll
  for (int i = 0; i < SPW; i++) {
    const int seg = seg0 + i;
    const int64_t cb = (int64_t)seg * 64 + tig * 16;
    const int64_t gi = (int64_t)seg * 8 + tig * 2;  // first of the two group scales
    qa[i] = va ? ldg_stream128(codes + ra * crow + cb) : make_uint4(0, 0, 0, 0);
    qb[i] = vb ? ldg_stream128(codes + rb * crow + cb) : make_uint4(0, 0, 0, 0);
    if (FMT == 2) {
      sa[i] = va ? ldg_stream32(scales + (ra * srow + gi) * 2) : 0u;
      sb[i] = vb ? ldg_stream32(scales + (rb * srow + gi) * 2) : 0u;
    } else if (FMT == 4) {  // the lane's 32 k are one MXFP4 group: one E8M0 byte (127 = 1 for rows past n)
      sa[i] = e8m0_f16_factor_pair(va ? ldg_stream8(scales + ra * (srow >> 1) + seg * 4 + tig) : 127u);
      sb[i] = e8m0_f16_factor_pair(vb ? ldg_stream8(scales + rb * (srow >> 1) + seg * 4 + tig) : 127u);
    } else {
      sa[i] = va ? e4m3x2_to_f16x2(ldg_stream16(scales + ra * srow + gi)) : 0u;
      sb[i] = vb ? e4m3x2_to_f16x2(ldg_stream16(scales + rb * srow + gi)) : 0u;
    }
  }
}

// WIDE (k % 256 == 0, SPW even, codes 32-byte aligned): each lane loads its
// bytes of two segments with one 256-bit load per row, and their scales with
// one load (8 B fp16, 4 B E4M3, 2 B E8M0), the segment pairing of
// ldg_tile_mma's WIDE layout.
// PRE < SPW (FP4-G16, 128-bit layout): only the first PRE segments of each
// warp are loaded before the dependency wait, the rest right after it, so
// that when the resident wave's CTAs are released together their remaining
// loads keep HBM busy while they decode what arrived (on B200 at PRE = 4 of
// 8: in_proj 9.83 vs 10.01 us per launch, out_proj 4.97 vs 5.26; at in_proj's
// configuration the 103 registers this takes leave 4 CTAs per SM instead of
// 5, part of the effect).
template <int FMT, int NT, int SPW, int WPC = kLdgWarps, int MINB = 2, bool WIDE = false, bool XW = false,
          int PRE = SPW>
__global__ void __launch_bounds__(WPC * 32, MINB)
    gemv_fp4_ldg_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                        const uint16_t* __restrict__ x, uint16_t* __restrict__ y, int n, int k, int m, float g) {
  static_assert(!WIDE || SPW % 2 == 0, "WIDE pairs segments");
  __shared__ float red[WPC][16][16];  // [warp][token][row]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 2, tig = lane & 3;
  const int n0 = blockIdx.x * 16;
  const int ra = n0 + grp, rb = ra + 8;
  const bool va = ra < n, vb = rb < n;
  const int seg0 = warp * SPW;
  const int64_t crow = k >> 1, srow = k >> 4;

  pdl_launch_dependents();
  uint4 qa[SPW], qb[SPW];
  uint32_t sa[SPW], sb[SPW];
  if (WIDE) {
#pragma unroll
    for (int p = 0; p < SPW / 2; p++) {
      const int64_t w2 = (seg0 >> 1) + p;  // 256-k span
      const int64_t cb = w2 * 128 + tig * 32;
      const uint4 z = make_uint4(0, 0, 0, 0);
      qa[2 * p] = z; qa[2 * p + 1] = z; qb[2 * p] = z; qb[2 * p + 1] = z;
      if (va) ldg_stream256(codes + ra * crow + cb, qa[2 * p], qa[2 * p + 1]);
      if (vb) ldg_stream256(codes + rb * crow + cb, qb[2 * p], qb[2 * p + 1]);
      if (FMT == 2) {  // four fp16 group scales: groups 16*w2 + 4*tig .. +3
        const uint2 s0 = va ? ldg_stream64(scales + (ra * srow + w2 * 16 + tig * 4) * 2) : make_uint2(0, 0);
        const uint2 s1 = vb ? ldg_stream64(scales + (rb * srow + w2 * 16 + tig * 4) * 2) : make_uint2(0, 0);
        sa[2 * p] = s0.x; sa[2 * p + 1] = s0.y; sb[2 * p] = s1.x; sb[2 * p + 1] = s1.y;
      } else if (FMT == 4) {  // two E8M0 bytes: MX groups 8*w2 + 2*tig, +1 (127 = 1 for rows past n)
        const uint32_t s0 = va ? ldg_stream16(scales + ra * (srow >> 1) + w2 * 8 + tig * 2) : 0x7F7Fu;
        const uint32_t s1 = vb ? ldg_stream16(scales + rb * (srow >> 1) + w2 * 8 + tig * 2) : 0x7F7Fu;
        sa[2 * p] = e8m0_f16_factor_pair(s0 & 0xFFu); sa[2 * p + 1] = e8m0_f16_factor_pair(s0 >> 8);
        sb[2 * p] = e8m0_f16_factor_pair(s1 & 0xFFu); sb[2 * p + 1] = e8m0_f16_factor_pair(s1 >> 8);
      } else {  // four E4M3 group scales
        const uint32_t s0 = va ? ldg_stream32(scales + ra * srow + w2 * 16 + tig * 4) : 0u;
        const uint32_t s1 = vb ? ldg_stream32(scales + rb * srow + w2 * 16 + tig * 4) : 0u;
        sa[2 * p] = e4m3x2_to_f16x2(s0 & 0xFFFFu); sa[2 * p + 1] = e4m3x2_to_f16x2(s0 >> 16);
        sb[2 * p] = e4m3x2_to_f16x2(s1 & 0xFFFFu); sb[2 * p + 1] = e4m3x2_to_f16x2(s1 >> 16);
      }
    }
  } else if constexpr (PRE < SPW && !WIDE && (FMT == 2 || FMT == 3)) {
    ldg_tile_load_part<FMT, SPW, 0, PRE, false>(qa, qb, sa, sb, codes, scales, ra, rb, va, vb, seg0, tig, crow, srow);
    pdl_wait();  // x may be the previous kernel's output; y may still be read by it
    ldg_tile_load_part<FMT, SPW, PRE, SPW, true>(qa, qb, sa, sb, codes, scales, ra, rb, va, vb, seg0, tig, crow, srow);
  } else {
    ldg_tile_load<FMT, SPW>(qa, qb, sa, sb, codes, scales, ra, rb, va, vb, seg0, tig, crow, srow);
  }
  if (PRE >= SPW || WIDE || !(FMT == 2 || FMT == 3)) pdl_wait();  // x may be the previous kernel's output
  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; j++)
#pragma unroll
    for (int c = 0; c < 4; c++) acc[j][c] = 0.f;
  if constexpr (FMT == 4) {
    // the common case, every scale of the warp's segments an fp16 value
    // (factor f1 = 1, low half 0x3C00), takes one multiply per pair; one
    // vote per warp and tile, so the branch never diverges
    bool one = true;
#pragma unroll
    for (int i = 0; i < SPW; i++) one = one && (sa[i] & 0xFFFFu) == 0x3C00u && (sb[i] & 0xFFFFu) == 0x3C00u;
    if (__all_sync(0xFFFFFFFFu, one))
      ldg_tile_mma<FMT, NT, SPW, WIDE, XW, true>(acc, qa, qb, sa, sb, seg0, grp, tig, x, k, m);
    else
      ldg_tile_mma<FMT, NT, SPW, WIDE, XW, false>(acc, qa, qb, sa, sb, seg0, grp, tig, x, k, m);
  } else {
    ldg_tile_mma<FMT, NT, SPW, WIDE, XW>(acc, qa, qb, sa, sb, seg0, grp, tig, x, k, m);
  }
  ldg_tile_store<FMT, NT, WPC>(red, acc, warp, grp, tig, n0, n, m, g, y);
}

// ---------------------------------------------------------------------------
// Split-K for narrow matrices.  When n has too few 16-row tiles to fill the
// GPU (out_proj: 256 tiles of k = 8192 on 148 SMs), the CS CTAs of a
// thread-block cluster (launch attribute, CS = 2..8) share one tile: CTA c
// of the cluster multiplies k range c of CS equal ranges (its WPC warps
// split it as in gemv_fp4_ldg, the same loads and MMAs), the CTA's warps are
// summed in warp order into `part`, and after a cluster barrier the CTAs
// read each other's `part` through distributed shared memory: CTA c adds, in
// rank order 0..CS-1, the outputs whose index is c mod CS and stores them.
// A second cluster barrier keeps every CTA's `part` alive until all reads
// are done.  The order of every sum is fixed, so results are deterministic.
// Programmatic dependent launch as in gemv_fp4_ldg (weights before the wait).
// ---------------------------------------------------------------------------
template <int FMT, int NT, int SPW, int WPC, int MINB, bool XW>
__global__ void __launch_bounds__(WPC * 32, MINB)
    gemv_fp4_splitk_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                           const uint16_t* __restrict__ x, uint16_t* __restrict__ y, int n, int k, int m, float g) {
  __shared__ float red[WPC][16][16];  // [warp][token][row]
  __shared__ float part[16][16];      // [token][row]: this CTA's k range, warps summed
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 2, tig = lane & 3;
  const int cs = (int)cluster_nctarank(), c = (int)cluster_ctarank();
  const int n0 = (blockIdx.x / cs) * 16;
  const int ra = n0 + grp, rb = ra + 8;
  const bool va = ra < n, vb = rb < n;
  const int seg0 = (c * WPC + warp) * SPW;
  const int64_t crow = k >> 1, srow = k >> 4;

  pdl_launch_dependents();
  uint4 qa[SPW], qb[SPW];
  uint32_t sa[SPW], sb[SPW];
  ldg_tile_load<FMT, SPW>(qa, qb, sa, sb, codes, scales, ra, rb, va, vb, seg0, tig, crow, srow);
  pdl_wait();  // x may be the previous kernel's output; y may still be read by it

  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; j++)
#pragma unroll
    for (int q = 0; q < 4; q++) acc[j][q] = 0.f;
  ldg_tile_mma<FMT, NT, SPW, false, XW>(acc, qa, qb, sa, sb, seg0, grp, tig, x, k, m);
#pragma unroll
  for (int j = 0; j < NT; j++) {
    const int t0 = 8 * j + 2 * tig;
    red[warp][t0][grp] = acc[j][0];
    red[warp][t0 + 1][grp] = acc[j][1];
    red[warp][t0][grp + 8] = acc[j][2];
    red[warp][t0 + 1][grp + 8] = acc[j][3];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < 16 * m; idx += WPC * 32) {
    const int row = idx & 15, tok = idx >> 4;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < WPC; w++) v += red[w][tok][row];
    part[tok][row] = v;
  }
  cluster_sync();
  const float gs = (FMT == 3) ? g : 1.0f;
  for (int idx = c + cs * (int)threadIdx.x; idx < 16 * m; idx += cs * WPC * 32) {
    const int row = idx & 15, tok = idx >> 4;
    float v = 0.f;
    for (int r = 0; r < cs; r++) v += ld_dsmem_f32(&part[tok][row], (uint32_t)r);
    if (n0 + row < n) y[(int64_t)tok * n + n0 + row] = f32_to_f16_bits(v * gs);
  }
  cluster_sync();
}

}  // namespace qmm
