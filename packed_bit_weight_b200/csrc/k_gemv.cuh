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
// Streaming FP4-G16 kernel: TMA ring, warp-specialised, persistent.
//
// Work unit = a tile of RT = 16*MT consecutive weight rows over the whole k.
// Its k range is cut into 256-wide chunks; chunk c goes to consumer warp
// c % 8, so the eight warps split k and every warp has its own ring of DEPTH
// stages.  A stage holds the chunk's codes (RT rows x 128 B, loaded by a
// 2-D tensor map with the 128-byte swizzle so that the eight rows a warp
// reads at once fall in different banks) and its scales (RT x 16).  One
// producer thread issues the loads; each consumer warp waits on its stage's
// "full" barrier, decodes 16 code bytes per row and lane into MMA fragments,
// and releases the stage.  At the end of a tile the eight partial sums meet
// in shared memory and are added in a fixed order (deterministic).
// Activations are read straight from global memory (64 contiguous bytes per
// lane per segment; they stay in L1/L2).
// ---------------------------------------------------------------------------
constexpr int kGemvConsumers = 8;
constexpr int kGemvThreads = (kGemvConsumers + 1) * 32;
constexpr int kChunkK = 256;

template <int FMT, int MT>
struct GemvTmaCfg {
  static constexpr int RT = 16 * MT;
  static constexpr int kCodeBytes = RT * 128;                       // one swizzled row of 128 B per weight row
  static constexpr int kScaleBytes = RT * 16 * (FMT == 2 ? 2 : 1);  // 16 scales per row per chunk
  static constexpr int kRedBytes = kGemvConsumers * 16 * RT * 4;    // [warp][token][row] fp32
  static size_t smem_bytes(int depth) {
    return 1024 /*alignment slack*/ + (size_t)kGemvConsumers * depth * (kCodeBytes + kScaleBytes) + kRedBytes +
           (size_t)2 * kGemvConsumers * depth * 8 /*barriers*/;
  }
};

template <int FMT, int MT, int NT>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_fp4_tma_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_scales,
                        const uint16_t* __restrict__ x, uint16_t* __restrict__ y, int n, int k, int m, float g,
                        int num_tiles, int depth) {
  using C = GemvTmaCfg<FMT, MT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  const uint32_t codes_s = base;
  const uint32_t scales_s = codes_s + kGemvConsumers * depth * C::kCodeBytes;
  const uint32_t red_s = scales_s + kGemvConsumers * depth * C::kScaleBytes;
  const uint32_t bars = red_s + C::kRedBytes;  // full[w][d] then empty[w][d]
  float* red = reinterpret_cast<float*>(smem_raw + (red_s - smem_addr(smem_raw)));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = k / kChunkK;
  __shared__ volatile int s_abort;  // set by a consumer warp whose wait ran out

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < kGemvConsumers * depth; i++) {
      mbar_init(bars + 8 * i, 1);                                   // full: producer arrive + tx
      mbar_init(bars + 8 * (kGemvConsumers * depth + i), 1);        // empty: one lane per consumer warp
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kGemvConsumers) {
    // ----------------------------- producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tm_codes);
      prefetch_tmap(&tm_scales);
      int issued[kGemvConsumers];
      for (int w = 0; w < kGemvConsumers; w++) issued[w] = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int c = 0; c < nchunks; c++) {
          const int w = c % kGemvConsumers;
          const int s = issued[w] % depth;
          const uint32_t ph = (uint32_t)(issued[w] / depth) & 1u;
          const uint32_t full = bars + 8 * (w * depth + s);
          const uint32_t empty = bars + 8 * (kGemvConsumers * depth + w * depth + s);
          if (!mbar_wait(empty, ph ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(full, C::kCodeBytes + C::kScaleBytes);
          tma_load_2d(codes_s + (w * depth + s) * C::kCodeBytes, &tm_codes, c * 128, tile * C::RT, full);
          tma_load_2d(scales_s + (w * depth + s) * C::kScaleBytes, &tm_scales, c * 16, tile * C::RT, full);
          issued[w]++;
        }
      }
      // Drain: every armed stage must have landed before the CTA may exit.
      for (int w = 0; w < kGemvConsumers; w++) {
        for (int s = 0; s < depth && s < issued[w]; s++) {
          const int last = issued[w] - 1 - ((issued[w] - 1 - s) % depth);  // last use of slot s
          mbar_wait(bars + 8 * (w * depth + s), (uint32_t)(last / depth) & 1u);
        }
      }
    }
    return;
  }

  // ------------------------------- consumers -------------------------------
  const int grp = lane >> 2, tig = lane & 3;
  const int w = warp;
  int used = 0;
  bool ok = true;
  for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
    float acc[MT][NT][4];
#pragma unroll
    for (int a = 0; a < MT; a++)
#pragma unroll
      for (int b = 0; b < NT; b++)
#pragma unroll
        for (int c = 0; c < 4; c++) acc[a][b][c] = 0.f;

    for (int c = w; c < nchunks && ok; c += kGemvConsumers) {
      const int s = used % depth;
      const uint32_t ph = (uint32_t)(used / depth) & 1u;
      const uint32_t full = bars + 8 * (w * depth + s);
      const uint32_t empty = bars + 8 * (kGemvConsumers * depth + w * depth + s);
      const uint32_t cs = codes_s + (w * depth + s) * C::kCodeBytes;
      const uint32_t ss = scales_s + (w * depth + s) * C::kScaleBytes;
#pragma unroll
      for (int sub = 0; sub < 2; sub++) {
        // activations of this lane's segment: k = c*256 + sub*128 + tig*32 .. +31
        const int kseg = c * kChunkK + sub * 128 + tig * 32;
        uint32_t xb[NT][16];
#pragma unroll
        for (int j = 0; j < NT; j++) {
          const int tok = grp + 8 * j;
          if (tok < m) {
            const uint16_t* xp = x + (size_t)tok * k + kseg;
#pragma unroll
            for (int q = 0; q < 4; q++) {
              const uint4 v = ldg_nc128(xp + 8 * q);
              xb[j][4 * q] = v.x; xb[j][4 * q + 1] = v.y; xb[j][4 * q + 2] = v.z; xb[j][4 * q + 3] = v.w;
            }
          } else {
#pragma unroll
            for (int q = 0; q < 16; q++) xb[j][q] = 0u;
          }
        }
        if (sub == 0) {
          if (!mbar_wait(full, ph)) {
            ok = false;
            s_abort = 1;
            break;
          }
        }
        const int chunk = sub * 4 + tig;          // 16-byte unit within the 128-byte row
        const int phys = (chunk ^ grp) * 16;      // 128-byte swizzle: row % 8 == grp
#pragma unroll
        for (int mt = 0; mt < MT; mt++) {
          const int ra = mt * 16 + grp, rb = ra + 8;
          const uint4 qa = lds128(cs + ra * 128 + phys);
          const uint4 qb = lds128(cs + rb * 128 + phys);
          uint32_t sa0, sa1, sb0, sb1;  // f16x2 broadcast scales for bytes 0-7 / 8-15
          if (FMT == 2) {
            const uint32_t va = lds32(ss + ra * 32 + (sub * 8 + tig * 2) * 2);
            const uint32_t vb = lds32(ss + rb * 32 + (sub * 8 + tig * 2) * 2);
            sa0 = bcast_lo(va); sa1 = bcast_hi(va); sb0 = bcast_lo(vb); sb1 = bcast_hi(vb);
          } else {
            const uint32_t ea = e4m3x2_to_f16x2(lds16(ss + ra * 16 + sub * 8 + tig * 2));
            const uint32_t eb = e4m3x2_to_f16x2(lds16(ss + rb * 16 + sub * 8 + tig * 2));
            sa0 = bcast_lo(ea); sa1 = bcast_hi(ea); sb0 = bcast_lo(eb); sb1 = bcast_hi(eb);
          }
          uint32_t wa[16], wb[16];
          e2m1x8_to_f16x2(qa.x, *reinterpret_cast<uint32_t(*)[4]>(&wa[0]));
          e2m1x8_to_f16x2(qa.y, *reinterpret_cast<uint32_t(*)[4]>(&wa[4]));
          e2m1x8_to_f16x2(qa.z, *reinterpret_cast<uint32_t(*)[4]>(&wa[8]));
          e2m1x8_to_f16x2(qa.w, *reinterpret_cast<uint32_t(*)[4]>(&wa[12]));
          e2m1x8_to_f16x2(qb.x, *reinterpret_cast<uint32_t(*)[4]>(&wb[0]));
          e2m1x8_to_f16x2(qb.y, *reinterpret_cast<uint32_t(*)[4]>(&wb[4]));
          e2m1x8_to_f16x2(qb.z, *reinterpret_cast<uint32_t(*)[4]>(&wb[8]));
          e2m1x8_to_f16x2(qb.w, *reinterpret_cast<uint32_t(*)[4]>(&wb[12]));
#pragma unroll
          for (int i = 0; i < 8; i++) {
            const uint32_t sA = (i < 4) ? sa0 : sa1, sB = (i < 4) ? sb0 : sb1;
            const uint32_t a0 = hmul2(wa[2 * i], sA), a2 = hmul2(wa[2 * i + 1], sA);
            const uint32_t a1 = hmul2(wb[2 * i], sB), a3 = hmul2(wb[2 * i + 1], sB);
#pragma unroll
            for (int j = 0; j < NT; j++) mma_16816(acc[mt][j], a0, a1, a2, a3, xb[j][2 * i], xb[j][2 * i + 1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty);
      used++;
    }

    // -------- cross-warp reduction of the tile (fixed order, deterministic)
#pragma unroll
    for (int mt = 0; mt < MT; mt++)
#pragma unroll
      for (int j = 0; j < NT; j++) {
        const int t0 = 8 * j + 2 * tig;
        const int ra = mt * 16 + grp, rb = ra + 8;
        float* r = red + (size_t)w * 16 * C::RT;
        r[t0 * C::RT + ra] = acc[mt][j][0];
        r[(t0 + 1) * C::RT + ra] = acc[mt][j][1];
        r[t0 * C::RT + rb] = acc[mt][j][2];
        r[(t0 + 1) * C::RT + rb] = acc[mt][j][3];
      }
    named_bar_sync(1, kGemvConsumers * 32);
    // Every consumer warp reads the abort flag after the same barrier, so all
    // of them leave the tile loop together (bar.sync has no time limit).
    const bool stop = s_abort != 0;
    const int n0 = tile * C::RT;
    const float gs = (FMT == 3) ? g : 1.0f;
    for (int idx = threadIdx.x; idx < C::RT * m; idx += kGemvConsumers * 32) {
      const int row = idx % C::RT, tok = idx / C::RT;
      float v = 0.f;
#pragma unroll
      for (int ww = 0; ww < kGemvConsumers; ww++) v += red[(size_t)ww * 16 * C::RT + tok * C::RT + row];
      if (n0 + row < n) y[(size_t)tok * n + n0 + row] = f32_to_f16_bits(v * gs);
    }
    named_bar_sync(1, kGemvConsumers * 32);
    if (stop) break;
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
template <int FMT, int NT, int SPW, bool WIDE = false, bool XW = false>
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
      if (FMT == 4) {  // the lane's one group: code * f1 exact, * f2 rounds once
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

// WIDE (k % 256 == 0, SPW even, codes 32-byte aligned): each lane loads its
// bytes of two segments with one 256-bit load per row, and their scales with
// one load (8 B fp16, 4 B E4M3, 2 B E8M0), the segment pairing of
// ldg_tile_mma's WIDE layout.
template <int FMT, int NT, int SPW, int WPC = kLdgWarps, int MINB = 2, bool WIDE = false, bool XW = false>
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
  } else {
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
  pdl_wait();  // x may be the previous kernel's output; y may still be read by it

  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; j++)
#pragma unroll
    for (int c = 0; c < 4; c++) acc[j][c] = 0.f;
  ldg_tile_mma<FMT, NT, SPW, WIDE, XW>(acc, qa, qb, sa, sb, seg0, grp, tig, x, k, m);
  ldg_tile_store<FMT, NT, WPC>(red, acc, warp, grp, tig, n0, n, m, g, y);
}

// ---------------------------------------------------------------------------
// Two tiles per CTA, all bytes in flight at once.  The CTA of block b loads
// tile 2b into registers exactly as gemv_fp4_ldg does, and thread 0 copies
// tile 2b+1 (its 16 code rows and 16 scale rows are two contiguous ranges)
// into shared memory with two bulk copies.  With half as many CTAs the whole
// matrix fits in one wave of resident CTAs (registers plus shared memory hold
// a tile each), so no second wave waits for the first wave's arithmetic.
// Tile 2b+1 is then read from shared memory in the same lane layout.
// ---------------------------------------------------------------------------
template <int FMT>
__host__ __device__ inline uint32_t dual_smem_bytes(int k) {
  return 16u * ((uint32_t)k / 2u + ((FMT == 2) ? (uint32_t)k / 8u : (uint32_t)k / 16u)) + 16u;
}

template <int FMT, int NT, int SPW, int WPC, int MINB>
__global__ void __launch_bounds__(WPC * 32, MINB)
    gemv_fp4_dual_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                         const uint16_t* __restrict__ x, uint16_t* __restrict__ y, int n, int k, int m, float g) {
  extern __shared__ __align__(128) uint8_t smem_dual[];
  __shared__ float red[WPC][16][16];  // [warp][token][row]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 2, tig = lane & 3;
  const int seg0 = warp * SPW;
  const int64_t crow = k >> 1, srow = k >> 4;
  const uint32_t sbytes = (FMT == 2) ? (uint32_t)k / 8u : (uint32_t)k / 16u;  // scale bytes per row
  const int n0 = blockIdx.x * 32, n1 = n0 + 16;
  const uint32_t sbase = smem_addr(smem_dual);
  const uint32_t bar = sbase + 16u * ((uint32_t)crow + sbytes);

  pdl_launch_dependents();
  uint4 qa[SPW], qb[SPW];
  uint32_t sa[SPW], sb[SPW];
  {
    const int ra = n0 + grp, rb = ra + 8;
    const bool va = ra < n, vb = rb < n;
#pragma unroll
    for (int i = 0; i < SPW; i++) {
      const int seg = seg0 + i;
      const int64_t cb = (int64_t)seg * 64 + tig * 16;
      const int64_t gi = (int64_t)seg * 8 + tig * 2;
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
  const int rows1 = min(16, n - n1);  // rows of the second tile (<= 0: none)
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    if (rows1 > 0) {
      mbar_arrive_expect_tx(bar, (uint32_t)rows1 * ((uint32_t)crow + sbytes));
      bulk_load(sbase, codes + (int64_t)n1 * crow, (uint32_t)rows1 * (uint32_t)crow, bar);
      bulk_load(sbase + 16u * (uint32_t)crow, scales + (int64_t)n1 * sbytes, (uint32_t)rows1 * sbytes, bar);
    }
  }
  __syncthreads();  // the barrier is initialised before anyone waits on it
  pdl_wait();       // x may be the previous kernel's output; y may still be read by it

  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; j++)
#pragma unroll
    for (int c = 0; c < 4; c++) acc[j][c] = 0.f;
  ldg_tile_mma<FMT, NT, SPW>(acc, qa, qb, sa, sb, seg0, grp, tig, x, k, m);
  ldg_tile_store<FMT, NT, WPC>(red, acc, warp, grp, tig, n0, n, m, g, y);
  if (rows1 <= 0) return;

  // second tile: every lane waits for the copies (bounded); the decision is
  // made warp-uniform so the MMAs never run in a diverged warp
  const bool ready = __all_sync(0xFFFFFFFFu, mbar_wait(bar, 0));
  if (ready) {
    const uint8_t* cs = smem_dual + grp * crow + tig * 16;
    const uint8_t* ss = smem_dual + 16 * crow + grp * sbytes;
#pragma unroll
    for (int i = 0; i < SPW; i++) {
      const int seg = seg0 + i;
      qa[i] = *reinterpret_cast<const uint4*>(cs + seg * 64);
      qb[i] = *reinterpret_cast<const uint4*>(cs + 8 * crow + seg * 64);
      if (FMT == 2) {
        sa[i] = *reinterpret_cast<const uint32_t*>(ss + seg * 16 + tig * 4);
        sb[i] = *reinterpret_cast<const uint32_t*>(ss + 8u * sbytes + seg * 16 + tig * 4);
      } else {
        sa[i] = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(ss + seg * 8 + tig * 2));
        sb[i] = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(ss + 8u * sbytes + seg * 8 + tig * 2));
      }
    }
#pragma unroll
    for (int j = 0; j < NT; j++)
#pragma unroll
      for (int c = 0; c < 4; c++) acc[j][c] = 0.f;
    ldg_tile_mma<FMT, NT, SPW>(acc, qa, qb, sa, sb, seg0, grp, tig, x, k, m);
  }
  // the first tile's sums have been read from `red`; the store below holds
  // barriers, so it runs in every thread or in none
  if (__syncthreads_and(ready)) ldg_tile_store<FMT, NT, WPC>(red, acc, warp, grp, tig, n1, n, m, g, y);
}

// ---------------------------------------------------------------------------
// Streaming FP4-G16 kernel with per-warp cp.async rings (persistent).
//
// Work unit = a tile of 16 weight rows over the whole k; its k range is split
// into WPC equal ranges, one per warp, of SPW segments (128 k each).  Each
// CTA loops over tiles; each warp walks the same k range of successive tiles,
// a linear stream of segments, and keeps DEPTH segments in flight with
// cp.async: per segment a lane copies its own 16 code bytes of rows grp and
// grp+8 and their 4-byte scale words into a lane-private slot of the warp's
// ring.  Only the issuing lane reads what it copied, so the ring needs no
// barrier (cp.async.wait_group is per thread) and its layout is lane-major,
// conflict-free.  Loads in flight hold no registers, so two CTAs of WPC
// warps per SM keep ~2*WPC*DEPTH*1.3 KB streaming while the warps decode.
// At the end of a tile the WPC partial sums meet in shared memory (fixed
// order) and the tile's rows are stored.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One ring slot (one segment of one warp), lane-major per field so every
// cp.async destination is aligned to its size: codes of row a [32 lanes][16 B]
// at 0, codes of row b at 512, scale words of row a [32][4 B] at 1024, of
// row b at 1152.
constexpr int kCpaSlotBytes = 1280;
constexpr int kCpaCodesB = 512, kCpaScalesA = 1024, kCpaScalesB = 1152;

// Walks one warp's linear stream of (tile, segment) elements with pointers
// that advance by constant strides; rows past n are clamped once per tile.
template <int FMT>
struct CpaCursor {
  const uint8_t* ca;  // codes, row a, this lane's 16 bytes
  const uint8_t* cb;
  const uint8_t* sa;  // this lane's scale word, row a
  const uint8_t* sb;
  int seg;            // segment within the tile's warp range
  int tile;

  __device__ __forceinline__ void at_tile(const uint8_t* codes, const uint8_t* scales, int t, int n, int64_t crow,
                                          int64_t srow, int seg_lo, int grp, int tig) {
    tile = t;
    seg = 0;
    const int64_t ra = min((int64_t)t * 16 + grp, (int64_t)n - 1);
    const int64_t rb = min((int64_t)t * 16 + grp + 8, (int64_t)n - 1);
    ca = codes + ra * crow + seg_lo * 64 + tig * 16;
    cb = codes + rb * crow + seg_lo * 64 + tig * 16;
    if (FMT == 2) {
      sa = scales + (ra * srow + seg_lo * 8 + tig * 2) * 2;
      sb = scales + (rb * srow + seg_lo * 8 + tig * 2) * 2;
    } else {  // the aligned word holding this lane's two E4M3 bytes
      sa = scales + ra * srow + seg_lo * 8 + (tig & 2) * 2;
      sb = scales + rb * srow + seg_lo * 8 + (tig & 2) * 2;
    }
  }
  __device__ __forceinline__ void next(const uint8_t* codes, const uint8_t* scales, int spw, int G, int n,
                                       int64_t crow, int64_t srow, int seg_lo, int grp, int tig) {
    if (++seg == spw) {
      at_tile(codes, scales, tile + G, n, crow, srow, seg_lo, grp, tig);
    } else {
      ca += 64;
      cb += 64;
      sa += (FMT == 2) ? 16 : 8;
      sb += (FMT == 2) ? 16 : 8;
    }
  }
};

template <int FMT, int NT, int WPC, int DEPTH, int MINB = 2>
__global__ void __launch_bounds__(WPC * 32, MINB)
    gemv_fp4_cpa_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                        const uint16_t* __restrict__ x, uint16_t* __restrict__ y, int n, int k, int m, float g,
                        int num_tiles) {
  static_assert((DEPTH & (DEPTH - 1)) == 0, "ring depth must be a power of two");
  extern __shared__ __align__(16) uint8_t smem_cpa[];
  float* red = reinterpret_cast<float*>(smem_cpa);  // [WPC][16 tokens][16 rows]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 2, tig = lane & 3;
  const uint32_t ring = smem_addr(smem_cpa) + WPC * 16 * 16 * 4 + warp * DEPTH * kCpaSlotBytes;
  const int spw = (k >> 7) / WPC;  // segments per warp and tile
  const int seg_lo = warp * spw;
  const int G = (int)gridDim.x;
  const int64_t crow = k >> 1, srow = k >> 4;
  const int my_tiles = (num_tiles - (int)blockIdx.x + G - 1) / G;
  const int total = my_tiles * spw;  // this warp's element stream

  CpaCursor<FMT> in;  // next element to copy
  in.at_tile(codes, scales, (int)blockIdx.x, n, crow, srow, seg_lo, grp, tig);
  int issued = 0;
  auto issue_one = [&]() {
    if (issued < total) {
      const uint32_t slot = ring + (uint32_t)(issued & (DEPTH - 1)) * kCpaSlotBytes;
      cp_async16(slot + lane * 16, in.ca);
      cp_async16(slot + kCpaCodesB + lane * 16, in.cb);
      cp_async4(slot + kCpaScalesA + lane * 4, in.sa);
      cp_async4(slot + kCpaScalesB + lane * 4, in.sb);
      in.next(codes, scales, spw, G, n, crow, srow, seg_lo, grp, tig);
    }
    issued++;
    cp_async_commit();  // one group per element (empty past the end)
  };
#pragma unroll 1
  for (int j = 0; j < DEPTH - 1; j++) issue_one();

  float acc[NT][4];
  const float gs = (FMT == 3) ? g : 1.0f;
  int tile = (int)blockIdx.x, seg = 0;
  const uint16_t* xrow[NT];
#pragma unroll
  for (int t = 0; t < NT; t++) xrow[t] = (grp + 8 * t < m) ? x + (int64_t)(grp + 8 * t) * k + seg_lo * 128 + tig * 32 : nullptr;
#pragma unroll 1
  for (int j = 0; j < total; j++) {
    if (seg == 0) {
#pragma unroll
      for (int a = 0; a < NT; a++)
#pragma unroll
        for (int c = 0; c < 4; c++) acc[a][c] = 0.f;
    }
    issue_one();
    uint32_t xb[NT][16];
#pragma unroll
    for (int t = 0; t < NT; t++) {
      if (xrow[t]) {
        const uint16_t* xp = xrow[t] + seg * 128;
#pragma unroll
        for (int q = 0; q < 4; q++) {
          const uint4 v = ldg_x128(xp + 8 * q);
          xb[t][4 * q] = v.x; xb[t][4 * q + 1] = v.y; xb[t][4 * q + 2] = v.z; xb[t][4 * q + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < 16; q++) xb[t][q] = 0u;
      }
    }
    cp_async_wait<DEPTH - 1>();  // element j has landed (this lane's copies)
    const uint32_t slot = ring + (uint32_t)(j & (DEPTH - 1)) * kCpaSlotBytes;
    const uint4 qa = lds128(slot + lane * 16), qb = lds128(slot + kCpaCodesB + lane * 16);
    uint32_t sa = lds32(slot + kCpaScalesA + lane * 4), sb = lds32(slot + kCpaScalesB + lane * 4);
    if (FMT == 3) {
      sa = e4m3x2_to_f16x2((tig & 1) ? (sa >> 16) : sa);
      sb = e4m3x2_to_f16x2((tig & 1) ? (sb >> 16) : sb);
    }
    const uint32_t sa0 = bcast_lo(sa), sa1 = bcast_hi(sa), sb0 = bcast_lo(sb), sb1 = bcast_hi(sb);
    uint32_t wa[16], wb[16];
    e2m1x8_to_f16x2(qa.x, *reinterpret_cast<uint32_t(*)[4]>(&wa[0]));
    e2m1x8_to_f16x2(qa.y, *reinterpret_cast<uint32_t(*)[4]>(&wa[4]));
    e2m1x8_to_f16x2(qa.z, *reinterpret_cast<uint32_t(*)[4]>(&wa[8]));
    e2m1x8_to_f16x2(qa.w, *reinterpret_cast<uint32_t(*)[4]>(&wa[12]));
    e2m1x8_to_f16x2(qb.x, *reinterpret_cast<uint32_t(*)[4]>(&wb[0]));
    e2m1x8_to_f16x2(qb.y, *reinterpret_cast<uint32_t(*)[4]>(&wb[4]));
    e2m1x8_to_f16x2(qb.z, *reinterpret_cast<uint32_t(*)[4]>(&wb[8]));
    e2m1x8_to_f16x2(qb.w, *reinterpret_cast<uint32_t(*)[4]>(&wb[12]));
#pragma unroll
    for (int st = 0; st < 8; st++) {
      const uint32_t sA = (st < 4) ? sa0 : sa1, sB = (st < 4) ? sb0 : sb1;
      const uint32_t a0 = hmul2(wa[2 * st], sA), a2 = hmul2(wa[2 * st + 1], sA);
      const uint32_t a1 = hmul2(wb[2 * st], sB), a3 = hmul2(wb[2 * st + 1], sB);
#pragma unroll
      for (int t = 0; t < NT; t++) mma_16816(acc[t], a0, a1, a2, a3, xb[t][2 * st], xb[t][2 * st + 1]);
    }
    if (++seg == spw) {  // tile done: meet the other warps
      seg = 0;
      float* r = red + warp * 256;
#pragma unroll
      for (int t = 0; t < NT; t++) {
        const int t0 = 8 * t + 2 * tig;
        r[t0 * 16 + grp] = acc[t][0];
        r[(t0 + 1) * 16 + grp] = acc[t][1];
        r[t0 * 16 + grp + 8] = acc[t][2];
        r[(t0 + 1) * 16 + grp + 8] = acc[t][3];
      }
      __syncthreads();
      const int n0 = tile * 16;
      for (int idx = threadIdx.x; idx < 16 * m; idx += WPC * 32) {
        const int row = idx & 15, tok = idx >> 4;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < WPC; w++) v += red[w * 256 + tok * 16 + row];
        if (n0 + row < n) y[(int64_t)tok * n + n0 + row] = f32_to_f16_bits(v * gs);
      }
      __syncthreads();
      tile += G;
    }
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// Persistent streaming FP4-G16 kernel with a register prefetch ring.
//
// Tiles of 16 rows; WPC warps split each tile's k into ranges of spw
// segments (128 k).  Every warp walks the linear stream of its segments over
// the CTA's tiles and keeps P of them in flight in registers: the loads of
// element j+P are issued right after element j is decoded, into the registers
// element j just freed, so each SM always has WPC*P*1.25 KB per CTA streaming
// and no CTA ever waits for a whole tile to arrive.  Addresses advance by
// constant strides (64 code bytes, 8 scales per segment) and are clamped to
// row n-1 once per tile.  With programmatic dependent launch the weight loads
// of the first P elements are issued before griddepcontrol.wait, so they
// overlap the tail of the kernel that precedes this one on the stream;
// activations are read and outputs written only after the wait.
// ---------------------------------------------------------------------------
template <int FMT>
struct SegRegs {
  uint4 qa, qb;
  uint32_t sa, sb;
};

template <int FMT>
struct StreamCursor {
  const uint8_t* ca;
  const uint8_t* cb;
  const uint8_t* sa;
  const uint8_t* sb;
  int seg, tile;
  __device__ __forceinline__ void at_tile(const uint8_t* codes, const uint8_t* scales, int t, int n, int64_t crow,
                                          int64_t srow, int seg_lo, int grp, int tig) {
    tile = t;
    seg = 0;
    const int64_t ra = min((int64_t)t * 16 + grp, (int64_t)n - 1);
    const int64_t rb = min((int64_t)t * 16 + grp + 8, (int64_t)n - 1);
    ca = codes + ra * crow + seg_lo * 64 + tig * 16;
    cb = codes + rb * crow + seg_lo * 64 + tig * 16;
    sa = scales + (ra * srow + seg_lo * 8 + tig * 2) * (FMT == 2 ? 2 : 1);
    sb = scales + (rb * srow + seg_lo * 8 + tig * 2) * (FMT == 2 ? 2 : 1);
  }
  __device__ __forceinline__ void load(SegRegs<FMT>& r) const {
    r.qa = ldg_stream128(ca);
    r.qb = ldg_stream128(cb);
    if (FMT == 2) {
      r.sa = ldg_stream32(sa);
      r.sb = ldg_stream32(sb);
    } else {
      r.sa = ldg_stream16(sa);
      r.sb = ldg_stream16(sb);
    }
  }
  __device__ __forceinline__ void next(const uint8_t* codes, const uint8_t* scales, int spw, int G, int n,
                                       int64_t crow, int64_t srow, int seg_lo, int grp, int tig) {
    if (++seg == spw) {
      at_tile(codes, scales, tile + G, n, crow, srow, seg_lo, grp, tig);
    } else {
      ca += 64;
      cb += 64;
      sa += (FMT == 2) ? 16 : 8;
      sb += (FMT == 2) ? 16 : 8;
    }
  }
};

template <int FMT, int NT>
__device__ __forceinline__ void seg_mma(float (&acc)[NT][4], const SegRegs<FMT>& r, const uint16_t* const (&xrow)[NT],
                                        int off) {
  uint32_t xb[NT][16];
#pragma unroll
  for (int t = 0; t < NT; t++) {
    if (xrow[t]) {
      const uint16_t* xp = xrow[t] + off;
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const uint4 v = ldg_x128(xp + 8 * q);
        xb[t][4 * q] = v.x; xb[t][4 * q + 1] = v.y; xb[t][4 * q + 2] = v.z; xb[t][4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 16; q++) xb[t][q] = 0u;
    }
  }
  uint32_t sa = r.sa, sb = r.sb;
  if (FMT == 3) {
    sa = e4m3x2_to_f16x2(sa);
    sb = e4m3x2_to_f16x2(sb);
  }
  const uint32_t sa0 = bcast_lo(sa), sa1 = bcast_hi(sa), sb0 = bcast_lo(sb), sb1 = bcast_hi(sb);
  uint32_t wa[16], wb[16];
  e2m1x8_to_f16x2(r.qa.x, *reinterpret_cast<uint32_t(*)[4]>(&wa[0]));
  e2m1x8_to_f16x2(r.qa.y, *reinterpret_cast<uint32_t(*)[4]>(&wa[4]));
  e2m1x8_to_f16x2(r.qa.z, *reinterpret_cast<uint32_t(*)[4]>(&wa[8]));
  e2m1x8_to_f16x2(r.qa.w, *reinterpret_cast<uint32_t(*)[4]>(&wa[12]));
  e2m1x8_to_f16x2(r.qb.x, *reinterpret_cast<uint32_t(*)[4]>(&wb[0]));
  e2m1x8_to_f16x2(r.qb.y, *reinterpret_cast<uint32_t(*)[4]>(&wb[4]));
  e2m1x8_to_f16x2(r.qb.z, *reinterpret_cast<uint32_t(*)[4]>(&wb[8]));
  e2m1x8_to_f16x2(r.qb.w, *reinterpret_cast<uint32_t(*)[4]>(&wb[12]));
#pragma unroll
  for (int st = 0; st < 8; st++) {
    const uint32_t sA = (st < 4) ? sa0 : sa1, sB = (st < 4) ? sb0 : sb1;
    const uint32_t a0 = hmul2(wa[2 * st], sA), a2 = hmul2(wa[2 * st + 1], sA);
    const uint32_t a1 = hmul2(wb[2 * st], sB), a3 = hmul2(wb[2 * st + 1], sB);
#pragma unroll
    for (int t = 0; t < NT; t++) mma_16816(acc[t], a0, a1, a2, a3, xb[t][2 * st], xb[t][2 * st + 1]);
  }
}

template <int FMT, int NT, int WPC, int P, int MINB>
__global__ void __launch_bounds__(WPC * 32, MINB)
    gemv_fp4_stream_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                           const uint16_t* __restrict__ x, uint16_t* __restrict__ y, int n, int k, int m, float g,
                           int num_tiles) {
  __shared__ float red[WPC][16][16];  // [warp][token][row]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, grp = lane >> 2, tig = lane & 3;
  const int spw = (k >> 7) / WPC;
  const int seg_lo = warp * spw;
  const int G = (int)gridDim.x;
  const int64_t crow = k >> 1, srow = k >> 4;
  const int my_tiles = (num_tiles - (int)blockIdx.x + G - 1) / G;
  const int total = my_tiles * spw;

  pdl_launch_dependents();
  StreamCursor<FMT> in;
  in.at_tile(codes, scales, (int)blockIdx.x, n, crow, srow, seg_lo, grp, tig);
  SegRegs<FMT> buf[P];
#pragma unroll
  for (int u = 0; u < P; u++) {
    if (u < total) {
      in.load(buf[u]);
      in.next(codes, scales, spw, G, n, crow, srow, seg_lo, grp, tig);
    }
  }
  pdl_wait();  // the previous kernel's outputs (our x) are visible from here on

  const uint16_t* xrow[NT];
#pragma unroll
  for (int t = 0; t < NT; t++)
    xrow[t] = (grp + 8 * t < m) ? x + (int64_t)(grp + 8 * t) * k + seg_lo * 128 + tig * 32 : nullptr;
  const float gs = (FMT == 3) ? g : 1.0f;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; t++)
#pragma unroll
    for (int c = 0; c < 4; c++) acc[t][c] = 0.f;
  int tile = (int)blockIdx.x, seg = 0;
#pragma unroll 1
  for (int j0 = 0; j0 < total; j0 += P) {
#pragma unroll
    for (int u = 0; u < P; u++) {
      const int j = j0 + u;
      if (j < total) {
        seg_mma<FMT, NT>(acc, buf[u], xrow, seg * 128);
        if (j + P < total) {
          in.load(buf[u]);
          in.next(codes, scales, spw, G, n, crow, srow, seg_lo, grp, tig);
        }
        if (++seg == spw) {  // tile done: meet the other warps, store, reset
          seg = 0;
#pragma unroll
          for (int t = 0; t < NT; t++) {
            const int t0 = 8 * t + 2 * tig;
            red[warp][t0][grp] = acc[t][0];
            red[warp][t0 + 1][grp] = acc[t][1];
            red[warp][t0][grp + 8] = acc[t][2];
            red[warp][t0 + 1][grp + 8] = acc[t][3];
#pragma unroll
            for (int c = 0; c < 4; c++) acc[t][c] = 0.f;
          }
          __syncthreads();
          const int n0 = tile * 16;
          for (int idx = threadIdx.x; idx < 16 * m; idx += WPC * 32) {
            const int row = idx & 15, tok = idx >> 4;
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < WPC; w++) v += red[w][tok][row];
            if (n0 + row < n) y[(int64_t)tok * n + n0 + row] = f32_to_f16_bits(v * gs);
          }
          __syncthreads();
          tile += G;
        }
      }
    }
  }
}

}  // namespace qmm
