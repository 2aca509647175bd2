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

}  // namespace qmm
