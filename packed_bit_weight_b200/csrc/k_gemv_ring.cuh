// k_gemv_ring.cuh -- persistent FP4-G16 decode GEMV: whole 16-row weight
// tiles streamed into a shared-memory ring by the TMA engine, chained across
// launches.
//
// Format ("Mamb2_8B_FP4_Recall_SQ3.25", section "Representation"): E2M1 codes,
// two per byte along k (low nibble first), and one scale per 16 consecutive k
// (fp16, or E4M3FN with an fp32 global scale g applied to the fp32 sum).
//
// One CTA per SM walks the 16-row tiles t = blockIdx.x, blockIdx.x + grid, ...
// Sixteen consecutive rows are one contiguous range of the code array
// (16 * k/2 bytes) and one of the scale array, so a ring stage (one tile) is
// filled by two bulk copies: the copy engine's cost is per operation, and
// per-row copies measured at less than half the bandwidth.
//
//   warp 0 (producer): lane 0 bulk-copies the tile's codes, lane 1 its scales
//     (cp.async.bulk, L2 evict-first, no multicast), both completing on the
//     stage's barrier.  It never waits on the previous kernel: the weights are
//     read-only inputs.
//   warps 1..CW (consumers): a tile has k/128 segments of 128 k; consumer warp
//     w takes segments w, w+CW, ...  For a segment, lane (grp, tig) reads 16
//     code bytes (32 k) of rows grp and grp+8 and their two group scales (all
//     of the warp's segments into registers, then the stage is released),
//     decodes with the E2M1 convert, scales with one f16x2 multiply (the
//     bit-exact decoded weights), and issues 8 legacy m16n8k16 MMAs (rows as
//     M, tokens as N) into the segment's own fp32 accumulator set (independent
//     MMA chains, added at the end of the tile).  Activations are staged once per CTA
//     in shared memory when they take at most 16 KB, else read from global
//     memory (L1-resident: at most 16 rows of k fp16).  After the tile the warps'
//     partial sums meet in shared memory (two buffers, used by alternate
//     tiles) and are added in warp order: deterministic.
//
// The launch uses programmatic dependent launch: every CTA signals its
// dependents at once, so the next GEMV on the stream becomes resident beside
// this one (each uses under half of an SM's shared memory, registers and
// threads) and fills its ring while this one drains; consumers execute
// griddepcontrol.wait before they read x or write y.  So the weights must not
// be written by the kernel that immediately precedes the call on the stream.
//
// Every mbarrier wait is bounded (%globaltimer): on a timeout the error word
// is raised, the consumers leave together through a barrier that ORs their
// failure flags, and the producer waits (bounded) for its own copies.
#pragma once
#include "qmm_dev.cuh"

namespace qmm {

constexpr int kRingMaxStages = 4;
constexpr uint32_t kRingStageBudget = 96u * 1024u;  // ring bytes per CTA: two CTAs share an SM

// Bytes of one tile stage: codes [16][k/2] then scales [16][k/8] (fp16) or
// [16][k/16] (E4M3), each part a multiple of 16 bytes for k % 256 == 0.
__host__ __device__ inline uint32_t ring_stage_bytes(int fmt, int k) {
  return 8u * (uint32_t)k + 16u * ((fmt == 2) ? (uint32_t)k / 8u : (uint32_t)k / 16u);
}

template <int CW, int NT>
__host__ __device__ constexpr uint32_t ring_red_bytes() {
  return 2u * CW * (8u * NT) * 16u * 4u;  // [tile parity][warp][token][row] fp32
}

// Activations staged in shared memory when they are this small (m <= 2 at
// k = 4096): read once per CTA instead of once per tile from L1/L2.
constexpr uint32_t kRingXsMax = 16384u;

template <int CW, int NT>
__host__ __device__ inline uint32_t ring_smem_bytes(int fmt, int k, int stages, uint32_t xs_bytes) {
  return (uint32_t)stages * ring_stage_bytes(fmt, k) + ring_red_bytes<CW, NT>() + xs_bytes + 16u * (uint32_t)stages;
}

// Bulk copy with an L2 evict-first policy: each weight byte is read once.
__device__ __forceinline__ void bulk_load_stream(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Decode and multiply one 128-k segment already in registers: code bytes qa /
// qb of rows grp and grp+8 (32 k each), their group-scale words wa / wb (two
// fp16 scales, or two E4M3 bytes in the low half), activations of tokens grp
// and grp+8 (when < m) at k = kx .. kx+31 from x (shared memory when XSM,
// else global memory).
template <int FMT, int NT, bool XSM>
__device__ __forceinline__ void ring_mma_segment(float (&acc)[NT][4], const uint4& qa, const uint4& qb, uint32_t wa_s,
                                                 uint32_t wb_s, int grp, const uint16_t* __restrict__ x, int k, int m,
                                                 int kx) {
  uint32_t sa0, sa1, sb0, sb1;
  if (FMT == 2) {
    sa0 = bcast_lo(wa_s); sa1 = bcast_hi(wa_s); sb0 = bcast_lo(wb_s); sb1 = bcast_hi(wb_s);
  } else {
    const uint32_t ea = e4m3x2_to_f16x2(wa_s), eb = e4m3x2_to_f16x2(wb_s);
    sa0 = bcast_lo(ea); sa1 = bcast_hi(ea); sb0 = bcast_lo(eb); sb1 = bcast_hi(eb);
  }
  uint32_t xb[NT][16];
#pragma unroll
  for (int j = 0; j < NT; j++) {
    const int tok = grp + 8 * j;
    if (tok < m) {
      const uint16_t* xp = x + (int64_t)tok * k + kx;
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const uint4 v = XSM ? *reinterpret_cast<const uint4*>(xp + 8 * q) : ldg_x128(xp + 8 * q);
        xb[j][4 * q] = v.x; xb[j][4 * q + 1] = v.y; xb[j][4 * q + 2] = v.z; xb[j][4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 16; q++) xb[j][q] = 0u;
    }
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
  for (int st = 0; st < 8; st++) {
    const uint32_t sA = (st < 4) ? sa0 : sa1, sB = (st < 4) ? sb0 : sb1;
    const uint32_t a0 = hmul2(wa[2 * st], sA), a2 = hmul2(wa[2 * st + 1], sA);
    const uint32_t a1 = hmul2(wb[2 * st], sB), a3 = hmul2(wb[2 * st + 1], sB);
#pragma unroll
    for (int j = 0; j < NT; j++) mma_16816(acc[j], a0, a1, a2, a3, xb[j][2 * st], xb[j][2 * st + 1]);
  }
}

// CW consumer warps, NT MMA token tiles (m <= 8 * NT), at most SPW segments
// per consumer warp per tile (k <= 128 * CW * SPW).  MINB = 2 lets the next
// launch's CTA share the SM.
template <int FMT, int NT, int CW, int SPW, bool XSM>
__global__ void __maxnreg__((65536 / (2 * 32 * (CW + 1))) & ~7)
    gemv_fp4_ring_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                         const uint16_t* __restrict__ x, uint16_t* __restrict__ y, int n, int k, int m, float g,
                         int stages) {
  extern __shared__ __align__(128) uint8_t smem_ring[];
  constexpr int TOK = 8 * NT;
  const uint32_t S = (uint32_t)stages;
  const uint32_t stage_bytes = ring_stage_bytes(FMT, k);
  const uint32_t crow = (uint32_t)k / 2u;                                // code bytes per row
  const uint32_t srow = (FMT == 2) ? (uint32_t)k / 8u : (uint32_t)k / 16u;  // scale bytes per row
  const uint32_t sbase = smem_addr(smem_ring);
  const uint32_t red_off = S * stage_bytes;
  float* red = reinterpret_cast<float*>(smem_ring + red_off);
  const uint32_t xs_off = red_off + ring_red_bytes<CW, NT>();
  const uint32_t xs_bytes = XSM ? 2u * (uint32_t)m * (uint32_t)k : 0u;
  const uint32_t full = sbase + xs_off + xs_bytes, empty = full + 8u * S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = (n + 15) / 16;

  asm volatile("griddepcontrol.launch_dependents;" :::);
  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < S; s++) {
      mbar_init(full + 8u * s, 1);
      mbar_init(empty + 8u * s, CW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane >= 2) return;
    const uint64_t pol = l2_evict_first_policy();
    uint32_t it = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const uint32_t rows = (uint32_t)min(16, n - t * 16);
      const uint32_t slot = it % S;
      bool ok = true;
      if (lane == 0) {
        if (it >= S) ok = mbar_wait(empty + 8u * slot, ((it / S) & 1u) ^ 1u);
        if (ok) mbar_arrive_expect_tx(full + 8u * slot, rows * (crow + srow));
      }
      if (!__shfl_sync(0x3u, ok, 0)) break;  // also orders lane 1 after lane 0's wait
      const uint32_t st0 = sbase + slot * stage_bytes;
      if (lane == 0)
        bulk_load_stream(st0, codes + (int64_t)t * 16 * crow, rows * crow, full + 8u * slot, pol);
      else
        bulk_load_stream(st0 + 16u * crow, scales + (int64_t)t * 16 * srow, rows * srow, full + 8u * slot, pol);
      it++;
    }
    // the last copy into every stage has landed before the CTA may exit
    if (lane == 0)
      for (uint32_t s = 0; s < S && s < it; s++) {
      const uint32_t last = s + S * ((it - 1u - s) / S);
      mbar_wait(full + 8u * s, (last / S) & 1u);
    }
    return;
  }

  // ---------------- consumers ----------------
  const int cw = warp - 1, grp = lane >> 2, tig = lane & 3;
  const int ctid = threadIdx.x - 32;
  const int segs = k >> 7;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // x may be the previous kernel's output; y its input
  const uint16_t* xr = x;
  if (XSM) {  // stage the activations once for all of this CTA's tiles
    uint4* xs = reinterpret_cast<uint4*>(smem_ring + xs_off);
    for (uint32_t i = (uint32_t)ctid; i < xs_bytes / 16u; i += CW * 32) xs[i] = ldg_x128(x + 8 * i);
    named_bar_sync(2, CW * 32);
    xr = reinterpret_cast<const uint16_t*>(smem_ring + xs_off);
  }
  const float gs = (FMT == 3) ? g : 1.0f;
  uint32_t it = 0, tpar = 0;
  bool fail = false;
  for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
    float acc[SPW][NT][4];  // one accumulator chain per segment
#pragma unroll
    for (int i = 0; i < SPW; i++)
#pragma unroll
      for (int j = 0; j < NT; j++)
#pragma unroll
        for (int c = 0; c < 4; c++) acc[i][j][c] = 0.f;
    const uint32_t slot = it % S;
    // every lane waits (each needs the copies visible); the decision is made
    // warp-uniform so the MMAs below never run in a diverged warp
    const bool ready = __all_sync(0xFFFFFFFFu, !fail && mbar_wait(full + 8u * slot, (it / S) & 1u));
    // this warp's segments s = cw + i*CW (at most SPW, k <= 128*CW*SPW) are read
    // into registers first and the stage is released before any decoding, so
    // the producer refills it while the warp computes
    uint4 qa[SPW], qb[SPW];
    uint32_t wsa[SPW], wsb[SPW];
    if (ready) {
      const uint8_t* st0 = smem_ring + slot * stage_bytes;
      const uint8_t* ca = st0 + grp * crow + tig * 16;
      const uint8_t* sa = st0 + 16u * crow + grp * srow;
#pragma unroll
      for (int i = 0; i < SPW; i++) {
        const int s = cw + i * CW;
        if (s < segs) {
          qa[i] = *reinterpret_cast<const uint4*>(ca + s * 64);
          qb[i] = *reinterpret_cast<const uint4*>(ca + 8u * crow + s * 64);
          if (FMT == 2) {
            wsa[i] = *reinterpret_cast<const uint32_t*>(sa + s * 16 + tig * 4);
            wsb[i] = *reinterpret_cast<const uint32_t*>(sa + 8u * srow + s * 16 + tig * 4);
          } else {
            wsa[i] = *reinterpret_cast<const uint16_t*>(sa + s * 8 + tig * 2);
            wsb[i] = *reinterpret_cast<const uint16_t*>(sa + 8u * srow + s * 8 + tig * 2);
          }
        }
      }
    } else {
      fail = true;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + 8u * slot);
    it++;
    if (ready) {
      const int kx0 = tig * 32;
#pragma unroll
      for (int i = 0; i < SPW; i++) {
        const int s = cw + i * CW;
        if (s < segs) {
          ring_mma_segment<FMT, NT, XSM>(acc[i], qa[i], qb[i], wsa[i], wsb[i], grp, xr, k, m, kx0 + s * 128);
        }
      }
    }
#pragma unroll
    for (int i = 1; i < SPW; i++)
#pragma unroll
      for (int j = 0; j < NT; j++)
#pragma unroll
        for (int c = 0; c < 4; c++) acc[0][j][c] += acc[i][j][c];
    float* rw = red + (tpar * CW + (uint32_t)cw) * (TOK * 16);
#pragma unroll
    for (int j = 0; j < NT; j++) {
      const int t0 = 8 * j + 2 * tig;
      if (t0 < m) {
        rw[t0 * 16 + grp] = acc[0][j][0];
        rw[t0 * 16 + grp + 8] = acc[0][j][2];
      }
      if (t0 + 1 < m) {
        rw[(t0 + 1) * 16 + grp] = acc[0][j][1];
        rw[(t0 + 1) * 16 + grp + 8] = acc[0][j][3];
      }
    }
    fail = named_bar_or(1, CW * 32, fail);
    if (fail) break;
    const float* rr = red + tpar * CW * (TOK * 16);
    for (int idx = ctid; idx < 16 * m; idx += CW * 32) {
      const int row = idx & 15, tok = idx >> 4;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < CW; w++) v += rr[(w * TOK + tok) * 16 + row];
      if (t * 16 + row < n) y[(int64_t)tok * n + t * 16 + row] = f32_to_f16_bits(v * gs);
    }
    tpar ^= 1u;
  }
}

}  // namespace qmm
