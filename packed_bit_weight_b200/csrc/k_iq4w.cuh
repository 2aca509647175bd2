// k_iq4w.cuh -- IQ4_NL routed-expert kernel in which each warp owns whole
// 16-row tiles ("Mark-Experimental-V3-8B", section "Mixture-of-Experts
// (MoE)": 32 routed experts, 4 active per token; section "Quantization":
// IQ4_NL blocks of 32 weights, one fp16 scale d and 16 bytes of 4-bit indices
// into the printed 16-entry table; expert weights one contiguous 3-D tensor
// per projection).  Also serves the plain IQ4_NL product of up to 16 rows.
//
// Work items are (expert, group of up to 16 of its routed pairs, two 16-row
// tiles: the gate and up tiles of the same rows for the SwiGLU pass, else two
// neighbouring tiles), enumerated expert-major after the routing sort
// (offsets/perm of route_kernel).  Warp w of the grid takes items w, w +
// warps, ...: the warps of one CTA work on neighbouring tiles of the same
// expert and share its activation rows through L1.  A warp multiplies its two
// tiles over the whole k, so it needs no partial-sum exchange and no barrier:
// lane (grp, tig) owns block 4s + tig of rows grp and grp+8 of both tiles at
// super-step s (128 k), decodes each index byte through a 256-entry table of
// exact f16x2 pairs (w_j, w_{j+16}) replicated across the 32 banks,
// multiplies by the block scale (one f16x2 multiply: the bit-exact decoded
// weight) and feeds legacy m16n8k16 MMAs with the token rows, whose fragments
// the two tiles share.  The weight words of super-step s+1 are loaded before
// super-step s is decoded, so each warp keeps one step (2.5 KB) of HBM reads
// in flight while it computes; activations come from L1/L2.
//
// Epilogues (IQ_* modes of k_grouped.cuh): fp16 product; SiLU(gate) * up
// with the gate and up tiles of the same rows multiplied by the same warp
// (SiLU(z) = z / (1 + e^-z) in fp32); or g-scaled fp32 for the down
// projection.  Every output element is written by exactly one lane.
#pragma once
#include "k_grouped.cuh"
#include "qmm_dev.cuh"

namespace qmm {

constexpr int kIqwWarps = 8;  // warps per CTA; two CTAs per SM share it
constexpr int kIqwMaxExperts = 256;

struct IqwArgs {
  const uint8_t* data0;  // expert stack (gate when SWIGLU)
  const uint8_t* data1;  // SWIGLU: the up stack
  int64_t dstride0, dstride1;
  const uint16_t* x;
  int x_per_pair, topk;
  const int32_t* offsets;  // [E+1] pair offsets per expert (nullptr: plain product of m_plain rows)
  const int32_t* perm;     // [P] pair ids sorted by expert
  int m_plain;
  void* y;
  const float* gw;  // IQ_SCALED_F32: per-pair weights
  int n, k, E;
};

// The five 4-byte words that hold block b (18 bytes, starting 2 bytes into
// the first word when b is odd) of rows ra and rb of both sources of an item.
struct IqwWords {
  uint32_t w[2][2][5];  // [source][row grp / grp+8][word]
};

__device__ __forceinline__ void iqw_load(IqwWords& w, const uint8_t* const (&rp)[2][2], int blk, int tig) {
  const int64_t boff = (int64_t)blk * 18 - ((tig & 1) ? 2 : 0);  // 4-byte aligned start
#pragma unroll
  for (int s = 0; s < 2; s++)
#pragma unroll
    for (int r = 0; r < 2; r++) {
      const uint32_t* q = reinterpret_cast<const uint32_t*>(rp[s][r] + boff);
#pragma unroll
      for (int i = 0; i < 5; i++) w.w[s][r][i] = __ldg(q + i);
    }
}

// A block's scale (as f16x2 d,d) and its index word i from its five words,
// without a divergent branch: an odd block starts 2 bytes in (a funnel shift
// by 32, clamped, is the next word).
__device__ __forceinline__ uint32_t iqw_scale(const uint32_t (&w)[5], uint32_t fs) {
  const uint32_t d = (w[0] >> (fs - 16u)) & 0xFFFFu;
  return d | (d << 16);
}
__device__ __forceinline__ uint32_t iqw_qword(const uint32_t (&w)[5], int i, uint32_t fs) {
  return __funnelshift_rc(w[i], w[i + 1], fs);
}

// Decode one super-step of both sources (rows grp, grp+8; block blk, 32 k)
// and multiply it with the same 32 k of token columns grp (xr0) and grp+8
// (xr1): the activation fragments are shared by the two sources' MMAs.
template <int NT>
__device__ __forceinline__ void iqw_block(float (&acc)[2][2][4], const IqwWords& w, int tig, const uint16_t* xr0,
                                          const uint16_t* xr1, int blk, uint32_t lut_lane) {
  uint32_t xw[NT][16];
#pragma unroll
  for (int j = 0; j < NT; j++) {
    const uint16_t* xp = (j ? xr1 : xr0) + blk * 32;
#pragma unroll
    for (int q = 0; q < 4; q++) {
      const uint4 v = ldg_x128(xp + 8 * q);
      xw[j][4 * q] = v.x; xw[j][4 * q + 1] = v.y; xw[j][4 * q + 2] = v.z; xw[j][4 * q + 3] = v.w;
    }
  }
  const uint32_t fs = (tig & 1) ? 32u : 16u;
  uint32_t dd[2][2];
#pragma unroll
  for (int s = 0; s < 2; s++)
#pragma unroll
    for (int r = 0; r < 2; r++) dd[s][r] = iqw_scale(w.w[s][r], fs);
#pragma unroll
  for (int i = 0; i < 8; i++) {  // index bytes 2i, 2i+1 of the block
    uint32_t b0[NT], b1[NT];
#pragma unroll
    for (int j = 0; j < NT; j++) {
      b0[j] = __byte_perm(xw[j][i], xw[j][i + 8], 0x5410);  // (x_2i, x_2i+16)
      b1[j] = __byte_perm(xw[j][i], xw[j][i + 8], 0x7632);  // (x_2i+1, x_2i+17)
    }
    const int bs = (i & 1) * 2;
#pragma unroll
    for (int s = 0; s < 2; s++) {
      const uint32_t qwa = iqw_qword(w.w[s][0], i >> 1, fs), qwb = iqw_qword(w.w[s][1], i >> 1, fs);
      const uint32_t a0 = hmul2(lds32(lut_addr(qwa, bs, lut_lane)), dd[s][0]);
      const uint32_t a2 = hmul2(lds32(lut_addr(qwa, bs + 1, lut_lane)), dd[s][0]);
      const uint32_t a1 = hmul2(lds32(lut_addr(qwb, bs, lut_lane)), dd[s][1]);
      const uint32_t a3 = hmul2(lds32(lut_addr(qwb, bs + 1, lut_lane)), dd[s][1]);
#pragma unroll
      for (int j = 0; j < NT; j++) mma_16816(acc[s][j], a0, a1, a2, a3, b0[j], b1[j]);
    }
  }
}

// Both sources of an item over the whole k: super-steps of 128 k, the next
// step's weight words loaded before this step is decoded.
template <int NT>
__device__ __forceinline__ void iqw_tile(float (&acc)[2][2][4], const uint8_t* const (&rp)[2][2], int steps, int tig,
                                         const uint16_t* xr0, const uint16_t* xr1, uint32_t lut_lane) {
  IqwWords cur, nxt;
  iqw_load(cur, rp, tig, tig);
  for (int s = 0; s < steps; s++) {
    const int blk = 4 * s + tig;
    if (s + 1 < steps) iqw_load(nxt, rp, blk + 4, tig);
    iqw_block<NT>(acc, cur, tig, xr0, xr1, blk, lut_lane);
    cur = nxt;
  }
}

// Work item = (expert, group of up to 16 of its routed pairs, pair of 16-row
// tiles): with IQ_SWIGLU the gate and up tiles of the same rows, otherwise
// two neighbouring tiles of the matrix (the second one absent past n: its
// loads re-read the first tile and nothing of it is stored).
template <int MODE>
__global__ void __launch_bounds__(kIqwWarps * 32, 2) iq4_warp_kernel(const IqwArgs a) {
  extern __shared__ __align__(16) uint8_t smem_iqw[];
  __shared__ int s_items[kIqwMaxExperts + 1];  // first item of each expert
  const uint32_t lut = smem_addr(smem_iqw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, grp = lane >> 2, tig = lane & 3;
  for (int i = threadIdx.x; i < 256 * 32; i += kIqwWarps * 32) {
    const int v = i >> 5;
    const uint32_t lo = __half_as_ushort(__int2half_rn(c_iq4nl_kv[v & 15]));
    const uint32_t hi = __half_as_ushort(__int2half_rn(c_iq4nl_kv[v >> 4]));
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(lut + 4u * i), "r"(lo | (hi << 16)) : "memory");
  }
  const int tiles = (a.n + 15) / 16;
  const int pairs = (MODE == IQ_SWIGLU) ? tiles : (tiles + 1) / 2;  // items per token group
  const int E = a.offsets ? a.E : 1;
  if (warp == 0) {  // items per expert: ceil(pairs / 16) token groups x tile pairs, scanned
    int run = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      int c = 0;
      if (e < E) c = a.offsets ? a.offsets[e + 1] - a.offsets[e] : a.m_plain;
      int it = ((c + 15) / 16) * pairs, v = it;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += u;
      }
      if (e < E) s_items[e] = run + v - it;
      run += __shfl_sync(0xFFFFFFFFu, v, 31);
    }
    if (lane == 0) s_items[E] = run;
  }
  __syncthreads();
  const uint32_t lut_lane = lut + 4u * lane;
  const int items = s_items[E];
  const int steps = a.k >> 7;
  const int64_t rowb = (int64_t)(a.k >> 5) * 18;
  const int nwarps = gridDim.x * kIqwWarps;
  int e = 0;
  for (int item = blockIdx.x * kIqwWarps + warp; item < items; item += nwarps) {
    while (s_items[e + 1] <= item) e++;
    const int local = item - s_items[e], g = local / pairs, pr2 = local - g * pairs;
    const int start = (a.offsets ? a.offsets[e] : 0) + 16 * g;
    const int cnt = a.offsets ? a.offsets[e + 1] - a.offsets[e] : a.m_plain;
    const int ng = min(16, cnt - 16 * g);
    // activation rows of token columns grp and grp+8 (columns past ng read
    // the group's first row: their outputs are never stored)
    const uint16_t* xr[2];
#pragma unroll
    for (int j = 0; j < 2; j++) {
      const int slot = (grp + 8 * j < ng) ? grp + 8 * j : 0;
      const int pr = a.offsets ? a.perm[start + slot] : start + slot;
      const int row = (a.offsets && !a.x_per_pair) ? pr / a.topk : pr;
      xr[j] = a.x + (int64_t)row * a.k;
    }
    // first row of each source's tile; source 1 absent (= source 0) past n
    int row0[2];
    const uint8_t* base[2];
    if (MODE == IQ_SWIGLU) {
      row0[0] = row0[1] = pr2 * 16;
      base[0] = a.data0 + (int64_t)e * a.dstride0;
      base[1] = a.data1 + (int64_t)e * a.dstride1;
    } else {
      row0[0] = 2 * pr2 * 16;
      row0[1] = (2 * pr2 + 1 < tiles) ? row0[0] + 16 : row0[0];
      base[0] = base[1] = a.data0 + (int64_t)e * a.dstride0;
    }
    const uint8_t* rp[2][2];
#pragma unroll
    for (int s2 = 0; s2 < 2; s2++) {
      rp[s2][0] = base[s2] + (int64_t)min(row0[s2] + grp, a.n - 1) * rowb;
      rp[s2][1] = base[s2] + (int64_t)min(row0[s2] + grp + 8, a.n - 1) * rowb;
    }
    float acc[2][2][4];
#pragma unroll
    for (int s2 = 0; s2 < 2; s2++)
#pragma unroll
      for (int j = 0; j < 2; j++)
#pragma unroll
        for (int c = 0; c < 4; c++) acc[s2][j][c] = 0.f;
    if (ng <= 8) iqw_tile<1>(acc, rp, steps, tig, xr[0], xr[1], lut_lane);
    else iqw_tile<2>(acc, rp, steps, tig, xr[0], xr[1], lut_lane);
    // acc[s][j][c]: row grp (c = 0, 1) or grp+8 (c = 2, 3) of source s's
    // tile, token slot 8j + 2tig + (c & 1)
    const bool has1 = MODE != IQ_SWIGLU && row0[1] != row0[0];
#pragma unroll
    for (int s2 = 0; s2 < 2; s2++) {
      if (MODE == IQ_SWIGLU && s2 == 1) break;  // gate and up meet in source 0's loop
      if (s2 == 1 && !has1) break;
#pragma unroll
      for (int j = 0; j < 2; j++) {
#pragma unroll
        for (int c = 0; c < 4; c++) {
          const int slot = 8 * j + 2 * tig + (c & 1);
          const int row = row0[s2] + grp + ((c & 2) ? 8 : 0);
          if (slot >= ng || row >= a.n) continue;
          const int64_t pr = a.offsets ? a.perm[start + slot] : start + slot;
          const float v = acc[s2][j][c];
          if (MODE == IQ_SCALED_F32) {
            static_cast<float*>(a.y)[pr * a.n + row] = a.gw[pr] * v;
          } else if (MODE == IQ_SWIGLU) {
            static_cast<uint16_t*>(a.y)[pr * a.n + row] = f32_to_f16_bits(v / (1.0f + expf(-v)) * acc[1][j][c]);
          } else {
            static_cast<uint16_t*>(a.y)[pr * a.n + row] = f32_to_f16_bits(v);
          }
        }
      }
    }
  }
}

}  // namespace qmm
