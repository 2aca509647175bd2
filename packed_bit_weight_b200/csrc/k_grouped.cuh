// k_grouped.cuh -- routed-expert grouped GEMV ("Mark-Experimental-V3-8B",
// section "Mixture-of-Experts (MoE)": 32 routed experts, 4 active per token,
// y = ... + sum_i g_i F_i(x); expert weights stored as one contiguous 3-D
// tensor per projection, section "Quantization").
//
// Step 1 (route): a stable counting sort of the t*topk (token, slot) pairs by
// expert id -- offsets[E+1] and a pair permutation -- in one CTA.
// Step 2 (grouped GEMV): one warp per (expert, 16-row tile); the warp decodes
// its weight tile once per k16 step into MMA fragments and multiplies it with
// up to 32 gathered activation rows (4 MMA n-tiles) routed to that expert, so
// every expert's weights are read once for all of its pairs.  Outputs go to
// y[token][slot][:] of each pair.
#pragma once
#include "k_gemv.cuh"
#include "qmm_dev.cuh"

namespace qmm {

constexpr int kRouteMaxExperts = 256;
constexpr int kRouteThreads = 1024;

// Stable bucket sort of pair indices p = token*topk + slot by ids[p].  Ids
// outside [0, E) are left out and raise ERR_BAD_EXPERT.
__global__ void __launch_bounds__(kRouteThreads, 1)
    route_kernel(const int32_t* __restrict__ ids, int P, int E, int32_t* __restrict__ offsets,
                 int32_t* __restrict__ perm) {
  __shared__ int cnt[kRouteMaxExperts];
  __shared__ int fill[kRouteMaxExperts];
  __shared__ int wcnt[kRouteThreads / 32][kRouteMaxExperts];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // a kernel launched after this one with programmatic dependent launch may
  // start now (it waits for this kernel's results before reading them)
  asm volatile("griddepcontrol.launch_dependents;" :::);
  for (int e = tid; e < E; e += kRouteThreads) cnt[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int p = tid; p < P; p += kRouteThreads) {
    const int e = ids[p];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    else bad = true;
  }
  if (bad) raise_error(ERR_BAD_EXPERT);
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < E; e++) {
      fill[e] = run;
      offsets[e] = run;
      run += cnt[e];
    }
    offsets[E] = run;
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int c0 = 0; c0 < P; c0 += kRouteThreads) {
    const int p = c0 + tid;
    const int e = (p < P) ? ids[p] : -1;
    const bool valid = (e >= 0 && e < E);
    const int key = valid ? e : -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
    const int rank = __popc(peers & lt);
    for (int i = tid; i < (kRouteThreads / 32) * E; i += kRouteThreads) wcnt[i / E][i % E] = 0;
    __syncthreads();
    if (valid && (__ffs(peers) - 1) == lane) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    if (valid) {
      int base = fill[e];
      for (int w = 0; w < warp; w++) base += wcnt[w][e];
      perm[base + rank] = p;
    }
    __syncthreads();
    for (int i = tid; i < E; i += kRouteThreads) {
      int s = 0;
      for (int w = 0; w < kRouteThreads / 32; w++) s += wcnt[w][i];
      fill[i] += s;
    }
    __syncthreads();
  }
}

// One warp per (expert, 16-row tile).  x rows: x[token] (x_per_pair == 0,
// [t][k]) or x[pair] (x_per_pair == 1, [t*topk][k]).
template <int FMT>
__global__ void __launch_bounds__(128) grouped_gemv_kernel(
    const uint8_t* __restrict__ data, int64_t dstride, const uint8_t* __restrict__ scales, int64_t sstride,
    float g, const uint16_t* __restrict__ x, int x_per_pair, int topk, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ perm, uint16_t* __restrict__ y, int64_t n, int64_t k, int E) {
  __shared__ uint32_t kvh[16];
  if (threadIdx.x < 16) kvh[threadIdx.x] = __half_as_ushort(__int2half_rn(c_iq4nl_kv[threadIdx.x]));
  __syncthreads();
  const int lane = threadIdx.x & 31, grp = lane >> 2, tig = lane & 3;
  const int64_t tiles = (n + 15) / 16;
  const int64_t item = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int64_t e = item / tiles, tile = item % tiles;
  if (e >= E) return;
  const int start = offsets[e];
  const int cnt = offsets[e + 1] - start;
  if (cnt <= 0) return;
  const uint8_t* de = data + e * dstride;
  const uint8_t* se = scales ? scales + e * sstride : nullptr;
  const int64_t r0 = tile * 16 + grp, r1 = r0 + 8;
  const float gs = (FMT == 3) ? g : 1.0f;
  for (int tok0 = 0; tok0 < cnt; tok0 += 32) {
    const int ng = min(32, cnt - tok0);
    // activation rows of this lane's B fragments (token slots grp + 8j)
    const uint16_t* xr[4];
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const int slot = grp + 8 * j;
      xr[j] = nullptr;
      if (slot < ng) {
        const int pair = perm[start + tok0 + slot];
        xr[j] = x + (int64_t)(x_per_pair ? pair : pair / topk) * k;
      }
    }
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; j++)
#pragma unroll
      for (int c = 0; c < 4; c++) acc[j][c] = 0.f;
    for (int64_t k0 = 0; k0 < k; k0 += 16) {
      const int64_t ka = k0 + 2 * tig, kb = ka + 8;
      const uint32_t a0 = generic_pair<FMT>(de, se, r0, n, k, ka, kvh);
      const uint32_t a1 = generic_pair<FMT>(de, se, r1, n, k, ka, kvh);
      const uint32_t a2 = generic_pair<FMT>(de, se, r0, n, k, kb, kvh);
      const uint32_t a3 = generic_pair<FMT>(de, se, r1, n, k, kb, kvh);
#pragma unroll
      for (int j = 0; j < 4; j++) {
        if (8 * j < ng) {
          uint32_t b0 = 0, b1 = 0;
          if (xr[j]) {
            b0 = *reinterpret_cast<const uint32_t*>(xr[j] + ka);
            b1 = *reinterpret_cast<const uint32_t*>(xr[j] + kb);
          }
          mma_16816(acc[j], a0, a1, a2, a3, b0, b1);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const int s0 = 8 * j + 2 * tig, s1 = s0 + 1;
      if (s0 < ng) {
        const int64_t pr = perm[start + tok0 + s0];
        if (r0 < n) y[pr * n + r0] = f32_to_f16_bits(acc[j][0] * gs);
        if (r1 < n) y[pr * n + r1] = f32_to_f16_bits(acc[j][2] * gs);
      }
      if (s1 < ng) {
        const int64_t pr = perm[start + tok0 + s1];
        if (r0 < n) y[pr * n + r0] = f32_to_f16_bits(acc[j][1] * gs);
        if (r1 < n) y[pr * n + r1] = f32_to_f16_bits(acc[j][3] * gs);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// IQ4_NL streaming kernel for the grouped GEMV (and, with offsets == nullptr,
// the plain GEMV: one "expert", m tokens in order).
//
// Work item = (expert, 16-row tile); persistent CTAs of IQW warps loop over
// items.  The warps split the tile's k into ranges of "super-steps" of four
// blocks (128 k).  In a super-step lane (grp, tig) owns block 4s+tig of rows
// grp and grp+8: it reads the 18-byte block with five 4-byte loads (blocks of
// even index start 4-byte aligned, odd ones 2 bytes past; with an even block
// count per row the five words never leave the row), takes the scale d and
// the 16 index bytes, and turns each index byte j into the pair
// (w_j, w_{j+16}) = d * (kv[lo], kv[hi]) with one lookup in a 256-entry
// table of exact f16x2 pairs (replicated across the 32 banks, so each lane
// reads its own bank) and one f16x2 multiply -- the bit-exact decoded
// weights.  MMA step i uses bytes 2i and 2i+1; the matching activation pairs
// (x_2i, x_2i+16) and (x_2i+1, x_2i+17) are one byte permute each.
// ---------------------------------------------------------------------------
constexpr int kIqWarps = 4;
constexpr int kIqLutBytes = 256 * 32 * 4;  // [byte][lane] f16x2
constexpr int kIqRedBytes = kIqWarps * 32 * 16 * 4;

// Shared address of the table entry for byte `b` (compile-time 0..3) of q:
// one byte permute (zero-extended byte) and one multiply-add.
__device__ __forceinline__ uint32_t lut_addr(uint32_t q, int b, uint32_t lut_lane) {
  const uint32_t byte = __byte_perm(q, 0u, 0x4440u | (uint32_t)b);
  uint32_t a;
  asm("mad.lo.u32 %0, %1, 128, %2;" : "=r"(a) : "r"(byte), "r"(lut_lane));
  return a;
}

// One pass of a warp over its super-steps (at most SMAX) for up to 8*NT
// tokens.  All block loads of the pass are issued first, so a warp has up to
// SMAX * 1.25 KB in flight before it decodes anything.
template <int NT, int SMAX>
__device__ __forceinline__ void iq4_pass(float (&acc)[4][4], const uint8_t* __restrict__ de, int64_t rowb, int ra,
                                         int rb, int s_lo, int s_hi, int tig, const uint16_t* const (&xr)[4],
                                         uint32_t lut_lane) {
  uint32_t wa[SMAX][5], wb[SMAX][5];
  uint32_t xs[SMAX][NT][16];  // the pass's activation words, loaded with the weights
#pragma unroll
  for (int u = 0; u < SMAX; u++) {
    if (s_lo + u < s_hi) {
      const int b = 4 * (s_lo + u) + tig;
      const int64_t boff = (int64_t)b * 18 - ((tig & 1) ? 2 : 0);  // 4-byte aligned start
      const uint32_t* pa = reinterpret_cast<const uint32_t*>(de + (int64_t)ra * rowb + boff);
      const uint32_t* pb = reinterpret_cast<const uint32_t*>(de + (int64_t)rb * rowb + boff);
#pragma unroll
      for (int i = 0; i < 5; i++) {
        wa[u][i] = __ldg(pa + i);
        wb[u][i] = __ldg(pb + i);
      }
#pragma unroll
      for (int j = 0; j < NT; j++) {
        if (xr[j]) {
          const uint16_t* xp = xr[j] + b * 32;
#pragma unroll
          for (int q = 0; q < 4; q++) {
            const uint4 v = ldg_x128(xp + 8 * q);
            xs[u][j][4 * q] = v.x; xs[u][j][4 * q + 1] = v.y; xs[u][j][4 * q + 2] = v.z; xs[u][j][4 * q + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 16; q++) xs[u][j][q] = 0u;
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < SMAX; u++) {
    if (s_lo + u >= s_hi) break;
    uint32_t da, db, qa[4], qb[4];
    if (tig & 1) {  // block starts 2 bytes into word 0
      da = wa[u][0] >> 16;
      db = wb[u][0] >> 16;
#pragma unroll
      for (int i = 0; i < 4; i++) { qa[i] = wa[u][i + 1]; qb[i] = wb[u][i + 1]; }
    } else {
      da = wa[u][0] & 0xFFFFu;
      db = wb[u][0] & 0xFFFFu;
#pragma unroll
      for (int i = 0; i < 4; i++) {
        qa[i] = __funnelshift_r(wa[u][i], wa[u][i + 1], 16);
        qb[i] = __funnelshift_r(wb[u][i], wb[u][i + 1], 16);
      }
    }
    const uint32_t dda = da | (da << 16), ddb = db | (db << 16);
    const uint32_t (&xw)[NT][16] = xs[u];  // this block's 32 activations per n-tile, as 16 words
#pragma unroll
    for (int i = 0; i < 8; i++) {  // index bytes 2i, 2i+1 of the block
      const uint32_t qwa = qa[i >> 1], qwb = qb[i >> 1];
      const int bs = (i & 1) * 2;  // byte of the word
      const uint32_t a0 = hmul2(lds32(lut_addr(qwa, bs, lut_lane)), dda);
      const uint32_t a2 = hmul2(lds32(lut_addr(qwa, bs + 1, lut_lane)), dda);
      const uint32_t a1 = hmul2(lds32(lut_addr(qwb, bs, lut_lane)), ddb);
      const uint32_t a3 = hmul2(lds32(lut_addr(qwb, bs + 1, lut_lane)), ddb);
#pragma unroll
      for (int j = 0; j < NT; j++) {
        const uint32_t b0 = __byte_perm(xw[j][i], xw[j][i + 8], 0x5410);  // (x_2i, x_2i+16)
        const uint32_t b1 = __byte_perm(xw[j][i], xw[j][i + 8], 0x7632);  // (x_2i+1, x_2i+17)
        mma_16816(acc[j], a0, a1, a2, a3, b0, b1);
      }
    }
  }
}

// Passes over a warp range longer than SMAX super-steps are split in chunks.
template <int NT>
__device__ __forceinline__ void iq4_range(float (&acc)[4][4], const uint8_t* __restrict__ de, int64_t rowb, int ra,
                                          int rb, int s_lo, int s_hi, int tig, const uint16_t* const (&xr)[4],
                                          uint32_t lut_lane) {
  constexpr int SMAX = (NT == 1) ? 2 : 1;  // super-steps per pass (their weights and activations in registers)
  for (int s0 = s_lo; s0 < s_hi; s0 += SMAX)
    iq4_pass<NT, SMAX>(acc, de, rowb, ra, rb, s0, min(s0 + SMAX, s_hi), tig, xr, lut_lane);
}

// Epilogue of the IQ4_NL expert kernel.
//   IQ_OUT_F16: y[pair][row] = fp16(acc)                        (plain product)
//   IQ_SWIGLU:  the item multiplies the same 16-row tile of two matrices (gate,
//               up) and writes y[pair][row] = fp16(SiLU(gate) * up), with
//               SiLU(z) = z / (1 + e^-z) in fp32 ("Mark-Experimental-V3-8B",
//               section "Mixture-of-Experts (MoE)": F = (SiLU(x W_gate) *
//               (x W_up)) W_down).
//   IQ_SCALED_F32: yf[pair][row] = gw[pair] * acc in fp32 (the routing weight
//               g_i of the pair applied in the down projection; the slots of a
//               token are added by combine_kernel).
enum { IQ_OUT_F16 = 0, IQ_SWIGLU = 1, IQ_SCALED_F32 = 2 };
constexpr int kIqGateBytes = 16 * 16 * 4;  // [token slot][row] fp32 gate values

template <int MODE>
__global__ void __launch_bounds__(kIqWarps * 32, 4)
    grouped_iq4_kernel(const uint8_t* __restrict__ data, int64_t dstride, const uint8_t* __restrict__ data2,
                       int64_t dstride2, const uint16_t* __restrict__ x, int x_per_pair, int topk,
                       const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm, int m_plain,
                       void* __restrict__ yout, const float* __restrict__ gw, int n, int k, int E) {
  extern __shared__ __align__(16) uint8_t smem_iq[];
  const uint32_t lut = smem_addr(smem_iq);
  float* red = reinterpret_cast<float*>(smem_iq + kIqLutBytes);  // [warp][32 token slots][16 rows]
  float* gsm = reinterpret_cast<float*>(smem_iq + kIqLutBytes + kIqRedBytes);  // IQ_SWIGLU gate values
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, grp = lane >> 2, tig = lane & 3;
  for (int i = threadIdx.x; i < 256 * 32; i += kIqWarps * 32) {
    const int v = i >> 5;
    const uint32_t lo = __half_as_ushort(__int2half_rn(c_iq4nl_kv[v & 15]));
    const uint32_t hi = __half_as_ushort(__int2half_rn(c_iq4nl_kv[v >> 4]));
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(lut + 4u * i), "r"(lo | (hi << 16)) : "memory");
  }
  __syncthreads();
  const uint32_t lut_lane = lut + 4u * lane;
  const int tiles = (n + 15) / 16;
  const int steps = k >> 7;  // super-steps per row
  const int s_lo = warp * steps / kIqWarps, s_hi = (warp + 1) * steps / kIqWarps;
  const int64_t rowb = (int64_t)(k >> 5) * 18;  // bytes per row
  const int items = tiles * E;
  constexpr int kHalves = (MODE == IQ_SWIGLU) ? 2 : 1;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int e = item / tiles, tile = item % tiles;
    int start = 0, cnt = m_plain;
    if (offsets) {
      start = offsets[e];
      cnt = offsets[e + 1] - start;
    }
    if (cnt <= 0) continue;  // uniform across the CTA
    const int ra = min(tile * 16 + grp, n - 1), rb = min(tile * 16 + grp + 8, n - 1);
    for (int tok0 = 0; tok0 < cnt; tok0 += 16) {  // up to 16 gathered tokens per pass
      const int ng = min(16, cnt - tok0);
      const uint16_t* xr[4];
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const int slot = grp + 8 * j;
        xr[j] = nullptr;
        if (slot < ng) {
          const int pr = offsets ? perm[start + tok0 + slot] : tok0 + slot;
          xr[j] = x + (int64_t)((offsets && !x_per_pair) ? pr / topk : pr) * k;
        }
      }
#pragma unroll 1
      for (int half = 0; half < kHalves; half++) {
        const uint8_t* de = half ? data2 + (int64_t)e * dstride2 : data + (int64_t)e * dstride;
        float acc[4][4];
#pragma unroll
        for (int j = 0; j < 4; j++)
#pragma unroll
          for (int c = 0; c < 4; c++) acc[j][c] = 0.f;
        if (ng <= 8) iq4_range<1>(acc, de, rowb, ra, rb, s_lo, s_hi, tig, xr, lut_lane);
        else iq4_range<2>(acc, de, rowb, ra, rb, s_lo, s_hi, tig, xr, lut_lane);
        // meet the other warps: red[warp][token slot][row] (used token tiles only)
        float* r = red + warp * (32 * 16);
#pragma unroll
        for (int j = 0; j < 2; j++) {
          if (8 * j < ng) {
            const int t0 = 8 * j + 2 * tig;
            r[t0 * 16 + grp] = acc[j][0];
            r[(t0 + 1) * 16 + grp] = acc[j][1];
            r[t0 * 16 + grp + 8] = acc[j][2];
            r[(t0 + 1) * 16 + grp + 8] = acc[j][3];
          }
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < 16 * ng; idx += kIqWarps * 32) {
          const int row = idx & 15, slot = idx >> 4;
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kIqWarps; w++) v += red[w * 512 + slot * 16 + row];
          if (MODE == IQ_SWIGLU && half == 0) {
            gsm[idx] = v;  // gate value, kept for the up pass
            continue;
          }
          const int grow = tile * 16 + row;
          if (grow < n) {
            const int64_t pr = offsets ? perm[start + tok0 + slot] : tok0 + slot;
            if (MODE == IQ_SCALED_F32) {
              static_cast<float*>(yout)[pr * n + grow] = gw[pr] * v;
            } else {
              float o = v;
              if (MODE == IQ_SWIGLU) {
                const float gv = gsm[idx];
                o = gv / (1.0f + expf(-gv)) * v;
              }
              static_cast<uint16_t*>(yout)[pr * n + grow] = f32_to_f16_bits(o);
            }
          }
        }
        __syncthreads();
      }
    }
  }
}

}  // namespace qmm
