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

}  // namespace qmm
