// k_iq4p.cuh -- persistent, warp-specialised IQ4_NL kernel for the routed
// experts ("Mark-Experimental-V3-8B", section "Mixture-of-Experts (MoE)":
// 32 routed experts, 4 active per token; section "Quantization": IQ4_NL
// blocks of 32 weights, one fp16 scale and 16 bytes of 4-bit indices into a
// 16-entry table; expert weights stored as one contiguous 3-D tensor per
// projection) and for the plain IQ4_NL product of up to 16 rows.
//
// One CTA per SM.  Every CTA first buckets the routing ids itself (a count,
// two warp scans and a stable scatter in shared memory, so all CTAs hold the
// same permutation), so no separate routing kernel or global permutation is
// needed.  The work items are
// (expert, group of up to 16 tokens, 16-row tile); each CTA takes a
// contiguous range of the items that exist, in expert-major order, so
// consecutive items share their activation rows.
//
//   warp 0, lane 0 (producer): for each item, bulk-copies the weight tile
//     (16 consecutive rows are one contiguous byte range of 16 * k/32 * 18
//     bytes) of each matrix the item multiplies into a ring of S stages, and
//     when the token group changes, the group's activation rows into one of
//     XB row buffers (one bulk copy per row).  TMA engine, no multicast.
//   warps 1..W (consumers): split the tile's k into ranges of 128 (four
//     blocks per lane: lane (grp, tig) owns block 4s+tig of rows grp and
//     grp+8), decode each index byte through a 256-entry table of exact f16x2
//     pairs (w_j, w_{j+16}) replicated across the 32 banks, multiply by the
//     block scale (one f16x2 multiply: the bit-exact decoded weight) and feed
//     legacy m16n8k16 MMAs with the token rows read from shared memory.  A
//     warp releases a stage as soon as it has read it; partial sums meet in
//     shared memory and are added in warp order (deterministic).
//
// Every wait is bounded (%globaltimer); on a timeout the error word is
// raised, all warps leave their loops together (a barrier with an OR
// reduction) and the producer waits for its own copies before exiting.
#pragma once
#include "k_grouped.cuh"
#include "qmm_dev.cuh"

namespace qmm {

constexpr int kPxMaxWarps = 11;    // consumer warps (12 warps: up to 168 registers a thread)
constexpr int kPxMaxStages = 8;
constexpr int kPxMaxXBuf = 2;
constexpr int kPxMaxPairs = 4096;  // routing pairs bucketed in shared memory
constexpr int kPxMaxThreads = 32 * (kPxMaxWarps + 1);

struct PxArgs {
  const uint8_t* data0;  // first (or only) matrix stack
  const uint8_t* data1;  // IQ_SWIGLU: the up stack
  int64_t dstride0, dstride1;
  const uint16_t* x;
  int x_per_pair, topk;
  const int32_t* ids;  // [P] expert ids; nullptr: plain product of m_plain rows
  int P, m_plain;
  void* y;
  const float* gw;  // IQ_SCALED_F32: per-pair weights
  int n, k, E;
  int W, S, XB;  // consumer warps, ring stages, activation buffers
};

struct PxLayout {
  uint32_t lut, xbuf, ring, red, cnt, off, ip, pid, perm, bars, total;
  uint32_t x_stride, tile_bytes;
};

// Shared-memory layout, computed identically on host and device.
__host__ __device__ inline PxLayout px_layout(int k, int E, int P, int W, int S, int XB, int halves) {
  PxLayout L;
  const uint32_t rowb = (uint32_t)(k / 32) * 18u;
  L.tile_bytes = 16u * rowb;
  L.x_stride = 2u * (uint32_t)k + 16u;  // pad: token rows start in different banks
  uint32_t o = 0;
  L.lut = o;
  o += 256u * 32u * 4u;
  L.xbuf = o;
  o += (uint32_t)XB * 16u * L.x_stride;
  L.ring = o;
  o += (uint32_t)S * L.tile_bytes;
  L.red = o;
  o += (uint32_t)halves * (uint32_t)W * 16u * 16u * 4u;
  L.cnt = o;
  o += 4u * (uint32_t)(E + 1);
  o = (o + 15u) & ~15u;
  L.off = o;
  o += 4u * (uint32_t)(E + 1);
  o = (o + 15u) & ~15u;
  L.ip = o;
  o += 4u * (uint32_t)(E + 1);
  o = (o + 15u) & ~15u;
  L.pid = o;
  o += 4u * (uint32_t)(P > 0 ? P : 1);
  o = (o + 15u) & ~15u;
  L.perm = o;
  o += 4u * (uint32_t)(P > 0 ? P : 1);
  o = (o + 15u) & ~15u;
  L.bars = o;
  o += 8u * (uint32_t)(2 * S + 2 * XB);
  L.total = o;
  return L;
}

// Decode and multiply the super-steps [s_lo, s_hi) of one 16-row tile held in
// shared memory at `tile` against up to 8*NT token rows at xrow0 (slot grp)
// and xrow1 (slot grp+8).  Two super-steps are loaded before either is used.
template <int NT>
__device__ __forceinline__ void px_range(float (&acc)[2][4], uint32_t tile, uint32_t rowb, int grp, int tig, int s_lo,
                                         int s_hi, uint32_t xrow0, uint32_t xrow1, uint32_t lut_lane) {
  const uint32_t pa = tile + (uint32_t)grp * rowb, pb = pa + 8u * rowb;
  for (int s0 = s_lo; s0 < s_hi; s0 += 2) {
    uint32_t wa[2][5], wb[2][5], xw[2][NT][16];
#pragma unroll
    for (int u = 0; u < 2; u++) {
      if (s0 + u < s_hi) {
        const int b = 4 * (s0 + u) + tig;
        const uint32_t boff = (uint32_t)b * 18u - ((tig & 1) ? 2u : 0u);  // 4-byte aligned start
#pragma unroll
        for (int i = 0; i < 5; i++) {
          wa[u][i] = lds32(pa + boff + 4u * i);
          wb[u][i] = lds32(pb + boff + 4u * i);
        }
#pragma unroll
        for (int j = 0; j < NT; j++) {
          const uint32_t xp = (j ? xrow1 : xrow0) + (uint32_t)b * 64u;
#pragma unroll
          for (int q = 0; q < 4; q++) {
            const uint4 v = lds128(xp + 16u * q);
            xw[u][j][4 * q] = v.x;
            xw[u][j][4 * q + 1] = v.y;
            xw[u][j][4 * q + 2] = v.z;
            xw[u][j][4 * q + 3] = v.w;
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 2; u++) {
      if (s0 + u >= s_hi) break;
      uint32_t da, db, qa[4], qb[4];
      if (tig & 1) {  // block starts 2 bytes into word 0
        da = wa[u][0] >> 16;
        db = wb[u][0] >> 16;
#pragma unroll
        for (int i = 0; i < 4; i++) {
          qa[i] = wa[u][i + 1];
          qb[i] = wb[u][i + 1];
        }
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
#pragma unroll
      for (int i = 0; i < 8; i++) {  // index bytes 2i, 2i+1 of the block
        const uint32_t qwa = qa[i >> 1], qwb = qb[i >> 1];
        const int bs = (i & 1) * 2;
        const uint32_t a0 = hmul2(lds32(lut_addr(qwa, bs, lut_lane)), dda);
        const uint32_t a2 = hmul2(lds32(lut_addr(qwa, bs + 1, lut_lane)), dda);
        const uint32_t a1 = hmul2(lds32(lut_addr(qwb, bs, lut_lane)), ddb);
        const uint32_t a3 = hmul2(lds32(lut_addr(qwb, bs + 1, lut_lane)), ddb);
#pragma unroll
        for (int j = 0; j < NT; j++) {
          const uint32_t b0 = __byte_perm(xw[u][j][i], xw[u][j][i + 8], 0x5410);  // (x_2i, x_2i+16)
          const uint32_t b1 = __byte_perm(xw[u][j][i], xw[u][j][i + 8], 0x7632);  // (x_2i+1, x_2i+17)
          mma_16816(acc[j], a0, a1, a2, a3, b0, b1);
        }
      }
    }
  }
}

template <int MODE>
__global__ void __launch_bounds__(kPxMaxThreads, 1) iq4_persist_kernel(const PxArgs a) {
  extern __shared__ __align__(128) uint8_t smem_px[];
  constexpr int H = (MODE == IQ_SWIGLU) ? 2 : 1;
  const int W = a.W, S = a.S, XB = a.XB, k = a.k;
  const int E = a.ids ? a.E : 1;
  const PxLayout L = px_layout(k, E, a.P, W, S, XB, H);
  const uint32_t sb = smem_addr(smem_px);
  int* cnt = reinterpret_cast<int*>(smem_px + L.cnt);
  int* off = reinterpret_cast<int*>(smem_px + L.off);
  int* ip = reinterpret_cast<int*>(smem_px + L.ip);
  int* pid = reinterpret_cast<int*>(smem_px + L.pid);
  int* perm = reinterpret_cast<int*>(smem_px + L.perm);
  float* red = reinterpret_cast<float*>(smem_px + L.red);
  const uint32_t full = sb + L.bars, empty = full + 8u * S, xfull = empty + 8u * S, xempty = xfull + 8u * XB;
  __shared__ volatile int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nthr = blockDim.x;

  // exact f16x2 table [index byte][lane]: (kv[lo nibble], kv[hi nibble])
  for (int i = tid; i < 256 * 32; i += nthr) {
    const int v = i >> 5;
    const uint32_t lo = __half_as_ushort(__int2half_rn(c_iq4nl_kv[v & 15]));
    const uint32_t hi = __half_as_ushort(__int2half_rn(c_iq4nl_kv[v >> 4]));
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(sb + L.lut + 4u * i), "r"(lo | (hi << 16)) : "memory");
  }
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < S; s++) {
      mbar_init(full + 8u * s, 1);
      mbar_init(empty + 8u * s, (uint32_t)W);
    }
    for (int b = 0; b < XB; b++) {
      mbar_init(xfull + 8u * b, 1);
      mbar_init(xempty + 8u * b, (uint32_t)W);
    }
    fence_mbar_init();
  }
  // -- routing: count, scan, scatter (all in shared memory) --
  for (int e = tid; e <= E; e += nthr) cnt[e] = 0;
  __syncthreads();
  if (a.ids) {
    bool bad = false;
    for (int p = tid; p < a.P; p += nthr) {
      const int e = a.ids[p];
      pid[p] = e;
      if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
      else bad = true;
    }
    if (bad && blockIdx.x == 0) raise_error(ERR_BAD_EXPERT);
  } else if (tid == 0) {
    cnt[0] = a.m_plain;
  }
  __syncthreads();
  const int tiles = a.n / 16;
  if (warp == 0) {
    int run = 0, irun = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int c = e < E ? cnt[e] : 0;
      const int it = ((c + 15) / 16) * tiles;
      int v = c, w = it;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v2 = __shfl_up_sync(0xFFFFFFFFu, v, o), w2 = __shfl_up_sync(0xFFFFFFFFu, w, o);
        if (lane >= o) {
          v += v2;
          w += w2;
        }
      }
      if (e < E) {
        off[e] = run + v - c;
        ip[e] = irun + w - it;
      }
      run += __shfl_sync(0xFFFFFFFFu, v, 31);
      irun += __shfl_sync(0xFFFFFFFFu, w, 31);
    }
    if (lane == 0) {
      off[E] = run;
      ip[E] = irun;
    }
  }
  __syncthreads();
  if (a.ids) {
    for (int e = tid; e < E; e += nthr) cnt[e] = off[e];  // scatter cursors
    __syncthreads();
    // Stable scatter by warp 0, in ascending pair order.  Every CTA must build
    // the same permutation: an item (expert, token group, row tile) names its
    // pairs by position in it, and the row tiles of one group are spread over
    // CTAs.
    if (warp == 0) {
      const unsigned lt = (1u << lane) - 1u;
      for (int p0 = 0; p0 < a.P; p0 += 32) {
        const int p = p0 + lane;
        const int e = p < a.P ? pid[p] : -1;
        const bool ok = e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, ok ? e : -1);
        if (ok) perm[cnt[e] + __popc(peers & lt)] = p;
        __syncwarp();
        if (ok && (peers >> lane) == 1u) cnt[e] += __popc(peers);  // the group's highest lane
        __syncwarp();
      }
    }
  }
  __syncthreads();

  const int items = ip[E];
  const int i0 = (int)((int64_t)blockIdx.x * items / gridDim.x);
  const int i1 = (int)((int64_t)(blockIdx.x + 1) * items / gridDim.x);
  const uint32_t tb = L.tile_bytes, xs = L.x_stride;

  if (warp == 0) {
    if (lane != 0) return;
    // ---------------- producer ----------------
    uint32_t st = 0, xf = 0;
    int e = 0, ce = -1, cg = -1;
    for (int i = i0; i < i1 && !s_abort; i++) {
      while (ip[e + 1] <= i) e++;
      const int local = i - ip[e], g = local / tiles, tile = local - g * tiles;
      bool stop = false;
#pragma unroll
      for (int h = 0; h < H; h++) {
        const uint32_t slot = st % (uint32_t)S;
        if (st >= (uint32_t)S && !mbar_wait(empty + 8u * slot, ((st / S) & 1u) ^ 1u)) {
          stop = true;
          break;
        }
        mbar_arrive_expect_tx(full + 8u * slot, tb);
        const uint8_t* src = (h ? a.data1 + (int64_t)e * a.dstride1 : a.data0 + (int64_t)e * a.dstride0) +
                             (int64_t)tile * tb;
        bulk_load(sb + L.ring + slot * tb, src, tb, full + 8u * slot);
        st++;
      }
      if (!stop && (e != ce || g != cg)) {
        const uint32_t xb = xf % (uint32_t)XB;
        if (xf >= (uint32_t)XB && !mbar_wait(xempty + 8u * xb, ((xf / XB) & 1u) ^ 1u)) {
          stop = true;
        } else {
          const int start = off[e] + 16 * g;
          const int ng = min(16, off[e + 1] - start);
          mbar_arrive_expect_tx(xfull + 8u * xb, (uint32_t)ng * 2u * (uint32_t)k);
          for (int s = 0; s < ng; s++) {
            const int pr = a.ids ? perm[start + s] : start + s;
            const int row = (a.ids && !a.x_per_pair) ? pr / a.topk : pr;
            bulk_load(sb + L.xbuf + xb * 16u * xs + (uint32_t)s * xs, a.x + (int64_t)row * k, 2u * (uint32_t)k,
                      xfull + 8u * xb);
          }
          xf++;
          ce = e;
          cg = g;
        }
      }
      if (stop) {
        s_abort = 1;
        break;
      }
    }
    // drain: the last copy into every stage and row buffer has landed
    for (uint32_t s = 0; s < (uint32_t)S && s < st; s++) {
      const uint32_t last = s + (uint32_t)S * ((st - 1u - s) / (uint32_t)S);
      mbar_wait(full + 8u * s, (last / S) & 1u);
    }
    for (uint32_t b = 0; b < (uint32_t)XB && b < xf; b++) {
      const uint32_t last = b + (uint32_t)XB * ((xf - 1u - b) / (uint32_t)XB);
      mbar_wait(xfull + 8u * b, (last / XB) & 1u);
    }
    return;
  }

  // ---------------- consumers ----------------
  const int cw = warp - 1, grp = lane >> 2, tig = lane & 3;
  const uint32_t lut_lane = sb + L.lut + 4u * lane;
  const uint32_t rowb = (uint32_t)(k / 32) * 18u;
  const int steps = k >> 7;
  const int s_lo = cw * steps / W, s_hi = (cw + 1) * steps / W;
  const int cthreads = W * 32, ctid = tid - 32;
  uint32_t st = 0, xf = 0, xbase = 0;
  int e = 0, ce = -1, cg = -1;
  for (int i = i0; i < i1; i++) {
    while (ip[e + 1] <= i) e++;
    const int local = i - ip[e], g = local / tiles, tile = local - g * tiles;
    const int start = off[e] + 16 * g;
    const int ng = min(16, off[e + 1] - start);
    bool fail = false;
    if (e != ce || g != cg) {
      if (xf > 0 && lane == 0) mbar_arrive(xempty + 8u * ((xf - 1u) % (uint32_t)XB));
      const uint32_t xb = xf % (uint32_t)XB;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(xfull + 8u * xb, (xf / XB) & 1u))) fail = true;
      xbase = sb + L.xbuf + xb * 16u * xs;
      xf++;
      ce = e;
      cg = g;
    }
    const uint32_t xrow0 = xbase + (uint32_t)grp * xs, xrow1 = xrow0 + 8u * xs;
    float acc[H][2][4];
#pragma unroll
    for (int h = 0; h < H; h++)
#pragma unroll
      for (int j = 0; j < 2; j++)
#pragma unroll
        for (int c = 0; c < 4; c++) acc[h][j][c] = 0.f;
#pragma unroll
    for (int h = 0; h < H; h++) {
      const uint32_t slot = st % (uint32_t)S;
      if (__all_sync(0xFFFFFFFFu, !fail && !s_abort && mbar_wait(full + 8u * slot, (st / S) & 1u))) {
        const uint32_t t0 = sb + L.ring + slot * tb;
        if (ng <= 8) px_range<1>(acc[h], t0, rowb, grp, tig, s_lo, s_hi, xrow0, xrow1, lut_lane);
        else px_range<2>(acc[h], t0, rowb, grp, tig, s_lo, s_hi, xrow0, xrow1, lut_lane);
      } else {
        fail = true;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + 8u * slot);
      st++;
    }
    // partial sums of this warp: red[h][cw][token slot][row] (used token tiles only)
#pragma unroll
    for (int h = 0; h < H; h++) {
      float* r = red + ((h * W + cw) * 16) * 16;
#pragma unroll
      for (int j = 0; j < 2; j++) {
        if (8 * j < ng) {
          const int t0 = 8 * j + 2 * tig;
          r[t0 * 16 + grp] = acc[h][j][0];
          r[(t0 + 1) * 16 + grp] = acc[h][j][1];
          r[t0 * 16 + grp + 8] = acc[h][j][2];
          r[(t0 + 1) * 16 + grp + 8] = acc[h][j][3];
        }
      }
    }
    if (fail) s_abort = 1;
    named_bar_sync(1, cthreads);
    for (int idx = ctid; idx < 16 * ng; idx += cthreads) {
      const int row = idx & 15, slot = idx >> 4;
      float v[H];
#pragma unroll
      for (int h = 0; h < H; h++) {
        float sum = 0.f;
        for (int w = 0; w < W; w++) sum += red[((h * W + w) * 16 + slot) * 16 + row];
        v[h] = sum;
      }
      const int grow = tile * 16 + row;
      const int64_t pr = a.ids ? perm[start + slot] : start + slot;
      if (MODE == IQ_SCALED_F32) {
        static_cast<float*>(a.y)[pr * a.n + grow] = a.gw[pr] * v[0];
      } else if (MODE == IQ_SWIGLU) {
        const float gv = v[0];
        static_cast<uint16_t*>(a.y)[pr * a.n + grow] = f32_to_f16_bits(gv / (1.0f + expf(-gv)) * v[H - 1]);
      } else {
        static_cast<uint16_t*>(a.y)[pr * a.n + grow] = f32_to_f16_bits(v[0]);
      }
    }
    if (named_bar_or(2, cthreads, s_abort != 0)) break;
  }
}

}  // namespace qmm
