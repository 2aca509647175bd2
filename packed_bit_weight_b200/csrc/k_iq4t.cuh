// k_iq4t.cuh -- IQ4_NL routed-expert GEMV with the item's weights resident in
// registers ("Mark-Experimental-V3-8B", section "Mixture-of-Experts (MoE)":
// 32 routed experts, 4 active per token, F = (SiLU(x W_gate) * (x W_up))
// W_down; section "Quantization": IQ4_NL blocks of 32 weights, one fp16 scale
// d and 16 bytes of 4-bit indices into the printed 16-entry table; expert
// weights one contiguous 3-D tensor per projection).  Also serves the plain
// IQ4_NL product (one "expert", m tokens in order).
//
// One CTA per work item = (expert, S sources): with IQ_SWIGLU the gate and
// up tiles of S/2 neighbouring 16-row tiles, otherwise S neighbouring 16-row
// tiles of the matrix.  The CTA's WPC warps split k into ranges of SPW
// super-steps (128 k = four 18-byte blocks per row); in a super-step lane
// (grp, tig) owns block 4s + tig of rows grp and grp+8 of every source.  Each
// lane issues all of its weight loads at once (S * SPW * 2 blocks, each read
// as the 24-byte window around it with 16- and 8-byte streaming loads that do
// not allocate in L1), so a CTA has its whole item in flight, the way the FP4
// register GEMV keeps HBM busy.  The IQ4_NL kernels are bound by L1
// wavefronts rather than by DRAM or issue, so the weight loads are as wide as
// the 18-byte blocks allow (two or three loads per block instead of five
// 4-byte ones).  Measured slower and left out: 256-bit activation loads
// (their aligned 8-register destinations made the kernel spill) and a
// byte-permute codebook in registers instead of the table (about 1.5x the
// decode instructions cost more than the table's wavefronts).
// When the routing makes it likely that every expert has pairs, the loads are
// issued before griddepcontrol.wait (programmatic dependent launch) and
// overlap the routing kernel; otherwise after it, once the expert is known to
// have pairs.
//
// Decode: every index byte j becomes the pair (w_j, w_{j+16}) = d * (kv[lo],
// kv[hi]) through a 256-entry table of exact f16x2 pairs replicated across the
// 32 shared-memory banks and one f16x2 multiply (the bit-exact decoded
// weights); legacy m16n8k16 MMAs multiply them with up to 16 gathered token
// rows, whose fragments all S sources share.  The WPC partial sums meet in
// shared memory and are added in warp order (deterministic); token groups
// beyond 16 pairs re-decode the weights still held in registers.
//
// Epilogues (IQ_* modes of k_grouped.cuh): fp16 product; SiLU(gate) * up in
// fp32 (SiLU(z) = z / (1 + e^-z)); or g-scaled fp32 for the down projection.
#pragma once
#include "k_grouped.cuh"
#include "qmm_dev.cuh"

namespace qmm {

// The bank-replicated pair table in device memory, generated at compile
// time: entry (v, lane) at word 32 v + lane is the f16x2 pair (kv[v & 15],
// kv[v >> 4]) of the printed IQ4_NL table (every value an integer, so its
// fp16 is exact).  A CTA brings it into shared memory with one bulk copy
// instead of 2048 stores and conversions.
constexpr int8_t kIqKv[16] = {-127, -104, -83, -65, -49, -35, -22, -10, 1, 13, 25, 38, 53, 69, 89, 113};
constexpr uint32_t iq_f16_of_int(int v) {  // fp16 bits of a small integer (|v| < 2048), exact
  if (v == 0) return 0u;
  const uint32_t sgn = v < 0 ? 0x8000u : 0u;
  uint32_t a = (uint32_t)(v < 0 ? -v : v);
  int e = 0;
  while ((a >> (e + 1)) != 0u) e++;                       // a in [2^e, 2^(e+1))
  const uint32_t mant = ((a << 10) >> e) & 0x3FFu;        // the 10 fraction bits (exact: e <= 10)
  return sgn | ((uint32_t)(e + 15) << 10) | mant;
}
struct IqPairTable {
  uint32_t w[256 * 32];
  constexpr IqPairTable() : w() {
    for (int i = 0; i < 256 * 32; i++) {
      const int v = i >> 5;
      w[i] = iq_f16_of_int(kIqKv[v & 15]) | (iq_f16_of_int(kIqKv[v >> 4]) << 16);
    }
  }
};
__device__ __align__(128) const IqPairTable g_iq_pair_table = IqPairTable();

constexpr int kIqtGroup = 16;      // token slots per pass (two MMA n-tiles)
constexpr int kIqtMaxPairs = 1024;  // in-kernel routing: at most this many (token, slot) pairs
// ... and the dispatch uses it up to one warp's worth: warp 0 reads the ids
// 32 at a time, each read after the previous ballot, so at 256 pairs (64
// tokens, top-4) the eight dependent reads per CTA cost more than the routing
// pass they replace (routed experts 108 vs 92 us); at 4 pairs it saves the
// pass (MoE block t = 1 34.9 vs 36.1 us).
constexpr int kIqtInKernelRoutePairs = 32;

struct IqtArgs {
  const uint8_t* data0;  // expert stack (gate when IQ_SWIGLU)
  const uint8_t* data1;  // IQ_SWIGLU: the up stack
  int64_t dstride0, dstride1;
  const uint16_t* x;
  int x_per_pair, topk;
  const int32_t* offsets;  // [E+1] pair offsets per expert (nullptr: plain product of m_plain rows, or ids)
  const int32_t* perm;     // [P] pair ids sorted by expert
  const int32_t* ids;      // [P] expert of each pair: the CTA finds its expert's pairs itself (offsets unused)
  int P;
  int m_plain;
  void* y;
  const float* gw;  // IQ_SCALED_F32: per-pair weights
  int n, k, E;
  int items_per_expert;  // CTAs per expert
  int spec;              // 1: weight loads before the dependency wait
  int compact;           // ids with P <= 32 and P < E: CTA slot j takes the j-th distinct expert in the ids
  int withhold;          // test switch (qmm_debug_set, from the host): the bulk copies are not issued
};

// Shared memory: the pair table, then the partial sums [warp][source][slot][row].
__host__ __device__ constexpr uint32_t iqt_smem_bytes(int S, int wpc) {
  return (uint32_t)kIqLutBytes + (uint32_t)wpc * (uint32_t)S * kIqtGroup * 16u * 4u;
}

// A block's scale as f16x2 (d, d) and its index word i from its five words,
// without a divergent branch: an odd block starts 2 bytes into its first word
// (a funnel shift by 32, clamped, is the next word).
__device__ __forceinline__ uint32_t iqt_scale(const uint32_t (&w)[5], uint32_t fs) {
  const uint32_t d = (w[0] >> (fs - 16u)) & 0xFFFFu;
  return d | (d << 16);
}
__device__ __forceinline__ uint32_t iqt_qword(const uint32_t (&w)[5], int i, uint32_t fs) {
  return __funnelshift_rc(w[i], w[i + 1], fs);
}

// One super-step of all S sources (block blk of rows grp, grp+8) against the
// same 32 k of token columns grp (xr0) and grp+8 (xr1).
template <int S, int NT>
__device__ __forceinline__ void iqt_step(float (&acc)[S][2][4], const uint32_t (&win)[S][2][6], int tig,
                                         const uint16_t* xr0, const uint16_t* xr1, int blk, uint32_t lut_lane) {
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
  // the block's five words: the 8-byte-aligned window holds it 2*tig bytes in
  uint32_t w[S][2][5];
#pragma unroll
  for (int s = 0; s < S; s++)
#pragma unroll
    for (int r = 0; r < 2; r++)
#pragma unroll
      for (int i = 0; i < 5; i++) w[s][r][i] = (tig & 2) ? win[s][r][i + 1] : win[s][r][i];
  const uint32_t fs = (tig & 1) ? 32u : 16u;
  uint32_t dd[S][2];
#pragma unroll
  for (int s = 0; s < S; s++)
#pragma unroll
    for (int r = 0; r < 2; r++) dd[s][r] = iqt_scale(w[s][r], fs);
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
    for (int s = 0; s < S; s++) {
      const uint32_t qwa = iqt_qword(w[s][0], i >> 1, fs), qwb = iqt_qword(w[s][1], i >> 1, fs);
      const uint32_t a0 = hmul2(lds32(lut_addr(qwa, bs, lut_lane)), dd[s][0]);
      const uint32_t a2 = hmul2(lds32(lut_addr(qwa, bs + 1, lut_lane)), dd[s][0]);
      const uint32_t a1 = hmul2(lds32(lut_addr(qwb, bs, lut_lane)), dd[s][1]);
      const uint32_t a3 = hmul2(lds32(lut_addr(qwb, bs + 1, lut_lane)), dd[s][1]);
#pragma unroll
      for (int j = 0; j < NT; j++) mma_16816(acc[s][j], a0, a1, a2, a3, b0[j], b1[j]);
    }
  }
}

// The 24-byte window that holds block blk of a row: it starts at the
// block's offset rounded down to 8 bytes (18 * blk mod 8 = 2 * tig, the row
// starts 8-byte aligned), so the block sits 2*tig bytes in.  W16 (rows
// 16-byte aligned, k % 256 == 0): the window is a 16-byte and an 8-byte load
// (in the order its alignment allows: 72 * s mod 16 = 8 * (s mod 2)),
// otherwise three 8-byte loads.
template <bool W16>
__device__ __forceinline__ void iqt_window(uint32_t (&win)[6], const uint8_t* row, int blk, int s) {
  const uint8_t* p = row + (((int64_t)blk * 18) & ~(int64_t)7);
  if (W16 && !(s & 1)) {
    const uint4 a = ldg_stream128(p);
    const uint2 b = ldg_stream64(p + 16);
    win[0] = a.x; win[1] = a.y; win[2] = a.z; win[3] = a.w; win[4] = b.x; win[5] = b.y;
  } else if (W16) {
    const uint2 a = ldg_stream64(p);
    const uint4 b = ldg_stream128(p + 8);
    win[0] = a.x; win[1] = a.y; win[2] = b.x; win[3] = b.y; win[4] = b.z; win[5] = b.w;
  } else {
    const uint2 a = ldg_stream64(p), b = ldg_stream64(p + 8), c = ldg_stream64(p + 16);
    win[0] = a.x; win[1] = a.y; win[2] = b.x; win[3] = b.y; win[4] = c.x; win[5] = c.y;
  }
}

// The same 24-byte window read from the CTA's shared-memory copy of the tile
// (row = shared address of the row; rows 16-byte aligned when W16, so the
// window's alignment is the global one).
template <bool W16>
__device__ __forceinline__ void iqt_window_smem(uint32_t (&win)[6], uint32_t row, int blk, int s) {
  const uint32_t p = row + ((uint32_t)(blk * 18) & ~7u);
  if (W16 && !(s & 1)) {
    const uint4 a = lds128(p);
    const uint2 b = lds64(p + 16);
    win[0] = a.x; win[1] = a.y; win[2] = a.z; win[3] = a.w; win[4] = b.x; win[5] = b.y;
  } else if (W16) {
    const uint2 a = lds64(p);
    const uint4 b = lds128(p + 8);
    win[0] = a.x; win[1] = a.y; win[2] = b.x; win[3] = b.y; win[4] = b.z; win[5] = b.w;
  } else {
    const uint2 a = lds64(p), b = lds64(p + 8), c = lds64(p + 16);
    win[0] = a.x; win[1] = a.y; win[2] = b.x; win[3] = b.y; win[4] = c.x; win[5] = c.y;
  }
}

template <int S, int SPW, bool W16>
__device__ __forceinline__ void iqt_load_smem(uint32_t (&w)[SPW][S][2][6], const uint32_t (&rs)[S][2], int s0,
                                              int tig) {
#pragma unroll
  for (int u = 0; u < SPW; u++) {
    const int blk = 4 * (s0 + u) + tig;
#pragma unroll
    for (int s = 0; s < S; s++)
#pragma unroll
      for (int r = 0; r < 2; r++) iqt_window_smem<W16>(w[u][s][r], rs[s][r], blk, s0 + u);
  }
}

template <int S, int SPW, bool W16>
__device__ __forceinline__ void iqt_load(uint32_t (&w)[SPW][S][2][6], const uint8_t* const (&rp)[S][2], int s0,
                                         int tig) {
#pragma unroll
  for (int u = 0; u < SPW; u++) {
    const int blk = 4 * (s0 + u) + tig;
#pragma unroll
    for (int s = 0; s < S; s++)
#pragma unroll
      for (int r = 0; r < 2; r++) iqt_window<W16>(w[u][s][r], rp[s][r], blk, s0 + u);
  }
}

// Threads a CTA of this register budget may have.
__host__ __device__ constexpr int iqt_max_threads(int maxreg) { return (65536 / maxreg) & ~31; }

// In-kernel routing (a.ids): warp 0 collects the pairs p whose id is this
// CTA's expert, in increasing p (the order of the stable routing sort), into
// shared memory; any id outside [0, E) raises ERR_BAD_EXPERT and is left out.
// Compact grids (a.compact, P <= 32): the CTA's expert slot e is replaced by
// the e-th distinct valid id in order of first occurrence (none: -1, no
// pairs), so only as many experts' CTAs are launched as there are pairs.
// Returns the count to every thread and e through *s_e (ends with a barrier).
__device__ __forceinline__ int iqt_collect_pairs(const IqtArgs& a, int& e, int* s_pairs, int* s_cnt, int* s_e) {
  if ((threadIdx.x >> 5) == 0) {
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    if (a.compact) {
      const int id = lane < a.P ? a.ids[lane] : -1;
      const bool valid = lane < a.P && id >= 0 && id < a.E;
      const unsigned same = __match_any_sync(0xFFFFFFFFu, valid ? id : -1 - lane);  // invalid lanes: own keys
      const bool first = valid && (__ffs(same) - 1) == lane;
      const unsigned firsts = __ballot_sync(0xFFFFFFFFu, first);
      const unsigned mine = __ballot_sync(0xFFFFFFFFu, first && __popc(firsts & lt) == e);
      const int ej = mine ? __shfl_sync(0xFFFFFFFFu, id, __ffs(mine) - 1) : -1;
      const unsigned mask = __ballot_sync(0xFFFFFFFFu, valid && id == ej && ej >= 0);
      if (valid && id == ej && ej >= 0) s_pairs[__popc(mask & lt)] = lane;
      const bool bad = lane < a.P && !valid;
      if (__any_sync(0xFFFFFFFFu, bad) && lane == 0 && e == 0 && blockIdx.x == 0) raise_error(ERR_BAD_EXPERT);
      if (lane == 0) {
        *s_cnt = __popc(mask);
        *s_e = ej;
      }
    } else {
      int n = 0;
      bool bad = false;
      for (int p0 = 0; p0 < a.P; p0 += 32) {
        const int p = p0 + lane;
        const int id = p < a.P ? a.ids[p] : -1;
        bad |= p < a.P && (id < 0 || id >= a.E);
        const unsigned mask = __ballot_sync(0xFFFFFFFFu, id == e);
        if (id == e) s_pairs[n + __popc(mask & lt)] = p;
        n += __popc(mask);
      }
      if (__any_sync(0xFFFFFFFFu, bad) && lane == 0 && e == 0 && blockIdx.x == 0) raise_error(ERR_BAD_EXPERT);
      if (lane == 0) {
        *s_cnt = n;
        *s_e = e;
      }
    }
  }
  __syncthreads();
  e = *s_e;
  return *s_cnt;
}

// STG: the item's tiles (16 rows of each source, one contiguous byte range
// each) are brought into shared memory by the copy engine (one bulk copy per
// source, completing on an mbarrier) instead of each lane loading its
// windows from global memory: a warp's window loads from global memory touch
// eight rows' lines each and were the largest share of the L1 data-pipe
// wavefronts; from shared memory a 16-byte window load of eight rows costs
// the minimum four.  The copies are issued when the global loads would have
// been (before the dependency wait when speculative), and every exit waits
// for them, so no copy is in flight when the CTA leaves.
template <int MODE, int S, int SPW, int MAXREG, bool W16, bool STG = false>
__global__ void __launch_bounds__(iqt_max_threads(MAXREG)) __maxnreg__(MAXREG) iq4_tile_kernel(const IqtArgs a) {
  __shared__ int s_pairs[kIqtMaxPairs];
  __shared__ int s_cnt, s_e;
  __shared__ __align__(8) unsigned long long s_wbar;
  static_assert(MODE != IQ_SWIGLU || S % 2 == 0, "SwiGLU items are gate and up tiles of the same rows");
  constexpr int kOut = (MODE == IQ_SWIGLU) ? S / 2 : S;  // output tiles per item
  extern __shared__ __align__(16) uint8_t smem_iqt[];
  const uint32_t lut = smem_addr(smem_iqt);
  float* red = reinterpret_cast<float*>(smem_iqt + kIqLutBytes);  // [warp][source][slot][row]
  const int wpc = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, grp = lane >> 2, tig = lane & 3;
  int e = blockIdx.x / a.items_per_expert;  // compact grids: a slot, made an expert by iqt_collect_pairs
  const int item = blockIdx.x - e * a.items_per_expert;
  const int64_t rowb = (int64_t)(a.k >> 5) * 18;
  // STG: shared-memory copy of the sources after the table and the partial
  // sums; source s holds its 16 rows contiguously (rows past n hold stale
  // bytes: their outputs are never stored)
  const uint32_t stage = lut + (uint32_t)kIqLutBytes + (uint32_t)wpc * S * kIqtGroup * 16u * 4u;
  const uint32_t wbar = smem_addr(&s_wbar);
  auto issue_copies = [&]() {  // thread 0
    uint32_t bytes[S];
    uint32_t total = 0;
#pragma unroll
    for (int s = 0; s < S; s++) {
      const int r0 = (MODE == IQ_SWIGLU) ? (item * kOut + (s >> 1)) * 16 : (item * S + s) * 16;
      const int rows = max(0, min(16, a.n - r0));
      bytes[s] = (uint32_t)(rows * rowb);
      total += bytes[s];
    }
    mbar_arrive_expect_tx(wbar, total + (uint32_t)kIqLutBytes);
    if (a.withhold) return;  // test switch: the copies never come
    bulk_load(lut, &g_iq_pair_table, (uint32_t)kIqLutBytes, wbar);
#pragma unroll
    for (int s = 0; s < S; s++) {
      if (!bytes[s]) continue;
      const int r0 = (MODE == IQ_SWIGLU) ? (item * kOut + (s >> 1)) * 16 : (item * S + s) * 16;
      const uint8_t* base = (MODE == IQ_SWIGLU && (s & 1)) ? a.data1 + (int64_t)e * a.dstride1
                                                            : a.data0 + (int64_t)e * a.dstride0;
      bulk_load(stage + (uint32_t)s * 16u * (uint32_t)rowb, base + (int64_t)r0 * rowb, bytes[s], wbar);
    }
  };
  if (STG && threadIdx.x == 0) {
    mbar_init(wbar, 1);
    fence_mbar_init();
    if (a.spec) issue_copies();
  }
  pdl_launch_dependents();
  int start = 0, cnt = a.m_plain;
  if (!a.spec) {  // most experts may be empty: find out before any other work
    pdl_wait();
    if (a.ids) {
      cnt = iqt_collect_pairs(a, e, s_pairs, &s_cnt, &s_e);
    } else if (a.offsets) {
      start = a.offsets[e];
      cnt = a.offsets[e + 1] - start;
    }
    if (cnt <= 0) return;
    if (STG && threadIdx.x == 0) issue_copies();
  }
  // pair table: entry v (an index byte) = (kv[v & 15], kv[v >> 4]) as f16x2,
  // one copy per bank; each store covers four banks (STG: copied in with the
  // tiles instead)
  for (int i = threadIdx.x; !STG && i < 256 * 8; i += blockDim.x) {
    const int v = i >> 3;
    const uint32_t lo = __half_as_ushort(__int2half_rn(c_iq4nl_kv[v & 15]));
    const uint32_t hi = __half_as_ushort(__int2half_rn(c_iq4nl_kv[v >> 4]));
    const uint32_t p = lo | (hi << 16);
    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(lut + 16u * i), "r"(p) : "memory");
  }
  // rows grp and grp+8 of every source (clamped to n-1: a source past n
  // re-reads the last row and stores nothing)
  int row0[S];
  const uint8_t* rp[S][2];
#pragma unroll
  for (int s = 0; s < S; s++) {
    const uint8_t* base;
    if (MODE == IQ_SWIGLU) {  // sources 2q, 2q+1: gate and up of output tile q
      row0[s] = (item * kOut + (s >> 1)) * 16;
      base = ((s & 1) ? a.data1 + (int64_t)e * a.dstride1 : a.data0 + (int64_t)e * a.dstride0);
    } else {
      row0[s] = (item * S + s) * 16;
      base = a.data0 + (int64_t)e * a.dstride0;
    }
    rp[s][0] = base + (int64_t)min(row0[s] + grp, a.n - 1) * rowb;
    rp[s][1] = base + (int64_t)min(row0[s] + grp + 8, a.n - 1) * rowb;
  }
  const int s0 = warp * SPW;
  uint32_t w[SPW][S][2][6];
  if (a.spec) {
    if (!STG) iqt_load<S, SPW, W16>(w, rp, s0, tig);
    pdl_wait();  // routing, activations and the output buffer follow the previous kernel
    if (a.ids) {
      cnt = iqt_collect_pairs(a, e, s_pairs, &s_cnt, &s_e);
    } else if (a.offsets) {
      start = a.offsets[e];
      cnt = a.offsets[e + 1] - start;
    }
    if (cnt <= 0) {  // the whole CTA (cnt is the same in every thread): an expert without pairs
      if (STG) {       // let our copies land before leaving
        __syncthreads();  // (the barrier's initialisation is visible to every thread)
        mbar_wait(wbar, 0);
      }
      return;
    }
  } else if (!STG) {
    iqt_load<S, SPW, W16>(w, rp, s0, tig);
  }
  __syncthreads();  // the pair table is complete
  if (STG) {
    // the copies have landed (a wait that runs out raises the error word; the
    // CTA still waits, bounded again, before it reads or leaves)
    if (!mbar_wait(wbar, 0)) mbar_wait(wbar, 0);
    uint32_t rs[S][2];
#pragma unroll
    for (int s = 0; s < S; s++) {
      rs[s][0] = stage + (uint32_t)(s * 16 + grp) * (uint32_t)rowb;
      rs[s][1] = rs[s][0] + 8u * (uint32_t)rowb;
    }
    iqt_load_smem<S, SPW, W16>(w, rs, s0, tig);
  }
  const uint32_t lut_lane = lut + 4u * lane;

  for (int g0 = 0; g0 < cnt; g0 += kIqtGroup) {
    const int ng = min(kIqtGroup, cnt - g0);
    // activation rows of token columns grp and grp+8 (columns past ng read
    // the group's first row; their outputs are never stored)
    const uint16_t* xr[2];
#pragma unroll
    for (int j = 0; j < 2; j++) {
      const int slot = (grp + 8 * j < ng) ? grp + 8 * j : 0;
      const int pr = a.ids ? s_pairs[g0 + slot] : a.offsets ? a.perm[start + g0 + slot] : g0 + slot;
      const int row = ((a.ids || a.offsets) && !a.x_per_pair) ? pr / a.topk : pr;
      xr[j] = a.x + (int64_t)row * a.k;
    }
    float acc[S][2][4];
#pragma unroll
    for (int s = 0; s < S; s++)
#pragma unroll
      for (int j = 0; j < 2; j++)
#pragma unroll
        for (int c = 0; c < 4; c++) acc[s][j][c] = 0.f;
    if (ng <= 8) {
#pragma unroll
      for (int u = 0; u < SPW; u++) iqt_step<S, 1>(acc, w[u], tig, xr[0], xr[1], 4 * (s0 + u) + tig, lut_lane);
    } else {
#pragma unroll
      for (int u = 0; u < SPW; u++) iqt_step<S, 2>(acc, w[u], tig, xr[0], xr[1], 4 * (s0 + u) + tig, lut_lane);
    }
    // partial sums: red[warp][s][slot][row]; acc[s][j][c] is row grp (c < 2)
    // or grp+8, token slot 8j + 2tig + (c & 1)
#pragma unroll
    for (int s = 0; s < S; s++) {
      float* r = red + ((warp * S + s) * kIqtGroup) * 16;
#pragma unroll
      for (int j = 0; j < 2; j++) {
        const int t0 = 8 * j + 2 * tig;
        r[t0 * 16 + grp] = acc[s][j][0];
        r[(t0 + 1) * 16 + grp] = acc[s][j][1];
        r[t0 * 16 + grp + 8] = acc[s][j][2];
        r[(t0 + 1) * 16 + grp + 8] = acc[s][j][3];
      }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < kOut * 16 * ng; idx += blockDim.x) {
      const int row = idx & 15, slot = (idx >> 4) % ng, q = (idx >> 4) / ng;
      const int grow = (item * kOut + q) * 16 + row;
      if (grow >= a.n) continue;
      const int sv = (MODE == IQ_SWIGLU) ? 2 * q : q;  // source of the value (the gate for SwiGLU)
      float v = 0.f, u = 0.f;
      for (int wi = 0; wi < wpc; wi++) {
        v += red[((wi * S + sv) * kIqtGroup + slot) * 16 + row];
        if (MODE == IQ_SWIGLU) u += red[((wi * S + sv + 1) * kIqtGroup + slot) * 16 + row];
      }
      const int64_t pr = a.ids ? s_pairs[g0 + slot] : a.offsets ? a.perm[start + g0 + slot] : g0 + slot;
      if (MODE == IQ_SCALED_F32) {
        static_cast<float*>(a.y)[pr * a.n + grow] = a.gw[pr] * v;
      } else if (MODE == IQ_SWIGLU) {
        static_cast<uint16_t*>(a.y)[pr * a.n + grow] = f32_to_f16_bits(v / (1.0f + expf(-v)) * u);
      } else {
        static_cast<uint16_t*>(a.y)[pr * a.n + grow] = f32_to_f16_bits(v);
      }
    }
    __syncthreads();  // red is reused by the next token group
  }
}

}  // namespace qmm
