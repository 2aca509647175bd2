// k_gemm.cuh -- prefill GEMM on packed FP4-G16 weights with 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// Y[m][n] = sum_k X[m][k] W[n][k] for a prefill window (m = 2048 tokens in
// the model card's evaluation protocol, "Mamb2_8B_FP4_Recall_SQ3.25",
// section "Measured quality": windows of up to 2,048 targets).
//
// One CTA computes a 128 x BN tile of Y (128 tokens x BN weight rows).  Per
// 64-wide k step:
//   * warp 0 (one thread) loads the X tile [128 x 64] fp16 with a 2-D tensor
//     map, 128-byte swizzle -- the canonical K-major operand layout;
//   * warps 2-9 (256 threads, one weight row each) copy the packed codes and
//     scales of their row into a private cp.async ring PSLOTS steps ahead,
//     decode them to fp16 (E2M1 -> f16x2 convert, one multiply by the group
//     scale = the bit-exact dequantised weight) and store them into shared
//     memory in the same swizzled K-major layout;
//   * warp 1 (one thread) issues four tcgen05.mma (M=128, N=BN, K=16) per
//     step from the two shared-memory descriptors into the fp32 accumulator
//     in tensor memory and commits them to the stage's "empty" barrier.
// A ring of STAGES stages decouples the three.  After the last step the MMA
// thread commits to an "accumulator ready" barrier and warps 2-9 read the
// accumulator with tcgen05.ld (warp w owns TMEM lanes 32*(w%4).. = 32 tokens
// and half of the columns), round to fp16 and store Y.
//
// No TMA multicast is used.  Every wait is bounded (%globaltimer); on a
// timeout the kernel raises the error word, drains its own copies and MMAs,
// frees its tensor memory and returns.
#pragma once
#include "qmm_dev.cuh"

namespace qmm {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmDecodeWarps = 8;
constexpr int kGemmThreads = (2 + kGemmDecodeWarps) * 32;
constexpr int kGemmDecodeThreads = kGemmDecodeWarps * 32;
constexpr int kGemmPSlots = 5;  // packed-weight prefetch ring depth (k steps)

template <int BN, int STAGES>
struct GemmCfg {
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;  // 16 KB
  static constexpr int kBBytes = BN * kGemmBK * 2;        // 32 KB at BN=256
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = BN;                    // fp32 accumulator columns
  // packed ring slot: codes bytes 0-15 [BN][16], bytes 16-31 [BN][16], scales [BN][8]
  static constexpr int kPCodesHi = BN * 16, kPScales = 2 * BN * 16, kPSlotBytes = 2 * BN * 16 + BN * 8;
  static size_t smem_bytes() {
    return 1024 + (size_t)STAGES * kStageBytes + (size_t)kGemmPSlots * kPSlotBytes + 256;
  }
};

// --- tcgen05 wrappers --------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once all tcgen05.mma issued so far by this thread complete.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 B, 8-row groups 1024 B apart (SBO), LBO unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc_k128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Instruction descriptor, kind::f16: fp16 A and B (K-major), fp32 D, M=128.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void cp_async16_g(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8_g(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4_g(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit_g() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_g(int) {
  asm volatile("cp.async.wait_group %0;" ::"n"(kGemmPSlots - 1) : "memory");
}

// Copy the packed codes (32 bytes) and scales (8 or 4 bytes) of weight row
// `row` for the k step starting at k0 into this thread's ring slot.  Rows
// past n copy row n-1 (their outputs are never stored).
template <int FMT, int BN>
__device__ __forceinline__ void copy_rowpack(uint32_t slot, int t, const uint8_t* __restrict__ codes,
                                             const uint8_t* __restrict__ scales, int64_t row, int n, int k, int k0) {
  const int64_t r = row < n ? row : (int64_t)n - 1;
  const uint8_t* cp = codes + r * (int64_t)(k >> 1) + (k0 >> 1);
  cp_async16_g(slot + t * 16, cp);
  cp_async16_g(slot + BN * 16 + t * 16, cp + 16);
  if (FMT == 2) cp_async8_g(slot + 2 * BN * 16 + t * 8, scales + (r * (int64_t)(k >> 4) + (k0 >> 4)) * 2);
  else cp_async4_g(slot + 2 * BN * 16 + t * 8, scales + r * (int64_t)(k >> 4) + (k0 >> 4));
}

// Decode this thread's row (64 weights) from its ring slot and store it as 8
// swizzled 16-byte chunks of the B stage; rows past n store zeros.
template <int FMT, int BN>
__device__ __forceinline__ void store_row(uint32_t slot, int t, bool valid, uint32_t b_stage, int r) {
  const uint4 c0 = lds128(slot + t * 16), c1 = lds128(slot + BN * 16 + t * 16);
  const uint2 sv = lds64(slot + 2 * BN * 16 + t * 8);
  uint32_t sc[4];  // f16x2 broadcast scale per group of 16 (= two chunks)
  if (FMT == 2) {
    sc[0] = bcast_lo(sv.x); sc[1] = bcast_hi(sv.x); sc[2] = bcast_lo(sv.y); sc[3] = bcast_hi(sv.y);
  } else {
    const uint32_t e01 = e4m3x2_to_f16x2(sv.x & 0xFFFFu), e23 = e4m3x2_to_f16x2(sv.x >> 16);
    sc[0] = bcast_lo(e01); sc[1] = bcast_hi(e01); sc[2] = bcast_lo(e23); sc[3] = bcast_hi(e23);
  }
  if (!valid) sc[0] = sc[1] = sc[2] = sc[3] = 0u;
  const uint32_t q[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const uint32_t row_base = b_stage + (uint32_t)r * 128u;
  const uint32_t sw = (uint32_t)(r & 7);
#pragma unroll
  for (int c = 0; c < 8; c++) {  // chunk c = k 8c .. 8c+7 = code word q[c]
    uint32_t w[4];
    e2m1x8_to_f16x2(q[c], w);
    const uint32_t s = sc[c >> 1];
    sts128(row_base + ((c ^ sw) << 4), hmul2(w[0], s), hmul2(w[1], s), hmul2(w[2], s), hmul2(w[3], s));
  }
}

template <int FMT, int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_fp4_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const uint8_t* __restrict__ codes,
                       const uint8_t* __restrict__ scales, uint16_t* __restrict__ y, int m, int n, int k, float g) {
  using C = GemmCfg<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  const uint32_t a_s = base;                                  // STAGES x 16 KB
  const uint32_t b_s = a_s + STAGES * C::kABytes;             // STAGES x BN*128 B
  const uint32_t p_s = b_s + STAGES * C::kBBytes;             // packed ring, kGemmPSlots slots
  const uint32_t bars = p_s + kGemmPSlots * C::kPSlotBytes;   // full[S], empty[S], accum
  const uint32_t tmem_slot = bars + 8 * (2 * STAGES + 1);
  uint32_t* tmem_slot_ptr = reinterpret_cast<uint32_t*>(smem_raw + (tmem_slot - smem_addr(smem_raw)));
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (n + BN - 1) / BN;
  const int tile_n = blockIdx.x % n_tiles, tile_m = blockIdx.x / n_tiles;
  const int m0 = tile_m * kGemmBM, n0 = tile_n * BN;
  const int ksteps = k / kGemmBK;
  // the last weight-row tile may be half as wide: issue N = 128 there
  const int n_valid = min(BN, n - n0);
  const int n_mma = (n_valid <= BN / 2) ? BN / 2 : BN;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; s++) {
      mbar_init(bars + 8 * s, 1 + kGemmDecodeThreads);  // full: TMA arrive(+tx) + decode threads
      mbar_init(bars + 8 * (STAGES + s), 1);             // empty: MMA commit
    }
    mbar_init(bars + 8 * (2 * STAGES), 1);               // accumulator ready
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot_ptr;
  const uint32_t accum_bar = bars + 8 * (2 * STAGES);

  if (warp == 0) {
    // ---------------------------- X loader --------------------------------
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      int issued = 0;
      const int kissue = (g_test_flags & kTestWithholdXTiles) ? 0 : ksteps;  // test switch: issue nothing
      for (int ks = 0; ks < kissue; ks++) {
        const int s = ks % STAGES;
        const uint32_t ph = (uint32_t)(ks / STAGES) & 1u;
        if (s_abort || !mbar_wait(bars + 8 * (STAGES + s), ph ^ 1u)) { s_abort = 1; break; }
        mbar_arrive_expect_tx(bars + 8 * s, C::kABytes);
        tma_load_2d(a_s + s * C::kABytes, &tm_x, ks * kGemmBK, m0, bars + 8 * s);
        issued++;
      }
      // drain: the last use of every stage must have landed
      for (int s = 0; s < STAGES && s < issued; s++) {
        const int last = issued - 1 - ((issued - 1 - s) % STAGES);
        mbar_wait(bars + 8 * s, (uint32_t)(last / STAGES) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------------------- MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(n_mma);
      for (int ks = 0; ks < ksteps; ks++) {
        const int s = ks % STAGES;
        const uint32_t ph = (uint32_t)(ks / STAGES) & 1u;
        if (s_abort || !mbar_wait(bars + 8 * s, ph)) { s_abort = 1; break; }
        tc_fence_after();
        const uint64_t da = umma_desc_k128(a_s + s * C::kABytes);
        const uint64_t db = umma_desc_k128(b_s + s * C::kBBytes);
#pragma unroll
        for (int kk = 0; kk < kGemmBK / 16; kk++)  // +32 bytes per K=16 inside the swizzle row
          umma_f16(tmem, da + (uint64_t)(2 * kk), db + (uint64_t)(2 * kk), idesc, (ks | kk) != 0);
        umma_commit(bars + 8 * (STAGES + s));  // frees the stage when these MMAs are done
      }
      umma_commit(accum_bar);  // all issued MMAs complete -> accumulator ready
    }
  } else {
    // ---------------------- decode producers + epilogue ----------------------
    const int t = threadIdx.x - 64;  // 0..255: weight row t of the tile
    const int64_t row = (int64_t)n0 + t;
    const bool valid = row < n;
    // prologue: the first kGemmPSlots-1 steps in flight
#pragma unroll 1
    for (int j = 0; j < kGemmPSlots - 1; j++) {
      if (j < ksteps) copy_rowpack<FMT, BN>(p_s + j * C::kPSlotBytes, t, codes, scales, row, n, k, j * kGemmBK);
      cp_commit_g();
    }
    for (int ks = 0; ks < ksteps; ks++) {
      const int s = ks % STAGES;
      const uint32_t ph = (uint32_t)(ks / STAGES) & 1u;
      const int jn = ks + kGemmPSlots - 1;  // step to prefetch now
      if (jn < ksteps)
        copy_rowpack<FMT, BN>(p_s + (jn % kGemmPSlots) * C::kPSlotBytes, t, codes, scales, row, n, k, jn * kGemmBK);
      cp_commit_g();
      cp_wait_g(0);  // this thread's copies of step ks have landed
      if (s_abort || !mbar_wait(bars + 8 * (STAGES + s), ph ^ 1u)) { s_abort = 1; break; }
      store_row<FMT, BN>(p_s + (ks % kGemmPSlots) * C::kPSlotBytes, t, valid, b_s + s * C::kBBytes, t);
      fence_proxy_async_shared();  // generic-proxy stores -> visible to the tensor core
      mbar_arrive(bars + 8 * s);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    // epilogue: warp w owns TMEM lanes 32*(w%4) .. (tokens) and column half (w-2)/4
    const bool ready = mbar_wait(accum_bar, 0);
    tc_fence_after();
    if (ready && !s_abort) {
      const int q = warp & 3, half = (warp - 2) >> 2;
      const int mrow = m0 + 32 * q + lane;
      const float gs = (FMT == 3) ? g : 1.0f;
      const int ncols = n_mma / 2;  // columns of this warp
      for (int j = 0; j < ncols / 32; j++) {
        const int c0 = half * ncols + 32 * j;
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, r);
        tmem_ld_wait();
        const int col = n0 + c0;
        if (mrow < m && col < n) {
          uint32_t h[16];
#pragma unroll
          for (int i = 0; i < 16; i++)
            h[i] = f32x2_to_f16x2(__uint_as_float(r[2 * i]) * gs, __uint_as_float(r[2 * i + 1]) * gs);
          uint16_t* yp = y + (int64_t)mrow * n + col;
          if (col + 32 <= n && (n & 7) == 0) {
            uint4* y4 = reinterpret_cast<uint4*>(yp);
#pragma unroll
            for (int i = 0; i < 4; i++) y4[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
          } else {
            for (int i = 0; i < 32 && col + i < n; i++) yp[i] = (uint16_t)((h[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
          }
        }
      }
    }
  }

  // teardown: nothing of ours may still write shared or tensor memory
  if (warp == 1 && lane == 0 && s_abort) mbar_wait(accum_bar, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Persistent variant: one CTA per SM loops over tiles (tile = blockIdx.x +
// i * gridDim.x).  Tensor memory holds two 128 x 256 fp32 accumulators; the
// MMA thread fills accumulator i&1 while four epilogue warps (10-13) drain
// the other, so the store of tile i overlaps the main loop of tile i+1.  The
// operand ring and the decode warps' packed-weight prefetch run on across
// tile boundaries without a pause.  Barriers: full/empty per operand stage,
// acc_full/acc_empty per accumulator.
// ---------------------------------------------------------------------------
constexpr int kGemmPThreads = (2 + kGemmDecodeWarps + 4) * 32;
constexpr int kGemmChunkSteps = 4;  // k steps per cooperatively staged packed chunk (256 k)

// Staged packed chunk for BN=256 rows: codes [256][128 B] (16-byte unit u of
// row r at unit u ^ (r & 7), so the eight rows of a read phase hit eight
// different bank groups), then scales [256][32 B] (fp16: 16-byte half h at
// h ^ ((r >> 2) & 1); E4M3: the row's 16 bytes unswizzled).
constexpr int kStageCodes = 256 * 128;
constexpr int kStageScales = 256 * 32;
constexpr int kStageBytes = kStageCodes + kStageScales;

// IQ4_NL ("Mark-Experimental-V3-8B", section "Quantization": 18-byte blocks
// per 32 weights, fp16 d then 16 bytes of indices into the printed table):
// a 256-k chunk of a row is 8 blocks = 144 bytes, copied as 9 units into
// [256][144 B]; the 4 KB after them in staging slot 0 hold a 256-entry table
// of exact f16x2 pairs (kv[i & 15], kv[i >> 4]) in 4 bank-interleaved copies
// (copy c of entry i at word 4i + c; a thread reads copy lane & 3).
constexpr int kStageIq4Row = 144;
constexpr int kStageIq4Lut = 256 * kStageIq4Row;  // 36,864: table offset inside slot 0
static_assert(kStageIq4Lut + 256 * 4 * 4 <= kStageBytes, "IQ4_NL table fits in the staging slot");

// Decode the 16 index bytes Q[0..3] of one IQ4_NL block (scale dd, f16x2
// broadcast) into its 32 weights as four 8-weight chunks in k order: chunk 0
// = low nibbles of bytes 0..7 (weights 0..7), 1 = low of 8..15, 2 = high of
// 0..7 (weights 16..23), 3 = high of 8..15.  Two adjacent nibbles of the same
// kind form one table index, so each lookup yields two consecutive weights,
// exact; one f16x2 multiply by d rounds each once.
// LSH: log2 of a table entry's bytes (4 bytes per copy, 2^(LSH-2) copies).
template <int LSH = 4>
__device__ __forceinline__ void iq4_block_chunks(const uint32_t (&Q)[4], uint32_t dd, uint32_t lut_copy,
                                                 uint32_t (&out)[16]) {
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const uint32_t lo = Q[i] & 0x0F0F0F0Fu, hi = (Q[i] >> 4) & 0x0F0F0F0Fu;
    const uint32_t ul = lo | (lo >> 4), uh = hi | (hi >> 4);  // bytes 0 and 2: (n0 | n1 << 4), (n2 | n3 << 4)
    const uint32_t l0 = lds32(lut_copy + ((ul & 0xFFu) << LSH)), l1 = lds32(lut_copy + (((ul >> 16) & 0xFFu) << LSH));
    const uint32_t h0 = lds32(lut_copy + ((uh & 0xFFu) << LSH)), h1 = lds32(lut_copy + (((uh >> 16) & 0xFFu) << LSH));
    // bytes 4i..4i+3: low nibbles are weights 4i..4i+3, high ones 16+4i..
    out[(i >> 1) * 4 + (i & 1) * 2] = hmul2(l0, dd);
    out[(i >> 1) * 4 + (i & 1) * 2 + 1] = hmul2(l1, dd);
    out[8 + (i >> 1) * 4 + (i & 1) * 2] = hmul2(h0, dd);
    out[8 + (i >> 1) * 4 + (i & 1) * 2 + 1] = hmul2(h1, dd);
  }
}

__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// MH = 2: tiles of 256 tokens x BN = 128 weight rows, two M=128 MMAs per k16
// step that share the decoded weight tile and accumulate into two halves of
// the accumulator: half the weight decode per FLOP of MH = 1 (128 x 256),
// the same tensor memory (2 accumulators x 256 columns) and operand bytes
// per stage (32 + 16 KB instead of 16 + 32 KB).  With BN = 128 (either MH)
// decode thread t owns 32 of the 64 k of row t % 128.
template <int FMT, int BN, int STAGES, int MH = 1>
__global__ void __launch_bounds__(kGemmPThreads, 1)
    gemm_fp4_tc_persistent_kernel(const __grid_constant__ CUtensorMap tm_x, const uint8_t* __restrict__ codes,
                                  const uint8_t* __restrict__ scales, uint16_t* __restrict__ y, int m, int n, int k,
                                  float g) {
  using C = GemmCfg<BN, STAGES>;
  constexpr int TPR = kGemmDecodeThreads / BN;  // decode threads per weight row: 1, or 2 (32 k each)
  static_assert((TPR == 1 || TPR == 2) && BN * TPR == kGemmDecodeThreads, "one or two decode threads per row");
  // IQ4_NL pair table after the staged rows of slot 0: 16 word-interleaved
  // copies when 128 rows leave room (two lanes per copy), else 4
  constexpr int kLutC = (BN == 128) ? 16 : 4, kLutLsh = (BN == 128) ? 6 : 4;
  constexpr uint32_t kLutOff = (uint32_t)BN * kStageIq4Row;
  static_assert(kLutOff + 256u * kLutC * 4u <= (uint32_t)kStageBytes, "IQ4_NL table fits in staging slot 0");
  constexpr uint32_t kA = MH * C::kABytes;  // X bytes per stage
  constexpr int kBM = MH * kGemmBM;         // tokens per tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  const uint32_t a_s = base;
  const uint32_t b_s = a_s + STAGES * kA;
  const uint32_t p_s = b_s + STAGES * C::kBBytes;            // 2 staged packed chunks
  const uint32_t bars = p_s + 2 * kStageBytes;                // full[S] empty[S] accf[2] acce[2] done cf[2] ce[2]
  const uint32_t accf = bars + 8 * (2 * STAGES), acce = accf + 16, done_bar = acce + 16;
  const uint32_t cfull = done_bar + 8, cempty = cfull + 16;
  const uint32_t tmem_slot = cempty + 16;
  uint32_t* tmem_slot_ptr = reinterpret_cast<uint32_t*>(smem_raw + (tmem_slot - smem_addr(smem_raw)));
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (n + BN - 1) / BN;
  const int tiles = ((m + kBM - 1) / kBM) * n_tiles;
  const int ksteps = k / kGemmBK;
  const int G = (int)gridDim.x;
  const int my_tiles = (tiles - (int)blockIdx.x + G - 1) / G;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; s++) {
      mbar_init(bars + 8 * s, 1 + kGemmDecodeThreads);
      mbar_init(bars + 8 * (STAGES + s), 1);
    }
    for (int a = 0; a < 2; a++) {
      mbar_init(accf + 8 * a, 1);    // MMA commit
      mbar_init(acce + 8 * a, 128);  // every epilogue thread
    }
    mbar_init(done_bar, 1);
    for (int c = 0; c < 2; c++) {
      mbar_init(cfull + 8 * c, kGemmDecodeThreads);   // every decode thread's copies landed
      mbar_init(cempty + 8 * c, kGemmDecodeThreads);  // every decode thread done reading
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * MH * BN);
    tmem_relinquish();
  }
  if (FMT == 1) {  // IQ4_NL pair table, kLutC interleaved copies, in staging slot 0's spare tail
    for (int i = threadIdx.x; i < 256 * kLutC; i += blockDim.x) {
      const int v = i / kLutC;
      const uint32_t lo = __half_as_ushort(__int2half_rn(c_iq4nl_kv[v & 15]));
      const uint32_t hi = __half_as_ushort(__int2half_rn(c_iq4nl_kv[v >> 4]));
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(p_s + kLutOff + 4u * i), "r"(lo | (hi << 16)) : "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot_ptr;

  if (warp == 0) {
    // ---------------------------- X loader --------------------------------
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      int gs = 0, issued = 0;
      const int tissue = (g_test_flags & kTestWithholdXTiles) ? 0 : my_tiles;  // test switch: issue nothing
      for (int li = 0; li < tissue && !s_abort; li++) {
        const int tile = (int)blockIdx.x + li * G;
        const int m0 = (tile / n_tiles) * kBM;
        for (int ks = 0; ks < ksteps; ks++, gs++) {
          const int s = gs % STAGES;
          const uint32_t ph = (uint32_t)(gs / STAGES) & 1u;
          if (s_abort || !mbar_wait(bars + 8 * (STAGES + s), ph ^ 1u)) { s_abort = 1; break; }
          mbar_arrive_expect_tx(bars + 8 * s, kA);
          tma_load_2d(a_s + s * kA, &tm_x, ks * kGemmBK, m0, bars + 8 * s);  // box of kBM rows
          issued = gs + 1;
        }
      }
      for (int s = 0; s < STAGES && s < issued; s++) {  // drain our copies
        const int last = issued - 1 - ((issued - 1 - s) % STAGES);
        mbar_wait(bars + 8 * s, (uint32_t)(last / STAGES) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------------------- MMA issuer ------------------------------
    if (lane == 0) {
      int gs = 0;
      for (int li = 0; li < my_tiles && !s_abort; li++) {
        const int tile = (int)blockIdx.x + li * G;
        const int n0 = (tile % n_tiles) * BN;
        const int n_mma = (min(BN, n - n0) <= BN / 2) ? BN / 2 : BN;
        const uint32_t idesc = umma_idesc_f16(n_mma);
        const int a = li & 1;
        if (!mbar_wait(acce + 8 * a, (((uint32_t)li >> 1) & 1u) ^ 1u)) { s_abort = 1; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * MH * BN);
        bool ok = true;
        for (int ks = 0; ks < ksteps; ks++, gs++) {
          const int s = gs % STAGES;
          const uint32_t ph = (uint32_t)(gs / STAGES) & 1u;
          if (s_abort || !mbar_wait(bars + 8 * s, ph)) { s_abort = 1; ok = false; break; }
          tc_fence_after();
          const uint64_t db = umma_desc_k128(b_s + s * C::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; kk++)
#pragma unroll
            for (int h = 0; h < MH; h++)  // M-half h: X rows 128h.. of the stage, accumulator columns h*BN..
              umma_f16(d + (uint32_t)(h * BN), umma_desc_k128(a_s + s * kA + h * C::kABytes) + (uint64_t)(2 * kk),
                       db + (uint64_t)(2 * kk), idesc, (ks | kk) != 0);
          umma_commit(bars + 8 * (STAGES + s));
        }
        if (!ok) break;
        umma_commit(accf + 8 * a);
      }
      umma_commit(done_bar);  // every MMA we issued has completed when this arrives
    }
  } else if (warp < 2 + kGemmDecodeWarps) {
    // ------------------------- decode producers ---------------------------
    // Packed weights arrive in chunks of 4 k steps, copied cooperatively (8
    // threads per 128-byte row piece of codes, so a warp instruction touches
    // 4 cache lines) into a 2-slot staging ring; thread t then decodes row t.
    const int t = threadIdx.x - 64;
    const int rt = t % BN, hf = t / BN;  // row of the tile; with TPR = 2 the 32-k half of each step
    const int nck = ksteps / kGemmChunkSteps;  // chunks per tile
    const int total_ck = my_tiles * nck;
    const int64_t crow = k >> 1, srow = k >> 4;
    auto issue_chunk = [&](int c) -> bool {
      const int slot = c & 1;
      if (!mbar_wait(cempty + 8 * slot, (((uint32_t)c >> 1) & 1u) ^ 1u)) return false;
      const int tile = (int)blockIdx.x + (c / nck) * G;
      const int n0 = (tile % n_tiles) * BN;
      const int kc = (c % nck) * (kGemmChunkSteps * kGemmBK);  // first k of the chunk
      const uint32_t dst = p_s + slot * kStageBytes;
      if (FMT == 1) {  // IQ4_NL: BN rows x 9 units of 16 bytes (8 blocks of 18 bytes), unit-major [9][BN][16 B]
        const int64_t rowb = (int64_t)(k >> 5) * 18;
#pragma unroll
        for (int i = 0; i < (9 * BN + kGemmDecodeThreads - 1) / kGemmDecodeThreads; i++) {
          const int pc = i * kGemmDecodeThreads + t;
          if (pc >= 9 * BN) break;
          const int r = pc / 9, u = pc - r * 9;
          const int64_t gr = min((int64_t)n0 + r, (int64_t)n - 1);
          cp_async16_g(dst + u * (BN * 16) + r * 16, codes + gr * rowb + (int64_t)(kc >> 5) * 18 + u * 16);
        }
        cp_async_mbar_arrive_noinc(cfull + 8 * slot);
        return true;
      }
#pragma unroll
      for (int i = 0; i < 8 * BN / kGemmDecodeThreads; i++) {  // codes: BN rows x 8 units of 16 bytes
        const int pc = i * kGemmDecodeThreads + t;
        const int r = pc >> 3, u = pc & 7;
        const int64_t gr = min((int64_t)n0 + r, (int64_t)n - 1);
        cp_async16_g(dst + r * 128 + ((u ^ (r & 7)) << 4), codes + gr * crow + (kc >> 1) + u * 16);
      }
      if (FMT == 2) {
#pragma unroll
        for (int i = 0; i < 2 * BN / kGemmDecodeThreads; i++) {  // scales: BN rows x 2 halves of 16 bytes
          const int pc = i * kGemmDecodeThreads + t;
          const int r = pc >> 1, h = pc & 1;
          const int64_t gr = min((int64_t)n0 + r, (int64_t)n - 1);
          cp_async16_g(dst + kStageCodes + r * 32 + ((h ^ ((r >> 2) & 1)) << 4),
                       scales + (gr * srow + (kc >> 4)) * 2 + h * 16);
        }
      } else if (FMT == 4) {  // MXFP4: 8 E8M0 bytes per row (one per 32 k)
        const int r = t;
        const int64_t gr = min((int64_t)n0 + r, (int64_t)n - 1);
        if (r < BN) cp_async8_g(dst + kStageCodes + r * 32, scales + gr * (srow >> 1) + (kc >> 5));
      } else {  // E4M3: 16 bytes per row, copied whole; words read swizzled
        const int r = t;
        const int64_t gr = min((int64_t)n0 + r, (int64_t)n - 1);
        if (r < BN) cp_async16_g(dst + kStageCodes + r * 32, scales + gr * srow + (kc >> 4));
      }
      cp_async_mbar_arrive_noinc(cfull + 8 * slot);
      return true;
    };
    bool stop = !issue_chunk(0);
    int gs = 0;
    for (int c = 0; c < total_ck && !stop; c++) {
      if (c + 1 < total_ck && !issue_chunk(c + 1)) { s_abort = 1; break; }
      const int slot = c & 1;
      if (s_abort || !mbar_wait(cfull + 8 * slot, ((uint32_t)c >> 1) & 1u)) { s_abort = 1; break; }
      const int tile = (int)blockIdx.x + (c / nck) * G;
      const bool valid = (int64_t)(tile % n_tiles) * BN + rt < n;
      const uint32_t src = p_s + slot * kStageBytes;
#pragma unroll  // (IQ4_NL selects its words by j)
      for (int j = 0; j < kGemmChunkSteps; j++, gs++) {
        const int s = gs % STAGES;
        const uint32_t ph = (uint32_t)(gs / STAGES) & 1u;
        if (FMT == 1) {
          // this row's two blocks of step j: 36 bytes from byte 36j of the row,
          // inside its 16-byte units 2j .. 2j+2 (36j = 32j + 4j: the span
          // starts j words into unit 2j); a warp's 32 rows read each unit as
          // 512 contiguous bytes
          uint32_t uw[12];
#pragma unroll
          for (int u = 0; u < 3; u++) {
            const uint4 v = lds128(src + (2 * j + u) * (BN * 16) + rt * 16);
            uw[4 * u] = v.x; uw[4 * u + 1] = v.y; uw[4 * u + 2] = v.z; uw[4 * u + 3] = v.w;
          }
          uint32_t w[9];
#pragma unroll
          for (int i = 0; i < 9; i++) w[i] = (j == 0) ? uw[i] : (j == 1) ? uw[i + 1] : (j == 2) ? uw[i + 2] : uw[i + 3];
          uint32_t qa[4], qb[4];
#pragma unroll
          for (int i = 0; i < 4; i++) {
            qa[i] = __funnelshift_r(w[i], w[i + 1], 16);  // block 0: index bytes 2..17 of the 36
            qb[i] = w[5 + i];                              // block 1: bytes 20..35
          }
          uint32_t da = w[0] & 0xFFFFu, db = w[4] >> 16;
          da = valid ? (da | (da << 16)) : 0u;
          db = valid ? (db | (db << 16)) : 0u;
          if (s_abort || !mbar_wait(bars + 8 * (STAGES + s), ph ^ 1u)) { s_abort = 1; stop = true; break; }
          const uint32_t lut_copy = p_s + kLutOff + 4u * (uint32_t)(t & (kLutC - 1));
          const uint32_t row_base = b_s + s * C::kBBytes + (uint32_t)rt * 128u;
          const uint32_t swz = (uint32_t)(rt & 7);
          uint32_t o[16];
          if (TPR == 1 || hf == 0) {
            iq4_block_chunks<kLutLsh>(qa, da, lut_copy, o);
#pragma unroll
            for (int cc = 0; cc < 4; cc++)
              sts128(row_base + ((cc ^ swz) << 4), o[4 * cc], o[4 * cc + 1], o[4 * cc + 2], o[4 * cc + 3]);
          }
          if (TPR == 1 || hf == 1) {
            iq4_block_chunks<kLutLsh>(qb, db, lut_copy, o);
#pragma unroll
            for (int cc = 0; cc < 4; cc++)
              sts128(row_base + (((cc + 4) ^ swz) << 4), o[4 * cc], o[4 * cc + 1], o[4 * cc + 2], o[4 * cc + 3]);
          }
          fence_proxy_async_shared();
          mbar_arrive(bars + 8 * s);
          continue;
        }
        // this row's 32 code bytes (units 2j, 2j+1) and 4 scales of step j;
        // with TPR = 2 this thread takes unit 2j + hf (chunks 4hf .. 4hf+3)
        constexpr int kCh = 8 / TPR;                // 16-byte output chunks of this thread
        const int ch0 = (TPR == 2) ? 4 * hf : 0;    // its first chunk
        uint32_t q[8];
        {
          const uint4 c0 = lds128(src + rt * 128 + (((2 * j + (TPR == 2 ? hf : 0)) ^ (rt & 7)) << 4));
          q[0] = c0.x; q[1] = c0.y; q[2] = c0.z; q[3] = c0.w;
          if (TPR == 1) {
            const uint4 c1 = lds128(src + rt * 128 + (((2 * j + 1) ^ (rt & 7)) << 4));
            q[4] = c1.x; q[5] = c1.y; q[6] = c1.z; q[7] = c1.w;
          }
        }
        uint32_t sc[4];
        bool mx_wide = false;  // MXFP4 scale that is not an fp16 value: two fp16 factors
        uint32_t mx0a = 0u, mx0b = 0u, mx1a = 0u, mx1b = 0u;
        if (FMT == 2) {
          const uint32_t half = (uint32_t)((j >> 1) ^ ((rt >> 2) & 1));
          const uint2 sv = lds64(src + kStageCodes + rt * 32 + (half << 4) + (j & 1) * 8);
          sc[0] = bcast_lo(sv.x); sc[1] = bcast_hi(sv.x); sc[2] = bcast_lo(sv.y); sc[3] = bcast_hi(sv.y);
        } else if (FMT == 4) {  // two E8M0 bytes for this step's 64 k
          const uint32_t sw = lds32(src + kStageCodes + rt * 32 + (j >> 1) * 4) >> ((j & 1) * 16);
          const uint32_t b0 = sw & 0xFFu, b1 = (sw >> 8) & 0xFFu;
          mx_wide = !(e8m0_f16_ok(b0) && e8m0_f16_ok(b1));
          if (mx_wide) {  // rare: two fp16 factors per group
            e8m0_f16_factors(b0, mx0a, mx0b);
            e8m0_f16_factors(b1, mx1a, mx1b);
          }
          const int v0 = (int)b0 - 127, v1 = (int)b1 - 127;  // the power itself when it is an fp16 value
          sc[0] = sc[1] = f16x2_pow2(v0 < -24 ? -24 : (v0 > 15 ? 15 : v0));
          sc[2] = sc[3] = f16x2_pow2(v1 < -24 ? -24 : (v1 > 15 ? 15 : v1));
        } else {
          const uint32_t sw = lds32(src + kStageCodes + rt * 32 + j * 4);
          const uint32_t e01 = e4m3x2_to_f16x2(sw & 0xFFFFu), e23 = e4m3x2_to_f16x2(sw >> 16);
          sc[0] = bcast_lo(e01); sc[1] = bcast_hi(e01); sc[2] = bcast_lo(e23); sc[3] = bcast_hi(e23);
        }
        if (!valid) sc[0] = sc[1] = sc[2] = sc[3] = 0u;
        if (s_abort || !mbar_wait(bars + 8 * (STAGES + s), ph ^ 1u)) { s_abort = 1; stop = true; break; }
        const uint32_t row_base = b_s + s * C::kBBytes + (uint32_t)rt * 128u;
        const uint32_t swz = (uint32_t)(rt & 7);
        if (FMT == 4 && mx_wide) {
          if (!valid) mx0a = mx0b = mx1a = mx1b = 0u;
#pragma unroll
          for (int c = 0; c < kCh; c++) {
            const int cc = ch0 + c;
            uint32_t w4[4];
            e2m1x8_to_f16x2(q[c], w4);
            const uint32_t fa = (cc < 4) ? mx0a : mx1a, fb = (cc < 4) ? mx0b : mx1b;
            sts128(row_base + ((cc ^ swz) << 4), hmul2(hmul2(w4[0], fa), fb), hmul2(hmul2(w4[1], fa), fb),
                   hmul2(hmul2(w4[2], fa), fb), hmul2(hmul2(w4[3], fa), fb));
          }
        } else {
#pragma unroll
          for (int c = 0; c < kCh; c++) {
            const int cc = ch0 + c;
            uint32_t w4[4];
            e2m1x8_to_f16x2(q[c], w4);
            const uint32_t sv = sc[cc >> 1];
            sts128(row_base + ((cc ^ swz) << 4), hmul2(w4[0], sv), hmul2(w4[1], sv), hmul2(w4[2], sv),
                   hmul2(w4[3], sv));
          }
        }
        fence_proxy_async_shared();
        mbar_arrive(bars + 8 * s);
      }
      mbar_arrive(cempty + 8 * slot);  // this thread is done with the staged chunk
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else {
    // ------------------------------ epilogue ------------------------------
    const int q = warp & 3;  // TMEM lanes 32q .. 32q+31
    const float gs = (FMT == 3) ? g : 1.0f;
    for (int li = 0; li < my_tiles; li++) {
      const int tile = (int)blockIdx.x + li * G;
      const int m0 = (tile / n_tiles) * kBM, n0 = (tile % n_tiles) * BN;
      const int n_mma = (min(BN, n - n0) <= BN / 2) ? BN / 2 : BN;
      const int a = li & 1;
      if (s_abort || !mbar_wait(accf + 8 * a, ((uint32_t)li >> 1) & 1u)) { s_abort = 1; break; }
      tc_fence_after();
      for (int jj = 0; jj < MH * (n_mma / 32); jj++) {
        const int mh = jj / (n_mma / 32), j = jj - mh * (n_mma / 32);  // M-half, 32-column group
        const int mrow = m0 + 128 * mh + 32 * q + lane;
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * MH * BN + mh * BN + 32 * j), r);
        tmem_ld_wait();
        const int col = n0 + 32 * j;
        if (mrow < m && col < n) {
          uint32_t h[16];
#pragma unroll
          for (int i = 0; i < 16; i++)
            h[i] = f32x2_to_f16x2(__uint_as_float(r[2 * i]) * gs, __uint_as_float(r[2 * i + 1]) * gs);
          uint16_t* yp = y + (int64_t)mrow * n + col;
          if (col + 32 <= n && (n & 7) == 0) {
            uint4* y4 = reinterpret_cast<uint4*>(yp);
#pragma unroll
            for (int i = 0; i < 4; i++) y4[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
          } else {
            for (int i = 0; i < 32 && col + i < n; i++) yp[i] = (uint16_t)((h[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acce + 8 * a);  // accumulator a may be overwritten
    }
  }

  // teardown: no MMA of ours may still be writing tensor memory
  if (warp == 1 && lane == 0) mbar_wait(done_bar, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * MH * BN);
  }
}

}  // namespace qmm
