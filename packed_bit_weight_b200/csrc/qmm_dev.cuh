// qmm_dev.cuh -- device-side helpers shared by the sm_100a kernels of libqmm:
// nibble decoders, the legacy-MMA wrapper, mbarrier/TMA wrappers with
// bounded waits, and the per-device error word.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace qmm {

// Error word bits (read and cleared by qmm_sync_check).
enum : unsigned { ERR_TIMEOUT = 1u, ERR_BAD_EXPERT = 2u };

// One word per device that loads the library.
__device__ unsigned int g_err_word;

// A pipeline wait gives up after this many nanoseconds of %globaltimer
// (2 s; a test may lower it through qmm_debug_set).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
__device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;

// Test switches (qmm_debug_set), 0 in normal use.  kTestWithholdXTiles: the
// tensor-core GEMMs' activation loader issues no tile load, so the MMA
// issuer's wait for the first stage runs out and the kernel takes its
// timeout path (raise the error word, drain, free tensor memory, return).
// (The routed-expert tile kernel's switch, which withholds its bulk copies,
// is a launch argument instead: IqtArgs::withhold.)
enum : unsigned { kTestWithholdXTiles = 1u };
__device__ unsigned int g_test_flags;

__device__ __forceinline__ void raise_error(unsigned bits) { atomicOr(&g_err_word, bits); }

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// fp16 / E2M1 / E4M3 conversions (hardware cvt; lane order checked on B200:
// the low nibble / low byte lands in the low f16 half).
// ---------------------------------------------------------------------------

// Four bytes of packed E2M1 pairs -> four f16x2 (byte b -> out[b], low nibble
// in the low half).  Values are the exact E2M1 magnitudes with sign.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t q, uint32_t (&o)[4]) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(q));
}

// One byte of packed E2M1 pair (low 8 bits of the word) -> f16x2, by integer
// bit placement instead of the hardware convert: with only one byte of the
// .b8 unpack live, the convert returned zeros on B200, so the single-byte
// decoder avoids it.  E2M1 s|e1 e0|m placed at fp16 bits 15|11 10|9 is the
// code value times 2^-14 (exact, subnormal for e = 0); one exact f16x2
// multiply by 2^14 restores it.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte_in_low8) {
  const uint32_t b = byte_in_low8 & 0xFFu;
  const uint32_t lo = ((b & 0x7u) << 9) | ((b & 0x8u) << 12);
  const uint32_t hi = ((b & 0x70u) << 21) | ((b & 0x80u) << 24);
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(lo | hi), "r"(0x74007400u));  // 2^14 = 0x7400
  return d;
}

// Two E4M3FN bytes (low 16 bits) -> f16x2, exact (every E4M3 value is an fp16).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
  uint32_t o;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(o) : "h"((unsigned short)(two_bytes & 0xFFFFu)));
  return o;
}

// a * b on f16x2, round to nearest even, subnormals kept.
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// MXFP4 group scale: an OCP E8M0 byte b is 2^(b-127); 0xFF is NaN.
// e8m0_f16_ok: 2^(b-127) is an fp16 value (2^-24 .. 2^15, b in [103, 142]),
// so one f16x2 multiply by e8m0_to_f16x2(b) rounds code * scale exactly once.
__device__ __forceinline__ bool e8m0_f16_ok(uint32_t b) { return b - 103u <= 39u; }
__device__ __forceinline__ uint32_t e8m0_to_f16x2(uint32_t b) {
  const int s = (int)b - 127;
  const uint32_t h = (s >= -14) ? (uint32_t)(s + 15) << 10 : 1u << (s + 24);  // normal or subnormal 2^s
  return h | (h << 16);
}
// Any E8M0 byte as two fp16 factors f1, f2 (f16x2 broadcasts) such that
// fp16((code * f1) * f2) == fp16(code * 2^(b-127)) for every E2M1 code with
// the first product exact: 2^(b-127) = f1 * f2 when that fits (f1 = 1 inside
// the fp16 range; f1 = 2^-14 below it; f1 = 2^15 above it, where a first
// product that overflows means the true one does too); below 2^-38 and
// above 2^30 the clamped factors round to the same zero / infinity; 0xFF
// gives f2 = NaN.
__device__ __forceinline__ uint32_t f16x2_pow2(int v) {  // 2^v, v in [-24, 15]
  const uint32_t h = (v >= -14) ? (uint32_t)(v + 15) << 10 : 1u << (v + 24);
  return h | (h << 16);
}
__device__ __forceinline__ void e8m0_f16_factors(uint32_t b, uint32_t& f1, uint32_t& f2) {
  const int s = (int)b - 127;
  const int a = (s < -24) ? -14 : ((s > 15) ? 15 : 0);
  int r = s - a;
  r = r < -24 ? -24 : (r > 15 ? 15 : r);
  f1 = f16x2_pow2(a);
  f2 = (b == 255u) ? 0x7E007E00u : f16x2_pow2(r);
}

// The two factors of e8m0_f16_factors packed as two fp16 halves (f1 low).
__device__ __forceinline__ uint32_t e8m0_f16_factor_pair(uint32_t b) {
  uint32_t f1, f2;
  e8m0_f16_factors(b, f1, f2);
  return (f1 & 0xFFFFu) | (f2 << 16);
}

// 2^(b-127) as fp32 for every byte (b = 0: the fp32 subnormal 2^-127).
__device__ __forceinline__ float e8m0_to_f32(uint32_t b) {
  return b == 0u ? __uint_as_float(0x00400000u) : (b == 255u ? __uint_as_float(0x7FC00000u) : __uint_as_float(b << 23));
}

// Broadcast the low / high f16 of a word to both halves.
__device__ __forceinline__ uint32_t bcast_lo(uint32_t v) { return __byte_perm(v, v, 0x1010); }
__device__ __forceinline__ uint32_t bcast_hi(uint32_t v) { return __byte_perm(v, v, 0x3232); }

// f16x2 -> two f32 (exact).
__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  return __half22float2(h);
}

// two f32 -> f16x2 with round to nearest even (lo in the low half).
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ uint16_t f32_to_f16_bits(float v) {
  return __half_as_ushort(__float2half_rn(v));
}

// ---------------------------------------------------------------------------
// Legacy warp MMA: D(16x8, f32) += A(16x16, f16, row) * B(16x8, f16, col).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// fp16(code * scale) for the two exact code values of f16x2 c and any MXFP4
// scale s (fp32 from e8m0_to_f32): the fp32 product is exact (two
// significant bits times a power of two, fp32 subnormals kept), the narrowing
// rounds once.
__device__ __forceinline__ uint32_t mx_scale_any(uint32_t c, float s) {
  const float2 f = f16x2_to_f32x2(c);
  return f32x2_to_f16x2(f.x * s, f.y * s);
}

// ---------------------------------------------------------------------------
// Shared-memory / global loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 ldg_nc128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ---------------------------------------------------------------------------
// mbarrier + TMA (no cluster multicast anywhere in this library)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n}" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n}" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Gives up after
// g_wait_limit_ns, raises ERR_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  const unsigned long long limit = *(volatile unsigned long long*)&g_wait_limit_ns;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit) {
      raise_error(ERR_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled TMA load global -> this CTA's shared memory, completing on `bar`.
// c0 is the innermost coordinate (in elements); callers keep c0 * element
// size a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Contiguous bulk copy global -> this CTA's shared memory through the copy
// engine, completing `bytes` of transaction on `bar`.  Both addresses 16-byte
// aligned, bytes a multiple of 16 (callers check).  No multicast.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters: rank, barrier, distributed shared memory reads
// (plain loads from a peer CTA's shared memory on this GPU; no multicast).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster arrives, then waits for all: the
// shared-memory writes before it are visible cluster-wide after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// fp64 at the same shared-memory offset as `local` in the CTA of rank r.
__device__ __forceinline__ double ld_dsmem_f64(const double* local, uint32_t r) {
  uint32_t remote;
  double v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(r));
  asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(remote) : "memory");
  return v;
}
// fp32 at the same shared-memory offset as `local` in the CTA of rank r.
__device__ __forceinline__ float ld_dsmem_f32(const float* local, uint32_t r) {
  uint32_t remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(r));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// bar.sync on a named barrier that also returns the OR of every thread's flag.
__device__ __forceinline__ bool named_bar_or(int id, int threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace qmm
