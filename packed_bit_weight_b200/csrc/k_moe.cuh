// k_moe.cuh -- the pieces around the routed-expert GEMVs of a mixture-of-
// experts layer ("Mark-Experimental-V3-8B", section "Mixture-of-Experts
// (MoE)": s = Softmax(x W_router + b), top-4 experts with weights g_i,
// F(x) = (SiLU(x W_gate) * (x W_up)) W_down, routed output sum_i g_i F_i(x)).
//
// router_topk_kernel: one thread-block cluster of CS CTAs of 32 warps per
//   token; the CTAs split k, warps take experts, lanes split each CTA's k;
//   every fp16 x fp16 product is exact in fp32 and the dot product is
//   accumulated in fp64, then rounded once, with the bias, to an fp32 logit;
//   softmax in fp32;
//   the top-k is taken on the fp32 logits, larger first, ties to the lower
//   expert index; g = the softmax score of each chosen expert.
// combine_kernel: out[t][j] = sum_s g[t][s] * y[t][s][j]: the down
//   projection's epilogue already scaled each slot by g in fp32; the slots are
//   added in slot order (deterministic) and rounded once to fp16.
// (SiLU(gate) * up is fused into the grouped IQ4_NL kernel's epilogue.)
#pragma once
#include "qmm_dev.cuh"

namespace qmm {

constexpr int kRouterMaxExperts = 256;
constexpr int kRouterMaxTopk = 16;

// Router logits: a cluster of CS CTAs per token (launch attribute; CS = 1
// without one); CTA c of the cluster takes the 256-wide k chunks c, c + CS,
// ...; in each CTA warp w takes experts w, w+32, ..., and lanes take 8
// consecutive k of every chunk.  Each fp16 x fp16 product is exact in fp32
// and is added in fp64, into two partial sums (alternate chunks: two
// independent add chains); four chunks' loads are issued before their
// products.  The CTAs' fp64 partial sums meet in CTA 0 through distributed
// shared memory and are added in rank order (deterministic), then rounded
// once with the bias.  (Eight warps with four experts each measured 11 us
// per token: the fp64 adds and conversions are long-latency and two warps
// per scheduler did not hide them.  One CTA per token: 7.0 us per launch at
// one token, the cluster spreads that over CS SMs.)
constexpr int kRouterThreads = 1024;

__device__ __forceinline__ void router_acc8(double& s, const uint4& xv, const uint4& wv) {
  const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w}, ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const float2 xf = f16x2_to_f32x2(xs[i]), wf = f16x2_to_f32x2(ws[i]);
    s += (double)(xf.x * wf.x);  // exact product
    s += (double)(xf.y * wf.y);
  }
}

__global__ void __launch_bounds__(kRouterThreads) router_topk_kernel(const uint16_t* __restrict__ x,
                                                                     const uint16_t* __restrict__ w,
                                                                     const float* __restrict__ b, int k, int E,
                                                                     int topk, int32_t* __restrict__ ids,
                                                                     float* __restrict__ g,
                                                                     float* __restrict__ logits_out) {
  __shared__ float z[kRouterMaxExperts];
  __shared__ double zp[kRouterMaxExperts];  // this CTA's partial sums
  // a kernel launched after this one with programmatic dependent launch (the
  // routed-expert kernels) may start now; it waits for these results
  asm volatile("griddepcontrol.launch_dependents;" :::);
  const int cs = (int)cluster_nctarank(), c = (int)cluster_ctarank();
  const int tok = (int)blockIdx.x / cs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kWarps = kRouterThreads / 32;
  const uint16_t* xr = x + (int64_t)tok * k;
  const int step = 256 * cs;
  for (int e = warp; e < E; e += kWarps) {
    const uint16_t* wr = w + (int64_t)e * k;
    double s0 = 0.0, s1 = 0.0;
    int kk = 256 * c + lane * 8;
    for (; kk + 3 * step < k; kk += 4 * step) {
      uint4 xv[4], wv[4];
#pragma unroll
      for (int u = 0; u < 4; u++) {
        xv[u] = *reinterpret_cast<const uint4*>(xr + kk + u * step);
        wv[u] = *reinterpret_cast<const uint4*>(wr + kk + u * step);
      }
      router_acc8(s0, xv[0], wv[0]);
      router_acc8(s1, xv[1], wv[1]);
      router_acc8(s0, xv[2], wv[2]);
      router_acc8(s1, xv[3], wv[3]);
    }
    for (; kk < k; kk += step)
      router_acc8(s0, *reinterpret_cast<const uint4*>(xr + kk), *reinterpret_cast<const uint4*>(wr + kk));
    double v = s0 + s1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    if (lane == 0) zp[e] = v;
  }
  cluster_sync();  // every CTA's partials are written (also a CTA barrier)
  if (c == 0) {
    for (int e = threadIdx.x; e < E; e += kRouterThreads) {
      double v = 0.0;
      for (int r = 0; r < cs; r++) v += ld_dsmem_f64(&zp[e], (uint32_t)r);
      const float zz = __double2float_rn(v + (double)b[e]);
      z[e] = zz;
      if (logits_out) logits_out[(int64_t)tok * E + e] = zz;
    }
  }
  cluster_sync();  // the partials stay until CTA 0 has read them; z is complete
  if (c != 0 || warp != 0) return;
  float mx = -INFINITY;
  for (int e = lane; e < E; e += 32) mx = fmaxf(mx, z[e]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
  float den = 0.f;
  for (int e = lane; e < E; e += 32) den += expf(z[e] - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xFFFFFFFFu, den, off);
  uint32_t taken = 0u;  // bit i: expert lane + 32 i already chosen
  for (int j = 0; j < topk; j++) {
    float bv = -INFINITY;
    int be = E;  // larger logit first, ties to the lower index
    for (int i = 0, e = lane; e < E; i++, e += 32) {
      if ((taken >> i) & 1u) continue;
      const float v = z[e];
      if (v > bv || (v == bv && e < be)) { bv = v; be = e; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
      const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == 0) {
      ids[(int64_t)tok * topk + j] = be;
      g[(int64_t)tok * topk + j] = expf(bv - mx) / den;
    }
  }
}

// out[t][j] = fp16(sum_s yg[t][s][j]): the slots' g-scaled fp32 outputs
// added in slot order, 8 outputs per thread (n % 8 == 0).  Slots whose
// expert id is out of range were never computed and are left out.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ yg, const int32_t* __restrict__ ids,
                                                      int E, int t, int topk, int n, uint16_t* __restrict__ out) {
  // launched with programmatic dependent launch: resident while the down
  // pass finishes, reads its output only after it (MoE block t = 4 44.4 vs
  // 45.2 us on B200; the router launched the same way measured 0.6 us slower
  // at t = 1 and stays a plain launch)
  asm volatile("griddepcontrol.launch_dependents;" :::);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t per_tok = n / 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (int64_t)t * per_tok;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tok = i / per_tok;
    const int j = (int)(i % per_tok) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < topk; s++) {
      const int e = ids[tok * topk + s];
      if (e < 0 || e >= E) continue;
      const float* src = yg + (tok * topk + s) * n + j;
      const float4 v0 = *reinterpret_cast<const float4*>(src);
      const float4 v1 = *reinterpret_cast<const float4*>(src + 4);
      acc[0] += v0.x; acc[1] += v0.y; acc[2] += v0.z; acc[3] += v0.w;
      acc[4] += v1.x; acc[5] += v1.y; acc[6] += v1.z; acc[7] += v1.w;
    }
    uint4 o;
    o.x = f32x2_to_f16x2(acc[0], acc[1]);
    o.y = f32x2_to_f16x2(acc[2], acc[3]);
    o.z = f32x2_to_f16x2(acc[4], acc[5]);
    o.w = f32x2_to_f16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(out + tok * n + j) = o;
  }
}

}  // namespace qmm
