// qmm_lib.cu -- libqmm.so: the C ABI declared in include/qmm.h.
//
// Host side: argument validation, kernel-variant selection, TMA descriptor
// encoding and launches.  All arithmetic of the path runs in the sm_100a
// kernels included below; there is no host or CPU fallback.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/qmm.h"
#include "k_dequant.cuh"
#include "k_gemv.cuh"
#include "k_gemm.cuh"
#include "k_grouped.cuh"
#include "k_iq4t.cuh"
#include "k_quant.cuh"
#include "k_moe.cuh"

namespace qmm {

static thread_local char t_variant[160] = "";

static void set_variant(const char* fmt, ...) __attribute__((format(printf, 1, 2)));
static void prefix_variant(const char* prefix);
static void set_variant(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_variant, sizeof(t_variant), fmt, ap);
  va_end(ap);
}

// Record the dispatch path in front of the kernel variant just recorded.
static void prefix_variant(const char* prefix) {
  char kern[sizeof(t_variant)];
  snprintf(kern, sizeof(kern), "%s", t_variant);
  snprintf(t_variant, sizeof(t_variant), "%s%s", prefix, kern);
}

struct DevInfo {
  bool init = false;
  bool sm100 = false;
  int sms = 0;
  size_t smem_optin = 0;
};
static DevInfo g_dev[64];
// qmm_debug_set(QMM_DEBUG_WITHHOLD_TILE_COPIES): passed to the tile kernel as
// a launch argument (process-wide; tests only)
static bool g_withhold_tile_copies = false;
static std::mutex g_mu;

static qmm_status device_info(DevInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QMM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0, sms = 0, optin = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return QMM_ERR_CUDA;
    d.sm100 = (major == 10 && minor == 0);
    d.sms = sms;
    d.smem_optin = (size_t)optin;
    d.init = true;
  }
  *out = &d;
  return d.sm100 ? QMM_OK : QMM_ERR_NOT_SM100;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool valid_fmt(int32_t f) {
  return f == QMM_FMT_IQ4_NL || f == QMM_FMT_FP4G16_F16 || f == QMM_FMT_FP4G16_E4M3 || f == QMM_FMT_MXFP4;
}
static int64_t fmt_group(int32_t f) { return (f == QMM_FMT_IQ4_NL || f == QMM_FMT_MXFP4) ? 32 : 16; }

static qmm_status check_weights(const qmm_weights* w, bool allow_experts) {
  if (!w) return QMM_ERR_INVALID_ARG;
  if (!valid_fmt(w->fmt) || w->reserved != 0 || w->reserved2 != 0) return QMM_ERR_INVALID_ARG;
  if (w->n < 0 || w->k < 0 || w->num_experts < 1) return QMM_ERR_INVALID_ARG;
  if (!allow_experts && w->num_experts != 1) return QMM_ERR_INVALID_ARG;
  if (w->n > INT32_MAX || w->k > INT32_MAX) return QMM_ERR_UNSUPPORTED_SHAPE;
  if (w->k % fmt_group(w->fmt)) return QMM_ERR_UNSUPPORTED_SHAPE;
  if (w->n > 0 && w->k > 0) {
    if (!w->data) return QMM_ERR_INVALID_ARG;
    if (w->fmt != QMM_FMT_IQ4_NL && !w->scales) return QMM_ERR_INVALID_ARG;
    if (!aligned16(w->data) || (w->scales && !aligned16(w->scales))) return QMM_ERR_MISALIGNED;
  }
  return QMM_OK;
}

static qmm_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? QMM_OK : QMM_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched through the runtime, so the
// library needs no link-time libcuda).
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

static bool get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return false;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

// 2-D map over a row-major [rows][cols] array of `elem`-byte elements.
static bool make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem, uint64_t cols,
                        uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  if (!get_encoder()) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)elem};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Launch with programmatic dependent launch (the kernel waits on the previous
// one with griddepcontrol.wait before touching its outputs).
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

static int grid_for(int64_t items, int per_block, int sms, int waves = 8) {
  int64_t b = (items + per_block - 1) / per_block;
  int64_t cap = (int64_t)sms * waves;
  if (b > cap) b = cap;
  if (b < 1) b = 1;
  return (int)b;
}

// An empty kernel: launched without programmatic dependent launch after a
// kernel that writes packed weights, so that a following kernel which reads
// weights before its dependency wait overlaps nothing that writes them.
__global__ void ordering_kernel() {}

// ---------------------------------------------------------------------------
// GEMV dispatch
// ---------------------------------------------------------------------------
template <int FMT, int NT, int SPW, int WPC = kLdgWarps, int MINB = 2, bool WIDE = false, bool XW = false>
static qmm_status launch_gemv_ldg(const qmm_weights* w, const uint16_t* x, int m, uint16_t* y, cudaStream_t st,
                                  const DevInfo* di) {
  const int n = (int)w->n, k = (int)w->k;
  const int tiles = (n + 15) / 16;
  // half of each warp's 8 segments after the dependency wait (FP4-G16, the
  // 4- and 8-warp configurations of k = 4096 and 8192: in_proj 9.83 vs 10.01
  // us, out_proj 4.97 vs 5.26 us per launch on B200; also at two n-tiles)
  constexpr int kPre = (SPW == 8 && (WPC == 4 || WPC == 8) && !WIDE && (FMT == 2 || FMT == 3)) ? 4 : SPW;
  auto kern = gemv_fp4_ldg_kernel<FMT, NT, SPW, WPC, MINB, WIDE, XW, kPre>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles);
  cfg.blockDim = dim3(WPC * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint8_t* codes = static_cast<const uint8_t*>(w->data);
  const uint8_t* scales = static_cast<const uint8_t*>(w->scales);
  const float g = w->global_scale;
  if (cudaLaunchKernelEx(&cfg, kern, codes, scales, x, y, n, k, m, g) != cudaSuccess) return QMM_ERR_CUDA;
  set_variant("gemv_fp4_ldg<fmt=%d,nt=%d,spw=%d,wpc=%d,minb=%d,wide=%d,xw=%d,pre=%d,tiles=%d>", FMT, NT, SPW, WPC,
              MINB, WIDE ? 1 : 0, XW ? 1 : 0, kPre, tiles);
  return launch_status();
}

// The 256-bit-load layout where the shape and alignment allow it (k % 256 ==
// 0 for segment pairs, an even segment count per warp, 32-byte-aligned codes)
// and it measured faster: MXFP4 (one 2-byte scale load instead of two 1-byte
// loads per pair; in_proj m = 1 12.2 vs 13.1 us on B200).  For FP4-G16 it
// measured slower at every shape (in_proj m = 1 11.3 vs 10.4 us: 109 vs 98
// registers).  QMM_GEMV_WIDE=0/1 forces either layout (measurement knob).
static bool ldg_wide_ok(const qmm_weights* w) {
  if (w->k % 256 != 0 || (reinterpret_cast<uintptr_t>(w->data) & 31u) != 0) return false;
  const char* e = getenv("QMM_GEMV_WIDE");
  if (e && e[0]) return e[0] == '1';
  return w->fmt == QMM_FMT_MXFP4;
}

template <int FMT, int NT, int SPW, int WPC, int MINB>
static qmm_status launch_gemv_ldg_pick(bool wide, const qmm_weights* w, const uint16_t* x, int m, uint16_t* y,
                                       cudaStream_t st, const DevInfo* di) {
  // 256-bit activation loads when x is 32-byte aligned (QMM_GEMV_XW=0 turns
  // them off: measurement knob)
  const char* xe = getenv("QMM_GEMV_XW");
  const bool xw = (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && !(xe && xe[0] == '0');
  if constexpr (SPW % 2 == 0) {
    if (wide && xw) return launch_gemv_ldg<FMT, NT, SPW, WPC, MINB, true, true>(w, x, m, y, st, di);
    if (wide) return launch_gemv_ldg<FMT, NT, SPW, WPC, MINB, true>(w, x, m, y, st, di);
  }
  if (xw) return launch_gemv_ldg<FMT, NT, SPW, WPC, MINB, false, true>(w, x, m, y, st, di);
  return launch_gemv_ldg<FMT, NT, SPW, WPC, MINB, false>(w, x, m, y, st, di);
}

// Pick the warps per tile (WPC) and segments per warp (SPW <= 8) for k =
// 128 * WPC * SPW (k <= 16384 at m <= 8, k <= 8192 at m <= 16); fewer,
// fuller warps keep more bytes in flight per register.  Returns
// UNSUPPORTED_SHAPE for other k.
template <int FMT, int NT>
static qmm_status gemv_ldg_auto(const qmm_weights* w, const uint16_t* x, int m, uint16_t* y, cudaStream_t st,
                                const DevInfo* di) {
  const int segs = (int)(w->k / 128);
  if (w->k % 128) return QMM_ERR_UNSUPPORTED_SHAPE;
  const bool wide = ldg_wide_ok(w);
  if (NT == 1) {
    if (segs % 4 == 0 && segs / 4 <= 8) {
      switch (segs / 4) {
        case 1: return launch_gemv_ldg_pick<FMT, 1, 1, 4, 4>(wide, w, x, m, y, st, di);
        case 2: return launch_gemv_ldg_pick<FMT, 1, 2, 4, 4>(wide, w, x, m, y, st, di);
        case 3: return launch_gemv_ldg_pick<FMT, 1, 3, 4, 4>(wide, w, x, m, y, st, di);
        case 4: return launch_gemv_ldg_pick<FMT, 1, 4, 4, 4>(wide, w, x, m, y, st, di);
        case 5: return launch_gemv_ldg_pick<FMT, 1, 5, 4, 4>(wide, w, x, m, y, st, di);
        case 6: return launch_gemv_ldg_pick<FMT, 1, 6, 4, 4>(wide, w, x, m, y, st, di);
        case 7: return launch_gemv_ldg_pick<FMT, 1, 7, 4, 4>(wide, w, x, m, y, st, di);
        default: return launch_gemv_ldg_pick<FMT, 1, 8, 4, 4>(wide, w, x, m, y, st, di);
      }
    }
    if (segs % 8 == 0 && segs / 8 <= 8) {
      switch (segs / 8) {
        case 5: return launch_gemv_ldg_pick<FMT, 1, 5, 8, 2>(wide, w, x, m, y, st, di);
        case 6: return launch_gemv_ldg_pick<FMT, 1, 6, 8, 2>(wide, w, x, m, y, st, di);
        case 7: return launch_gemv_ldg_pick<FMT, 1, 7, 8, 2>(wide, w, x, m, y, st, di);
        case 8: return launch_gemv_ldg_pick<FMT, 1, 8, 8, 2>(wide, w, x, m, y, st, di);
        default: break;  // smaller counts took the 4-warp path
      }
    }
    if (segs % 16 == 0 && segs / 16 <= 8) {
      switch (segs / 16) {
        case 5: return launch_gemv_ldg_pick<FMT, 1, 5, 16, 1>(wide, w, x, m, y, st, di);
        case 6: return launch_gemv_ldg_pick<FMT, 1, 6, 16, 1>(wide, w, x, m, y, st, di);
        case 7: return launch_gemv_ldg_pick<FMT, 1, 7, 16, 1>(wide, w, x, m, y, st, di);
        case 8: return launch_gemv_ldg_pick<FMT, 1, 8, 16, 1>(wide, w, x, m, y, st, di);
        default: break;
      }
    }
  } else {
    // 9..16 tokens: the same shapes as one n-tile (4 warps of up to 8
    // segments, then 8 warps), which keep twice the segments in flight per
    // warp of the earlier 8-warp / 16-warp choice at 4 segments (on B200:
    // LM head m = 16 224 vs 254 us, out_proj 8.5 vs 9.9 us, in_proj 17.0 vs
    // 19.1 us, 8192 x 2048 4.7 vs 6.3 us).  k > 8192 is left to split-K.
    if (segs % 4 == 0 && segs / 4 <= 8) {
      switch (segs / 4) {
        case 1: return launch_gemv_ldg_pick<FMT, 2, 1, 4, 4>(wide, w, x, m, y, st, di);
        case 2: return launch_gemv_ldg_pick<FMT, 2, 2, 4, 4>(wide, w, x, m, y, st, di);
        case 3: return launch_gemv_ldg_pick<FMT, 2, 3, 4, 4>(wide, w, x, m, y, st, di);
        case 4: return launch_gemv_ldg_pick<FMT, 2, 4, 4, 4>(wide, w, x, m, y, st, di);
        case 5: return launch_gemv_ldg_pick<FMT, 2, 5, 4, 4>(wide, w, x, m, y, st, di);
        case 6: return launch_gemv_ldg_pick<FMT, 2, 6, 4, 4>(wide, w, x, m, y, st, di);
        case 7: return launch_gemv_ldg_pick<FMT, 2, 7, 4, 4>(wide, w, x, m, y, st, di);
        default: return launch_gemv_ldg_pick<FMT, 2, 8, 4, 4>(wide, w, x, m, y, st, di);
      }
    }
    if (segs % 8 == 0 && segs / 8 <= 8) {
      switch (segs / 8) {
        case 5: return launch_gemv_ldg_pick<FMT, 2, 5, 8, 2>(wide, w, x, m, y, st, di);
        case 6: return launch_gemv_ldg_pick<FMT, 2, 6, 8, 2>(wide, w, x, m, y, st, di);
        case 7: return launch_gemv_ldg_pick<FMT, 2, 7, 8, 2>(wide, w, x, m, y, st, di);
        case 8: return launch_gemv_ldg_pick<FMT, 2, 8, 8, 2>(wide, w, x, m, y, st, di);
        default: break;  // smaller counts took the 4-warp path
      }
    }
  }
  return QMM_ERR_UNSUPPORTED_SHAPE;
}

// Split-K GEMV (k_gemv.cuh, gemv_fp4_splitk_kernel): clusters of cs CTAs
// share a 16-row tile, 4 warps per CTA, spw segments per warp.
template <int FMT, int NT, int SPW, bool XW>
static qmm_status launch_gemv_splitk(const qmm_weights* w, const uint16_t* x, int m, uint16_t* y, cudaStream_t st,
                                     int cs) {
  const int n = (int)w->n, k = (int)w->k;
  const int64_t tiles = (n + 15) / 16;
  if (tiles * cs > INT32_MAX) return QMM_ERR_UNSUPPORTED_SHAPE;
  constexpr int kMinb = NT == 1 ? 4 : 2;
  auto kern = gemv_fp4_splitk_kernel<FMT, NT, SPW, 4, kMinb, XW>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles * cs));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)cs;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, kern, static_cast<const uint8_t*>(w->data), static_cast<const uint8_t*>(w->scales), x,
                         y, n, k, m, w->global_scale) != cudaSuccess)
    return QMM_ERR_CUDA;
  set_variant("gemv_fp4_splitk<fmt=%d,nt=%d,spw=%d,wpc=4,cs=%d,xw=%d,tiles=%lld>", FMT, NT, SPW, cs, XW ? 1 : 0,
              (long long)tiles);
  return launch_status();
}

// Clusters per tile (0 = no split), from a sweep on B200 (per-launch time,
// n x k at m = 1: 256 x 4096 3.35 -> 2.47 us at cs = 4, 256 x 8192 3.86 ->
// 2.74 at cs = 8, 1024 x 4096 3.62 -> 3.12 at cs = 4, 2048 x 4096 4.36 ->
// 3.33 at cs = 2; 4096 x 8192 (out_proj) 5.25 unsplit, 6.4-11.8 split).  At
// m <= 8 a matrix of at most 64 tiles takes cs = 256 / tiles rounded down to
// a power of two, at most 8 and at most k / 1024 (two or more segments per
// warp); 65..128 tiles with k <= 4096 take cs = 2.  At m > 8 the split lost
// everywhere the unsplit kernel has a configuration, so it serves only the
// shapes that kernel does not take (k = 16384 at m = 16: 646 -> 3.9 us,
// instead of the generic kernel).  Each choice needs whole 4-warp CTAs of
// 1..8 segments per warp (1..4 at m > 8).  QMM_GEMV_SPLITK=<cs> forces a
// count (0 turns split-K off); a count the shape does not divide is ignored.
static bool splitk_fits(int64_t k, int m, int cs) {
  const int64_t segs = k / 128;
  const int max_spw = m > 8 ? 4 : 8;
  return k % 128 == 0 && segs % (4 * cs) == 0 && segs / (4 * cs) >= 1 && segs / (4 * cs) <= max_spw &&
         (segs / (4 * cs)) != 3 && (segs / (4 * cs)) != 5 && (segs / (4 * cs)) != 6 && (segs / (4 * cs)) != 7;
}
static int splitk_clusters(int64_t n, int64_t k, int m, bool unsplit_ok) {
  const int64_t tiles = (n + 15) / 16;
  if (const char* e = getenv("QMM_GEMV_SPLITK")) {
    const int cs = atoi(e);
    return (cs == 2 || cs == 4 || cs == 8) && splitk_fits(k, m, cs) ? cs : 0;
  }
  if (!unsplit_ok) {  // the shape has no unsplit configuration: any count that fits
    for (int cs = 2; cs <= 8; cs *= 2)
      if (splitk_fits(k, m, cs)) return cs;
    return 0;
  }
  if (m > 8) return 0;
  int cs = 0;
  if (tiles <= 64) {
    for (int c = 8; c >= 2 && !cs; c /= 2)
      if (tiles * c <= 256 && k / 1024 >= c && splitk_fits(k, m, c)) cs = c;
  } else if (tiles <= 128 && k <= 4096 && splitk_fits(k, m, 2)) {
    cs = 2;
  }
  return cs;
}

// Whether gemv_ldg_auto has a configuration for this k and batch (its cases).
static bool ldg_config_exists(int64_t k, int m) {
  if (k % 128) return false;
  const int64_t segs = k / 128;
  if (m <= 8)
    return (segs % 4 == 0 && segs / 4 >= 1 && segs / 4 <= 8) || (segs % 8 == 0 && segs / 8 >= 5 && segs / 8 <= 8) ||
           (segs % 16 == 0 && segs / 16 >= 5 && segs / 16 <= 8);
  return (segs % 4 == 0 && segs / 4 >= 1 && segs / 4 <= 8) || (segs % 8 == 0 && segs / 8 >= 5 && segs / 8 <= 8);
}

template <int FMT, int NT>
static qmm_status gemv_splitk_auto(const qmm_weights* w, const uint16_t* x, int m, uint16_t* y, cudaStream_t st,
                                   int cs) {
  const int spw = (int)(w->k / 128) / (4 * cs);
  const bool xw = (reinterpret_cast<uintptr_t>(x) & 31u) == 0;
  switch (spw) {
    case 1: return xw ? launch_gemv_splitk<FMT, NT, 1, true>(w, x, m, y, st, cs) : launch_gemv_splitk<FMT, NT, 1, false>(w, x, m, y, st, cs);
    case 2: return xw ? launch_gemv_splitk<FMT, NT, 2, true>(w, x, m, y, st, cs) : launch_gemv_splitk<FMT, NT, 2, false>(w, x, m, y, st, cs);
    case 4: return xw ? launch_gemv_splitk<FMT, NT, 4, true>(w, x, m, y, st, cs) : launch_gemv_splitk<FMT, NT, 4, false>(w, x, m, y, st, cs);
    case 8:
      if constexpr (NT == 1)
        return xw ? launch_gemv_splitk<FMT, NT, 8, true>(w, x, m, y, st, cs) : launch_gemv_splitk<FMT, NT, 8, false>(w, x, m, y, st, cs);
      return QMM_ERR_UNSUPPORTED_SHAPE;
    default: return QMM_ERR_UNSUPPORTED_SHAPE;
  }
}

// Kernel override, for tests that cover the kernels a shape does not reach by
// default: QMM_GEMV_VARIANT=ldg|generic (FP4 formats), iq4|iq4t (IQ4_NL:
// streaming or tile-resident kernel).  Unset: the default dispatch.
enum { PICK_DEFAULT = 0, PICK_LDG = 2, PICK_GENERIC = 3, PICK_IQ4_STREAM = 5, PICK_IQ4_TILE = 10 };
static int gemv_variant_env() {
  const char* v = getenv("QMM_GEMV_VARIANT");
  if (!v) return PICK_DEFAULT;
  if (!strcmp(v, "ldg")) return PICK_LDG;
  if (!strcmp(v, "generic")) return PICK_GENERIC;
  if (!strcmp(v, "iq4")) return PICK_IQ4_STREAM;
  if (!strcmp(v, "iq4t")) return PICK_IQ4_TILE;
  return PICK_DEFAULT;
}

// Tile-resident IQ4_NL kernel (k_iq4t.cuh); UNSUPPORTED_SHAPE launches nothing.
template <int MODE>
static qmm_status launch_iq4_tile(const qmm_weights* w0, const qmm_weights* w1, const uint16_t* x, int x_per_pair,
                                  int64_t topk, const int32_t* offsets, const int32_t* perm, int64_t P, int m_plain,
                                  void* y, const float* gw, cudaStream_t st, const int32_t* ids = nullptr);

static qmm_status launch_iq4_stream(const qmm_weights* w, const uint16_t* x, int x_per_pair, int64_t topk,
                                   const int32_t* offsets, const int32_t* perm, int m_plain, uint16_t* y,
                                   cudaStream_t st, const DevInfo* di);

template <int FMT>
static qmm_status gemv_fmt(const qmm_weights* w, const uint16_t* x, int m, uint16_t* y, cudaStream_t st,
                           const DevInfo* di) {
  const int64_t n = w->n, k = w->k;
  const int pick = gemv_variant_env();
  if constexpr (FMT != 1) {  // the register kernels decode E2M1 codes only
    if (pick == PICK_DEFAULT) {
      const int cs = splitk_clusters(n, k, m, ldg_config_exists(k, m));
      if (cs) {
        const qmm_status s = (m <= 8) ? gemv_splitk_auto<FMT, 1>(w, x, m, y, st, cs)
                                      : gemv_splitk_auto<FMT, 2>(w, x, m, y, st, cs);
        if (s != QMM_ERR_UNSUPPORTED_SHAPE) return s;
      }
    }
    if (pick == PICK_DEFAULT || pick == PICK_LDG) {
      const qmm_status s = (m <= 8) ? gemv_ldg_auto<FMT, 1>(w, x, m, y, st, di) : gemv_ldg_auto<FMT, 2>(w, x, m, y, st, di);
      if (s != QMM_ERR_UNSUPPORTED_SHAPE) return s;
    }
  }
  // Plain IQ4_NL GEMV: the tile-resident kernel, except where the streaming
  // one measured faster on B200 (us per launch, streaming / tile): very tall
  // matrices at small m (LM head 256000 x 4096 m = 1 / 4: 269 / 325, 312 /
  // 340; in_proj 18560 x 4096 m = 1: 24.0 / 24.8) and short rows at m > 8
  // (256 x 512 m = 16: 3.6 / 5.0; 2560 x 896: 5.9 / 6.6).  Elsewhere the
  // tile kernel leads: 256 x 512 m = 1 2.5 vs 3.1, 4096 x 4096 m = 1 6.2 vs
  // 10.6, in_proj m = 16 32.6 vs 41.0, LM head m = 16 430 vs 513.
  if constexpr (FMT == 1) {
    const int64_t tiles = (n + 15) / 16;
    const bool stream_first = (m > 8 && k < 2048) || (tiles >= 4096 && m <= 8) || (tiles >= 1024 && m == 1);
    if (pick == PICK_IQ4_TILE || (pick == PICK_DEFAULT && !stream_first)) {
      const qmm_status s = launch_iq4_tile<IQ_OUT_F16>(w, nullptr, x, 0, 1, nullptr, nullptr, 0, m, y, nullptr, st);
      if (s != QMM_ERR_UNSUPPORTED_SHAPE) return s;
    }
  }
  if (FMT == 1 && k % 128 == 0 && (pick == PICK_DEFAULT || pick == PICK_IQ4_STREAM)) {
    const qmm_status s = launch_iq4_stream(w, x, 0, 1, nullptr, nullptr, m, y, st, di);
    set_variant("gemv_iq4_stream");
    return s;
  }
  const int64_t tiles = (n + 15) / 16;
  const int64_t blocks = (tiles + 3) / 4;
  if (blocks > INT32_MAX) return QMM_ERR_UNSUPPORTED_SHAPE;
  gemv_generic_kernel<FMT><<<(unsigned)blocks, 128, 0, st>>>(static_cast<const uint8_t*>(w->data),
                                                             static_cast<const uint8_t*>(w->scales), w->global_scale,
                                                             x, y, n, k, m);
  set_variant("gemv_generic<fmt=%d>", FMT);
  return launch_status();
}

// ---------------------------------------------------------------------------
// GEMM dispatch
// ---------------------------------------------------------------------------
template <int FMT>
static qmm_status launch_gemm_tc(const qmm_weights* w, const uint16_t* x, int m, uint16_t* y, cudaStream_t st,
                                 const DevInfo* di) {
  constexpr int BN = 256, STAGES = 3;
  using C = GemmCfg<BN, STAGES>;
  const int n = (int)w->n, k = (int)w->k;
  CUtensorMap tx;
  if (!make_map_2d(&tx, x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)k, (uint64_t)m, kGemmBK, kGemmBM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return QMM_ERR_CUDA;
  const size_t smem = C::smem_bytes();
  if (smem > di->smem_optin - 1024) return QMM_ERR_CUDA;
  auto kern = gemm_fp4_tc_kernel<FMT, BN, STAGES>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QMM_ERR_CUDA;
  const int64_t tiles = (int64_t)((m + kGemmBM - 1) / kGemmBM) * ((n + BN - 1) / BN);
  if (tiles > INT32_MAX) return QMM_ERR_UNSUPPORTED_SHAPE;
  kern<<<(unsigned)tiles, kGemmThreads, smem, st>>>(tx, static_cast<const uint8_t*>(w->data),
                                                    static_cast<const uint8_t*>(w->scales), y, m, n, k,
                                                    w->global_scale);
  set_variant("gemm_fp4_tc<fmt=%d,bm=128,bn=%d,bk=64,stages=%d,tiles=%lld>", FMT, BN, STAGES, (long long)tiles);
  return launch_status();
}

// MH = 1: 128-token x 256-row tiles; MH = 2: 256 x 128 (half the weight
// decode per FLOP, two MMAs per k16 step sharing the decoded weights).
template <int FMT, int MH, int BN = 256 / MH>
static qmm_status launch_gemm_tc_persistent_mh(const qmm_weights* w, const uint16_t* x, int m, uint16_t* y,
                                               cudaStream_t st, const DevInfo* di) {
  constexpr int STAGES = 3, BM = kGemmBM * MH;
  using C = GemmCfg<BN, STAGES>;
  const int n = (int)w->n, k = (int)w->k;
  CUtensorMap tx;
  if (!make_map_2d(&tx, x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (uint64_t)k, (uint64_t)m, kGemmBK, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return QMM_ERR_CUDA;
  const size_t smem = 1024 + (size_t)STAGES * (MH * C::kABytes + C::kBBytes) + 2 * (size_t)kStageBytes + 256;
  if (smem > di->smem_optin) return QMM_ERR_CUDA;
  auto kern = gemm_fp4_tc_persistent_kernel<FMT, BN, STAGES, MH>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QMM_ERR_CUDA;
  const int64_t tiles = (int64_t)((m + BM - 1) / BM) * ((n + BN - 1) / BN);
  if (tiles > INT32_MAX) return QMM_ERR_UNSUPPORTED_SHAPE;
  const int grid = tiles < di->sms ? (int)tiles : di->sms;
  kern<<<grid, kGemmPThreads, smem, st>>>(tx, static_cast<const uint8_t*>(w->data),
                                          static_cast<const uint8_t*>(w->scales), y, m, n, k, w->global_scale);
  set_variant("gemm_fp4_tc_persistent<fmt=%d,bm=%d,bn=%d,bk=64,stages=%d,grid=%d,tiles=%lld>", FMT, BM, BN, STAGES,
              grid, (long long)tiles);
  return launch_status();
}

// 256-token tiles from m = 256 up (2048 x 18560 x 4096 on B200: FP4-G16
// 949 vs 871 TFLOP/s, E4M3 995 vs 882, MXFP4 957 vs 766, IQ4_NL 685 vs 470),
// 128-token tiles below.  QMM_GEMM_MH=1/2 forces either (measurement knob).
template <int FMT>
static qmm_status launch_gemm_tc_persistent(const qmm_weights* w, const uint16_t* x, int m, uint16_t* y,
                                            cudaStream_t st, const DevInfo* di) {
  const char* e = getenv("QMM_GEMM_MH");
  const bool two = (e && e[0]) ? e[0] == '2' : m >= 256;
  if (two) return launch_gemm_tc_persistent_mh<FMT, 2>(w, x, m, y, st, di);
  return launch_gemm_tc_persistent_mh<FMT, 1>(w, x, m, y, st, di);
}

// Any shape the tensor-core kernel does not take, and small batches: the
// decode GEMV dispatch (register kernels, split-K, IQ4_NL kernels) over
// 16-token slices of x, one launch per slice.  Slice j reads x rows
// [16j, 16j + 16) and writes the same rows of y; both stay 32-byte aligned
// (16 rows of k or n fp16 values are 32 k or 32 n bytes).
// (A four-n-tile register kernel over 32-token slices measured no better:
// in_proj m = 32 39.0 vs 37.6 us, LM head 519 vs 508 us, out_proj 18.7 vs
// 19.8 us on B200.)
template <int FMT>
static qmm_status gemm_by_gemv(const qmm_weights* w, const uint16_t* x, int64_t m, uint16_t* y, cudaStream_t st,
                               const DevInfo* di) {
  const int64_t slices = (m + 15) / 16;
  for (int64_t m0 = 0; m0 < m; m0 += 16) {
    const int mm = (int)((m - m0) < 16 ? (m - m0) : 16);
    const qmm_status s = gemv_fmt<FMT>(w, x + m0 * w->k, mm, y + m0 * w->n, st, di);
    if (s != QMM_OK) return s;
  }
  char pre[64];
  snprintf(pre, sizeof(pre), "gemm_by_gemv[slices=%lld]:", (long long)slices);
  prefix_variant(pre);
  return QMM_OK;
}

// IQ4_NL streaming kernel (k % 128 == 0): persistent CTAs over (expert, tile).
// MODE selects the epilogue (IQ_OUT_F16, IQ_SWIGLU with w2 the up matrix,
// IQ_SCALED_F32 with gw the per-pair weights and an fp32 output).
template <int MODE>
static qmm_status launch_iq4_mode(const qmm_weights* w, const qmm_weights* w2, const uint16_t* x, int x_per_pair,
                                  int64_t topk, const int32_t* offsets, const int32_t* perm, int m_plain, void* y,
                                  const float* gw, cudaStream_t st, const DevInfo* di) {
  const size_t smem = kIqLutBytes + kIqRedBytes + kIqGateBytes;
  if (cudaFuncSetAttribute(grouped_iq4_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return QMM_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, grouped_iq4_kernel<MODE>, kIqWarps * 32, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return QMM_ERR_CUDA;
  const int64_t items = ((w->n + 15) / 16) * w->num_experts;
  const int64_t grid = items < (int64_t)per_sm * di->sms ? items : (int64_t)per_sm * di->sms;
  grouped_iq4_kernel<MODE><<<(unsigned)grid, kIqWarps * 32, smem, st>>>(
      static_cast<const uint8_t*>(w->data), w->expert_data_stride,
      w2 ? static_cast<const uint8_t*>(w2->data) : nullptr, w2 ? w2->expert_data_stride : 0, x, x_per_pair,
      (int)topk, offsets, perm, m_plain, y, gw, (int)w->n, (int)w->k, (int)w->num_experts);
  return launch_status();
}

// Tile-resident IQ4_NL kernel (k_iq4t.cuh): one CTA per (expert, item of S
// tiles), programmatic dependent launch.  The weights are loaded before the
// dependency wait when most experts are expected to have pairs (P >= 4E:
// fewer than 2 % of the experts empty for uniform routing) or for the plain
// product; QMM_IQ4T_SPEC=0/1 forces either (measurement knob).
template <int MODE, int S, int SPW, int kMaxReg, bool W16, bool STG = false>
static qmm_status launch_iq4_tile_cfg(const qmm_weights* w0, const qmm_weights* w1, const uint16_t* x, int x_per_pair,
                                      int64_t topk, const int32_t* offsets, const int32_t* perm, int64_t P,
                                      int m_plain, void* y, const float* gw, cudaStream_t st, const int32_t* ids) {
  const int steps = (int)(w0->k / 128), wpc = steps / SPW;
  const int64_t tiles = (w0->n + 15) / 16;
  constexpr int kOut = (MODE == IQ_SWIGLU) ? S / 2 : S;  // output tiles per item
  const int64_t ipe = (tiles + kOut - 1) / kOut;
  if (wpc * 32 > iqt_max_threads(kMaxReg)) return QMM_ERR_UNSUPPORTED_SHAPE;
  const int64_t E = (offsets || ids) ? w0->num_experts : 1;
  // in-kernel routing with fewer pairs than experts (decode: one token's
  // top-k): CTAs only for as many experts as there are pairs, each slot
  // taking the next distinct expert of the ids (MoE block t = 1: 224 instead
  // of 1,792 gate/up CTAs)
  const bool compact = ids && P <= 32 && P < E;
  const int64_t grid = (compact ? P : E) * ipe;
  if (ids && P > kIqtMaxPairs) return QMM_ERR_UNSUPPORTED_SHAPE;
  if (grid < 1 || grid > INT32_MAX) return QMM_ERR_UNSUPPORTED_SHAPE;
  auto kern = iq4_tile_kernel<MODE, S, SPW, kMaxReg, W16, STG>;
  const uint32_t smem = iqt_smem_bytes(S, wpc) + (STG ? (uint32_t)S * 16u * (uint32_t)(w0->k / 32 * 18) : 0u);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return QMM_ERR_CUDA;
  IqtArgs a;
  a.data0 = static_cast<const uint8_t*>(w0->data);
  a.data1 = w1 ? static_cast<const uint8_t*>(w1->data) : nullptr;
  a.dstride0 = w0->expert_data_stride;
  a.dstride1 = w1 ? w1->expert_data_stride : 0;
  a.x = x;
  a.x_per_pair = x_per_pair;
  a.topk = (int)topk;
  a.offsets = ids ? nullptr : offsets;
  a.perm = ids ? nullptr : perm;
  a.ids = ids;
  a.P = (int)P;
  a.m_plain = m_plain;
  a.y = y;
  a.gw = gw;
  a.n = (int)w0->n;
  a.k = (int)w0->k;
  a.E = (int)E;
  a.items_per_expert = (int)ipe;
  a.spec = ((!offsets && !ids) || P >= 4 * E) ? 1 : 0;
  if (const char* e = getenv("QMM_IQ4T_SPEC")) a.spec = (e[0] == '1') ? 1 : 0;
  a.compact = compact ? 1 : 0;
  a.withhold = g_withhold_tile_copies ? 1 : 0;
  if (compact) a.spec = 0;  // a slot's expert is known only after the ids are read
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(wpc * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return QMM_ERR_CUDA;
  set_variant("iq4_tile<mode=%d,s=%d,spw=%d,wpc=%d,w16=%d,stg=%d,spec=%d,route=%s,grid=%d>", MODE, S, SPW, wpc,
              W16 ? 1 : 0, STG ? 1 : 0, a.spec, compact ? "in_kernel_compact" : ids ? "in_kernel" : offsets ? "sorted" : "none",
              (int)grid);
  return launch_status();
}

// Needs k % 256 == 0 and k <= 5376 (at most 21 warps of two super-steps)
// or k % 128 == 0 and k <= 2048 (at most 16 warps of one); returns
// QMM_ERR_UNSUPPORTED_SHAPE, having launched nothing, otherwise.
template <int MODE>
static qmm_status launch_iq4_tile(const qmm_weights* w0, const qmm_weights* w1, const uint16_t* x, int x_per_pair,
                                  int64_t topk, const int32_t* offsets, const int32_t* perm, int64_t P, int m_plain,
                                  void* y, const float* gw, cudaStream_t st, const int32_t* ids) {
  if (w0->fmt != QMM_FMT_IQ4_NL || (w1 && w1->fmt != QMM_FMT_IQ4_NL)) return QMM_ERR_UNSUPPORTED_SHAPE;
  const int64_t k = w0->k, n = w0->n;
  if (k % 128 || k < 128 || n < 1 || n > INT32_MAX / 2) return QMM_ERR_UNSUPPORTED_SHAPE;
  const int64_t steps = k / 128;
  // Items of S tiles (sources) whose activation fragments are shared; each
  // warp holds S * SPW blocks per row pair in registers.  k % 256 == 0 (rows
  // 16-byte aligned): two tiles, two super-steps per warp, 96 registers (two
  // CTAs of up to 10 warps per SM).  Otherwise four tiles, one super-step per
  // warp, 128 registers.  Four tiles at one super-step per warp for k = 2560
  // would need 20 warps of ~128 registers (more than an SM holds).
  // Shared-memory staging of the tiles (k_iq4t.cuh, STG) wherever every
  // source tile is a whole number of 16-byte units (rows * 9k/16 bytes:
  // whole tiles, an even k / 128, or an even number of rows in the last
  // tile).  QMM_IQ4T_STAGE=0/1 forces it off / on where it fits.
  const int64_t rem = n % 16;
  bool stg = rem == 0 || (steps % 2 == 0) || (rem % 2 == 0);
  if (const char* e = getenv("QMM_IQ4T_STAGE")) stg = stg && e[0] == '1';
  if (steps % 2 == 0 && steps / 2 <= iqt_max_threads(96) / 32) {
    if (stg)
      return launch_iq4_tile_cfg<MODE, 2, 2, 96, true, true>(w0, w1, x, x_per_pair, topk, offsets, perm, P, m_plain, y,
                                                             gw, st, ids);
    return launch_iq4_tile_cfg<MODE, 2, 2, 96, true>(w0, w1, x, x_per_pair, topk, offsets, perm, P, m_plain, y, gw,
                                                     st, ids);
  }
  if (steps <= iqt_max_threads(128) / 32) {
    if (stg)
      return launch_iq4_tile_cfg<MODE, 4, 1, 128, false, true>(w0, w1, x, x_per_pair, topk, offsets, perm, P, m_plain,
                                                               y, gw, st, ids);
    return launch_iq4_tile_cfg<MODE, 4, 1, 128, false>(w0, w1, x, x_per_pair, topk, offsets, perm, P, m_plain, y, gw,
                                                       st, ids);
  }
  return QMM_ERR_UNSUPPORTED_SHAPE;
}

static qmm_status launch_iq4_stream(const qmm_weights* w, const uint16_t* x, int x_per_pair, int64_t topk,
                                   const int32_t* offsets, const int32_t* perm, int m_plain, uint16_t* y,
                                   cudaStream_t st, const DevInfo* di) {
  return launch_iq4_mode<IQ_OUT_F16>(w, nullptr, x, x_per_pair, topk, offsets, perm, m_plain, y, nullptr, st, di);
}

template <int FMT>
static qmm_status launch_grouped(const qmm_weights* w, const uint16_t* x, int x_per_pair, int64_t topk,
                                 const int32_t* offsets, const int32_t* perm, uint16_t* y, cudaStream_t st) {
  const int64_t tiles = (w->n + 15) / 16;
  const int64_t items = tiles * w->num_experts;
  const int64_t blocks = (items + 3) / 4;
  if (blocks > INT32_MAX) return QMM_ERR_UNSUPPORTED_SHAPE;
  grouped_gemv_kernel<FMT><<<(unsigned)blocks, 128, 0, st>>>(
      static_cast<const uint8_t*>(w->data), w->expert_data_stride, static_cast<const uint8_t*>(w->scales),
      w->expert_scale_stride, w->global_scale, x, x_per_pair, (int)topk, offsets, perm, y, w->n, w->k,
      (int)w->num_experts);
  return launch_status();
}

// ---------------------------------------------------------------------------
// Fixed device scratch for qmm_grouped_gemv_noalloc
// ---------------------------------------------------------------------------
// Routing offsets (first kNoAllocOffsetInts words) and the pair permutation
// (next kNoAllocMaxPairs words) for callers that cannot hand the library a
// workspace.  Every GPU that loads the library holds this array (258 KiB)
// until the process exits; all calls on a device share it.
constexpr int64_t kNoAllocMaxPairs = 65536;
constexpr int kNoAllocOffsetInts = 512;  // >= kRouteMaxExperts + 1; keeps the permutation 256-byte aligned
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocOffsetInts + kNoAllocMaxPairs];
static int32_t* g_noalloc_addr[64];  // device address of g_noalloc_scratch, per device

// The host-side name g_noalloc_scratch is only a stand-in; the kernels need
// the device address, fetched once per device with that device current.
static qmm_status noalloc_scratch(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QMM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return QMM_ERR_CUDA;
    g_noalloc_addr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_noalloc_addr[dev];
  return QMM_OK;
}

}  // namespace qmm

using namespace qmm;

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

size_t qmm_data_bytes(int32_t fmt, int64_t n, int64_t k) {
  if (!valid_fmt(fmt) || n < 0 || k < 0) return 0;
  if (k % fmt_group(fmt)) return 0;
  if (fmt == QMM_FMT_IQ4_NL) return (size_t)n * (size_t)(k / 32) * 18u;
  return (size_t)n * (size_t)(k / 2);
}

size_t qmm_scale_bytes(int32_t fmt, int64_t n, int64_t k) {
  if (!valid_fmt(fmt) || n < 0 || k < 0 || fmt == QMM_FMT_IQ4_NL || (k % fmt_group(fmt))) return 0;
  if (fmt == QMM_FMT_MXFP4) return (size_t)n * (size_t)(k / 32);
  return (size_t)n * (size_t)(k / 16) * (fmt == QMM_FMT_FP4G16_F16 ? 2u : 1u);
}

size_t qmm_packed_bytes(int32_t fmt, int64_t n, int64_t k) {
  return qmm_data_bytes(fmt, n, k) + qmm_scale_bytes(fmt, n, k) + (fmt == QMM_FMT_FP4G16_E4M3 ? 4u : 0u);
}

const char* qmm_status_string(int32_t s) {
  switch (s) {
    case QMM_OK: return "ok";
    case QMM_ERR_INVALID_ARG: return "invalid argument";
    case QMM_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case QMM_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case QMM_ERR_NOT_SM100: return "current device is not sm_100 (B200)";
    case QMM_ERR_CUDA: return "CUDA runtime error";
    case QMM_ERR_TIMEOUT: return "a kernel pipeline wait timed out";
    case QMM_ERR_DEVICE_FAULT: return "bad data seen on the device (expert id out of range)";
    case QMM_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

const char* qmm_last_variant(void) { return t_variant; }

const char* qmm_version(void) { return "qmm 0.1 (sm_100a)"; }

qmm_status qmm_dequant(const qmm_weights* w, uint16_t* out, void* stream) {
  qmm_status s = check_weights(w, false);
  if (s != QMM_OK) return s;
  DevInfo* di = nullptr;
  if ((s = device_info(&di)) != QMM_OK) return s;
  const int64_t total = w->n * w->k;
  if (total == 0) return QMM_OK;
  if (!out) return QMM_ERR_INVALID_ARG;
  if (!aligned16(out)) return QMM_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint8_t* data = static_cast<const uint8_t*>(w->data);
  const uint8_t* sc = static_cast<const uint8_t*>(w->scales);
  if (w->fmt == QMM_FMT_IQ4_NL) {
    const int64_t nb = total / 32;
    dequant_iq4nl_kernel<<<grid_for(nb, 256, di->sms), 256, 0, st>>>(data, out, nb);
    set_variant("dequant_iq4nl");
  } else if (w->fmt == QMM_FMT_FP4G16_F16) {
    const int64_t ng = total / 16;
    dequant_fp4_kernel<2><<<grid_for(ng, 256, di->sms), 256, 0, st>>>(data, sc, 1.0f, out, ng);
    set_variant("dequant_fp4<fmt=2>");
  } else if (w->fmt == QMM_FMT_MXFP4) {
    const int64_t ng = total / 32;
    dequant_mxfp4_kernel<<<grid_for(ng, 256, di->sms), 256, 0, st>>>(data, sc, out, ng);
    set_variant("dequant_mxfp4");
  } else {
    const int64_t ng = total / 16;
    dequant_fp4_kernel<3><<<grid_for(ng, 256, di->sms), 256, 0, st>>>(data, sc, w->global_scale, out, ng);
    set_variant("dequant_fp4<fmt=3>");
  }
  return launch_status();
}

qmm_status qmm_quantize(int32_t fmt, const uint16_t* w, int64_t n, int64_t k, void* data, void* scales, void* stream) {
  if (!valid_fmt(fmt) || n < 0 || k < 0) return QMM_ERR_INVALID_ARG;
  if (fmt == QMM_FMT_FP4G16_E4M3) return QMM_ERR_UNSUPPORTED_SHAPE;  // needs a matrix-wide global scale: not encoded
  if (k % fmt_group(fmt) || n > INT32_MAX || k > INT32_MAX) return QMM_ERR_UNSUPPORTED_SHAPE;
  qmm_status s;
  DevInfo* di = nullptr;
  if ((s = device_info(&di)) != QMM_OK) return s;
  const int64_t total = n * k;
  if (total == 0) return QMM_OK;
  if (!w || !data || (fmt != QMM_FMT_IQ4_NL && !scales)) return QMM_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(data) || (scales && !aligned16(scales))) return QMM_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* d = static_cast<uint8_t*>(data);
  uint8_t* sc = static_cast<uint8_t*>(scales);
  if (fmt == QMM_FMT_IQ4_NL) {
    const int64_t nb = total / 32;
    quantize_iq4nl_kernel<<<grid_for(nb, 128, di->sms), 128, 0, st>>>(w, d, nb);
    set_variant("quantize_iq4nl");
  } else if (fmt == QMM_FMT_MXFP4) {
    const int64_t ng = total / 32;
    quantize_fp4_kernel<4><<<grid_for(ng, 128, di->sms), 128, 0, st>>>(w, d, sc, ng);
    set_variant("quantize_fp4<fmt=4>");
  } else {
    const int64_t ng = total / 16;
    quantize_fp4_kernel<2><<<grid_for(ng, 128, di->sms), 128, 0, st>>>(w, d, sc, ng);
    set_variant("quantize_fp4<fmt=2>");
  }
  if (cudaGetLastError() != cudaSuccess) return QMM_ERR_CUDA;
  // The GEMV and expert kernels read W before their dependency wait, so the
  // kernel right before them must not be the one that wrote W: this empty
  // kernel (plain launch, it starts after the encoder has finished) takes
  // that place.
  ordering_kernel<<<1, 32, 0, st>>>();
  return launch_status();
}

static qmm_status zero_output(uint16_t* y, int64_t count, cudaStream_t st, const DevInfo* di) {
  zero_fill_kernel<<<grid_for(count, 256, di->sms), 256, 0, st>>>(y, count);
  set_variant("zero_fill");
  return launch_status();
}

qmm_status qmm_gemv(const qmm_weights* w, const uint16_t* x, int64_t m, uint16_t* y, void* ws, size_t ws_bytes,
                    void* stream) {
  (void)ws;
  (void)ws_bytes;
  qmm_status s = check_weights(w, false);
  if (s != QMM_OK) return s;
  if (m < 0) return QMM_ERR_INVALID_ARG;
  if (m > 16) return QMM_ERR_UNSUPPORTED_SHAPE;
  DevInfo* di = nullptr;
  if ((s = device_info(&di)) != QMM_OK) return s;
  if (m == 0 || w->n == 0) return QMM_OK;
  if (!y || (w->k > 0 && !x)) return QMM_ERR_INVALID_ARG;
  if (!aligned16(y) || (x && !aligned16(x))) return QMM_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (w->k == 0) return zero_output(y, m * w->n, st, di);
  switch (w->fmt) {
    case QMM_FMT_IQ4_NL: return gemv_fmt<1>(w, x, (int)m, y, st, di);
    case QMM_FMT_FP4G16_F16: return gemv_fmt<2>(w, x, (int)m, y, st, di);
    case QMM_FMT_MXFP4: return gemv_fmt<4>(w, x, (int)m, y, st, di);
    default: return gemv_fmt<3>(w, x, (int)m, y, st, di);
  }
}

// Device address of bytes [p, p + bytes) of page-locked host memory mapped
// into the current device's address space (16-byte aligned), else nullptr
// (pageable memory, or a range whose ends are not in the same mapping).
static void* mapped_host_alias(const void* p, size_t bytes) {
  if (!p || bytes == 0) return nullptr;
  cudaPointerAttributes a, b;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || !a.devicePointer || (reinterpret_cast<uintptr_t>(a.devicePointer) & 15u))
    return nullptr;
  const char* last = static_cast<const char*>(p) + bytes - 1;
  if (cudaPointerGetAttributes(&b, last) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (b.type != cudaMemoryTypeHost || !b.devicePointer ||
      static_cast<char*>(b.devicePointer) - static_cast<char*>(a.devicePointer) != (ptrdiff_t)(bytes - 1))
    return nullptr;
  return a.devicePointer;
}

qmm_status qmm_gemv_host(const qmm_weights* w, const uint16_t* x_host, int64_t m, uint16_t* y_host, uint16_t* x_dev,
                         uint16_t* y_dev, void* stream) {
  qmm_status s = check_weights(w, false);
  if (s != QMM_OK) return s;
  if (m < 0) return QMM_ERR_INVALID_ARG;
  if (m > 16) return QMM_ERR_UNSUPPORTED_SHAPE;
  if (m == 0 || w->n == 0) return QMM_OK;
  if (!y_host || !y_dev || (w->k > 0 && (!x_host || !x_dev))) return QMM_ERR_INVALID_ARG;
  if (!aligned16(y_dev) || (x_dev && !aligned16(x_dev))) return QMM_ERR_MISALIGNED;  // before anything is queued
  DevInfo* di = nullptr;
  if ((s = device_info(&di)) != QMM_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t xb = 2 * (size_t)m * (size_t)w->k, yb = 2 * (size_t)m * (size_t)w->n;
  // Page-locked host buffers are used in place through their device mapping:
  // a copy kernel brings x in (the GEMV's weight stream starts meanwhile) and
  // the GEMV stores y straight to host memory.  Pageable buffers go through
  // the copy engine.
  const void* xa = mapped_host_alias(x_host, xb);
  void* ya = mapped_host_alias(y_host, yb);
  if (xb) {
    if (xa && xb % 16 == 0) {
      const int64_t n16 = (int64_t)(xb / 16);  // at most 16 x 2^30 / 16: the grid covers it
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)((n16 + 255) / 256));
      cfg.blockDim = dim3(256);
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaLaunchKernelEx(&cfg, fetch16_kernel, static_cast<const uint4*>(xa), reinterpret_cast<uint4*>(x_dev),
                             n16) != cudaSuccess)
        return QMM_ERR_CUDA;
    } else if (cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, st) != cudaSuccess) {
      return QMM_ERR_CUDA;
    }
  }
  if (ya) return qmm_gemv(w, x_dev, m, static_cast<uint16_t*>(ya), nullptr, 0, stream);
  if ((s = qmm_gemv(w, x_dev, m, y_dev, nullptr, 0, stream)) != QMM_OK) return s;
  if (cudaMemcpyAsync(y_host, y_dev, yb, cudaMemcpyDeviceToHost, st) != cudaSuccess) return QMM_ERR_CUDA;
  return QMM_OK;
}

// Batches under 256 tokens: tensor-core GEMM or the decode GEMV over 16-token
// slices, whichever a cost model calibrated on B200 puts first.  The GEMM
// (128 x 256 tiles, one per SM at a time) is decode-bound at about 22,800
// weights per us per SM, so it costs its waves of tiles whatever m is; the
// GEMV streams the packed bytes once per slice at about 2.9 TB/s (the 16-token
// rate) plus ~3 us of launch and tail.  qmm_gemm per launch, us, tc / slices:
// in_proj 18560x4096 m = 32: 46.0 / 37.7, m = 48: 46.7 / 55.7; out_proj
// 4096x8192 (16 tiles) m = 128: 87.7 / 75.7; LM head 256000x4096 m = 17:
// 292 / 365.  From 256 tokens the GEMM's 256-token tiles always lead.
static bool gemm_prefers_tc(int64_t m, int64_t n, int64_t k, size_t packed_bytes, int sms) {
  if (m >= 256) return true;
  const double tiles = (double)((m + 127) / 128) * (double)((n + 255) / 256);
  const double waves = ceil(tiles / (double)sms);
  const double tc_us = 5.0 + waves * 256.0 * (double)k / 22800.0;
  const double gemv_us = (double)((m + 15) / 16) * (3.0 + (double)packed_bytes / 2.9e6);
  return tc_us < gemv_us;
}

qmm_status qmm_gemm(const qmm_weights* w, const uint16_t* x, int64_t m, uint16_t* y, void* ws, size_t ws_bytes,
                    void* stream) {
  (void)ws;
  (void)ws_bytes;
  qmm_status s = check_weights(w, false);
  if (s != QMM_OK) return s;
  if (m < 0) return QMM_ERR_INVALID_ARG;
  if (m > INT32_MAX) return QMM_ERR_UNSUPPORTED_SHAPE;
  DevInfo* di = nullptr;
  if ((s = device_info(&di)) != QMM_OK) return s;
  if (m == 0 || w->n == 0) return QMM_OK;
  if (!y || (w->k > 0 && !x)) return QMM_ERR_INVALID_ARG;
  if (!aligned16(y) || (x && !aligned16(x))) return QMM_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (w->k == 0) return zero_output(y, m * w->n, st, di);
  // QMM_GEMM_VARIANT=tc / gemv forces either path at any m (measurements),
  // =tile the one-tile-per-CTA tensor-core kernel.
  const char* gv = getenv("QMM_GEMM_VARIANT");
  const bool force_tc = gv && (!strcmp(gv, "tc") || !strcmp(gv, "tile"));
  const bool force_gemv = gv && !strcmp(gv, "gemv");
  const size_t packed = qmm_packed_bytes(w->fmt, w->n, w->k);
  const bool tc = w->k % kGemmBK == 0 && !force_gemv &&
                  (force_tc || gemm_prefers_tc(m, w->n, w->k, packed, di->sms));
  // persistent kernel when k is a multiple of its 256-wide staging chunk
  const bool persist = !(gv && !strcmp(gv, "tile")) && w->k % (kGemmChunkSteps * kGemmBK) == 0;
  switch (w->fmt) {
    case QMM_FMT_IQ4_NL:  // the persistent kernel only (256-wide staging chunk = 8 blocks = 144 bytes a row)
      if (!tc || !persist) return gemm_by_gemv<1>(w, x, m, y, st, di);
      return launch_gemm_tc_persistent<1>(w, x, (int)m, y, st, di);
    case QMM_FMT_FP4G16_F16:
      if (!tc) return gemm_by_gemv<2>(w, x, m, y, st, di);
      return persist ? launch_gemm_tc_persistent<2>(w, x, (int)m, y, st, di) : launch_gemm_tc<2>(w, x, (int)m, y, st, di);
    case QMM_FMT_MXFP4:  // the persistent kernel only (its 256-wide staging chunk holds 8 E8M0 bytes a row)
      if (!tc || !persist) return gemm_by_gemv<4>(w, x, m, y, st, di);
      return launch_gemm_tc_persistent<4>(w, x, (int)m, y, st, di);
    default:
      if (!tc) return gemm_by_gemv<3>(w, x, m, y, st, di);
      return persist ? launch_gemm_tc_persistent<3>(w, x, (int)m, y, st, di) : launch_gemm_tc<3>(w, x, (int)m, y, st, di);
  }
}

static size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

static qmm_status check_routing(const int32_t* ids, int64_t t, int64_t topk, int64_t num_experts) {
  if (t < 0 || topk < 0 || num_experts < 1) return QMM_ERR_INVALID_ARG;
  // bound the factors before multiplying them (no int64 overflow)
  if (num_experts > kRouteMaxExperts || (topk > 0 && t > (INT32_MAX / 2) / topk)) return QMM_ERR_UNSUPPORTED_SHAPE;
  if (t * topk > 0 && !ids) return QMM_ERR_INVALID_ARG;
  if (ids && !aligned16(ids)) return QMM_ERR_MISALIGNED;
  return QMM_OK;
}

qmm_status qmm_route(const int32_t* topk_ids, int64_t t, int64_t topk, int64_t num_experts, int32_t* expert_offsets,
                     int32_t* pair_perm, void* ws, size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  qmm_status s = check_routing(topk_ids, t, topk, num_experts);
  if (s != QMM_OK) return s;
  if (!expert_offsets || (t * topk > 0 && !pair_perm)) return QMM_ERR_INVALID_ARG;
  if (!aligned16(expert_offsets) || (pair_perm && !aligned16(pair_perm))) return QMM_ERR_MISALIGNED;
  DevInfo* di = nullptr;
  if ((s = device_info(&di)) != QMM_OK) return s;
  route_kernel<<<1, kRouteThreads, 0, static_cast<cudaStream_t>(stream)>>>(topk_ids, (int)(t * topk),
                                                                          (int)num_experts, expert_offsets, pair_perm);
  set_variant("route_stable_counting_sort");
  return launch_status();
}

static qmm_status check_expert_strides(const qmm_weights* w) {
  const size_t db = qmm_data_bytes(w->fmt, w->n, w->k), sb = qmm_scale_bytes(w->fmt, w->n, w->k);
  if (w->num_experts > 1) {
    if (w->expert_data_stride < (int64_t)db || (sb && w->expert_scale_stride < (int64_t)sb)) return QMM_ERR_INVALID_ARG;
    if ((w->expert_data_stride & 15) || (sb && (w->expert_scale_stride & 15))) return QMM_ERR_MISALIGNED;
  }
  return QMM_OK;
}

qmm_status qmm_grouped_gemv(const qmm_weights* experts, const uint16_t* x, int32_t x_per_pair, const int32_t* topk_ids,
                            int64_t t, int64_t topk, uint16_t* y, void* ws, size_t ws_bytes, void* stream) {
  qmm_status s = check_weights(experts, true);
  if (s != QMM_OK) return s;
  if ((s = check_expert_strides(experts)) != QMM_OK) return s;
  if ((s = check_routing(topk_ids, t, topk, experts->num_experts)) != QMM_OK) return s;
  if (x_per_pair != 0 && x_per_pair != 1) return QMM_ERR_INVALID_ARG;
  DevInfo* di = nullptr;
  if ((s = device_info(&di)) != QMM_OK) return s;
  const int64_t P = t * topk;
  if (P == 0 || experts->n == 0) return QMM_OK;
  if (!y || (experts->k > 0 && !x)) return QMM_ERR_INVALID_ARG;
  if (!aligned16(y) || (x && !aligned16(x))) return QMM_ERR_MISALIGNED;
  const size_t need = qmm_workspace_bytes(QMM_OP_GROUPED, experts, 0, t, topk);
  if (!ws || ws_bytes < need) return QMM_ERR_WORKSPACE;
  if (!aligned16(ws)) return QMM_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int pick = gemv_variant_env();
  // IQ4_NL: the tile-resident kernel (its weight loads overlap the previous
  // kernel when most experts have pairs); up to kIqtInKernelRoutePairs pairs
  // each CTA finds its expert's pairs itself, so no routing pass runs.
  // QMM_GEMV_VARIANT=iq4 keeps the streaming kernel.
  const bool iq4_tile = pick == PICK_IQ4_TILE || pick == PICK_DEFAULT;
  if (experts->fmt == QMM_FMT_IQ4_NL && experts->k > 0 && iq4_tile && P <= kIqtInKernelRoutePairs) {
    s = launch_iq4_tile<IQ_OUT_F16>(experts, nullptr, x, x_per_pair, topk, nullptr, nullptr, P, 0, y, nullptr, st,
                                    topk_ids);
    if (s != QMM_ERR_UNSUPPORTED_SHAPE) {
      prefix_variant("grouped_iq4_tile+in_kernel_route:");
      return s;
    }
  }
  int32_t* offsets = static_cast<int32_t*>(ws);
  int32_t* perm = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + align256(4 * (size_t)(experts->num_experts + 1)));
  route_kernel<<<1, kRouteThreads, 0, st>>>(topk_ids, (int)P, (int)experts->num_experts, offsets, perm);
  if (cudaGetLastError() != cudaSuccess) return QMM_ERR_CUDA;
  if (experts->k == 0) {
    // every routed pair's row is an empty sum
    zero_fill_kernel<<<grid_for(P * experts->n, 256, di->sms), 256, 0, st>>>(y, P * experts->n);
    set_variant("route+zero_fill");
    return launch_status();
  }
  if (experts->fmt == QMM_FMT_IQ4_NL && iq4_tile) {  // more pairs: after the routing sort
    s = launch_iq4_tile<IQ_OUT_F16>(experts, nullptr, x, x_per_pair, topk, offsets, perm, P, 0, y, nullptr, st);
    if (s != QMM_ERR_UNSUPPORTED_SHAPE) {
      prefix_variant("route+grouped_iq4_tile:");
      return s;
    }
  }
  if (experts->fmt == QMM_FMT_IQ4_NL && experts->k % 128 == 0 && (pick == PICK_DEFAULT || pick == PICK_IQ4_STREAM)) {
    s = launch_iq4_stream(experts, x, x_per_pair, topk, offsets, perm, 0, y, st, di);
    set_variant("route+grouped_iq4_stream");
    return s;
  }
  switch (experts->fmt) {
    case QMM_FMT_IQ4_NL: s = launch_grouped<1>(experts, x, x_per_pair, topk, offsets, perm, y, st); break;
    case QMM_FMT_FP4G16_F16: s = launch_grouped<2>(experts, x, x_per_pair, topk, offsets, perm, y, st); break;
    case QMM_FMT_MXFP4: s = launch_grouped<4>(experts, x, x_per_pair, topk, offsets, perm, y, st); break;
    default: s = launch_grouped<3>(experts, x, x_per_pair, topk, offsets, perm, y, st); break;
  }
  set_variant("route+grouped_gemv_generic<fmt=%d>", experts->fmt);
  return s;
}

size_t qmm_workspace_bytes(int32_t op, const qmm_weights* w, int64_t m, int64_t t, int64_t topk) {
  if (op == QMM_OP_GROUPED || op == QMM_OP_MOE) {
    if (!w || w->num_experts < 1 || t < 0 || topk < 0 || w->n < 0 || w->k < 0) return 0;
    if (topk > 0 && t > (INT32_MAX / 2) / topk) return 0;  // the call itself refuses these sizes
    size_t b = align256(4 * (size_t)(w->num_experts + 1)) + align256(4 * (size_t)(t * topk));
    if (op == QMM_OP_MOE)  // h [t*topk][f] fp16, g-scaled slot outputs [t*topk][d] fp32
      b += align256(2 * (size_t)(t * topk) * (size_t)w->n) + align256(4 * (size_t)(t * topk) * (size_t)w->k);
    return b;
  }
  (void)m;
  return 0;
}

qmm_status qmm_grouped_gemv_noalloc(const qmm_weights* experts, const uint16_t* x, int32_t x_per_pair,
                                    const int32_t* topk_ids, int64_t t, int64_t topk, uint16_t* y, void* stream) {
  qmm_status s = check_weights(experts, true);
  if (s != QMM_OK) return s;
  if ((s = check_expert_strides(experts)) != QMM_OK) return s;
  if ((s = check_routing(topk_ids, t, topk, experts->num_experts)) != QMM_OK) return s;
  if (x_per_pair != 0 && x_per_pair != 1) return QMM_ERR_INVALID_ARG;
  if (t * topk > kNoAllocMaxPairs) return QMM_ERR_UNSUPPORTED_SHAPE;  // beyond the fixed scratch
  DevInfo* di = nullptr;
  if ((s = device_info(&di)) != QMM_OK) return s;
  const int64_t P = t * topk;
  if (P == 0 || experts->n == 0) return QMM_OK;
  if (!y || (experts->k > 0 && !x)) return QMM_ERR_INVALID_ARG;
  if (!aligned16(y) || (x && !aligned16(x))) return QMM_ERR_MISALIGNED;
  int32_t* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != QMM_OK) return s;
  // The routing kernel rewrites offsets[0..E] and every permutation slot the
  // grouped kernel reads, so nothing in the shared array has to be cleared.
  int32_t* offsets = scratch;
  int32_t* perm = scratch + kNoAllocOffsetInts;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  route_kernel<<<1, kRouteThreads, 0, st>>>(topk_ids, (int)P, (int)experts->num_experts, offsets, perm);
  if (cudaGetLastError() != cudaSuccess) return QMM_ERR_CUDA;
  if (experts->k == 0) {
    zero_fill_kernel<<<grid_for(P * experts->n, 256, di->sms), 256, 0, st>>>(y, P * experts->n);
    set_variant("noalloc:route+zero_fill");
    return launch_status();
  }
  switch (experts->fmt) {
    case QMM_FMT_IQ4_NL: s = launch_grouped<1>(experts, x, x_per_pair, topk, offsets, perm, y, st); break;
    case QMM_FMT_FP4G16_F16: s = launch_grouped<2>(experts, x, x_per_pair, topk, offsets, perm, y, st); break;
    case QMM_FMT_MXFP4: s = launch_grouped<4>(experts, x, x_per_pair, topk, offsets, perm, y, st); break;
    default: s = launch_grouped<3>(experts, x, x_per_pair, topk, offsets, perm, y, st); break;
  }
  set_variant("noalloc:route+grouped_gemv_generic<fmt=%d>", experts->fmt);
  return s;
}

qmm_status qmm_router_topk(const uint16_t* x, const uint16_t* w_router, const float* bias, int64_t t, int64_t k,
                           int64_t num_experts, int64_t topk, int32_t* topk_ids, float* topk_weights, float* logits,
                           void* stream) {
  if (t < 0 || k < 0 || num_experts < 1 || topk < 1 || topk > num_experts) return QMM_ERR_INVALID_ARG;
  if (num_experts > kRouterMaxExperts || k % 8 || t > INT32_MAX) return QMM_ERR_UNSUPPORTED_SHAPE;
  DevInfo* di = nullptr;
  qmm_status s = device_info(&di);
  if (s != QMM_OK) return s;
  if (t == 0) return QMM_OK;
  if (!bias || !topk_ids || !topk_weights || (k > 0 && (!x || !w_router))) return QMM_ERR_INVALID_ARG;
  if ((x && !aligned16(x)) || (w_router && !aligned16(w_router)) || !aligned16(bias) || !aligned16(topk_ids) ||
      !aligned16(topk_weights) || (logits && !aligned16(logits)))
    return QMM_ERR_MISALIGNED;
  // a cluster of cs CTAs per token splits k: 8 for a few tokens, 2 for more
  // (router alone on B200, us per launch at cs = 1 / 2 / 4 / 8: one token
  // 7.8 / 6.4 / 6.2 / 5.8; 64 tokens 8.4 / 7.0 / 10.2 / 17.0).
  // QMM_ROUTER_CS=1/2/4/8 forces a size (measurement knob).
  int cs = t <= 4 ? 8 : 2;
  if (const char* e = getenv("QMM_ROUTER_CS")) {
    const int v = atoi(e);
    if (v == 1 || v == 2 || v == 4 || v == 8) cs = v;
  }
  if ((int64_t)t * cs > INT32_MAX) cs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(t * cs));
  cfg.blockDim = dim3(kRouterThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, router_topk_kernel, x, w_router, bias, (int)k, (int)num_experts, (int)topk, topk_ids,
                         topk_weights, logits) != cudaSuccess)
    return QMM_ERR_CUDA;
  set_variant("router_topk<cs=%d>", cs);
  return launch_status();
}

qmm_status qmm_moe_routed(const qmm_weights* gate, const qmm_weights* up, const qmm_weights* down, const uint16_t* x,
                          const int32_t* topk_ids, const float* topk_weights, int64_t t, int64_t topk, uint16_t* out,
                          void* ws, size_t ws_bytes, void* stream) {
  qmm_status s;
  for (const qmm_weights* w : {gate, up, down}) {
    if ((s = check_weights(w, true)) != QMM_OK) return s;
    if ((s = check_expert_strides(w)) != QMM_OK) return s;
    if (w->fmt != QMM_FMT_IQ4_NL) return QMM_ERR_UNSUPPORTED_SHAPE;
  }
  const int64_t f = gate->n, d = gate->k, E = gate->num_experts;
  if (up->n != f || up->k != d || down->n != d || down->k != f || up->num_experts != E || down->num_experts != E)
    return QMM_ERR_INVALID_ARG;
  if ((s = check_routing(topk_ids, t, topk, E)) != QMM_OK) return s;
  if (d % 128 || f % 128 || d > INT32_MAX / 2 || f > INT32_MAX / 2) return QMM_ERR_UNSUPPORTED_SHAPE;
  DevInfo* di = nullptr;
  if ((s = device_info(&di)) != QMM_OK) return s;
  const int64_t P = t * topk;
  if (P == 0 || d == 0) return QMM_OK;
  if (!out || !x || !topk_weights) return QMM_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(x) || !aligned16(topk_weights)) return QMM_ERR_MISALIGNED;
  const size_t need = qmm_workspace_bytes(QMM_OP_MOE, gate, 0, t, topk);
  if (!ws || ws_bytes < need) return QMM_ERR_WORKSPACE;
  if (!aligned16(ws)) return QMM_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* p = static_cast<char*>(ws);
  int32_t* offsets = reinterpret_cast<int32_t*>(p);
  p += align256(4 * (size_t)(E + 1));
  int32_t* perm = reinterpret_cast<int32_t*>(p);
  p += align256(4 * (size_t)P);
  uint16_t* h = reinterpret_cast<uint16_t*>(p);
  p += align256(2 * (size_t)P * (size_t)f);
  float* yg = reinterpret_cast<float*>(p);
  // tile-resident kernels (measured faster than the streaming ones at 1, 4,
  // 16 and 64 tokens); up to kIqtInKernelRoutePairs pairs each CTA finds its
  // expert's pairs itself, so no routing pass runs.  QMM_GEMV_VARIANT=iq4
  // keeps the streaming kernels.
  const int pick = gemv_variant_env();
  const bool tile = pick == PICK_IQ4_TILE || pick == PICK_DEFAULT;
  if (f > 0 && tile && P <= kIqtInKernelRoutePairs) {
    s = launch_iq4_tile<IQ_SWIGLU>(gate, up, x, 0, topk, nullptr, nullptr, P, 0, h, nullptr, st, topk_ids);
    if (s == QMM_OK)
      s = launch_iq4_tile<IQ_SCALED_F32>(down, nullptr, h, 1, topk, nullptr, nullptr, P, 0, yg, topk_weights, st,
                                         topk_ids);
    if (s == QMM_OK) {
      if (launch_pdl(combine_kernel, dim3((unsigned)grid_for(t * (d / 8), 256, di->sms)), dim3(256), 0, st,
                     (const float*)yg, topk_ids, (int)E, (int)t, (int)topk, (int)d, out) != cudaSuccess)
        return QMM_ERR_CUDA;
      set_variant("moe:gate_up_swiglu_iq4_tile+down_scaled_iq4_tile+combine(in-kernel routing)");
      return launch_status();
    }
    if (s != QMM_ERR_UNSUPPORTED_SHAPE) return s;
  }
  route_kernel<<<1, kRouteThreads, 0, st>>>(topk_ids, (int)P, (int)E, offsets, perm);
  if (cudaGetLastError() != cudaSuccess) return QMM_ERR_CUDA;
  if (f == 0) {
    // h is empty: every slot output is an empty sum
    zero_fill_kernel<<<grid_for(t * d, 256, di->sms), 256, 0, st>>>(out, t * d);
    set_variant("moe:route+zero_fill");
    return launch_status();
  }
  if (tile) {  // more pairs: after the routing sort
    s = launch_iq4_tile<IQ_SWIGLU>(gate, up, x, 0, topk, offsets, perm, P, 0, h, nullptr, st);
    if (s == QMM_OK)
      s = launch_iq4_tile<IQ_SCALED_F32>(down, nullptr, h, 1, topk, offsets, perm, P, 0, yg, topk_weights, st);
    if (s == QMM_OK) {
      if (launch_pdl(combine_kernel, dim3((unsigned)grid_for(t * (d / 8), 256, di->sms)), dim3(256), 0, st,
                     (const float*)yg, topk_ids, (int)E, (int)t, (int)topk, (int)d, out) != cudaSuccess)
        return QMM_ERR_CUDA;
      set_variant("moe:route+gate_up_swiglu_iq4_tile+down_scaled_iq4_tile+combine");
      return launch_status();
    }
    if (s != QMM_ERR_UNSUPPORTED_SHAPE) return s;
  }
  if ((s = launch_iq4_mode<IQ_SWIGLU>(gate, up, x, 0, topk, offsets, perm, 0, h, nullptr, st, di)) != QMM_OK)
    return s;
  if ((s = launch_iq4_mode<IQ_SCALED_F32>(down, nullptr, h, 1, topk, offsets, perm, 0, yg, topk_weights, st, di)) !=
      QMM_OK)
    return s;
  if (launch_pdl(combine_kernel, dim3((unsigned)grid_for(t * (d / 8), 256, di->sms)), dim3(256), 0, st,
                 (const float*)yg, topk_ids, (int)E, (int)t, (int)topk, (int)d, out) != cudaSuccess)
    return QMM_ERR_CUDA;
  set_variant("moe:route+gate_up_swiglu_iq4+down_scaled_iq4+combine");
  return launch_status();
}

qmm_status qmm_debug_set(int32_t what, int64_t value) {
  DevInfo* di = nullptr;
  qmm_status s = device_info(&di);
  if (s != QMM_OK) return s;
  if (what == QMM_DEBUG_WAIT_LIMIT_NS) {
    if (value < 1000 || value > 10000000000ll) return QMM_ERR_INVALID_ARG;
    const unsigned long long v = (unsigned long long)value;
    return cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? QMM_OK : QMM_ERR_CUDA;
  }
  if (what == QMM_DEBUG_WITHHOLD_X_TILES) {
    if (value != 0 && value != 1) return QMM_ERR_INVALID_ARG;
    const unsigned int v = value ? kTestWithholdXTiles : 0u;
    return cudaMemcpyToSymbol(g_test_flags, &v, sizeof(v)) == cudaSuccess ? QMM_OK : QMM_ERR_CUDA;
  }
  if (what == QMM_DEBUG_WITHHOLD_TILE_COPIES) {  // a launch argument of the tile kernel (no device read)
    if (value != 0 && value != 1) return QMM_ERR_INVALID_ARG;
    g_withhold_tile_copies = value != 0;
    return QMM_OK;
  }
  return QMM_ERR_INVALID_ARG;
}

qmm_status qmm_sync_check(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return QMM_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_err_word, sizeof(v)) != cudaSuccess) return QMM_ERR_CUDA;
  if (v == 0) return QMM_OK;
  if (cudaMemcpyToSymbol(g_err_word, &zero, sizeof(zero)) != cudaSuccess) return QMM_ERR_CUDA;
  if (v & ERR_TIMEOUT) return QMM_ERR_TIMEOUT;
  return QMM_ERR_DEVICE_FAULT;
}

}  // extern "C"
