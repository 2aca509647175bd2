/*
 * qmm.h -- C ABI of the packed 4-bit weight matmul library (libqmm.so) for
 * NVIDIA B200 (sm_100a).
 *
 * The library decodes and multiplies weights that stay packed in GPU memory:
 *
 *   IQ4_NL      18-byte blocks of 32 weights: a little-endian fp16 scale d,
 *               then 16 bytes of 4-bit indices into the 16-entry non-linear
 *               table {-127,-104,-83,-65,-49,-35,-22,-10,1,13,25,38,53,69,89,
 *               113}; the low nibble of byte j is weight j of the block, the
 *               high nibble weight j+16.  A row of k weights is k/32
 *               consecutive blocks; rows follow each other.
 *               ("Mark-Experimental-V3-8B", section "Quantization".)
 *   FP4G16_F16  E2M1 codes, two per byte (low nibble = even k), row-major
 *               [n][k/2]; one fp16 scale per 16 consecutive k, row-major
 *               [n][k/16].  Weight = fp16(code * scale).
 *   FP4G16_E4M3 the same codes; one E4M3FN byte scale per 16 consecutive k,
 *               row-major [n][k/16], and one fp32 global scale g per matrix.
 *               Weight = fp16(fp32(code * e4m3 * g)).
 *               ("Mamb2_8B_FP4_Recall_SQ3.25", section "Representation",
 *               paragraph "Weights": E2M1 codes with magnitudes 0, 0.5, 1,
 *               1.5, 2, 3, 4, 6, 16-element groups along the input axis, an
 *               E4M3FN block scale per group and an FP32 scale per matrix.)
 *
 * A weight matrix W is [n][k]: n output rows, k input columns; groups run
 * along k.  Activations x are fp16 [m][k] row-major, outputs y are fp16
 * [m][n] row-major (y = x W^T), accumulated in fp32.  fp16 values are passed
 * as uint16_t bit patterns.
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument marked "device" must point to GPU global memory
 *     of the current device; the caller allocates and owns all of it.  The
 *     library allocates nothing on the device; its only device memory is its
 *     fixed error word and the fixed scratch array of
 *     qmm_grouped_gemv_noalloc, and it keeps no pointer after a call returns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); all work
 *     is enqueued on it and the call returns without synchronising.
 *   - Argument checks happen on the host before anything is enqueued; on
 *     failure nothing is launched and the status says why.  There is no CPU
 *     fallback and no silent fallback: a shape or layout that no kernel
 *     supports returns QMM_ERR_UNSUPPORTED_SHAPE.
 *   - Errors that can only be seen on the device (a pipeline wait that ran
 *     out, an expert id out of range) set a per-device error word;
 *     qmm_sync_check() reports and clears it.
 *   - Device base pointers must be 16-byte aligned (QMM_ERR_MISALIGNED
 *     otherwise).
 *   - Calls on different streams may run concurrently.  What they share:
 *     the per-device error word; the fixed scratch array of
 *     qmm_grouped_gemv_noalloc (two calls of that entry point whose kernels
 *     overlap race on it); and nothing else on the device.  The record read
 *     by qmm_last_variant() is kept per host thread.
 */
#ifndef QMM_H_
#define QMM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QMM_OK = 0,
  QMM_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad format */
  QMM_ERR_UNSUPPORTED_SHAPE = 2, /* k not a multiple of the group, m out of range */
  QMM_ERR_MISALIGNED = 3,        /* a device pointer is not 16-byte aligned */
  QMM_ERR_NOT_SM100 = 4,         /* current device is not compute capability 10.0 */
  QMM_ERR_CUDA = 5,              /* a CUDA runtime call failed (launch, attribute) */
  QMM_ERR_TIMEOUT = 6,           /* a kernel wait ran out (reported by qmm_sync_check) */
  QMM_ERR_DEVICE_FAULT = 7,      /* bad data seen on the device, e.g. expert id out of range */
  QMM_ERR_WORKSPACE = 8          /* workspace missing or smaller than qmm_workspace_bytes() */
} qmm_status;

typedef enum {
  QMM_FMT_IQ4_NL = 1,
  QMM_FMT_FP4G16_F16 = 2,
  QMM_FMT_FP4G16_E4M3 = 3,
  /* E2M1 codes laid out as for FP4-G16 plus one OCP E8M0 scale byte per 32
   * consecutive k, a separate [n][k/32] array ("1bit.gg zyphra", section
   * "What these numbers say": MXFP4 experts, E8M0 scale bytes and 32 E2M1
   * codes per group).  w = fp16(code * 2^(e-127)), one rounding; e = 0xFF
   * is NaN.  k % 32 == 0. */
  QMM_FMT_MXFP4 = 4
} qmm_format;

/* One packed matrix, or a stack of `num_experts` packed matrices of equal
 * shape (the routed-expert tensor of the IQ4_NL model card: one contiguous
 * [E][n][k] tensor per projection, "Mark-Experimental-V3-8B", section
 * "Quantization", last bullet). */
typedef struct {
  int32_t fmt;            /* qmm_format */
  int32_t reserved;       /* must be 0 */
  int64_t n;              /* output rows */
  int64_t k;              /* input columns: k % 32 == 0 (IQ4_NL, MXFP4), k % 16 == 0 (FP4-G16) */
  const void* data;       /* device: IQ4_NL blocks, or FP4 codes [n][k/2] */
  const void* scales;     /* device: FP4-G16 scales [n][k/16] (fp16 or E4M3FN), MXFP4 [n][k/32]
                           * E8M0 bytes; NULL for IQ4_NL */
  float global_scale;     /* FP4G16_E4M3 only (fp32 g); ignored otherwise */
  int32_t reserved2;      /* must be 0 */
  int64_t num_experts;    /* 1 for a plain matrix */
  int64_t expert_data_stride;  /* bytes between experts in `data` (>= qmm_data_bytes) */
  int64_t expert_scale_stride; /* bytes between experts in `scales` */
} qmm_weights;

/* Bytes of the code/block array of one [n][k] matrix (IQ4_NL: n*k/32*18;
 * FP4: n*k/2).  Returns 0 for an invalid format or shape. */
size_t qmm_data_bytes(int32_t fmt, int64_t n, int64_t k);

/* Bytes of the separate scale array of one matrix (IQ4_NL: 0; FP4G16_F16:
 * n*k/16*2; FP4G16_E4M3: n*k/16; MXFP4: n*k/32). */
size_t qmm_scale_bytes(int32_t fmt, int64_t n, int64_t k);

/* qmm_data_bytes + qmm_scale_bytes (+4 for the FP4G16_E4M3 global scale, as
 * the storage table of the FP4-G16 model card counts it). */
size_t qmm_packed_bytes(int32_t fmt, int64_t n, int64_t k);

/* Decode a packed matrix to resident fp16, bit-exactly as defined above (one
 * rounding to fp16, round to nearest even, fp16 subnormals kept; for E4M3 the
 * product is rounded to fp32 and then to fp16).  This is what the published
 * runtime of the FP4-G16 model card does at load time
 * ("Mamb2_8B_FP4_Recall_SQ3.25", section "Storage and runtime memory": all
 * decoded FP16 weights stay resident).
 *   w       weights (num_experts must be 1)
 *   out     device, [n][k] fp16, written completely
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, NOT_SM100, CUDA. */
qmm_status qmm_dequant(const qmm_weights* w, uint16_t* out, void* stream);

/* Encode resident fp16 weights into a packed format (the inverse direction
 * of qmm_dequant, for callers that hold fp16 checkpoints).  The formats are
 * the pages' ("Mamb2_8B_FP4_Recall_SQ3.25", section "Representation";
 * "1bit.gg zyphra", MXFP4 experts; "Mark-Experimental-V3-8B", section
 * "Quantization"); the pages do not give the quantiser, so the scale is the
 * plainest reading: FP4G16_F16 s = fp16(amax / 6) per 16; MXFP4 E8M0 e =
 * floor(log2 amax) - 2 + 127 in [0, 254] per 32 (0 for an all-zero group,
 * 254 when amax is infinite); IQ4_NL d = fp16(m / -127) per 32, m the first
 * element of largest |w| (it maps to the table's -127 entry).  Each weight
 * then takes the code whose decoded value (exactly as qmm_dequant decodes
 * it) is nearest, the lowest code on equal distance, code 0 for NaN.
 *   fmt     QMM_FMT_FP4G16_F16, QMM_FMT_MXFP4 or QMM_FMT_IQ4_NL
 *           (FP4G16_E4M3: UNSUPPORTED_SHAPE, its global scale is matrix-wide)
 *   w       device, [n][k] fp16 (k a multiple of the format's group)
 *   data    device, qmm_data_bytes(fmt, n, k) bytes, written completely
 *   scales  device, qmm_scale_bytes(fmt, n, k) bytes (NULL for IQ4_NL)
 * The call ends with an empty kernel launched without programmatic
 * dependent launch, so a qmm_gemv or expert call that follows on the same
 * stream (those read W before their dependency wait) starts only after the
 * encoded bytes are complete and visible.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, NOT_SM100, CUDA. */
qmm_status qmm_quantize(int32_t fmt, const uint16_t* w, int64_t n, int64_t k, void* data, void* scales,
                        void* stream);

/* Fused dequantise-and-multiply for decode batches: y[m][n] = sum_k
 * x[m][k] * W[n][k] with the decoded fp16 weights, fp32 accumulation, one
 * rounding of the sum to fp16.  The weights are the FP16-decoded ones the
 * FP4-G16 model card's runtime holds resident ("Mamb2_8B_FP4_Recall_SQ3.25",
 * section "Storage and runtime memory": the decoded FP16 weights stay
 * resident and no packed-resident FP4 matmul kernel is provided); this call
 * is that product with W left packed in GPU memory and decoded inside the
 * kernel.  For FP4G16_E4M3 the global scale g is applied to the fp32 sum
 * instead of to each weight (the difference from the per-weight definition
 * is one fp16 rounding of each weight).
 * The FP4 kernels are launched with programmatic dependent launch: they start
 * reading W while the kernel before them on the stream is still running (x
 * and y wait for it).  So W must not be written by the kernel that
 * immediately precedes this call on the stream; any other operation in
 * between (a copy, an event, another library call) restores full ordering.
 *   x       device, [m][k] fp16
 *   m       1..16
 *   y       device, [m][n] fp16
 *   ws      device workspace of ws_bytes (qmm_workspace_bytes(QMM_OP_GEMV, ...));
 *           may be NULL when that is 0
 * Errors: as qmm_dequant, plus WORKSPACE. */
qmm_status qmm_gemv(const qmm_weights* w, const uint16_t* x, int64_t m, uint16_t* y, void* ws,
                    size_t ws_bytes, void* stream);

/* qmm_gemv with host-resident activations and outputs, in one call (a
 * serving step's whole round trip), enqueued on `stream`: x_host reaches
 * x_dev, the product is formed, y lands in y_host.  Page-locked host buffers
 * (cudaHostAlloc, torch pin_memory) are used in place through their device
 * mapping: a copy kernel reads x_host into x_dev while the GEMV, launched
 * with programmatic dependent launch, already streams W, and the GEMV stores
 * y straight into y_host (y_dev is then unused).  The copy kernel is itself
 * launched with programmatic dependent launch: it reads x_host while the
 * kernel before it on the stream still runs and writes x_dev only after that
 * kernel has finished, so x_host must not be written by the kernel
 * immediately preceding this call on the stream (any other operation in
 * between restores full ordering).  Pageable buffers go through
 * cudaMemcpyAsync (synchronous to the host) and y_dev.  y_host holds the
 * result once the stream reaches the end of this call's work.
 *   x_host  host, [m][k] fp16 (16-byte aligned for the in-place path)
 *   y_host  host, [m][n] fp16 (16-byte aligned for the in-place path)
 *   x_dev   device, [m][k] fp16 staging buffer (16-byte aligned)
 *   y_dev   device, [m][n] fp16 staging buffer (16-byte aligned)
 * The whole [m][k] and [m][n] ranges must lie in the buffers the caller
 * passes (a page-locked range is read and written by the GPU directly).
 * Errors: as qmm_gemv; CUDA when a copy cannot be enqueued (the kernel may
 * then already be queued). */
qmm_status qmm_gemv_host(const qmm_weights* w, const uint16_t* x_host, int64_t m, uint16_t* y_host,
                         uint16_t* x_dev, uint16_t* y_dev, void* stream);

/* The same product for a prefill window: every token of a window of m
 * tokens at once (the FP4-G16 model card scores 2,048-token windows,
 * "Mamb2_8B_FP4_Recall_SQ3.25", section "Measured quality"; the weights are
 * the decoded ones of section "Storage and runtime memory", as for
 * qmm_gemv).  m may be any size.  From 256 tokens (k % 64 == 0) the kernel
 * is a tensor-core GEMM that decodes weight tiles into shared memory; below
 * that either that GEMM or the qmm_gemv kernels over 16-token slices of x,
 * whichever a cost model of the two puts first for the shape (few rows or
 * few tokens favour the slices); qmm_last_variant names the path taken.
 *   x       device, [m][k] fp16;  y device, [m][n] fp16
 * Errors: as qmm_gemv. */
qmm_status qmm_gemm(const qmm_weights* w, const uint16_t* x, int64_t m, uint16_t* y, void* ws,
                    size_t ws_bytes, void* stream);

/* Bucket the t*topk (token, slot) pairs of a top-k routing by expert: a
 * counting sort ("Mark-Experimental-V3-8B", section "Mixture-of-Experts
 * (MoE)": 32 routed experts, top-4 per token).
 *   topk_ids        device, [t][topk] int32 expert ids
 *   expert_offsets  device, [num_experts+1] int32: pairs of expert e are
 *                   pair_perm[offsets[e] .. offsets[e+1]-1]
 *   pair_perm       device, [t*topk] int32 pair indices p = token*topk+slot,
 *                   grouped by expert (order within an expert unspecified);
 *                   ids outside [0, num_experts) are left out, their count is
 *                   t*topk - offsets[num_experts], and the device error word
 *                   records QMM_ERR_DEVICE_FAULT
 *   ws              device workspace (qmm_workspace_bytes(QMM_OP_ROUTE, ...))
 * Errors: INVALID_ARG, MISALIGNED, NOT_SM100, CUDA, WORKSPACE. */
qmm_status qmm_route(const int32_t* topk_ids, int64_t t, int64_t topk, int64_t num_experts,
                     int32_t* expert_offsets, int32_t* pair_perm, void* ws, size_t ws_bytes,
                     void* stream);

/* Routed-expert grouped GEMV: for every (token, slot) with e =
 * topk_ids[token][slot] in range, y[token][slot][:] = W_e x_row, where x_row
 * is x[token] (x_per_pair = 0, x is [t][k]) or x[token][slot]
 * (x_per_pair = 1, x is [t][topk][k]).  Each expert's weights are read once
 * for all of the pairs routed to it.  Pairs with an id out of range leave
 * their y row untouched and set QMM_ERR_DEVICE_FAULT in the error word.
 * IQ4_NL experts are launched with programmatic dependent launch (their
 * weights may be read while the kernel before them on the stream still
 * runs, as for qmm_gemv: the experts must not be written by that kernel).
 *   experts   a stack of num_experts matrices (expert_*_stride set)
 *   y         device, [t][topk][n] fp16
 *   ws        device workspace (qmm_workspace_bytes(QMM_OP_GROUPED, ...));
 *             scratch for the routing sort (IQ4_NL with at most 32 pairs
 *             routes inside the expert kernel and leaves it untouched)
 * Errors: as qmm_gemv. */
qmm_status qmm_grouped_gemv(const qmm_weights* experts, const uint16_t* x, int32_t x_per_pair,
                            const int32_t* topk_ids, int64_t t, int64_t topk, uint16_t* y, void* ws,
                            size_t ws_bytes, void* stream);

/* Allocation-free variant of qmm_grouped_gemv.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory, so cannot supply the routing workspace qmm_grouped_gemv
 * asks for -- for example a host runtime that hands out all device memory
 * from its own fixed pool and forbids other allocations, or a latency-bound
 * serving loop that must not block in the allocator.
 *
 * Same arguments and result as qmm_grouped_gemv, minus the workspace.  The
 * routing offsets and pair permutation live instead in one fixed array of
 * the library's own device memory (258 KiB, held by every GPU that loads the
 * library until the process exits).  Limits: t*topk <= 65536 pairs and
 * num_experts <= 256; larger calls return QMM_ERR_UNSUPPORTED_SHAPE and
 * launch nothing.  The call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it; make that
 * first call before any stream capture.  The cache holds one address per
 * device for the life of the process: after cudaDeviceReset (or anything
 * else that destroys and recreates the device's primary context) the
 * address is stale, so do not call this entry point again in that process.
 * The expert products run on the library's generic grouped kernel (one warp
 * per 16-row tile, any format), not on the IQ4_NL kernels qmm_grouped_gemv
 * uses by default: the results agree within the same tolerance, the speed
 * does not.  Every call on a device uses the
 * same array and it keeps the last call's contents (each call rewrites every
 * entry it reads, so nothing needs clearing): two calls whose kernels
 * overlap on the GPU -- on different streams, or from different host
 * threads -- race on it and must be serialised by the caller.
 * Errors: as qmm_grouped_gemv, except QMM_ERR_WORKSPACE. */
qmm_status qmm_grouped_gemv_noalloc(const qmm_weights* experts, const uint16_t* x, int32_t x_per_pair,
                                    const int32_t* topk_ids, int64_t t, int64_t topk, uint16_t* y,
                                    void* stream);

/* Router of a mixture-of-experts layer ("Mark-Experimental-V3-8B", section
 * "Mixture-of-Experts (MoE)": s_{t,e} = Softmax(x_t W_router + b_e), the 4
 * experts of largest score are active, each weighted by g_i).
 * For every token: z_e = fp32(sum_k x[k] w_router[e][k] + bias[e]) with the
 * sum taken in fp64 (every fp16 product is exact there) and rounded once;
 * s = softmax(z) in fp32; topk_ids = the topk experts of largest z, larger
 * first, equal z to the lower index; topk_weights = their s (no
 * renormalisation over the chosen experts).
 *   x             device, [t][k] fp16 activations
 *   w_router      device, [num_experts][k] fp16 (a quantised router is
 *                 decoded once with qmm_dequant)
 *   bias          device, [num_experts] fp32 (the b_e of the formula)
 *   topk_ids      device, [t][topk] int32 out
 *   topk_weights  device, [t][topk] fp32 out
 *   logits        device, [t][num_experts] fp32 out (z), or NULL
 * Limits: 1 <= topk <= num_experts <= 256, k % 8 == 0.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, NOT_SM100, CUDA. */
qmm_status qmm_router_topk(const uint16_t* x, const uint16_t* w_router, const float* bias, int64_t t,
                           int64_t k, int64_t num_experts, int64_t topk, int32_t* topk_ids,
                           float* topk_weights, float* logits, void* stream);

/* Routed-expert block of a mixture-of-experts layer ("Mark-Experimental-V3-8B",
 * section "Mixture-of-Experts (MoE)": F_i(x) = (SiLU(x W_gate) * (x W_up))
 * W_down, output sum over the chosen experts of g_i F_i(x); the expert
 * weights are contiguous 3-D tensors ffn_gate_exps / ffn_up_exps /
 * ffn_down_exps, section "Quantization"):
 *   out[t][:] = sum_s topk_weights[t][s] * W_down,e (h_{t,s}),
 *   h_{t,s}   = fp16(SiLU(W_gate,e x_t) * (W_up,e x_t)),  e = topk_ids[t][s].
 * Three kernels after the routing sort (up to 32 pairs the expert kernels
 * route themselves and no sort runs): gate and up are multiplied in one
 * pass over the same row tiles with SiLU(gate) * up applied before the only
 * fp16 rounding of h; the down projection multiplies each expert's pairs,
 * scales them by g in fp32 and keeps them in fp32; a last pass adds a
 * token's slots in slot order and rounds once to fp16.  The shared experts
 * of the formula are this same call with ids {0, 1} and weights 1.  The
 * expert kernels use programmatic dependent launch: gate/up/down must not be
 * written by the kernel that immediately precedes this call.
 *   gate, up     IQ4_NL stacks of num_experts matrices [f][d] (same f, d, E)
 *   down         IQ4_NL stack of num_experts matrices [d][f]
 *   x            device, [t][d] fp16
 *   topk_ids     device, [t][topk] int32 (ids out of range: their pairs are
 *                left out, QMM_ERR_DEVICE_FAULT set in the error word)
 *   topk_weights device, [t][topk] fp32
 *   out          device, [t][d] fp16
 *   ws           device workspace (qmm_workspace_bytes(QMM_OP_MOE, gate, 0,
 *                t, topk)), laid out as offsets [E+1] int32 | pair_perm
 *                [t*topk] int32 | h [t*topk][f] fp16 | g-scaled slot outputs
 *                [t*topk][d] fp32, each part starting on a 256-byte
 *                boundary; after the call h is readable there (pairs with an
 *                out-of-range id hold stale data; offsets and pair_perm are
 *                written only when the routing sort runs)
 * Limits: d % 128 == 0, f % 128 == 0 (whole 4-block super-steps per row).
 * Errors: as qmm_grouped_gemv. */
qmm_status qmm_moe_routed(const qmm_weights* gate, const qmm_weights* up, const qmm_weights* down,
                          const uint16_t* x, const int32_t* topk_ids, const float* topk_weights,
                          int64_t t, int64_t topk, uint16_t* out, void* ws, size_t ws_bytes,
                          void* stream);

enum { QMM_OP_DEQUANT = 0, QMM_OP_GEMV = 1, QMM_OP_GEMM = 2, QMM_OP_ROUTE = 3, QMM_OP_GROUPED = 4,
       QMM_OP_MOE = 5 };

/* Device workspace bytes an operation needs for these sizes (0 = none).
 * `w` may be NULL for QMM_OP_ROUTE; `num_experts` is taken from `w` except
 * for QMM_OP_ROUTE, where it is passed in `m`.  For QMM_OP_MOE `w` is the
 * gate stack (f = w->n, d = w->k). */
size_t qmm_workspace_bytes(int32_t op, const qmm_weights* w, int64_t m, int64_t t, int64_t topk);

/* Synchronise `stream`, then read and clear this device's error word.
 * Returns QMM_OK, QMM_ERR_TIMEOUT, QMM_ERR_DEVICE_FAULT or QMM_ERR_CUDA. */
qmm_status qmm_sync_check(void* stream);

/* Test hooks for the failure path of the pipelined kernels (not needed in
 * normal use; the pages have no counterpart).  Every mbarrier wait of the
 * tensor-core GEMMs is bounded by a device-wide limit on %globaltimer; when
 * a wait runs out, the kernel sets QMM_ERR_TIMEOUT in the error word, lets
 * its own copies and MMAs finish, frees its tensor memory and returns, so
 * the context stays usable.  These hooks let a test exercise that path
 * without faulting anything:
 *   QMM_DEBUG_WAIT_LIMIT_NS     value = the limit in ns (1e3 .. 1e10;
 *                               2e9 by default)
 *   QMM_DEBUG_WITHHOLD_X_TILES  value = 1: the GEMMs' activation loader
 *                               issues no tile load, so their waits run out
 *                               (nothing is written to y); 0: normal
 *   QMM_DEBUG_WITHHOLD_TILE_COPIES  value = 1: the routed-expert tile kernel
 *                               issues none of its bulk copies, so its wait
 *                               for them runs out (y is left meaningless);
 *                               0: normal
 * The first two are device-wide (current device) and copied synchronously,
 * the third applies to every later launch of this process; all stay set
 * until changed.  Errors: INVALID_ARG (unknown hook or value), NOT_SM100,
 * CUDA. */
enum { QMM_DEBUG_WAIT_LIMIT_NS = 1, QMM_DEBUG_WITHHOLD_X_TILES = 2, QMM_DEBUG_WITHHOLD_TILE_COPIES = 3 };
qmm_status qmm_debug_set(int32_t what, int64_t value);

/* Static text for a status code. */
const char* qmm_status_string(int32_t status);

/* Name of the kernel variant the last successful call on this host thread
 * launched (for dispatch records next to timings); "" before any call. */
const char* qmm_last_variant(void);

/* Library version string. */
const char* qmm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QMM_H_ */
