/*
 * moe.h -- C ABI of libmoe_b200.so: the forward pass of a Mixture-of-Experts
 * SwiGLU FFN layer on NVIDIA B200 (sm_100a).
 *
 * The layer, per token t ("Fused MoE Triton kernel: 5 launches instead of
 * 24" page, list of fused steps: top-k routing weights, dispatch of tokens to
 * the chosen experts, parallel expert compute, weighted aggregation; "CUDA:
 * fuse shared experts into MMVQ" page, section on shared experts: always
 * active, added to every token):
 *
 *   l_e   = x_t . Wr[e] (+ b_e)                     router logits, fp32 FMA
 *   p     = softmax(l) over all E experts
 *   K     = the top_k experts with the largest l_e (ties: lower index)
 *   w_j   = p_j / sum_{K} p                         renormalised weights
 *   out_t = sum_{j in K} w_j FFN_j(x_t) + sum_s FFN_s(x_t)
 *   FFN(x) = Wd (SiLU(Wg x) * (Wu x)),  SiLU(z) = z / (1 + e^-z)
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers, owned by the caller, aligned to
 *    16 bytes (TMA requires 16-byte aligned bases and row pitches).  The
 *    library never copies or frees them.  Weights stay in place.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Compute entry points only enqueue work: they neither allocate nor
 *    synchronise, so they may be captured in a CUDA graph.
 *  - Every entry point returns a moe_status_t; nothing is thrown or aborted
 *    across the ABI.  Host-side argument checks run before any launch, so an
 *    invalid call enqueues nothing.
 *  - Matrices are row-major with the reduction dimension contiguous
 *    ("[out][in]"):  x [T][d] bf16;  router_w [E][d] fp32;  router_b [E] fp32;
 *    routed gate/up [E][F][d], down [E][d][F];  shared gate/up [S][Fs][d],
 *    down [S][d][Fs];  out [T][d] fp32.
 *  - bf16 values are raw IEEE bfloat16 bit patterns (uint16).
 *  - Host threads: the library keeps per-process state (each kernel's
 *    shared-memory limit, raised once per device) and per-plan state (the
 *    tensor-map caches, the launch count).  Calls must not run concurrently
 *    on several host threads; serialise them.  Work from one plan must also
 *    not overlap on the GPU (see moe_forward).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or shape */
    MOE_ERR_UNSUPPORTED = 2,   /* valid request outside what this build runs */
    MOE_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
    MOE_ERR_OOM = 4,           /* plan workspace allocation failed */
    MOE_ERR_DEVICE_FLAG = 5,   /* a kernel flagged an inconsistent state */
    MOE_ERR_TIMEOUT = 6        /* a bounded device-side wait ran out */
} moe_status_t;

/* Weight formats.
 * MOE_WFMT_BF16: every expert matrix is bf16 in the layouts above.
 * MOE_WFMT_Q4_0: blocks of 32 consecutive weights along the reduction dim,
 *   each an fp16 scale d and 32 codes q in 0..15, weight = d * (q - 8)
 *   (the 35B-A3B Q4_0 workload; the "MoE on RTX 5090 reaches 41% of
 *   bandwidth" page names Q4_0, measurement-setup paragraph; the MMVQ page
 *   asks that quantised weights be read once and never expanded, section
 *   "what MMVQ is").  The kernels read the packed form written by
 *   moe_q4_0_pack, not the canonical 18-byte blocks.
 * MOE_WFMT_Q8_0: blocks of 32 consecutive weights along the reduction dim,
 *   each an fp16 scale d and 32 signed 8-bit codes q, weight = d * q (the
 *   5090 page lists q8_0 among the formats of the 35B-A3B model it measures;
 *   it prints no layout, and the canonical 34-byte block is the reading
 *   taken).  The kernels read the packed form written by moe_q8_0_pack.
 * MOE_WFMT_Q5_0: blocks of 32 consecutive weights along the reduction dim,
 *   each an fp16 scale d and 32 codes q in 0..31, weight = d * (q - 16) (the
 *   5090 page lists q5_0 in the same list of formats; the canonical 22-byte
 *   block is the reading taken).  The kernels read the packed form written by
 *   moe_q5_0_pack.
 * MOE_WFMT_Q6_K: super-blocks of 256 consecutive weights along the reduction
 *   dim, each an fp16 scale d, 16 signed 8-bit sub-block scales (one per 16
 *   weights) and 256 6-bit codes q in 0..63, weight = d * sc * (q - 32) (the
 *   5090 page lists q6_K among the formats of the 35B-A3B model; the
 *   canonical 210-byte super-block is the reading taken).  The reduction dim
 *   must be a multiple of 256 and every matrix's row count of 16.  The
 *   kernels read the packed form written by moe_q6_k_pack.
 * MOE_WFMT_BF16_F16DOWN: gate and up matrices bf16, every down matrix
 *   (routed and shared) IEEE fp16 -- the bf16 weights rounded once to fp16
 *   with moe_bf16_to_f16, exact for 2^-17 <= |w| <= 65504 (below 2^-17 the
 *   rounding error is at most 2^-25).  The hidden activation h then travels
 *   between the two prefill GEMMs as fp16 (11 significant bits) instead of
 *   bf16 (8): the pages have no counterpart; it is the precision headroom of
 *   the bf16 layer's 2e-3 bound.  Both regimes run it.
 * The quantised formats run in the decode regime only (T <= MOE_DECODE_MAX_T). */
typedef enum moe_wfmt {
    MOE_WFMT_BF16 = 0,
    MOE_WFMT_Q4_0 = 1,
    MOE_WFMT_Q8_0 = 2,
    MOE_WFMT_Q5_0 = 3,
    MOE_WFMT_Q6_K = 4,
    MOE_WFMT_BF16_F16DOWN = 5
} moe_wfmt_t;

/* Execution regime.  AUTO picks DECODE for T <= MOE_DECODE_MAX_T (and for
 * every T with quantised weights, up to MOE_DECODE_MAX_T) and PREFILL otherwise.
 * DECODE streams every active expert's weights once, through a TMA ring,
 * with the <= 8 tokens of an expert as the N side of mma.sync and the
 * weighted combine fused.  PREFILL runs grouped GEMMs on tcgen05 tensor
 * cores with accumulators in tensor memory (bf16 only). */
typedef enum moe_regime {
    MOE_REGIME_AUTO = 0,
    MOE_REGIME_DECODE = 1,
    MOE_REGIME_PREFILL = 2
} moe_regime_t;

#define MOE_DECODE_MAX_T 8

typedef struct moe_config {
    int32_t t_max;        /* largest T any forward call will pass */
    int32_t d_model;      /* d; multiple of 128 */
    int32_t d_ff;         /* F, routed expert hidden size; multiple of 32
                             (of 64 for the prefill regime) */
    int32_t n_experts;    /* E >= 1 routed experts (<= 1024) */
    int32_t top_k;        /* 1 <= k <= min(E, 16) */
    int32_t n_shared;     /* S >= 0 shared experts (<= 8) */
    int32_t d_ff_shared;  /* Fs, hidden size of each shared expert (0 if S=0);
                             same multiples as d_ff */
    int32_t wfmt;         /* moe_wfmt_t */
    int32_t regime;       /* moe_regime_t */
    int32_t device;       /* CUDA device ordinal the plan lives on */
} moe_config_t;

/* One stack of expert matrices.  bf16: `data` is the bf16 stack, `scales`
 * must be NULL.  Q4_0 / Q8_0 / Q5_0: `data` = packed codes, `scales` = the
 * packed fp16 scales (Q5_0: the packed records of scales and fifth bits),
 * both from moe_q4_0_pack / moe_q8_0_pack / moe_q5_0_pack. */
typedef struct moe_matrix {
    const void* data;
    const void* scales;
} moe_matrix_t;

typedef struct moe_weights {
    const float* router_w;       /* [E][d] fp32 */
    const float* router_b;       /* [E] fp32, or NULL for no bias */
    moe_matrix_t gate, up, down; /* routed experts, E stacked */
    moe_matrix_t shared_gate, shared_up, shared_down; /* S stacked; ignored if S=0 */
} moe_weights_t;

/* Optional copies of the routing tables of the last call (device pointers,
 * each may be NULL).  ids/weights are [T][k] with each token's experts in
 * descending logit order, ties to the lower index; counts [E]; offsets
 * [E+1] exclusive prefix sums of counts; slot_pair [T*k]: slot s (ordered by
 * expert, then ascending token) holds the pair index t*k + j. */
typedef struct moe_routing {
    int32_t* ids;
    float* weights;
    int32_t* counts;
    int32_t* offsets;
    int32_t* slot_pair;
} moe_routing_t;

typedef struct moe_plan_s* moe_plan_t;

/* Validate `cfg`, select the device, size and allocate the plan workspace
 * for cfg->t_max tokens and resolve the driver's tensor-map encoder.  The
 * pages have no counterpart to the plan itself: it owns the tables that the
 * fused steps of the "Fused MoE Triton kernel: 5 launches instead of 24" page
 * pass between them (routing weights, the dispatch buckets), so that the
 * compute calls below allocate nothing.  On
 * success *out receives the plan; on failure *out is NULL and nothing is
 * left allocated.  This is the only entry point that allocates device
 * memory.  Errors: INVALID_ARG (shape limits above), UNSUPPORTED (PREFILL
 * regime with quantised weights, or a device that is not sm_100), CUDA,
 * OOM. */
moe_status_t moe_plan_create(const moe_config_t* cfg, moe_plan_t* out);

/* Free the plan's workspace.  The caller must make sure no work enqueued
 * with the plan is still running.  NULL is ignored.  (No counterpart on the
 * pages: the pair of moe_plan_create.) */
void moe_plan_destroy(moe_plan_t plan);

/* The whole layer: route, bucket, experts, weighted combine -- the four
 * fused steps of the "Fused MoE Triton kernel: 5 launches instead of 24"
 * page (list of fused steps), with the always-on shared experts of the
 * "CUDA: fuse shared experts into MMVQ" page (section on shared experts) in
 * the same pass.
 * x [T][d] bf16, out [T][d] fp32 (overwritten), 0 <= T <= t_max.
 * top_k and wfmt are the call's k and weight format (moe_wfmt_t); they must
 * equal the plan's (cfg->top_k, cfg->wfmt), else MOE_ERR_INVALID_ARG and
 * nothing is enqueued (the plan's workspace and tensor maps are sized and
 * built for one k and one format).
 * `routing` may be NULL; when given, the routing tables are copied to it
 * (device-to-device, on `stream`).  T = 0 enqueues nothing.
 * Launches: decode regime -- 1 cooperative kernel (router, top-k, buckets,
 * every routed and shared expert, weighted combine; each CTA waits for the
 * router logits of all others, tagged with the launch, before it routes);
 * if the device cannot co-schedule that grid, the
 * two-launch path of moe_route + moe_experts.  Prefill regime -- 4 kernels
 * (router, bucket scatter + row gather, gate/up GEMM, down GEMM with the
 * weighted combine).  Work enqueued with one plan must not overlap on the
 * GPU with other work of the same plan (they share the workspace). */
moe_status_t moe_forward(moe_plan_t plan, const moe_weights_t* w,
                         const void* x, int32_t T, int32_t top_k, int32_t wfmt,
                         float* out, moe_routing_t* routing, void* stream);

/* The same layer as moe_forward in two steps, for callers that time or
 * schedule them separately.  moe_route: router, top-k, buckets and work
 * list into the plan's workspace; also zero-fills `out` (decode: 1 kernel;
 * prefill: 2, including the gather of x rows per expert) -- the Triton
 * page's fused steps one and two (routing weights, dispatch; its launch
 * table's routing and dispatch rows).  moe_experts: expert FFNs and the
 * weighted combine into `out`, reading what moe_route wrote with the same T
 * (decode: 1 kernel; prefill: 2 GEMM kernels) -- the Triton page's steps
 * three and four (parallel expert compute, weighted aggregation), shared
 * experts in the same pass as on the MMVQ page.  top_k and wfmt as for
 * moe_forward. */
moe_status_t moe_route(moe_plan_t plan, const moe_weights_t* w,
                       const void* x, int32_t T, int32_t top_k, int32_t wfmt,
                       float* out, void* stream);
moe_status_t moe_experts(moe_plan_t plan, const moe_weights_t* w,
                         const void* x, int32_t T, int32_t top_k, int32_t wfmt,
                         float* out, void* stream);

/* moe_route_noalloc: moe_route for callers that cannot allocate device
 * memory (no plan needed).  The source pages have no counterpart to this
 * entry point; it exists for host programs that may not call cudaMalloc
 * while they serve a batch -- engines that forbid allocations on their hot
 * path, plugin interfaces whose enqueue step may only launch work, code that
 * runs while the allocator is locked.
 * It runs the decode-regime router kernel with its scratch (fp32 logits,
 * ticket, work list, slot maps, error word) in a 64 KiB file-scope device
 * array of the library instead of a plan workspace; it calls no cudaMalloc,
 * cudaFree or other allocating routine.  Each GPU that loads the library
 * holds that array until the process exits.
 * Inputs: cfg (d_model, n_experts, top_k, n_shared as for moe_plan_create;
 * t_max, d_ff, wfmt, regime and device are ignored), w->router_w/router_b,
 * x [T][d] bf16.  Outputs: out [T][d] zero-filled, and every member of
 * `routing` (all five required) filled as moe_routing_get would.
 * 0 <= T <= MOE_DECODE_MAX_T; a larger T returns MOE_ERR_INVALID_ARG (the
 * scratch array holds at most that many tokens).  Runs on the current
 * device.  The first call in a CUDA context resolves the array's device
 * address (cudaGetSymbolAddress) and caches it with the context's id; make
 * that first call before any stream capture.  With CUDA's lazy module
 * loading (the default) the first call on a device may also be the one that
 * loads the library's module, and loading a module allocates device memory
 * (for this array and the kernels): make a first call at start-up, outside
 * the section that must not allocate.
 * Every call on a device shares the one array, so calls whose work overlaps
 * on the GPU race: serialise them.  Device-side flags (an out-of-range id)
 * are not returned by this call; they stay in the array's error word until
 * moe_route_noalloc_status reads them. */
moe_status_t moe_route_noalloc(const moe_config_t* cfg, const moe_weights_t* w,
                               const void* x, int32_t T, float* out,
                               moe_routing_t* routing, void* stream);

/* Read and clear the error word of moe_route_noalloc on the current device
 * (synchronises the device): OK, or DEVICE_FLAG if a router kernel of an
 * earlier call saw an out-of-range id or an expert with more tokens than a
 * decode pass holds.  Allocates nothing.  No counterpart on the pages. */
moe_status_t moe_route_noalloc_status(void);

/* Copy the routing tables of the last moe_route/moe_forward (T tokens) from
 * the workspace to `routing` (device pointers; NULL members skipped): the
 * routing weights and dispatch buckets of the Triton page's fused steps one
 * and two. */
moe_status_t moe_routing_get(moe_plan_t plan, int32_t T, moe_routing_t* routing,
                             void* stream);

/* Number of kernels the last moe_forward/moe_route/moe_experts call enqueued
 * (what the Triton page's launch-count table counts: 24 launches per layer
 * for PyTorch, 16 for Megablocks, 5 for the fused kernel).  -1 for NULL. */
int32_t moe_last_launch_count(moe_plan_t plan);

/* Read and clear the sticky device error word (synchronises `plan`'s device).
 * The pages have no counterpart (they describe no failure handling).
 * OK, DEVICE_FLAG (a kernel saw an out-of-range id or count) or TIMEOUT (a
 * bounded wait -- of a pipeline stage, or of the fused kernel's wait for
 * the other CTAs' router logits -- gave up, after at most 2 s; the kernel
 * then skipped its remaining work, so that call's `out` is incomplete).  A
 * fused decode launch that starts while such a timeout is still unread does
 * no work at all: it writes NaN to its `out` and the next read of this word
 * also returns TIMEOUT (the launch ticket count a timeout leaves behind may
 * be mid-round, and computing on it could route on stale logits).  Reading
 * a TIMEOUT resets the plan's ticket count and logit words. */
moe_status_t moe_get_device_status(moe_plan_t plan);

/* Failure-path check (the pages have no counterpart): make the next fused
 * decode launch of `plan` unable to finish routing, by setting the plan's
 * launch ticket count to 1 (async memsets on `stream`), a value from which
 * the launch's CTAs derive two different tags, so that no CTA ever sees
 * every router logit carry its own tag.  Each waits the bounded 2 s, skips
 * its expert work, and exits, so the call's `out` is incomplete;
 * moe_get_device_status then returns MOE_ERR_TIMEOUT and resets the count,
 * after which the plan works normally again.  Nothing hangs and nothing
 * faults.  UNSUPPORTED if the device cannot run the fused (cooperative)
 * launch. */
moe_status_t moe_debug_stall_barrier(moe_plan_t plan, void* stream);

/* Bytes of the packed Q4_0 form of n_mats matrices of [rows][k] weights.
 * k must be a multiple of 32.  Returns INVALID_ARG otherwise.  (The 5090
 * page's Q4_0, measurement-setup paragraph; the sizes serve moe_q4_0_pack.) */
moe_status_t moe_q4_0_packed_bytes(int64_t n_mats, int64_t rows, int64_t k,
                                   size_t* code_bytes, size_t* scale_bytes);

/* Repack canonical Q4_0 blocks (the 5090 page's Q4_0, measurement-setup
 * paragraph; the MMVQ page's "read quantised weights once" is why the
 * kernels read this packed form directly) ([n_mats][rows][k/32] blocks of 18 bytes: a
 * little-endian fp16 scale, then 16 bytes whose byte j holds code j in the
 * low nibble and code j+16 in the high nibble) into the kernel layout:
 *   codes  [n_mats][k/32][rows][16 bytes], the 32 codes of each block
 *          permuted so one 32-bit word feeds one tensor-core fragment;
 *   scales [n_mats][k/32][rows] fp16.
 * Same 4.5 bits per weight.  All pointers are device pointers; `blocks`
 * needs no alignment, `codes`/`scales` 16 bytes.  Enqueued on `stream`. */
moe_status_t moe_q4_0_pack(const void* blocks, int64_t n_mats, int64_t rows,
                           int64_t k, void* codes, void* scales, void* stream);

/* Bytes of the packed Q8_0 form of n_mats matrices of [rows][k] weights
 * (32 code bytes and one fp16 scale per block).  k must be a multiple of 32.
 * Returns INVALID_ARG otherwise.  (q8_0 is in the 5090 page's list of the
 * model's formats; the sizes serve moe_q8_0_pack.) */
moe_status_t moe_q8_0_packed_bytes(int64_t n_mats, int64_t rows, int64_t k,
                                   size_t* code_bytes, size_t* scale_bytes);

/* Repack canonical Q8_0 blocks ([n_mats][rows][k/32] blocks of 34 bytes: a
 * little-endian fp16 scale, then 32 signed bytes, element j in byte j) into
 * the kernel layout:
 *   codes  [n_mats][k/32][rows][32 bytes]: one byte per code, biased to
 *          u = q + 128; byte 8t + n of a block row (t = 0..3, n = 0..7)
 *          holds element 2t + (n & 1) + 8 ((n >> 1) & 1) + 16 (n >> 2), so
 *          that t's first 4 bytes are elements 2t, 2t+1, 2t+8, 2t+9 and its
 *          last 4 the same plus 16;
 *   scales [n_mats][k/32][rows] fp16.
 * Same 8.5 bits per weight.  All pointers are device pointers; `blocks`
 * needs no alignment, `codes`/`scales` 16 bytes.  Enqueued on `stream`.
 * The pages have no counterpart to this repacking (it serves the kernels'
 * tensor-core fragments). */
moe_status_t moe_q8_0_pack(const void* blocks, int64_t n_mats, int64_t rows,
                           int64_t k, void* codes, void* scales, void* stream);

/* Bytes of the packed Q5_0 form of n_mats matrices of [rows][k] weights
 * (16 code bytes per block; 6 bytes of scale and fifth bits per block in
 * `scale_bytes`).  k must be a multiple of 32 and rows of 8 (every matrix of
 * a layer qualifies: d is a multiple of 128, F and Fs of 32).  Returns
 * INVALID_ARG otherwise.  (q5_0 is in the 5090 page's list of the model's
 * formats; the sizes serve moe_q5_0_pack.) */
moe_status_t moe_q5_0_packed_bytes(int64_t n_mats, int64_t rows, int64_t k,
                                   size_t* code_bytes, size_t* scale_bytes);

/* Repack canonical Q5_0 blocks ([n_mats][rows][k/32] blocks of 22 bytes: a
 * little-endian fp16 scale, a little-endian 32-bit word whose bit j is the
 * fifth bit of element j, then 16 bytes whose byte j holds the low 4 bits of
 * element j in the low nibble and of element j+16 in the high nibble) into
 * the kernel layout:
 *   codes  [n_mats][k/32][rows][16 bytes]: the low 4 bits, permuted exactly
 *          like the Q4_0 codes;
 *   scales [n_mats][k/32][rows/8][48 bytes]: for 8 consecutive rows their 8
 *          fp16 scales, then their 8 32-bit words of fifth bits; in a row's
 *          word, bits 4t+n and 16+4t+n (t, n = 0..3) are the fifth bits of
 *          the codes that bits 4n..4n+3 and 16+4n..16+4n+3 of the row's code
 *          word t hold.
 * Same 5.5 bits per weight.  All pointers are device pointers; `blocks`
 * needs no alignment, `codes`/`scales` 16 bytes.  Enqueued on `stream`.  The
 * pages have no counterpart to this repacking (it serves the kernels'
 * tensor-core fragments). */
moe_status_t moe_q5_0_pack(const void* blocks, int64_t n_mats, int64_t rows,
                           int64_t k, void* codes, void* scales, void* stream);

/* Bytes of the packed q6_K form of n_mats matrices of [rows][k] weights:
 * code_bytes = 16 per 32 weights (the low 4 bits), scale_bytes = 160 per 32
 * weights and 16 rows (high bits and sub-block scales) followed by 2 per row
 * and 256 weights (super-block scales).  k must be a multiple of 256 and rows
 * of 16 (every matrix of a q6_K layer qualifies: d a multiple of 256, F and
 * Fs multiples of 256).  Returns INVALID_ARG otherwise.  (q6_K is in the
 * 5090 page's list of the model's formats.) */
moe_status_t moe_q6_k_packed_bytes(int64_t n_mats, int64_t rows, int64_t k,
                                   size_t* code_bytes, size_t* scale_bytes);

/* Repack canonical q6_K super-blocks ([n_mats][rows][k/256] super-blocks of
 * 210 bytes: ql[128], qh[64], 16 int8 sub-block scales, fp16 scale; element
 * i = 128h + 32c + l takes its low 4 bits from the low (c < 2) or high
 * nibble of ql[64h + 32(c%2) + l] and its high 2 bits from bits 2c, 2c+1 of
 * qh[32h + l]) into the kernel layout:
 *   codes  [n_mats][k/32][rows][16 bytes]: the low 4 bits, permuted exactly
 *          like the Q4_0 codes;
 *   scales [n_mats][k/32][rows/16][160 bytes]: per block and 16-row group,
 *          32 words of high bits (word 4g+t: lane t's codes of rows g and
 *          g+8, the code in nibble n of row g's code word at bit
 *          {4,8,6,10,20,24,22,26}[n], row g+8's 8 bits higher, mod 32), then
 *          per g the two int8 sub-block scales of row g and of row g+8;
 *          followed by [n_mats][k/256][rows] fp16 super-block scales.
 * Same 6.5625 bits per weight.  Device pointers; `codes`/`scales` 16-byte
 * aligned.  Enqueued on `stream`.  The pages have no counterpart to this
 * repacking (it serves the kernels' tensor-core fragments). */
moe_status_t moe_q6_k_pack(const void* blocks, int64_t n_mats, int64_t rows, int64_t k,
                           void* codes, void* scales, void* stream);

/* Round n bf16 values (raw bits) to IEEE fp16 (nearest, ties to even) into
 * dst: the down matrices of MOE_WFMT_BF16_F16DOWN.  Exact for 2^-17 <= |w|
 * <= 65504 and for zeros; smaller values round to fp16 subnormals (error at
 * most 2^-25), larger ones to +-inf.  Device pointers, 2-byte aligned, no
 * overlap; enqueued on `stream`.  INVALID_ARG for n < 0 or NULL pointers
 * with n > 0.  No counterpart on the pages (see MOE_WFMT_BF16_F16DOWN). */
moe_status_t moe_bf16_to_f16(const void* src, int64_t n, void* dst, void* stream);

/* Static description of a status code (never NULL).  No counterpart on the
 * pages. */
const char* moe_status_string(moe_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
