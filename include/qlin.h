/*
 * qlin.h -- C ABI of the B200 (sm_100a) quantized linear layer library.
 *
 * The hot path of a quantized linear layer in LLM serving: dynamic activation
 * quantisation followed by a scaled GEMM whose epilogue applies the scales and
 * the bias and stores bf16,
 *
 *     C[m,n] = bf16( (sum_k A_q[m,k] * W_q[n,k]) * s_a[m] * s_w[n] + bias[n] )
 *
 * in the three formats named on the page "Helion in vLLM: A Unified Route to
 * Tunable Linear Kernels" (section "What the integration changes": FP8 dynamic
 * quantisation, W8A8 INT8 and Block-FP8), with the three GEMM strategies the
 * same section lists (ordinary GEMM, Split-K, Swap-AB) chosen per shape from a
 * dispatch table ("Algorithm choice becomes part of tuning", same section).
 *
 * Conventions shared by every entry point
 *   - Pointers named *_q, x, scale_*, bias, c_out and workspace are DEVICE
 *     pointers owned by the caller; the library allocates no device memory and
 *     keeps no pointer after a call returns.
 *   - All device work is enqueued on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and is asynchronous: outputs are valid once the
 *     stream has reached that point.  Apart from the table loader and
 *     qlin_sync_status, no entry point synchronises, allocates or compiles;
 *     the quantisers, qlin_scaled_mm and qlin_linear may be captured in a
 *     CUDA graph (the benchmark replays them that way).
 *   - Arguments are validated on the host before anything is launched; a bad
 *     argument returns an error status and launches nothing.  No entry point
 *     aborts the process.
 *   - Matrices are dense and row-major: A [M,K], W [N,K] (nn.Linear layout,
 *     so both GEMM operands are K-major), C [M,N].
 *   - bf16 data is IEEE bfloat16; e4m3 is the OCP FP8 E4M3 ("e4m3fn")
 *     encoding; int8 is two's complement.
 *   - Device kernels never wait unboundedly: a wait that exceeds its limit
 *     records QLIN_ERR_DEVICE_TIMEOUT, which qlin_sync_status() reports.
 */
#ifndef QLIN_H
#define QLIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QLIN_ABI_VERSION 7

#if defined(__GNUC__)
#define QLIN_API __attribute__((visibility("default")))
#else
#define QLIN_API
#endif

typedef void* qlin_stream_t; /* cudaStream_t */

typedef enum {
    QLIN_OK = 0,
    QLIN_ERR_INVALID_ARG = 1,   /* null pointer, bad enum, non-positive size, ... */
    QLIN_ERR_UNSUPPORTED = 2,   /* shape/format/variant combination not provided */
    QLIN_ERR_ALIGNMENT = 3,     /* pointer or stride not 16-byte aligned */
    QLIN_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
    QLIN_ERR_TABLE_IO = 5,      /* dispatch table file unreadable */
    QLIN_ERR_TABLE_FORMAT = 6,  /* dispatch table malformed or inconsistent */
    QLIN_ERR_TABLE_DEVICE = 7,  /* dispatch table made for another device */
    QLIN_ERR_CUDA = 8,          /* a CUDA runtime/driver call failed */
    QLIN_ERR_DEVICE_TIMEOUT = 9,/* a device-side wait gave up (see qlin_sync_status) */
    QLIN_ERR_NO_DEVICE = 10     /* no sm_100 device is current */
} qlin_status;

typedef enum {
    QLIN_FMT_INT8 = 0,       /* W8A8 INT8, per-token / per-channel scales, int32 accumulate */
    QLIN_FMT_FP8 = 1,        /* e4m3, per-token / per-channel scales, fp32 accumulate */
    QLIN_FMT_FP8_BLOCK = 2,  /* e4m3, 1x128 activation groups, 128x128 weight blocks */
    QLIN_FMT_BF16 = 3,       /* bf16 operands, no scales, fp32 accumulate (qlin_matmul_bf16 only;
                                also accepted by qlin_scaled_mm_workspace_size and
                                qlin_dispatch_query) */
    QLIN_FMT_MXFP8 = 4,      /* e4m3, one E8M0 scale per 32 elements of K (qlin_quantize_block_scaled,
                                qlin_block_scaled_mm; also qlin_scaled_mm_workspace_size and
                                qlin_dispatch_query) */
    QLIN_FMT_NVFP4 = 5       /* packed e2m1, one E4M3 scale per 16 elements of K and one fp32
                                scale per tensor (as QLIN_FMT_MXFP8) */
} qlin_format;

typedef enum {
    QLIN_VAR_AUTO = 0,          /* dispatch table entry, else the built-in rule */
    QLIN_VAR_PLAIN = 1,         /* one CTA per output tile, all K segments in it */
    QLIN_VAR_SPLITK = 2,        /* K segments of a tile spread over CTAs, fixed-order reduce */
    QLIN_VAR_SWAPAB = 3,        /* C^T = W A^T: N fills the 128-row MMA side, M the narrow side */
    QLIN_VAR_SWAPAB_SPLITK = 4, /* Swap-AB with the K segments spread over CTAs */
    QLIN_VAR_PAIR = 5           /* plain, 256-row tiles on a pair of CTAs (a cluster of 2): each CTA
                                   loads its 128 rows of A and half of the W tile, and one
                                   tcgen05.mma.cta_group::2 per K step fills both CTAs' accumulators.
                                   tile_n 256, INT8 and FP8; sums K in the plain variant's order */
} qlin_variant;

/* flags */
#define QLIN_OUT_I32ACC 1u /* qlin_scaled_mm, INT8 only: write the raw int32 accumulators instead of bf16 C */
/* Launch as a programmatic dependent of the previous kernel in the stream:
 * the kernel may start before that kernel has finished, waits for it before
 * reading activations or scales or writing outputs, and lets the next kernel
 * start early in turn.  qlin_scaled_mm streams weight tiles (w_q) before the
 * wait, so with this flag w_q must not be written by the kernel that
 * immediately precedes the call in the stream.  Accepted by every launching
 * entry point. */
#define QLIN_PDL 2u
/* Swap-AB Split-K with at most 8 (tile_n 16) or 4 (tile_n 32, 64) segments:
 * run the S segment CTAs of each tile as one thread-block cluster and reduce
 * in the shared memory of the first of them, over distributed shared memory,
 * instead of through the workspace (none is needed then).  Both paths add the
 * segments in the same order and give bitwise the same C.  Not the default:
 * in back-to-back launches the clusters start later than single CTAs and the
 * workspace reduction finishes first.  qlin_scaled_mm only. */
#define QLIN_SPLITK_CLUSTER 4u
/* qlin_linear: where the configuration allows, let the GEMM quantise its own
 * activation rows (one kernel) instead of running the stand-alone quantiser
 * first.  Not the default: measured on B200 the in-GEMM quantisation sits on
 * the MMA's critical path and the two-kernel sequence finishes first for the
 * per-token formats; for Block-FP8 at M = 1 the one kernel is ~3% faster. */
#define QLIN_FUSED 8u

/* A resolved GEMM configuration (what qlin_dispatch_query returns). */
typedef struct {
    int32_t variant;    /* qlin_variant, never AUTO */
    int32_t tile_n;     /* rows of the narrow MMA operand per tile: 16, 32, 64 (Swap-AB) or 128, 256 */
    int32_t k_segments; /* S: K is cut into S equal segments; fixed per (format, N, K) */
    int32_t stages;     /* shared-memory pipeline depth the kernel uses for tile_n */
    int64_t m_max;      /* upper bound of the table bucket (0 for the built-in rule) */
    int32_t from_table; /* 1 if the loaded table supplied the entry */
} qlin_config;

/*
 * qlin_quantize_per_token -- dynamic per-token activation quantisation
 * ("FP8 dynamic quantization" and "W8A8 INT8", page "Helion in vLLM: A Unified
 * Route to Tunable Linear Kernels", section "What the integration changes").
 *
 * For each row r: amax = max_c |x[r,c]|; scale_out[r] = amax / Qmax (IEEE
 * binary32 division; Qmax = 127 for INT8, 448 for FP8); q_out[r,c] =
 * round(x[r,c] / scale_out[r]) -- INT8: half-to-even, clamped to [-127,127];
 * FP8: clamped to [-448,448] then nearest e4m3, ties to even.  A row whose
 * amax is 0 gets scale 0 and all-zero codes.  Also quantises weights
 * per output channel (rows of W).
 *
 *   fmt        QLIN_FMT_INT8 or QLIN_FMT_FP8
 *   x          bf16 [rows, ld_x] (device); only the first `cols` of each row are read
 *   rows, cols rows >= 0 (0 is a no-op), cols >= 1, cols % 8 == 0
 *   ld_x       row stride of x in elements, >= cols, ld_x % 8 == 0
 *   q_out      int8 / e4m3 [rows, cols] dense (device)
 *   scale_out  fp32 [rows] (device)
 *   flags      0 or QLIN_PDL
 * Alignment: x, q_out 16-byte aligned; scale_out 4-byte aligned.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA (launch failure).
 */
QLIN_API qlin_status qlin_quantize_per_token(int fmt, const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                             void* q_out, float* scale_out, uint32_t flags, qlin_stream_t stream);

/*
 * qlin_quantize_block -- Block-FP8 quantisation ("Block-FP8", page "Helion in
 * vLLM: A Unified Route to Tunable Linear Kernels", section "What the
 * integration changes"): one scale per block of block_rows x block_cols
 * elements, scale = block amax / 448, codes as in qlin_quantize_per_token's
 * FP8 path.  block_rows = 1 gives the 1x128 activation groups (the dynamic,
 * per-call path); block_rows = 128 gives the 128x128 weight blocks (done once
 * per weight, offline).  A block on the bottom edge covers the rows that exist.
 *
 *   x           bf16 [rows, ld_x] (device)
 *   block_rows  1 or 128;  block_cols  128;  cols % 128 == 0
 *   q_out       e4m3 [rows, cols] dense (device)
 *   scale_out   fp32 [ceil(rows/block_rows), cols/128] row-major (device)
 *   flags       0 or QLIN_PDL
 * Alignment as qlin_quantize_per_token.
 * Errors: INVALID_ARG, UNSUPPORTED (other block shapes), ALIGNMENT, CUDA.
 */
QLIN_API qlin_status qlin_quantize_block(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int block_rows,
                                         int block_cols, void* q_out, float* scale_out, uint32_t flags,
                                         qlin_stream_t stream);

/*
 * qlin_scaled_mm -- the scaled GEMM with a fused scale / bias / bf16 epilogue,
 * strategies "ordinary GEMM", "Split-K" and "Swap-AB" (page "Helion in vLLM: A
 * Unified Route to Tunable Linear Kernels", section "What the integration
 * changes").  Runs as one persistent tcgen05 kernel (TMA-fed shared-memory
 * stages, accumulators in tensor memory).
 *
 *   INT8, FP8:  C[m,n] = bf16( ((float)acc[m,n] * s_a[m]) * s_w[n] + bias[n] )
 *               s_a fp32 [M], s_w fp32 [N]; acc exact int32 (INT8) or fp32 (FP8)
 *   FP8_BLOCK:  C[m,n] = bf16( sum_kb P_kb[m,n] * (s_a[m,kb] * s_w[n/128,kb]) )
 *               s_a fp32 [M, K/128], s_w fp32 [ceil(N/128), K/128]; bias must be NULL
 *
 * Determinism and batch invariance: K is cut into k_segments equal segments,
 * a fixed number per (format, N, K) in the dispatch table; every variant sums
 * the per-segment results in the same fixed order s = 0..S-1, so a row of C
 * depends only on that row of A and never on M, on the variant or on the
 * order in which CTAs finish.
 *
 *   fmt, variant        qlin_format, qlin_variant (AUTO = table / built-in rule)
 *   tile_n, k_segments  0 = take from the table / rule; otherwise forced
 *                       (a forced k_segments gives up invariance with calls that
 *                       use another value)
 *   M, N, K             M >= 0 (0 is a no-op), N >= 16, N % 16 == 0
 *                       (FP8_BLOCK: N % 128 == 0), K % 128 == 0, k_segments | K/128
 *   a_q, w_q            int8 / e4m3 [M,K] and [N,K] (device)
 *   bias                bf16 [N] (device) or NULL
 *   c_out               bf16 [M,N] (device); int32 [M,N] with QLIN_OUT_I32ACC
 *   flags               QLIN_OUT_I32ACC (INT8 only), QLIN_PDL, QLIN_SPLITK_CLUSTER
 *   workspace           device buffer of at least qlin_scaled_mm_workspace_size()
 *                       bytes (may be NULL when that size is 0, and for a
 *                       Split-K run as a cluster).  Its first
 *                       64 KiB hold the Split-K ticket words: they must be
 *                       zero-filled once when the buffer is allocated, and every
 *                       call that completes leaves them at zero again; the rest
 *                       holds partial tiles.  Calls that overlap in time must
 *                       not share a workspace.  After qlin_sync_status() has
 *                       reported QLIN_ERR_DEVICE_TIMEOUT, a CTA may have left a
 *                       ticket half-counted: zero the first 64 KiB again before
 *                       the buffer is used by another call.
 * Alignment: a_q, w_q, c_out, workspace 16-byte aligned; scales and bias 4 / 2.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_scaled_mm(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N, int64_t K,
                           const void* a_q, const float* s_a, const void* w_q, const float* s_w,
                           const void* bias, void* c_out, uint32_t flags, void* workspace,
                           size_t workspace_bytes, qlin_stream_t stream);

/*
 * qlin_matmul_bf16 -- the batch-invariant persistent bf16 matmul of the page
 * "[Kernel][Perf] Add Hopper (SM90) tuned config for batch-invariant
 * persistent matmul" (section "Summary": a per-shape tuned persistent matmul
 * whose outputs do not depend on the batch size; "Test Plan"), on the same
 * kernel family, tiles, strategies and dispatch table as qlin_scaled_mm:
 *
 *     C[m,n] = bf16( fp32( sum_k a[m,k] * w[n,k] ) + bias[n] )
 *
 * Determinism and batch invariance exactly as qlin_scaled_mm: K is cut into
 * k_segments segments fixed per (N, K) in the table; each segment is summed by
 * the tensor core in fp32 and the segments are added in order from +0, so a
 * row of C depends only on that row of a, never on M, the variant or CTA
 * timing.  A K block is 64 bf16 elements (128 bytes); k_segments | K/64.
 *
 *   variant, tile_n, k_segments   as qlin_scaled_mm (AUTO: table entry "bf16")
 *   M, N, K       M >= 0 (0 is a no-op), N >= 16, N % 16 == 0, K % 64 == 0
 *   a, w          bf16 [M, K] and [N, K] row-major (device)
 *   bias          bf16 [N] (device) or NULL
 *   c_out         bf16 [M, N] (device)
 *   flags         QLIN_PDL, QLIN_SPLITK_CLUSTER
 *   workspace     as qlin_scaled_mm (size from qlin_scaled_mm_workspace_size
 *                 with QLIN_FMT_BF16)
 * Alignment: a, w, c_out, workspace 16-byte aligned; bias 2.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_matmul_bf16(int variant, int tile_n, int k_segments, int64_t M, int64_t N, int64_t K,
                                      const void* a, const void* w, const void* bias, void* c_out, uint32_t flags,
                                      void* workspace, size_t workspace_bytes, qlin_stream_t stream);

/*
 * qlin_scaled_mm_noalloc -- qlin_scaled_mm for callers that cannot allocate
 * device memory and so cannot pass a workspace (no source page describes one;
 * this is a library convenience).  Typical caller: a plugin inside a serving
 * engine that owns the whole device-memory pool and forbids allocations it
 * does not make itself, so that every byte the engine hands out is accounted
 * for by the engine.
 *
 * Same arguments, flags (QLIN_OUT_I32ACC, QLIN_PDL, QLIN_SPLITK_CLUSTER),
 * arithmetic and results as qlin_scaled_mm, without the workspace: the Split-K
 * ticket words and partial tiles live in a device array of
 * QLIN_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.  The entry point allocates
 * nothing and calls no allocating routine.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current).
 *   - Each call that needs the array clears its ticket words on `stream`
 *     before the launch (the array keeps the previous call's contents).
 *   - All calls share the one array: calls whose kernels overlap in time on the
 *     GPU (e.g. on two streams) race on it and must be avoided.
 *   - M = 0 is a no-op that returns QLIN_OK after the shape checks.
 * Errors: as qlin_scaled_mm; QLIN_ERR_WORKSPACE when the resolved configuration
 * needs more scratch than QLIN_NOALLOC_SCRATCH_BYTES (force a smaller
 * k_segments, a non-Split-K variant, or QLIN_SPLITK_CLUSTER, which needs none).
 */
#define QLIN_NOALLOC_SCRATCH_BYTES (8u << 20) /* 8 MiB: 64 KiB of tickets + partial tiles */
QLIN_API qlin_status qlin_scaled_mm_noalloc(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N,
                                            int64_t K, const void* a_q, const float* s_a, const void* w_q,
                                            const float* s_w, const void* bias, void* c_out, uint32_t flags,
                                            qlin_stream_t stream);

/*
 * qlin_linear -- the whole quantized linear layer: dynamic activation
 * quantisation of bf16 x (per token for INT8 / FP8, 1x128 groups for
 * FP8_BLOCK, exactly as qlin_quantize_per_token / qlin_quantize_block) followed
 * by qlin_scaled_mm, in one call.  Results -- C, and the codes and scales
 * written to a_q / s_a -- are bitwise those of the two calls in sequence.
 *
 * By default the quantiser runs first and the GEMM is launched as its
 * programmatic dependent.  With QLIN_FUSED, Swap-AB configurations (small M)
 * whose work units fit the kernel's resident activation operand (at most 32,
 * 16 or 8 K blocks of 128 per unit for tile_n 16, 32, 64) run as ONE kernel:
 * each CTA quantises the bf16 rows of its unit into shared memory itself, so
 * the codes never make the round trip through HBM before the GEMM reads them
 * and there is no second launch; other configurations ignore the flag.
 *
 *   x          bf16 [M, K] (device), row stride ld_x elements (ld_x >= K, ld_x % 8 == 0)
 *   a_q, s_a   outputs: the activation codes [M, K] and scales (fp32 [M], or
 *              [M, K/128] for FP8_BLOCK), as the quantisers write them
 *   others     as qlin_scaled_mm (workspace: qlin_scaled_mm_workspace_size)
 *   flags      QLIN_PDL (applies to the first kernel), QLIN_FUSED,
 *              QLIN_OUT_I32ACC (INT8 only)
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_linear(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N, int64_t K,
                                 const void* x, int64_t ld_x, void* a_q, float* s_a, const void* w_q,
                                 const float* s_w, const void* bias, void* c_out, uint32_t flags, void* workspace,
                                 size_t workspace_bytes, qlin_stream_t stream);

/*
 * ---------------------------------------------------------------- FP8 MoE
 * The FP8 MoE layer run as one path of kernels chained with programmatic
 * dependent launch, as the page "vLLM and Tencent Hunyuan upstream two HPC
 * backends for NVIDIA Hopper GPUs" describes it (section "FP8 MoE pipeline as
 * a single execution path": routing, Gate-Up GEMM, activation function,
 * quantisation, Down GEMM, top-k reduction).  Dimensions: T tokens, hidden
 * size H, expert intermediate size I, E experts (1 .. 255), top-k (1 .. 32,
 * <= E); R = T * topk expert rows.  Each entry point below is one step; every
 * one accepts QLIN_PDL (launch as the previous kernel's programmatic
 * dependent) and is asynchronous on `stream`.
 */

/*
 * qlin_moe_route -- top-k routing and the expert row layout.  For token t:
 * the topk experts with the largest fp32 logits (descending; ties to the
 * lower expert index) into topk_ids [T, topk], and weights into topk_w
 * [T, topk]: w_j = e_j / (e_0 + ... ) in fp32 with e_j = fp32(exp(l_j - l_0))
 * (the exponential in binary64).  Then offsets [E + 1] = prefix sums of the
 * experts' row counts, and rows [T, topk] = the row of (t, j) in expert
 * topk_ids[t, j]'s group [offsets[e], offsets[e+1]) (any order inside a group;
 * results never depend on it).  logits fp32 [T, E]; all device pointers.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_moe_route(int64_t T, int E, int topk, const float* logits, int32_t* topk_ids,
                                    float* topk_w, int32_t* rows, int32_t* offsets, uint32_t flags,
                                    qlin_stream_t stream);

/*
 * qlin_moe_quantize_scatter -- per-token FP8 quantisation of x (bf16 [T, H],
 * H % 16 == 0; as qlin_quantize_per_token) written to each of the token's
 * expert rows: a_q [R, H] e4m3, s_a [R] fp32, rows as qlin_moe_route made them.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_moe_quantize_scatter(int64_t T, int64_t H, int topk, const void* x, const int32_t* rows,
                                               void* a_q, float* s_a, uint32_t flags, qlin_stream_t stream);

/*
 * qlin_moe_grouped_mm -- the scaled GEMM over experts: for each expert e and
 * each row r of its group [offsets[e], offsets[e+1]),
 *     C[r, n] = bf16( ((float)acc * s_a[r]) * s_w[e N + n] ),
 *     acc = sum_k A_q[r, k] W_q[e N + n, k]
 * (INT8 or FP8 per-token / per-channel, as qlin_scaled_mm without bias).  One
 * persistent tcgen05 kernel; the experts' tile counts are read from offsets
 * (device) after the dependency wait.  A row's result never depends on the
 * other rows of its tile or on the tiling (K is summed in one segment).
 *   fmt        QLIN_FMT_INT8 or QLIN_FMT_FP8
 *   variant    AUTO (Swap-AB when the average rows per expert is <= 64, else
 *              plain), QLIN_VAR_SWAPAB or QLIN_VAR_PLAIN; tile_n 0 or as
 *              qlin_scaled_mm
 *   a_q [R, K], s_a [R]; w_q [E N, K], s_w [E N]; c_out bf16 [R, N]
 *   N % 16 == 0, K % 128 == 0
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_moe_grouped_mm(int fmt, int variant, int tile_n, int E, int64_t R, int64_t N, int64_t K,
                                         const void* a_q, const float* s_a, const int32_t* offsets, const void* w_q,
                                         const float* s_w, void* c_out, uint32_t flags, qlin_stream_t stream);

/*
 * qlin_moe_act_quantize -- the activation and its quantisation: for each row
 * r of g (bf16 [R, 2I]: gate = g[:, :I], up = g[:, I:]), h = silu(gate) * up
 * in fp32 with silu(x) = x / (1 + fp32(exp(-x))) (the exponential in
 * binary64), then the per-token FP8 quantisation of h into h_q [R, I] and
 * s_h [R] (scale = amax / 448, codes as qlin_quantize_per_token).  I % 16 == 0.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_moe_act_quantize(int64_t R, int64_t I, const void* g, void* h_q, float* s_h,
                                           uint32_t flags, qlin_stream_t stream);

/*
 * qlin_moe_combine -- the top-k reduction: out[t, n] = bf16( sum_j topk_w[t, j]
 * * y[rows[t, j], n] ), summed in fp32 from +0 in routing order j = 0 ..
 * topk-1, each product and add separately rounded.  y bf16 [R, H], out bf16
 * [T, H], H % 16 == 0.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_moe_combine(int64_t T, int64_t H, int topk, const void* y, const float* topk_w,
                                      const int32_t* rows, void* out, uint32_t flags, qlin_stream_t stream);

/*
 * qlin_moe_workspace_size -- bytes of workspace qlin_moe_forward needs.  The
 * workspace holds, each at a 256-byte aligned offset in this order: topk_ids
 * [R] int32, topk_w [R] fp32, rows [R] int32, offsets [E + 1] int32, a_q [R, H]
 * e4m3, s_a [R], g [R, 2I] bf16, h_q [R, I] e4m3, s_h [R], y [R, H] bf16.
 * Errors: INVALID_ARG.
 */
QLIN_API qlin_status qlin_moe_workspace_size(int64_t T, int64_t H, int64_t I, int E, int topk, size_t* bytes_out);

/*
 * qlin_moe_forward -- the whole FP8 MoE layer: route, quantise-scatter,
 * grouped gate-up GEMM (N = 2I, K = H), activation + quantisation, grouped
 * down GEMM (N = H, K = I), combine; seven kernels, each after the first the
 * previous one's programmatic dependent.  x bf16 [T, H]; logits fp32 [T, E];
 * w1_q e4m3 [E, 2I, H] with s_w1 [E, 2I]; w2_q e4m3 [E, H, I] with s_w2
 * [E, H] (weights quantised per output channel, e.g. by
 * qlin_quantize_per_token on the [E * rows, cols] view); out bf16 [T, H].
 * H % 128 == 0, I % 128 == 0.  workspace: qlin_moe_workspace_size() bytes,
 * 16-byte aligned, no initialisation needed; calls that overlap in time must
 * not share one.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_moe_forward(int64_t T, int64_t H, int64_t I, int E, int topk, const void* x,
                                      const float* logits, const void* w1_q, const float* s_w1, const void* w2_q,
                                      const float* s_w2, void* out, uint32_t flags, void* workspace,
                                      size_t workspace_bytes, qlin_stream_t stream);

/*
 * qlin_scaled_mm_workspace_size -- bytes of workspace qlin_scaled_mm needs for
 * the same (fmt, variant, tile_n, k_segments, M, N, K): the Split-K partial
 * tiles plus one ticket word per output tile (0 for the other variants).  A
 * call with QLIN_SPLITK_CLUSTER that can run as a cluster needs none.
 * Host-only; resolves AUTO through the table exactly as qlin_scaled_mm does.
 * Errors: INVALID_ARG, UNSUPPORTED.
 */
QLIN_API qlin_status qlin_scaled_mm_workspace_size(int fmt, int variant, int tile_n, int k_segments, int64_t M,
                                          int64_t N, int64_t K, size_t* bytes_out);

/*
 * qlin_dispatch_table_load -- load a per-shape dispatch table written by the
 * offline sweep (format: see the sweep's source).  Per-shape configurations
 * are looked up at launch, as the page "[Kernel][Perf] Add Hopper (SM90) tuned
 * config for batch-invariant persistent matmul" describes (section "Summary":
 * the config lookup runs at kernel launch and at initialisation).  The table
 * header names the device it was measured on; a table from another device
 * (name, compute capability or SM count) is refused, the lesson of that page's
 * review thread about a table applied to the wrong Hopper parts.  Entries
 * whose shared-memory need exceeds the device's opt-in limit, or whose
 * k_segments differ between M buckets of one (format, N, K), are refused.
 * Replaces any previously loaded table; a failed load leaves the previous
 * table in place.  Blocking, host-only; call it before any graph capture.
 * Errors: INVALID_ARG, TABLE_IO, TABLE_FORMAT, TABLE_DEVICE, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_dispatch_table_load(const char* path);

/* Drop the loaded table (AUTO then uses the built-in rule).  Host-only. */
QLIN_API qlin_status qlin_dispatch_table_clear(void);

/*
 * qlin_dispatch_query -- the configuration AUTO resolves to for a shape: the
 * table entry for (fmt, N, K) with the smallest m_max >= M (the largest if M
 * exceeds them all), else the built-in rule (Swap-AB for M <= 64, Split-K when
 * the output tiles cannot fill the SMs, plain otherwise).  Host-only, no
 * allocation.
 * Errors: INVALID_ARG, UNSUPPORTED.
 */
QLIN_API qlin_status qlin_dispatch_query(int fmt, int64_t M, int64_t N, int64_t K, qlin_config* out);

/* Human-readable text for a status code (static storage; never NULL). */
QLIN_API const char* qlin_status_string(qlin_status status);

/*
 * qlin_sync_status -- synchronise `stream`, then report and clear the device
 * status word that kernels set when a bounded wait gives up.  Returns QLIN_OK,
 * QLIN_ERR_DEVICE_TIMEOUT or QLIN_ERR_CUDA.  Blocking.  After
 * QLIN_ERR_DEVICE_TIMEOUT the outputs of the calls since the previous check
 * are undefined and any Split-K workspace they used must have its 64 KiB
 * ticket prefix zeroed again before reuse.
 */
QLIN_API qlin_status qlin_sync_status(qlin_stream_t stream);

/*
 * qlin_selftest_wait_timeout -- exercise the failure path of the device-side
 * waits without faulting the GPU: enqueue a one-thread kernel that waits, for
 * at most limit_us microseconds (1 .. 1000000), on an mbarrier that nothing
 * arrives on.  The wait gives up, records QLIN_ERR_DEVICE_TIMEOUT and the
 * kernel returns; the next qlin_sync_status() on the stream reports (and
 * clears) it, and the context stays usable.  Asynchronous.
 * Errors: INVALID_ARG, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_selftest_wait_timeout(uint32_t limit_us, qlin_stream_t stream);

/*
 * Block-scaled formats.  The page "Helion in vLLM: A Unified Route to Tunable
 * Linear Kernels" (introduction) lists NVFP4 among the formats vLLM's quantized
 * linear layers serve; neither it nor MXFP8 is defined there.  These entry
 * points follow the formats' public definitions:
 *
 *   MXFP8 (OCP Microscaling Formats v1.0): blocks of 32 consecutive elements
 *     along K share one E8M0 scale X = 2^(code - 127).  Quantisation: amax =
 *     max |x| of the block; amax == 0 gives code 0 and zero elements;
 *     otherwise e = floor(log2(amax)) - 8, clamped to [-127, 127], code e + 127,
 *     q = e4m3(x * 2^-e) (nearest, ties to even, saturating at +-448).
 *   NVFP4: blocks of 16 elements along K share one E4M3 scale s, and the
 *     tensor has one fp32 decode scale g (x ~ q * s * g).  Quantisation: s =
 *     e4m3((amax / 6) / g) (two binary32 divisions, then nearest, saturating at
 *     448); d = s * g (binary32); d == 0 gives zero elements; otherwise q =
 *     e2m1(x / d) (binary32 division, nearest of +-{0, .5, 1, 1.5, 2, 3, 4, 6},
 *     ties to even, saturating at 6).  Two elements per byte, element 2i in
 *     the low nibble.
 *
 * Scale-factor layout ("tiled", what the tensor cores read): rows are grouped
 * by 128 and K by atoms of 4 scale factors (128 elements for MXFP8, 64 for
 * NVFP4).  Each (row group, atom) is one 512-byte block, stored row group
 * major, atom minor: sf[(r / 128) * atoms + a][512], and inside it the scale
 * of row r and sub-block j (0..3) of the atom sits at byte
 * (r % 32) * 16 + ((r / 32) % 4) * 4 + j.  atoms = K / 128 (MXFP8) or K / 64
 * (NVFP4); the buffer holds ceil(rows / 128) * atoms * 512 bytes.  The bytes
 * of rows past the last row are never written; whatever they hold only
 * reaches outputs that are not stored.
 */

/*
 * qlin_quantize_block_scaled -- MXFP8 or NVFP4 quantisation of a bf16 matrix
 * (activations per call; weights once, offline), arithmetic as above.
 *
 *   fmt        QLIN_FMT_MXFP8 or QLIN_FMT_NVFP4
 *   x          bf16 [rows, ld_x] (device)
 *   rows, cols rows >= 0 (0 is a no-op); cols % 128 == 0
 *   ld_x       row stride of x in elements, >= cols, ld_x % 8 == 0
 *   g          NVFP4: fp32 [1] (device), the tensor's decode scale, > 0 and
 *              finite; MXFP8: NULL
 *   q_out      MXFP8: e4m3 [rows, cols]; NVFP4: uint8 [rows, cols / 2] (device)
 *   sf_out     tiled scale factors, ceil(rows/128) * atoms * 512 bytes (device)
 *   flags      0 or QLIN_PDL
 * Inputs must be finite.  Alignment: x, q_out, sf_out 16-byte aligned; g 4.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA.
 */
QLIN_API qlin_status qlin_quantize_block_scaled(int fmt, const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                                const float* g, void* q_out, void* sf_out, uint32_t flags,
                                                qlin_stream_t stream);

/*
 * qlin_block_scaled_mm -- the GEMM of the block-scaled formats on the tcgen05
 * block-scaled MMA (kind::mxf8f6f4 with E8M0 scales, kind::mxf4nvf4 with E4M3
 * scales over 16-element blocks), which applies the scale factors inside the
 * tensor core:
 *
 *   MXFP8:  C[m,n] = bf16( acc[m,n] + bias[n] )
 *   NVFP4:  C[m,n] = bf16( ((acc[m,n] * g_a) * g_w) + bias[n] )
 *           acc[m,n] = sum over blocks of (block scales) * sum_k a_q w_q, fp32
 *
 * Plain tiles of 128 x 128 and, for M <= tile_n, Swap-AB tiles of 32 or 64
 * activation rows (one activation tile: its scales are the first rows of the
 * first 128-row atom; no tile 16, no pair tiles), each with Split-K.  K is cut into
 * k_segments segments added in order from +0, as in qlin_scaled_mm, so rows of
 * C do not depend on M or on the variant.  The dispatch table's entries are
 * keyed "mxfp8" / "nvfp4"; without one, M <= 64 runs Swap-AB and larger M
 * plain tiles, with one K segment.
 *
 *   fmt                 QLIN_FMT_MXFP8 or QLIN_FMT_NVFP4
 *   variant             AUTO, PLAIN, SPLITK, SWAPAB or SWAPAB_SPLITK
 *   tile_n              0, or 128 (plain) / 32, 64 (Swap-AB, M <= tile_n);  k_segments as
 *                       qlin_scaled_mm
 *   M, N, K             M >= 0 (0 is a no-op), N >= 16, N % 16 == 0;
 *                       K % 128 == 0 (MXFP8) or K % 256 == 0 (NVFP4)
 *   a_q, a_sf           A codes [M, K] (NVFP4: [M, K/2] packed) and tiled scales (device)
 *   w_q, w_sf           W codes [N, K] (NVFP4: [N, K/2]) and tiled scales (device)
 *   g_a, g_w            NVFP4: fp32 [1] each (device), the tensors' decode scales;
 *                       MXFP8: NULL
 *   bias                bf16 [N] (device) or NULL
 *   c_out               bf16 [M, N] (device)
 *   flags               QLIN_PDL
 *   workspace           as qlin_scaled_mm (size from qlin_scaled_mm_workspace_size
 *                       with the same fmt)
 * Alignment: a_q, a_sf, w_q, w_sf, c_out, workspace 16-byte aligned; g 4; bias 2.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA, NO_DEVICE.
 */
QLIN_API qlin_status qlin_block_scaled_mm(int fmt, int variant, int tile_n, int k_segments, int64_t M, int64_t N,
                                          int64_t K, const void* a_q, const void* a_sf, const void* w_q,
                                          const void* w_sf, const float* g_a, const float* g_w, const void* bias,
                                          void* c_out, uint32_t flags, void* workspace, size_t workspace_bytes,
                                          qlin_stream_t stream);

/* ABI version of the loaded library (QLIN_ABI_VERSION at build time). */
QLIN_API int qlin_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QLIN_H */
