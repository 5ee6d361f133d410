/*
 * lmoe.h -- C ABI of the LatentMoE layer forward for NVIDIA B200 (sm_100a).
 *
 * The layer (per token t, tokens independent):
 *   1. router logits l = W_r f_t (+ bias), f = x_t: the gate stays at the full
 *      width d ("LatentMoE: How MoE Made a Key Paradigm Leap in 2026", section 2,
 *      closing note); with latent_router = 1 the gate reads z_t instead
 *      (the same section's step 2 reading "routing happens in the latent").
 *   2. the top-K' logits (ties to the lower expert id) and their renormalised
 *      softmax weights w.
 *   3. z_t = W_down x_t, d -> latent ("How LatentMoE Works", step 1;
 *      Nemotron-3 article section 2.2, Figure 3b).
 *   4. per selected FFN expert e, in the latent width: o = W2_e act(W1_e z_t),
 *      act = relu(u)^2 or silu(gate) * up ("How LatentMoE Works", step 2);
 *      MoE++ zero / copy / constant experts return 0 / z_t / v_c without a GEMM
 *      (Nemotron-3 article section 3.2, Figure 1).
 *   5. yl_t = sum_k w_k o_k, aggregated in the latent width (Figure 3b).
 *   6. y_t = x_t + W_up yl_t, latent -> d ("How LatentMoE Works", step 3).
 * With has_proj = 0 (latent == d) there is no W_down / W_up: the standard MoE
 * of Figure 3a, y_t = x_t + yl_t.
 * With shared_m > 0 a shared expert at the full width d (it stays at d like the
 * gate: "LatentMoE: How MoE Made a Key Paradigm Leap in 2026", section 2,
 * closing note) adds Ws2 act(Ws1 x_t), act as for the routed experts; it runs
 * on a stream of the handle's own, concurrently with the routed path.
 * With expert_fmt = LMOE_FMT_MXFP8 or LMOE_FMT_MXFP4 the FFN experts' W1 / W2
 * are stored block-scaled (Open Compute Project Microscaling v1.0; the pages
 * name MXFP4 as the Kimi K3 serving format, in the comparison table of "Two
 * Teams, Two Practices"), and the rows those matrices multiply (z_t, and
 * act(W1_e z_t)) are encoded in MXFP8 from their bf16 values before the
 * multiply; see lmoe_mx_encode_weights for the format and layout.  With
 * LMOE_FMT_NVFP4 (the pages name it as Nemotron 3 Super's training format,
 * in the training note of the outlook section) the weights and those rows
 * are NVFP4; see lmoe_nvfp4_encode_weights.
 *
 * Conventions for every entry point:
 *   - all matrices are row-major; bf16 tensors are passed as `void *` (IEEE
 *     bfloat16 bit patterns), fp32 as `float *`, ids as `int32_t *`;
 *   - "device" pointers are CUDA global-memory addresses of the current
 *     device; "host" pointers are ordinary (preferably pinned) host memory;
 *   - every device pointer must be 16-byte aligned;
 *   - the caller owns every buffer; the library never allocates device memory
 *     for data and borrows the weights and the workspace for the handle's
 *     lifetime (the executable CUDA graphs of lmoe_forward are driver objects
 *     that the handle creates on the first forward of each launch sequence,
 *     at most 8; lmoe_destroy releases them);
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); work is
 *     enqueued asynchronously, nothing in lmoe_forward synchronises the host;
 *   - return values: LMOE_OK (0) or a negative LMOE_ERR_* status; a rejected
 *     call enqueues no work.
 */
#ifndef LMOE_H
#define LMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LMOE_API __attribute__((visibility("default")))
#else
#define LMOE_API
#endif

#define LMOE_OK 0
#define LMOE_ERR_INVALID_ARG (-1)       /* null / misaligned pointer, bad enum, x aliases y */
#define LMOE_ERR_UNSUPPORTED_SHAPE (-2) /* see lmoe_config */
#define LMOE_ERR_TOO_MANY_TOKENS (-3)   /* T > max_tokens, or T < 0 */
#define LMOE_ERR_CUDA (-4)              /* a CUDA runtime / driver call failed */
#define LMOE_ERR_TIMEOUT (-5)           /* device: a bounded wait inside a kernel gave up */
#define LMOE_ERR_BAD_INDEX (-6)         /* device: an expert id outside [0, n_total), or twice in one row */
#define LMOE_ERR_WORKSPACE (-7)         /* workspace missing or smaller than lmoe_workspace_bytes */
#define LMOE_ERR_BAD_COUNTS (-8)        /* device: received row counts of lmoe_ep_experts inconsistent */

#define LMOE_ACT_RELU2 0    /* h = relu(u)^2 (non-gated) */
#define LMOE_ACT_SWIGLU 1   /* W1_e rows [0,m) gate, [m,2m) up: h = silu(gate) * up */
#define LMOE_ACT_IDENTITY 2 /* h = u (test use) */

#define LMOE_FMT_BF16 0  /* expert weights in bf16 */
#define LMOE_FMT_MXFP8 1 /* E4M3 elements, one E8M0 scale per 32 along K */
#define LMOE_FMT_MXFP4 2 /* E2M1 elements, one E8M0 scale per 32 along K */
#define LMOE_FMT_NVFP4 3 /* E2M1 elements, one E4M3 scale per 16 along K, one fp32 scale per expert matrix */

/*
 * Layer shape.  Constraints (else LMOE_ERR_UNSUPPORTED_SHAPE): d, latent and m
 * multiples of 64 and at most 16384; 1 <= top_k <= min(32, n_total);
 * n_total = n_experts + n_zero + n_copy + n_const <= 1024; n_experts >= 1;
 * max_tokens >= 1; has_proj == 0 requires latent == d; shared_m is 0 or a
 * multiple of 64 up to 16384.  A block-scaled expert_fmt also requires
 * latent and m to be multiples of 128 (256 for NVFP4).  Block-scaled experts
 * always take the weight-streaming GEMM: an expert that received more than 32
 * rows streams its weights once per 32 rows, so they suit decode batches (at
 * T <= 32 each touched expert streams once).
 * Expert parallelism (see lmoe_ep_dispatch): ep_size 0 or 1 means none;
 * otherwise 2 <= ep_size <= n_experts, n_experts a multiple of ep_size,
 * 0 <= ep_rank < ep_size, expert_fmt == LMOE_FMT_BF16, and
 * ep_size * max_tokens * min(top_k, n_local) <= 2^30, with
 * n_local = n_experts / ep_size.
 */
typedef struct lmoe_config {
    int32_t d;             /* model width */
    int32_t latent;        /* latent width l (== d without projections) */
    int32_t m;             /* expert hidden width */
    int32_t n_experts;     /* routed FFN experts N' (ids 0 .. N'-1) */
    int32_t top_k;         /* experts per token K' */
    int32_t max_tokens;    /* largest T a forward may be called with */
    int32_t act;           /* LMOE_ACT_* */
    int32_t n_zero;        /* MoE++ zero experts (ids N' ..) */
    int32_t n_copy;        /* MoE++ copy experts (ids after the zero experts) */
    int32_t n_const;       /* MoE++ constant experts (last ids) */
    int32_t has_proj;      /* 1: LatentMoE with W_down / W_up; 0: standard MoE */
    int32_t latent_router; /* 1: the gate reads z (latent) instead of x (d) */
    int32_t shared_m;      /* hidden width of the shared expert at d; 0: no shared expert */
    int32_t expert_fmt;    /* LMOE_FMT_*: storage of the FFN experts' W1 / W2 */
    int32_t ep_size;       /* ranks the FFN experts are split over (0 or 1: all experts on this device) */
    int32_t ep_rank;       /* this rank: it holds FFN experts ep_rank * n_local .. (ep_rank + 1) * n_local - 1 */
} lmoe_config;

/*
 * Device pointers to the layer's weights (bf16 unless stated).  n_total as
 * above; n_local = n_experts / ep_size (n_experts without expert
 * parallelism): w1, w2 and their scales hold this rank's experts only, local
 * expert j being FFN expert ep_rank * n_local + j.  The router, projections,
 * constant vectors and shared expert are whole on every rank.
 */
typedef struct lmoe_weights {
    const void *w_router;     /* [n_total, d], or [n_total, latent] with latent_router */
    const float *router_bias; /* fp32 [n_total], added to the logits before selection; may be NULL */
    const void *w_down;       /* [latent, d]; NULL when has_proj == 0 */
    const void *w_up;         /* [d, latent]; NULL when has_proj == 0 */
    const void *w1;           /* [n_local, g*m, latent], g = 2 for SwiGLU else 1 (block-scaled: codes) */
    const void *w2;           /* [n_local, latent, m] (block-scaled: codes) */
    const void *const_vecs;   /* [n_const, latent]; may be NULL when n_const == 0 */
    const void *w_shared1;    /* [g*shared_m, d] (gate rows first when gated); NULL when shared_m == 0 */
    const void *w_shared2;    /* [d, shared_m]; NULL when shared_m == 0 */
    const void *w1_scales;    /* block-scaled only: scale atoms of w1 (lmoe_mx_encode_weights or
                                 lmoe_nvfp4_encode_weights: E8M0 or E4M3 bytes); else NULL */
    const void *w2_scales;    /* block-scaled only: scale atoms of w2; else NULL */
    const float *w1_gscale;   /* NVFP4 only: fp32 [n_local] tensor scale of each expert's W1_e; else NULL */
    const float *w2_gscale;   /* NVFP4 only: fp32 [n_local] tensor scale of each expert's W2_e; else NULL */
} lmoe_weights;

/*
 * Optional device buffers that receive copies of intermediate results after a
 * forward (enqueued on the same stream).  Every field may be NULL.
 */
typedef struct lmoe_debug {
    int32_t *topk_idx; /* [T, top_k] expert ids, slot order */
    float *topk_w;     /* [T, top_k] renormalised weights */
    int32_t *counts;   /* [n_total] tokens per expert */
    int32_t *offsets;  /* [n_total + 1] exclusive scan of counts */
    int32_t *perm;     /* [T * top_k] slot index t*K'+k at each sorted position */
    void *z;           /* bf16 [T, latent] latent tokens (has_proj == 1) */
    void *yl;          /* bf16 [T, latent] combined latent output (has_proj == 1) */
    float *logits;     /* fp32 [T, n_total] router logits, bias not included */
} lmoe_debug;

typedef struct lmoe_handle lmoe_handle;

/* Bytes of device workspace a handle for `cfg` needs (0 if cfg is invalid). */
LMOE_API size_t lmoe_workspace_bytes(const lmoe_config *cfg);

/*
 * Validate `cfg`, record the weight pointers, carve `workspace` (device,
 * 256-byte aligned, at least lmoe_workspace_bytes(cfg) bytes) and build the
 * TMA descriptors of the weights.  Uses the current CUDA device.  On success
 * *out receives a handle (host memory owned by the library until
 * lmoe_destroy).
 */
LMOE_API int lmoe_create(const lmoe_config *cfg, const lmoe_weights *w, void *workspace, size_t workspace_bytes,
                lmoe_handle **out);

/*
 * y = LatentMoE(x) for T tokens: x, y device bf16 [T, d], must not overlap.
 * Rejected (LMOE_ERR_INVALID_ARG) on a handle with ep_size > 1, which holds
 * only its rank's experts: use the lmoe_ep_* stages there.
 * 0 <= T <= max_tokens (T == 0 enqueues nothing and accepts NULL x / y).  Asynchronous on `stream`;
 * concurrent forwards on one handle share its workspace and must be ordered
 * by the caller (same stream).  Device-side faults (a bounded wait that gave
 * up, a bad expert id) are reported by lmoe_last_error after the stream is
 * synchronised.  Output is bit-identical from run to run.  `dbg` may be NULL.
 * By default, for a layer without a shared expert, the forward's launches
 * reach the GPU as one CUDA graph: they are captured on a stream of the
 * handle's own, and the handle's executable graph for that launch sequence is
 * updated and launched on `stream` (see lmoe_set_graph_launch).  The library
 * allocates no device memory and the host does not wait on the device.  The
 * executable graph is a driver object: its first instantiation (the first
 * graph-launched forward of a handle, or the first after a change of launch
 * sequence) left the free device memory that cudaMemGetInfo reports
 * unchanged on B200, for a decode-size and a prefill-path layer (measured to
 * its 2 MiB granularity), and replays of a kept graph take none.  With a shared expert (two streams), while
 * `stream` is itself being captured, with phase timing on, or with `dbg` set,
 * the launches go onto `stream` one by one; the results are the same bits.
 */
LMOE_API int lmoe_forward(lmoe_handle *h, const void *x, void *y, int32_t T, void *stream, const lmoe_debug *dbg);

/*
 * The same forward on HOST buffers: copies x_host [T, d] into the workspace,
 * runs the layer and copies y back to y_host [T, d].  The input copy runs on a
 * stream of the handle's own, into one of two workspace input buffers taken in
 * turn, and `stream` waits for it; the forward and the output copy run on
 * `stream`.  So calls issued back to back overlap each call's input copy with
 * the previous call's forward.  While `stream` is being captured, everything
 * runs on `stream`.  The host buffers should be pinned for the copies to be
 * asynchronous; the caller synchronises `stream` before reading y_host or
 * reusing x_host (that covers the input copy too).
 */
LMOE_API int lmoe_forward_host(lmoe_handle *h, const void *x_host, void *y_host, int32_t T, void *stream);

/*
 * Read and clear the device error word of the handle's workspace (blocking
 * copy; synchronise the forward's stream first).  Returns LMOE_OK,
 * LMOE_ERR_TIMEOUT, LMOE_ERR_BAD_INDEX or LMOE_ERR_BAD_COUNTS (the first set,
 * in that order), or LMOE_ERR_CUDA if the read failed.
 */
LMOE_API int lmoe_last_error(lmoe_handle *h);

/* Release the handle (not the caller's buffers).  NULL is ignored. */
LMOE_API void lmoe_destroy(lmoe_handle *h);

/* Static English text of a status code. */
LMOE_API const char *lmoe_status_string(int status);

/*
 * Kernel-phase timing.  With profiling on, every forward records CUDA events
 * around each phase on its stream (at most `max_forwards` forwards are kept).
 * lmoe_phase_times writes, for each phase, the summed milliseconds and the
 * number of kernel launches over the kept forwards into ms[i] / launches[i]
 * (arrays of lmoe_num_phases() entries; either may be NULL), then forgets
 * them.  Synchronise the stream(s) first.  The phase names are static.
 */
LMOE_API int lmoe_set_profiling(lmoe_handle *h, int enable, int max_forwards);
LMOE_API int lmoe_phase_times(lmoe_handle *h, float *ms, int32_t *launches);
LMOE_API int lmoe_num_phases(void);
LMOE_API const char *lmoe_phase_name(int phase);

/*
 * Sizes of the last forward's routing, read back from the device (blocking;
 * synchronise first).  After lmoe_ep_experts they describe the rows that
 * stage received for this rank's experts instead.  out8[0] rows routed to
 * FFN experts, [1] FFN experts with at least one row, [2] tensor-core
 * M-tiles, [3] experts on the weight-streaming path, [4] rows on that path,
 * [5] experts on the grouped tensor-core path, [6] rows on that path, [7] the
 * row threshold the forward used (see lmoe_set_small_rows).  Used to compute
 * the algorithmic work of a forward.  With block-scaled experts [3] counts the
 * entries of the weight-streaming list, 32 rows at most each: an expert with
 * more rows takes several, each streaming its weights.
 */
LMOE_API int lmoe_routing_stats(lmoe_handle *h, int32_t *out8);

/*
 * Expert-path threshold: FFN experts with at most `rows` routed rows (0..32,
 * default 16) take the weight-streaming GEMM (the expert's weights as the
 * 128-row tensor-core operand, its rows as a 16- or 32-row operand); the
 * others take the grouped GEMM in 128-row tiles.  A forward with T <= 32
 * tokens raises a nonzero threshold to 16 (T <= 16) or 32, so that every
 * expert streams and the grouped GEMM is not launched.  0 sends every expert
 * to the grouped GEMM.
 */
LMOE_API int lmoe_set_small_rows(lmoe_handle *h, int32_t rows);

/*
 * enable = 1 (default): lmoe_forward and lmoe_forward_host launch each forward
 * of a layer without a shared expert as one CUDA graph (captured per call on
 * the handle's own stream, replayed from an executable graph updated in place;
 * the handle keeps up to 8, one per launch sequence, since token counts can
 * change which kernels run); 0: the kernels are launched on the caller's
 * stream one by one.  Outputs are bit-identical.
 * Errors: LMOE_ERR_INVALID_ARG for a NULL handle or enable not 0 or 1.
 */
LMOE_API int lmoe_set_graph_launch(lmoe_handle *h, int enable);

/*
 * Kernel of the grouped (tensor-core) expert GEMMs, for the experts that get
 * more rows than the weight-streaming threshold.  kind = 0 (default):
 * single-CTA 128 x 256 tiles over 128-row slices of each expert's rows.
 * kind = 1: CTA pairs computing each expert's GEMM transposed, weight rows as
 * the 256-row operand split over the pair and the expert's token rows as
 * N <= 256 (taken when latent is a multiple of 256 and m of 256, or of 128
 * with SwiGLU, for bf16 experts; other shapes keep kind 0).  Kind 1 moves a
 * quarter fewer operand bytes from L2 and was faster on the Kimi-like skewed
 * layer, kind 0 on the Nemotron-like one (about 350 rows per expert); both
 * are deterministic and agree with each other to rounding.
 * Errors: LMOE_ERR_INVALID_ARG for a NULL handle or kind not 0 or 1.
 */
LMOE_API int lmoe_set_grouped_gemm(lmoe_handle *h, int kind);

/* Bound of every in-kernel wait, nanoseconds (default 1e9). */
LMOE_API int lmoe_set_wait_timeout(lmoe_handle *h, uint64_t ns);

/*
 * Failure-path self-test: launch one thread that waits, with the bounded wait
 * every kernel of the layer uses, on a barrier nothing ever arrives on.  After
 * `timeout_ns` (1 .. 2e9) it gives up and records a timeout in the handle's
 * device error word, so lmoe_last_error (after synchronising `stream`) returns
 * LMOE_ERR_TIMEOUT; the CUDA context stays usable.  Asynchronous.
 */
LMOE_API int lmoe_selftest_wait(lmoe_handle *h, uint64_t timeout_ns, void *stream);

/*
 * Plain GEMM on the layer's tensor-core kernel: C[M,N] = A[M,K] * B[N,K]^T,
 * bf16 in (device, row-major, K-major both), fp32 accumulate, bf16 out.
 * K a multiple of 64 (<= 65536), N a multiple of 64, M >= 0.  `err_word` is a
 * device int that collects device error bits (may be NULL: errors are then
 * not reported).  Asynchronous on `stream`.
 */
LMOE_API int lmoe_gemm_bf16(const void *A, const void *B, void *C, int32_t M, int32_t N, int32_t K, void *stream,
                   int *err_word);

/*
 * Expert counting sort without any caller-provided scratch.
 *
 * The pages have no counterpart to this entry point; it exists for callers that
 * cannot allocate device memory.  Examples are a plugin whose host framework
 * owns the whole device-memory budget and gives it no allocation hook, and a
 * latency-critical loop where the implicit device synchronisation of cudaMalloc
 * is unacceptable.  Such callers cannot provide the workspace that lmoe_create
 * needs.  This call does the same stable sort of the (token, slot) pairs by
 * expert as lmoe_forward's dispatch step.  It uses the same kernels, with its
 * scratch in a fixed device array of the library: a 2 MiB + 256 B bitmap /
 * prefix / header area that every device which loads the library holds until
 * the process exits.  It allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library call).
 *
 *   idx      device int32 [T, top_k]: expert ids in [0, n_total); the ids of
 *            one row (one token) must be distinct, as a top-K' selection's are
 *   counts   device int32 [n_total]: rows per expert
 *   offsets  device int32 [n_total + 1]: exclusive scan of counts
 *   perm     device int32 [T * top_k]: the slot index t*top_k+k at each sorted
 *            position
 *   inv      device int32 [T * top_k]: the sorted position of each slot
 *   err_word optional device int32 (NULL: not reported).  The call writes its
 *            device error bits there, 0 when the ids were valid:
 *              LMOE_DEVERR_BAD_INDEX       an id outside [0, n_total) was
 *                                          skipped: its slot's inv entry is not
 *                                          written, counts leave it out, and
 *                                          perm is filled only up to
 *                                          offsets[n_total] < T * top_k;
 *              LMOE_DEVERR_REPEATED_INDEX  a row named one expert twice: counts,
 *                                          perm and inv are then not a valid
 *                                          sort (every write still stays inside
 *                                          the buffers above).
 *
 * Limits: 0 <= T <= 8192 (else LMOE_ERR_TOO_MANY_TOKENS); 1 <= top_k <= 32,
 * top_k <= n_total <= 1024 (else LMOE_ERR_UNSUPPORTED_SHAPE).  A rejected call
 * enqueues no work.  T = 0 zeroes counts, offsets and *err_word.
 * The scratch array's device address is looked up (cudaGetSymbolAddress) by
 * the first call on a device, with that device current, and again whenever the
 * current context of that device has changed since (after cudaDeviceReset, for
 * instance); make that first call before any stream capture.  Every call on a
 * device shares the one scratch array, which keeps the last call's contents, so
 * calls whose work overlaps on the GPU (different streams, no ordering between
 * them) race and corrupt each other's results; order them on one stream.
 * Asynchronous on `stream`.
 */
#define LMOE_DEVERR_BAD_INDEX 2
#define LMOE_DEVERR_REPEATED_INDEX 8
LMOE_API int lmoe_dispatch_noalloc(const int32_t *idx, int32_t T, int32_t top_k, int32_t n_total, int32_t *counts,
                                   int32_t *offsets, int32_t *perm, int32_t *inv, int32_t *err_word, void *stream);

/*
 * Block-scaled (MX) encoding of a bf16 weight matrix, for lmoe_weights.w1 /
 * w2 with a block-scaled expert_fmt.  It follows the Open Compute Project
 * Microscaling specification v1.0 (the pages name the format only).  Each
 * row is split into blocks of 32 consecutive values along K.  A block shares
 * one scale 2^s, stored as the E8M0 byte s + 127, with
 * s = floor(log2 max|v|) - emax: emax is 8 for E4M3, 2 for E2M1; s is clamped
 * to [-127, 127]; an all-zero block gets s = -127.  Each element is v / 2^s
 * rounded to the nearest element value, ties to even, and saturated at
 * +-448 (E4M3) or +-6 (E2M1).
 *
 *   w       device bf16 [rows, K]: an expert tensor viewed as rows, e.g. W1
 *           as [n_experts * g * m, latent], W2 as [n_experts * latent, m]
 *   rows    multiple of 128;  K multiple of 128
 *   fmt     LMOE_FMT_MXFP8 or LMOE_FMT_MXFP4
 *   codes   device, [rows, K] bytes (E4M3), or [rows, K/2] bytes (E2M1: two
 *           per byte, element 2i in the low nibble of byte i)
 *   scales  device, rows * K / 32 bytes, in 512-byte atoms
 *           [rows/128][K/128][32][16]: byte (r, c) of atom (R, G) holds the
 *           scale of row 128R + 32(c/4) + r, block 4G + c%4 (the order in
 *           which the tensor cores read block scales)
 *
 * Bad sizes or format: LMOE_ERR_UNSUPPORTED_SHAPE; a NULL or misaligned
 * pointer: LMOE_ERR_INVALID_ARG.  Asynchronous on `stream`; deterministic.
 */
LMOE_API int lmoe_mx_encode_weights(const void *w, int64_t rows, int32_t K, int32_t fmt, void *codes, void *scales,
                                    void *stream);

/*
 * NVFP4 encoding of bf16 weight matrices, for lmoe_weights.w1 / w2 with
 * expert_fmt = LMOE_FMT_NVFP4.  It follows NVIDIA's published two-level
 * definition (the pages name the format only).  Each of the n_mats matrices
 * (an expert's W1_e or W2_e, rows_per_mat rows of K values) takes one fp32
 * tensor scale g = amax / (6 * 448), or 1 when all its values are zero.  Each
 * row is split into blocks of 16 consecutive values along K; a block shares
 * one positive E4M3 scale sb = E4M3(amax_block / (g * 6)), and each element
 * is E2M1(v / (sb * g)); both round to nearest even and saturate (448, 6),
 * and a block whose scale is zero encodes zeros.  The products g * 6 and
 * sb * g and both quotients are fp32 operations.  An element stands for
 * e2m1 * sb * g.
 *
 *   w             device bf16 [n_mats * rows_per_mat, K]
 *   n_mats        1 .. 65535;  rows_per_mat a multiple of 128;  K a multiple
 *                 of 64 (the layer's kernels need multiples of 256)
 *   codes         device, [n_mats * rows_per_mat, K/2] bytes, two elements
 *                 per byte, element 2i in the low nibble of byte i
 *   scales        device, rows * K / 16 bytes, in 512-byte atoms
 *                 [rows/128][K/64][32][16]: byte (r, c) of atom (R, G) holds
 *                 the scale of row 128R + 32(c/4) + r, block 4G + c%4 (one
 *                 atom per 64 values of 128 rows: the order in which the
 *                 tensor cores read the scales of one K = 64 MMA)
 *   gscale        device fp32 [n_mats]: the tensor scales (written)
 *
 * Bad sizes: LMOE_ERR_UNSUPPORTED_SHAPE; a NULL or misaligned pointer:
 * LMOE_ERR_INVALID_ARG.  Asynchronous on `stream`; deterministic.
 */
LMOE_API int lmoe_nvfp4_encode_weights(const void *w, int32_t n_mats, int64_t rows_per_mat, int32_t K, void *codes,
                                       void *scales, float *gscale, void *stream);

/*
 * Expert parallelism: the forward split at the two all-to-all exchanges that
 * the pages put between routing and the experts and between the experts and
 * the aggregation (Kimi K3 / Nemotron 3 Super article, "MoE 遇到了什么问题？";
 * Nemotron-3 article section 2.2: the exchanged rows are latent-wide, which is
 * the 4x saving in communication volume the LatentMoE design is built on).
 * The library does no communication: the caller moves the rows between the
 * stages (NCCL all-to-all over NVLink, for instance).  One forward on one rank:
 *
 *   lmoe_ep_dispatch   router, W_down, top-K', counting sort; the latent rows
 *                      of slots routed to FFN experts, grouped by expert id,
 *                      hence by destination rank, go to send_rows.
 *   (caller)           all-to-all of send_counts, then of the rows: rank r's
 *                      block of send_rows goes to rank r.
 *   lmoe_ep_experts    this rank's experts on the rows it received.
 *   (caller)           the reverse all-to-all of the expert outputs.
 *   lmoe_ep_combine    aggregation in the latent width (MoE++ bypass experts
 *                      included; they need no exchange), W_up and residual.
 *
 * The result of dispatch -> exchange -> experts -> exchange -> combine on
 * ep_size ranks equals, token for token, lmoe_forward of the whole layer.
 * The stages need expert_fmt == LMOE_FMT_BF16 (else LMOE_ERR_UNSUPPORTED_SHAPE).
 * The three stages keep state in the handle's workspace: a handle serves one
 * forward at a time, dispatch before combine, all on one stream.  The experts
 * stage uses workspace that dispatch and combine do not, so it may run
 * between them (it normally does: it serves the other ranks' tokens).
 */

/*
 * Stage 1.  x device bf16 [T, d], 0 <= T <= max_tokens, unchanged until
 * lmoe_ep_combine has run (the residual and the shared expert read it).
 *   send_rows    device bf16 [T * top_k, latent] (capacity): rows 0 .. n_send-1
 *                receive the latent rows (z_t, or x_t for the standard MoE)
 *                of every (token, slot) routed to an FFN expert, ordered by
 *                expert id, then token, then slot.  n_send = sum(send_counts).
 *   send_counts  device int32 [n_experts]: rows per FFN expert.  Viewed as
 *                [ep_size][n_local], row r counts the rows for rank r, which
 *                are the r-th consecutive block of send_rows.
 * T == 0 only zeroes send_counts.  Asynchronous on `stream`.
 */
LMOE_API int lmoe_ep_dispatch(lmoe_handle *h, const void *x, int32_t T, void *send_rows, int32_t *send_counts,
                              void *stream);

/*
 * Stage 2: this rank's FFN experts on the rows it received.
 *   recv_rows    device bf16 [n_recv, latent]: ep_size consecutive blocks,
 *                block s being rank s's rows for this rank (its send_rows
 *                block ep_rank), in rank s's order.
 *   recv_counts  device int32 [ep_size, n_local]: recv_counts[s][j] = rank s's
 *                send_counts[ep_rank * n_local + j].
 *   n_recv       sum of recv_counts (host value), 0 .. ep_size * max_tokens *
 *                min(top_k, n_local).
 *   rows_bound   an upper bound of the rows any one local expert received (for
 *                instance the tokens of all ranks together, or the exact
 *                maximum of the column sums of recv_counts).  At most 32 lets
 *                every expert take the weight-streaming GEMM (the same rule
 *                lmoe_set_small_rows states for T); above 32 the grouped GEMM
 *                runs too.  Must be >= 1 when n_recv > 0.
 *   out_rows     device bf16 [n_recv, latent]: row i = o_e(recv row i), e its
 *                expert.  May be recv_rows itself.
 * The device checks recv_counts: a negative count, a sum other than n_recv, or
 * an expert with more rows than rows_bound sets LMOE_ERR_BAD_COUNTS (see
 * lmoe_last_error) and the stage then computes nothing.  Asynchronous.
 */
LMOE_API int lmoe_ep_experts(lmoe_handle *h, const void *recv_rows, const int32_t *recv_counts, int32_t n_recv,
                             int32_t rows_bound, void *out_rows, void *stream);

/*
 * Stage 3.  ret_rows device bf16 [n_send, latent]: the expert outputs of
 * send_rows, in the same order (the reverse exchange's result).  y device
 * bf16 [T, d] (T of the dispatch), not overlapping x.  Requires a dispatch on
 * this handle since the last combine (else LMOE_ERR_INVALID_ARG).  With T == 0
 * it only closes the forward.  Asynchronous.
 */
LMOE_API int lmoe_ep_combine(lmoe_handle *h, const void *ret_rows, void *y, void *stream);

/*
 * The block exchange: the same three stages with fixed-size blocks, so that
 * no count has to reach the host during a forward.  Every (sending rank,
 * receiving rank) pair gets a block of block_rows rows, the same on every
 * rank, for instance lmoe_ep_block_rows(h) (max_tokens * min(top_k,
 * n_experts / ep_size), the most rows one rank can send one other rank: a
 * token's K' experts are distinct).  An all-to-all with equal splits of
 * block_rows rows (known before the forward) then moves every block, and the
 * counts (send_counts, device) only tell the receiver how many rows of each
 * block hold rows.  The blocks cost transfer volume (ep_size * block_rows
 * latent rows each way per rank, used or not), so the block exchange suits
 * decode-size batches; the packed stages above send only the routed rows but
 * need the counts on the host to size the exchange.
 *
 * lmoe_ep_dispatch_blocks: as lmoe_ep_dispatch, with send_blocks device bf16
 *   [ep_size * block_rows, latent]: rank r's rows (experts r * n_local ..,
 *   ordered as in send_rows) at rows r * block_rows ..; the other rows of
 *   each block are not written.  block_rows must be at least T * min(top_k,
 *   n_local) and at most lmoe_ep_block_rows(h) (else LMOE_ERR_INVALID_ARG).
 *   It uses the handle's gathered-row workspace to sort the rows.
 * lmoe_ep_experts_blocks: as lmoe_ep_experts, with recv_blocks device bf16
 *   [ep_size * block_rows, latent]: block s holds rank s's rows for this rank
 *   (its send_blocks block ep_rank), the first sum(recv_counts[s]) rows of it.
 *   out_blocks has the same layout (the rows past each block's count are not
 *   written) and may be recv_blocks.  A source whose counts add up to more
 *   than block_rows, a negative count, or an expert with more than rows_bound
 *   rows sets LMOE_ERR_BAD_COUNTS, and the stage computes nothing.
 * lmoe_ep_combine_blocks: as lmoe_ep_combine, with ret_blocks in the layout
 *   of send_blocks (the reverse exchange's result); it requires a
 *   lmoe_ep_dispatch_blocks since the last combine, as lmoe_ep_combine
 *   requires a lmoe_ep_dispatch.
 * All asynchronous on `stream`; the stages of one forward on one stream.
 * The result equals the packed stages' result bit for bit.
 */
LMOE_API int64_t lmoe_ep_block_rows(lmoe_handle *h);
LMOE_API int lmoe_ep_dispatch_blocks(lmoe_handle *h, const void *x, int32_t T, void *send_blocks, int32_t block_rows,
                                     int32_t *send_counts, void *stream);
LMOE_API int lmoe_ep_experts_blocks(lmoe_handle *h, const void *recv_blocks, int32_t block_rows,
                                    const int32_t *recv_counts, int32_t rows_bound, void *out_blocks, void *stream);
LMOE_API int lmoe_ep_combine_blocks(lmoe_handle *h, const void *ret_blocks, void *y, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LMOE_H */
