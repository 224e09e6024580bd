/*
 * moda.h -- C ABI of libmoda, the fused Mixture-of-Depths Attention (MoDA)
 * operator for NVIDIA B200 (sm_100a).
 *
 * The operator (paper summary of arXiv 2603.15619, section "Mixture-of-Depths
 * Attention (MoDA): The Unified Operator", joint-softmax equation and its two
 * masks): for batch b, query head h, token t, with KV head hk = floor(h / G)
 * and G = Hq / Hk (GQA by repeat_interleave, "moda-attention 0.1.0" PyPI page,
 * "Key Design Choices"),
 *
 *   s_j  = scale * <Q[b,h,t], K[b,hk,j]>              j = 0..t   (causal, incl. t)
 *   s'_l = scale * <Q[b,h,t], Kd[b,hk,t*L + l]>       l = 0..L-1 (own token only)
 *   P    = softmax over the concatenated row [s_0..s_t | s'_0..s'_{L-1}]
 *   O[b,h,t]   = sum_j P_j V[b,hk,j] + sum_l P'_l Vd[b,hk,t*L + l]
 *   LSE[b,h,t] = natural-log log-sum-exp of the row
 *
 * scale = 1/sqrt(d) unless moda_shape.softmax_scale > 0.  By default the
 * operator is causal as written above; MODA_FLAG_NONCAUSAL (the non-causal
 * kernel the pages list as unreleased) and moda_shape.depth_window (bounded
 * depth slots) change only which keys and depth rows a row sees.
 *
 * Conventions for every entry point:
 *  - Tensors are dense, contiguous, row-major, in device memory, with base
 *    addresses aligned to 16 bytes.  Layouts ("moda-attention 0.1.0" PyPI
 *    page, "Using the Kernel Directly"):
 *        Q, O, dO, dQ          [B, Hq, T, d]
 *        K, V, dK, dV          [B, Hk, T, d]
 *        Kd, Vd, dKd, dVd      [B, Hk, T*L, d], row t*L + l = layer l of token t
 *        LSE                   [B, Hq, T] float32
 *    Element type of every tensor but LSE is moda_shape.dtype.
 *  - The caller allocates and owns every buffer, including the workspace.
 *    The library never allocates, frees or synchronises; all work is queued
 *    on the caller's stream (NULL = legacy default stream).  Outputs are
 *    fully overwritten (no accumulate-into).  Inputs and outputs must not
 *    alias.
 *  - Errors are returned as moda_status; nothing is thrown across the ABI.
 *    On any error nothing has been queued.  moda_last_error_message() gives a
 *    one-line detail for the calling thread's most recent failure.
 *  - Kernel-side waits are bounded.  A wait that runs out sets a device
 *    status word and the kernel returns early; moda_check_status() reports it
 *    as MODA_ERR_TIMEOUT.
 *  - Thread-safe; calls on different streams may run concurrently.
 */
#ifndef MODA_H_
#define MODA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* moda_stream_t;

typedef enum moda_status {
    MODA_OK = 0,
    MODA_ERR_INVALID_ARG = 1,   /* NULL pointer, bad shape or enum value   */
    MODA_ERR_MISALIGNED = 2,    /* a pointer is not 16-byte aligned         */
    MODA_ERR_UNSUPPORTED = 3,   /* valid but not implemented (e.g. d=96 bf16) */
    MODA_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than required  */
    MODA_ERR_CUDA = 5,          /* a CUDA runtime / driver call failed      */
    MODA_ERR_TIMEOUT = 6        /* a kernel-side bounded wait ran out        */
} moda_status;

typedef enum moda_dtype {
    MODA_BF16 = 0,   /* bf16 in/out, fp32 accumulation and softmax statistics */
    MODA_FP32 = 1    /* fp32 everywhere (CUDA-core path)                       */
} moda_dtype;

/*
 * Depth layouts.  FLAT is the flash-compatible layout of the paper summary,
 * "Hardware-Efficient Implementation": token t's L rows contiguous at
 * [t*L, (t+1)*L).  CHUNKED is the chunk-aware view [B, Hk, T/C, C*L, d]: with
 * C counted in tokens, chunk c holds rows [c*C*L, (c+1)*C*L) of the FLAT
 * tensor, so it is the same bytes; CHUNKED only adds the check T % C == 0.
 *
 * LAYER is the natural layer-major depth cache itself (the input of
 * moda_repack_depth): Kd and Vd are [L, B, Hk, T, d], row (l, b, hk, t)
 * holding depth row t*L + l of (b, hk).  moda_fwd and moda_bwd read it in
 * place -- the tensor-map view (d, layer, token, b*Hk + hk) lands a box of
 * whole tokens in shared memory as rows t*L + l, so the transpose of the
 * repack happens inside the depth-tile loads -- and moda_bwd writes dKd and
 * dVd in the same layer-major layout.  Supported for bf16 when every depth
 * block holds whole tokens: with Tq = 128 / G and n(c) = min(c, Tq*L
 * rounded up to a multiple of 16), L must divide n(128) and n(64) (any power
 * of two L <= 64 qualifies); other shapes get MODA_ERR_UNSUPPORTED (repack
 * to FLAT instead).  The fp32 path takes FLAT or CHUNKED only.
 *
 * Results are bitwise identical for all three layouts and every C (dKd, dVd
 * in the layout of Kd, Vd).
 */
typedef enum moda_depth_layout {
    MODA_DEPTH_FLAT = 0,
    MODA_DEPTH_CHUNKED = 1,
    MODA_DEPTH_LAYER = 2
} moda_depth_layout;

/* moda_shape.flags bits. */
#define MODA_FLAG_NONCAUSAL 1  /* drop the sequence causal mask: every row sees
                                  keys 0..T-1 (ByteDance-Seed/MoDA README,
                                  "TODO": the non-causal MoDA kernel; vision use,
                                  paper summary, "7. Implications and Future
                                  Directions").  The depth matching mask stays. */

typedef struct moda_shape {
    int B;            /* batch, >= 0 (0 = nothing to do)                   */
    int Hq;           /* query heads, >= 1                                  */
    int Hk;           /* KV heads, >= 1, Hq % Hk == 0, G = Hq/Hk <= 128       */
    int T;            /* tokens, >= 0 (0 = nothing to do)                   */
    int d;            /* head dim: 64 or 128 for BF16; 1..128 for FP32       */
    int L;            /* depth rows per token, >= 0 (0: Kd/Vd may be NULL)  */
    int C;            /* chunk size in tokens (CHUNKED only; >= 1, T % C == 0) */
    moda_dtype dtype;
    moda_depth_layout depth_layout;
    float softmax_scale;  /* <= 0 selects 1/sqrt(d) */
    int flags;        /* MODA_FLAG_* bits; 0 = the causal operator           */
    int depth_window; /* 0 = all L depth rows; S in 1..L = each token attends
                         only to its last S depth rows t*L+L-S .. t*L+L-1
                         (bounded depth slots with a sliding-window policy,
                         paper summary, "6. Limitations and Trade-offs");
                         gradients of the other depth rows are zero          */
} moda_shape;

/*
 * Bytes of workspace for this shape:
 *   for_bwd = 0   moda_fwd (0: ws may be NULL);
 *   for_bwd = 1   moda_bwd at its fastest: the row statistics D plus, for
 *                 bf16 with d = 128, G in {1, 2, 4, 8} and at most 16 GiB of
 *                 them, the stored score gradients dS (16 KB per 128 query
 *                 rows x 64 keys), which the dQ kernel then reads instead of
 *                 recomputing the scores;
 *   for_bwd = 2   the least moda_bwd accepts: D only (4 bytes per query row,
 *                 rounded up to 256); the dQ kernel then recomputes S and dP.
 * Returns (size_t)-1 for a shape the corresponding call would reject or an
 * unknown for_bwd.
 */
size_t moda_workspace_size(const moda_shape* shape, int for_bwd);

/*
 * Depth-KV repack (paper summary, "Hardware-Efficient Implementation": the
 * natural depth cache is layer-major with stride T*d between layers; the
 * flash-compatible layout puts each token's L rows contiguously).
 *   src  [L, B, Hk, T, d]  layer-major cache (one tensor: K or V)
 *   dst  [B, Hk, T*L, d]   token-major; dst row t*L + l = src[l, b, hk, t]
 * A bytewise permutation: exact for any dtype.  Call once for K_depth and
 * once for V_depth.  L = 0, B = 0 or T = 0 is a no-op.
 */
moda_status moda_repack_depth(const moda_shape* shape, const void* src, void* dst,
                              moda_stream_t stream);

/*
 * Forward (the operator above, fused: one online softmax over the causal
 * sequence keys and the token's own depth rows).
 *   Q, K, V, Kd, Vd   inputs as laid out above (Kd, Vd may be NULL if L = 0)
 *   O                 output [B, Hq, T, d], dtype of the shape
 *   LSE               output [B, Hq, T] float32, natural log; needed by moda_bwd
 *   ws, ws_bytes      workspace of at least moda_workspace_size(shape, 0) bytes
 */
moda_status moda_fwd(const moda_shape* shape,
                     const void* Q, const void* K, const void* V,
                     const void* Kd, const void* Vd,
                     void* O, float* LSE,
                     void* ws, size_t ws_bytes, moda_stream_t stream);

/*
 * Backward of moda_fwd.  The pages give no backward formulas; this is the
 * derivative of the forward definition (one softmax over [seq | depth]):
 *   D = rowsum(dO * O),  dS = P * (dO . v - D),
 *   dQ = scale * (sum_j dS_j K_j + sum_l dS'_l Kd_l),
 *   dK[hk,j]  = scale * sum over the group's heads h and rows t >= j of dS q,
 *   dV[hk,j]  = sum over the same rows of P dO,
 *   dKd[hk,t*L+l] = scale * sum over the group's heads of dS' q[h,t],
 *   dVd[hk,t*L+l] = sum over the group's heads of P' dO[h,t].
 *   O, LSE            the outputs of moda_fwd for the same inputs
 *   dO                incoming gradient [B, Hq, T, d]
 *   dQ, dK, dV, dKd, dVd   outputs (fully overwritten; dKd/dVd may be NULL if L = 0)
 *   ws, ws_bytes      workspace: at least moda_workspace_size(shape, 2) bytes;
 *                     with moda_workspace_size(shape, 1) bytes or more the
 *                     faster stored-dS path runs (on token-major query rows,
 *                     read through a head-strided tensor-map view of Q and dO;
 *                     if the driver declines that view, the recomputing path
 *                     runs instead).  The two paths round dS the same way but
 *                     compute it in different kernels, so their results may
 *                     differ in the last bits.
 * Deterministic: no floating-point atomics; repeated calls with the same
 * ws_bytes give identical bits.
 */
moda_status moda_bwd(const moda_shape* shape,
                     const void* Q, const void* K, const void* V,
                     const void* Kd, const void* Vd,
                     const void* O, const float* LSE, const void* dO,
                     void* dQ, void* dK, void* dV, void* dKd, void* dVd,
                     void* ws, size_t ws_bytes, moda_stream_t stream);

/*
 * moda_bwd_noalloc: moda_bwd without a workspace argument.  The pages have no
 * counterpart; it exists for callers that cannot allocate device memory where
 * they run the backward -- for example a plugin whose host framework owns all
 * device memory and forbids allocation while it executes, or code replaying a
 * fixed memory plan -- and so cannot hand moda_bwd its workspace.
 *
 * Same arguments, layouts, results and errors as moda_bwd, minus ws/ws_bytes;
 * it allocates nothing and calls no allocating routine.  Its scratch (one fp32
 * per query row) is a fixed 16 MiB array inside the library, so it accepts at
 * most B*Hq*T = 4,194,304 query rows; larger problems get MODA_ERR_WORKSPACE.
 * Every device that loads the library holds that array until the process
 * exits.  Phase markers (moda_set_phase_events) apply as for moda_bwd.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  All calls share the one array, and each call
 * writes every row it reads before reading it, so nothing needs clearing
 * between calls -- but calls that overlap on the GPU (concurrent streams,
 * threads) race on it: serialise them.
 */
moda_status moda_bwd_noalloc(const moda_shape* shape,
                             const void* Q, const void* K, const void* V,
                             const void* Kd, const void* Vd,
                             const void* O, const float* LSE, const void* dO,
                             void* dQ, void* dK, void* dV, void* dKd, void* dVd,
                             moda_stream_t stream);

/*
 * Optional timing markers (observability; the pages have no counterpart).
 * After this call, every moda_fwd and moda_bwd call made by the calling
 * thread records events[0] on its stream before its first kernel launch and
 * events[k] right after its k-th launch: moda_fwd has one launch; moda_bwd
 * has three (row dots D = rowsum(dO*O), the dK/dV kernel, the dQ + depth-
 * gradient kernel), so it uses events[0..3].  Markers beyond n are skipped.
 *   events   array of n cudaEvent_t handles, created and owned by the caller
 *   n        0..8; 0 turns the markers off
 * Nothing is allocated; the library keeps only the handles (thread-local).
 */
moda_status moda_set_phase_events(void* const* events, int n);

/*
 * Synchronises `stream`, then reads and clears the current device's kernel
 * status word.  MODA_ERR_TIMEOUT if a kernel's bounded wait ran out since the
 * last check, MODA_ERR_CUDA if the stream reports an error, else MODA_OK.
 */
moda_status moda_check_status(moda_stream_t stream);

/*
 * Decoding: one new token per sequence attends to T cached keys and to its
 * own L depth rows under one softmax (paper summary of arXiv 2603.15619,
 * "Mixture-of-Depths Attention (MoDA): The Unified Operator", the newest query
 * position; "Complexity Analysis", Table 1: decoding costs O(L*T*D + L^2*D)
 * per token across the layers).
 *   shape     B, Hq, Hk, d, dtype, softmax_scale, depth_window as for
 *             moda_fwd; T = cached keys including the new token's own
 *             (T >= 1 when B > 0); L = depth rows of the new token; C, the
 *             depth layout and MODA_FLAG_NONCAUSAL have no effect.
 *             Supported: d in {64, 128}, G = Hq / Hk <= 16, bf16 or fp32.
 *   q         [B, Hq, d]     the new token's queries       (device)
 *   K, V      [B, Hk, T, d]  the cached keys and values    (device)
 *   Kd, Vd    [B, Hk, L, d]  the new token's depth rows    (device; NULL if L == 0)
 *   o         [B, Hq, d]     output, same dtype            (device)
 *   lse       [B, Hq]        fp32 natural-log LSE          (device)
 *   ws        moda_decode_workspace_size(shape) bytes      (device, caller-owned)
 * All buffers are contiguous and 16-byte aligned; nothing is allocated.  The
 * workspace holds fp32 partial results whose count follows the key split,
 * which depends on the current device's SM count: query the size with the
 * device that runs the call current (148 SMs are assumed without a device).
 * Returns MODA_ERR_INVALID_ARG / MODA_ERR_UNSUPPORTED for shapes outside the
 * above, MODA_ERR_MISALIGNED, MODA_ERR_WORKSPACE if ws_bytes is too small.
 */
size_t moda_decode_workspace_size(const moda_shape* shape);
moda_status moda_decode(const moda_shape* shape, const void* q, const void* K, const void* V,
                        const void* Kd, const void* Vd, void* o, float* lse,
                        void* ws, size_t ws_bytes, moda_stream_t stream);

/*
 * Failure-path self-test (the pages have no counterpart).  Queues on `stream`
 * one small kernel whose warps wait, through the same bounded mbarrier wait
 * the forward and backward kernels use, on a barrier that nothing arrives on.
 * The wait gives up after its time limit (2 s), the kernel records the
 * timeout in the device status word and returns normally; the next
 * moda_check_status(stream) then returns MODA_ERR_TIMEOUT (and clears the
 * word), and the device stays usable.  No memory is allocated or faulted.
 * Returns MODA_ERR_CUDA if the launch fails, else MODA_OK.
 */
moda_status moda_selftest_wait_timeout(moda_stream_t stream);

/* Static, human-readable name of a status code. */
const char* moda_status_string(moda_status status);

/* Detail of the calling thread's most recent failed call ("" if none). */
const char* moda_last_error_message(void);

/* Library version, major*10000 + minor*100 + patch. */
int moda_version(void);   /* 10200: adds MODA_DEPTH_LAYER (10100: flags and depth_window in moda_shape) */

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MODA_H_ */
