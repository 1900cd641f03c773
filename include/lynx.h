/*
 * lynx.h -- C ABI of the B200 (sm_100a) RT-Lynx online 2:4 activation-sparse
 * linear layer.
 *
 * The layer (RT-Lynx pages; "qingkeai.online article" = the RT-Lynx article on
 * qingkeai.online, "ai-feeds summary" = the ai-feeds.com summary of the paper):
 *
 *     Y = S(X) W^T + bias + (X A^T) B^T
 *
 *   - S(X): per token row, each group of 4 consecutive K-values keeps its 2
 *     largest magnitudes, ties to the lower position (qingkeai.online article
 *     section 02: Y = S(X) W^T with a 2:4 pattern made at run time; section 03:
 *     Top-K).  The kept values are multiplied by the norm-compensation factor
 *     s = sum|x| / sum|kept| of the row, computed in fp32 (section 03.1; ai-feeds
 *     summary, core module 1), and rounded to bf16.
 *   - (X A^T) B^T: LoRA residual of rank r on the dense X, frozen W (section
 *     03.2; the neuraltrendhub summary gives rank 64, the pages' setting).  Any
 *     r with r % 16 == 0 and 16 <= r <= 256 is accepted.
 *   - skip_sparsify: the layer stays dense, S(X) = X (section 03.3, selective
 *     layer skipping).
 *   - The sparse product runs on sparse tensor cores (tcgen05.mma.sp) with the
 *     compression, metadata layout, sparse GEMM and LoRA residual in CUDA
 *     kernels of this library (section 04).
 *
 * Conventions for every entry point:
 *   - Tensors are bf16 (bfloat16: the upper 16 bits of an IEEE fp32), row-major, contiguous,
 *     given as plain device pointers.  The caller owns and allocates every
 *     buffer; the library never allocates device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls only enqueue work and return; nothing synchronises except
 *     lynx_check_error.
 *   - Return value: a lynx_status.  Host-side checks run before anything is
 *     enqueued: on failure nothing is launched and no buffer is touched.
 *     Device-side failures (a bounded wait that gave up) are recorded in a
 *     status word of the stream the call was enqueued on, which
 *     lynx_check_error(stream) reports; a CUDA graph captured from a stream
 *     keeps recording into that stream's word when it is replayed.
 *   - Inputs must be finite; NaN/Inf inputs give unspecified (but memory-safe)
 *     results.
 *   - Shapes: M >= 1 tokens, K >= 64 with K % 64 == 0, N >= 8 with N % 8 == 0,
 *     and, when a LoRA branch is given, 16 <= r <= 256 with r % 16 == 0.
 *     Every pointer 16-byte aligned.
 *   - Thread safety: calls from several host threads on different streams are
 *     safe.  Calls whose device work overlaps must not share output buffers or
 *     a workspace.
 */
#ifndef LYNX_H_
#define LYNX_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LYNX_API __attribute__((visibility("default")))
#else
#define LYNX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lynx_status {
  LYNX_OK = 0,
  LYNX_ERR_INVALID_ARG = 1,         /* null pointer, A without B, bad flag */
  LYNX_ERR_UNSUPPORTED_SHAPE = 2,   /* M < 1, K % 64, N % 8, r % 16, r > 256, ... */
  LYNX_ERR_MISALIGNED = 3,          /* a pointer not 16-byte aligned */
  LYNX_ERR_WORKSPACE_TOO_SMALL = 4, /* workspace_bytes < lynx_workspace_bytes() */
  LYNX_ERR_CUDA = 5,                /* a CUDA runtime/driver call failed */
  LYNX_ERR_DEVICE_TIMEOUT = 6       /* a kernel gave up a bounded wait */
} lynx_status;

/* Human-readable name of a status code (static storage, never NULL). */
LYNX_API const char* lynx_status_string(int status);

/* ABI version: (major << 16) | minor. */
LYNX_API int lynx_version(void);

/* The LoRA rank the RT-Lynx pages use (64); the bindings' default. */
LYNX_API int lynx_lora_rank(void);

/* 1 if the kernels accept LoRA rank r (r % 16 == 0 and 16 <= r <= 256), else 0.
 * r is the N of the down-projection MMA (M = 128 rows, N a multiple of 16 up to
 * 256) and the K of the up-projection, which runs in steps of 32 (the last one
 * half empty when r % 32 == 16). */
LYNX_API int lynx_lora_rank_supported(int64_t r);

/* ---- sizes ------------------------------------------------------------- */

/* Bytes of the compressed values S(X): M x K/2 bf16 = M*K bytes. */
LYNX_API size_t lynx_vals_bytes(int64_t M, int64_t K);

/* Bytes of the 2:4 metadata in the tcgen05.mma.sp operand layout: one
 * 2048-byte block per 128 rows x 128 dense K; rows are padded to a multiple of
 * 256 (128-row blocks come in pairs, one per CTA of a CTA pair) and K to a
 * multiple of 128: ceil(M/256) * 2 * ceil(K/128) * 2048.
 * Layout: block (mb, kb) at byte (mb * ceil(K/128) + kb) * 2048; inside a
 * block, row m and dense column k (both relative to the block) map to TMEM
 * lane L = (m % 8) + 8 * ((k / 16) % 2) + 16 * (m / 16), 32-bit word
 * w = k / 32 of the lane's 16 bytes, bit b = (k % 16) + 16 * ((m / 8) % 2);
 * each group of 4 owns 4 bits: lo | hi << 2 (lo < hi its kept positions).
 * Padding rows hold the pattern of an all-zero row (lo = 0, hi = 1). */
LYNX_API size_t lynx_meta_bytes(int64_t M, int64_t K);

/* Bytes of the workspace lynx_linear needs (kept values, metadata, row scales,
 * the bf16 LoRA down-projection [M,r], per-range partial sums, one state word
 * per 32-row slice, alignment).  r = 0 (no LoRA) sizes it as for r = 64. */
LYNX_API size_t lynx_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r);

/* ---- the layer --------------------------------------------------------- */

/* Bytes of the scratch workspace lynx_sparsify needs (per-range partial row
 * sums and, when no row_scale buffer is given, s). */
LYNX_API size_t lynx_sparsify_workspace_bytes(int64_t M, int64_t K);

/* S(X) alone (qingkeai.online article sections 02-03.1; ai-feeds summary,
 * core module 1).
 *   X         [M,K] bf16, input activations (read only)
 *   vals      [M,K/2] bf16, out: kept values after compensation, two per group,
 *             ascending position (lynx_vals_bytes)
 *   meta      out: metadata blocks, lynx_meta_bytes(M,K) bytes (layout above);
 *             padding rows hold the pattern of an all-zero row
 *   row_scale [M] fp32, out: s per row, or NULL
 *   workspace caller-allocated scratch of workspace_bytes >=
 *             lynx_sparsify_workspace_bytes(M,K) */
LYNX_API int lynx_sparsify(const void* X, int64_t M, int64_t K, void* vals, void* meta,
                           float* row_scale, void* workspace, size_t workspace_bytes,
                           void* stream);

/* ---- S(X) without a caller workspace ---------------------------------- */

/* Largest M lynx_sparsify_noalloc accepts. */
#define LYNX_SPARSIFY_NOALLOC_MAX_ROWS 16384

/* lynx_sparsify with its scratch (the per-range partial row sums and, when
 * row_scale is NULL, s) in a fixed device array of the library instead of a
 * caller workspace: LYNX_SPARSIFY_NOALLOC_MAX_ROWS * (8 * 8 + 4) bytes
 * (1.06 MiB) per device.  The RT-Lynx pages have no counterpart of this entry
 * point; it exists for callers that cannot hand out a workspace: code behind a
 * fixed operator signature that receives only its inputs and outputs, and
 * latency-critical loops that must not call cudaMalloc (which can synchronise
 * the whole device) nor go through another runtime's allocator.
 *   Arguments, output layout, results and errors are those of lynx_sparsify.
 *   M > LYNX_SPARSIFY_NOALLOC_MAX_ROWS returns LYNX_ERR_WORKSPACE_TOO_SMALL
 *   before anything is launched.
 *   The call allocates no memory.  The first call on a device looks up the
 *   scratch's device address (cudaGetSymbolAddress) and the device's SM count;
 *   make that first call before any stream capture.
 *   Nothing in the scratch has to start at zero: every call writes all the
 *   partials it reads.
 *   All calls on one device share the one scratch array: two calls whose device
 *   work overlaps (different streams, or different host threads, without an
 *   ordering between them) race on it and give wrong results.  Calls in order
 *   on one stream are safe. */
LYNX_API int lynx_sparsify_noalloc(const void* X, int64_t M, int64_t K, void* vals, void* meta,
                                   float* row_scale, void* stream);

/* LYNX_SPARSIFY_NOALLOC_MAX_ROWS, for callers without the header. */
LYNX_API int64_t lynx_sparsify_noalloc_max_rows(void);

/* Y = S(X) W^T + bias + (X A^T) B^T  (S(X) = X when skip_sparsify != 0).
 *   X [M,K], W [N,K] (frozen backbone weight), bias [N] or NULL,
 *   A [r,K] and B [N,r] (LoRA, both or neither; r % 16 == 0, 16 <= r <= 256),
 *   Y [M,N] out.
 *   workspace: caller-allocated device buffer of workspace_bytes >=
 *   lynx_workspace_bytes(M,N,K,r), used as scratch; at 256-byte aligned
 *   offsets, in this order, it ends up holding the kept values before
 *   compensation [M,K/2] bf16, the metadata, s per row [M] fp32 and T/s [M,r]
 *   bf16 (T = X A^T).  The workspace needs no initial contents: every call
 *   writes what it reads, the GEMM's per-row-block state words included (the
 *   call's first kernel sets them to 0), so calls and replays of a captured
 *   CUDA graph that reuse one workspace in stream order are independent.
 *   The compensation factor s is applied to the fp32 accumulator row, so
 *   Y = bf16(s * (S0 W^T + (T/s) B^T) + bias) with S0 the uncompensated kept
 *   values: the same product as S(X) W^T + T B^T with one rounding fewer. */
LYNX_API int lynx_linear(const void* X, const void* W, const void* bias, const void* A, const void* B,
                int64_t M, int64_t N, int64_t K, int64_t r, int skip_sparsify, void* Y,
                void* workspace, size_t workspace_bytes, void* stream);

/* ---- the layer in two halves ------------------------------------------ */

/* lynx_linear_act split at its one internal hand-off, so that a caller can put
 * the halves on different streams (for example the next layer's pass beside
 * this layer's GEMM, each with its own workspace):
 *   lynx_linear_begin   the sparsify pass (S(X) kept values, metadata, the row
 *                       sums and T partials) into the workspace; on the dense
 *                       path (skip_sparsify) the LoRA-down pass, or nothing;
 *   lynx_linear_finish  the GEMM from that workspace into Y.
 * Both take lynx_linear_act's arguments and check them the same way.  finish
 * must run after begin has completed on the same workspace (the same stream in
 * order, or another stream that waits on an event recorded after begin), with
 * nothing else writing that workspace in between; then the pair computes
 * exactly what lynx_linear_act does (the same Y, bit for bit).  begin reads X
 * and A; finish reads X (dense path only), W, bias, B and the workspace. */
LYNX_API int lynx_linear_begin(const void* X, const void* W, const void* bias, const void* A,
                               const void* B, int64_t M, int64_t N, int64_t K, int64_t r,
                               int skip_sparsify, int act, void* Y, void* workspace,
                               size_t workspace_bytes, void* stream);
LYNX_API int lynx_linear_finish(const void* X, const void* W, const void* bias, const void* A,
                                const void* B, int64_t M, int64_t N, int64_t K, int64_t r,
                                int skip_sparsify, int act, void* Y, void* workspace,
                                size_t workspace_bytes, void* stream);

/* ---- an activation applied in the GEMM epilogue ------------------------ */

/* Activations lynx_linear_act applies to the finished output row. */
#define LYNX_ACT_NONE 0
/* GELU, tanh form (Hendrycks & Gimpel, "Gaussian Error Linear Units"):
 * gelu(v) = v/2 (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), the activation
 * between a DiT block's MLP up- and down-projections; the down-projection
 * (MLP.Down, the layer the qingkeai.online article takes as its example in
 * section 02) reads its output as the activation it sparsifies.  Not on the
 * RT-Lynx pages themselves, which fuse the sparsification steps so that no
 * intermediate goes back to memory (same article, section 04); this carries
 * that to the activation pass before the sparsified layer. */
#define LYNX_ACT_GELU_TANH 1

/* Y = act(S(X) W^T + bias + (X A^T) B^T): lynx_linear with the activation
 * applied in fp32 to each finished output value before its one bf16 rounding,
 * inside the GEMM's epilogue.  Saves the separate activation pass over Y (one
 * read and one write of M*N*2 bytes) that the layer feeding a sparsified
 * MLP down-projection otherwise needs.
 *   act: LYNX_ACT_NONE (then the call is lynx_linear) or LYNX_ACT_GELU_TANH;
 *   any other value returns LYNX_ERR_INVALID_ARG before anything is launched.
 *   Every other argument, the workspace and the errors are those of
 *   lynx_linear.  GELU is evaluated as v * sigmoid(2u), u = sqrt(2/pi)
 *   (v + 0.044715 v^3) (the same function: (1 + tanh u)/2 = sigmoid(2u)), with
 *   the hardware base-2 exponential and reciprocal approximations (a few fp32
 *   ulps; values whose magnitude falls below the fp32 normal range may come
 *   out as zero). */
LYNX_API int lynx_linear_act(const void* X, const void* W, const void* bias, const void* A,
                             const void* B, int64_t M, int64_t N, int64_t K, int64_t r,
                             int skip_sparsify, int act, void* Y, void* workspace,
                             size_t workspace_bytes, void* stream);

/* ---- the fully fused variant ------------------------------------------- */

/* Y = act(S(X) W^T + bias + (X A^T) B^T) like lynx_linear_act, with the 2:4
 * selection and compression inside the GEMM (qingkeai.online article, section
 * 04: selection, compression, the sparse operand layout, the sparse GEMM and the
 * LoRA residual fused, no compressed activations written back).  A slim first
 * pass reads X for the two row sums (s) and T = X A^T only; the GEMM then loads
 * the dense X tiles itself, selects and compresses them in shared memory into
 * the tcgen05.mma.sp operand (values and metadata) and multiplies.  The
 * selection is redone for every output tile of 256 columns, so on B200 this
 * variant is slower than lynx_linear whenever N is much more than 256 (the
 * selection work grows with N / 256); lynx_linear is the default path.
 * Results equal lynx_linear's within the same tolerance (the same s, the same
 * kept values).  Arguments, workspace and errors as lynx_linear_act without
 * skip_sparsify; shapes the CTA-pair GEMM does not take (M <= 128, N < 256,
 * K % 128 != 0) run lynx_linear_act. */
LYNX_API int lynx_linear_fused(const void* X, const void* W, const void* bias, const void* A,
                               const void* B, int64_t M, int64_t N, int64_t K, int64_t r, int act,
                               void* Y, void* workspace, size_t workspace_bytes, void* stream);

/* ---- the layer on host-memory activations ------------------------------ */

/* Bytes of the device workspace lynx_linear_host needs: device copies of X and
 * Y plus the layer workspace of one row chunk. */
LYNX_API size_t lynx_linear_host_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r);

/* lynx_linear with X [M,K] and Y [M,N] in host memory (page-locked for the copies
 * to run asynchronously); W, bias, A, B stay device pointers.  The rows are
 * processed in up to 8 chunks (multiples of 256 rows): the copy of chunk i+1 into
 * the device, the layer on chunk i and the copy of chunk i-1 back to the host run
 * at the same time, the two copy directions on internal streams of the library.
 * The work is ordered after everything already enqueued on `stream`, and
 * anything enqueued on `stream` afterwards (a synchronize included) sees Y
 * complete in host memory.  Results equal lynx_linear's, row for row.
 *   workspace: device buffer of workspace_bytes >= lynx_linear_host_workspace_bytes.
 *   Errors as lynx_linear.  The first call on a device creates its two streams
 *   and its events.  Enqueues from several host threads are serialised inside
 *   the call; each call needs its own workspace and Y. */
LYNX_API int lynx_linear_host(const void* X_host, const void* W, const void* bias, const void* A,
                              const void* B, int64_t M, int64_t N, int64_t K, int64_t r,
                              int skip_sparsify, void* Y_host, void* workspace,
                              size_t workspace_bytes, void* stream);

/* lynx_linear_host with an activation in the GEMM epilogue (lynx_linear_act's
 * act argument); same workspace and errors. */
LYNX_API int lynx_linear_host_act(const void* X_host, const void* W, const void* bias, const void* A,
                                  const void* B, int64_t M, int64_t N, int64_t K, int64_t r,
                                  int skip_sparsify, int act, void* Y_host, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* The dense path of a layer that selective layer skipping leaves dense
 * (qingkeai.online article section 03.3): Y = X W^T + bias + (X A^T) B^T.
 * Same arguments and workspace as lynx_linear. */
LYNX_API int lynx_linear_dense(const void* X, const void* W, const void* bias, const void* A,
                      const void* B, int64_t M, int64_t N, int64_t K, int64_t r, void* Y,
                      void* workspace, size_t workspace_bytes, void* stream);

/* The sparse product on an S(X) made earlier by lynx_sparsify (or the
 * workspace of lynx_linear):  Y = S(X) W^T + bias + T B^T.
 *   vals [M,K/2] and meta as written by lynx_sparsify; T [M,r] bf16 or NULL,
 *   B [N,r] or NULL (both or neither, r as for lynx_linear); other arguments as
 *   above. */
LYNX_API int lynx_sparse_gemm(const void* vals, const void* meta, const void* T, const void* W,
                     const void* bias, const void* B, int64_t M, int64_t N, int64_t K, int64_t r,
                     void* Y, void* stream);

/* ---- errors and metadata conversion ----------------------------------- */

/* Synchronises `stream`, then reports (and clears) the status word of that
 * stream on the current device: LYNX_ERR_DEVICE_TIMEOUT if a kernel launched on
 * it gave up a bounded wait since the last check, LYNX_ERR_CUDA if the stream
 * holds a CUDA error, else LYNX_OK.  Errors of calls on other streams stay in
 * their own words.  (A process uses at most 1023 words per device; the streams
 * after those share one more word, which any of them reports and clears.)
 * *device_code (may be NULL) receives the raw device code (0 if none). */
LYNX_API int lynx_check_error(void* stream, uint32_t* device_code);

/* Host-side conversions between the hardware metadata layout (above) and the
 * canonical one: row m owns K/8 bytes, group g is the nibble lo | hi << 2 in
 * byte m*K/8 + g/2, low nibble for even g.  Host pointers; K % 8 == 0.
 * canonical_to_hw fills padding rows with the all-zero-row pattern (lo=0,hi=1)
 * and padding K with zero bits. */
LYNX_API int lynx_meta_hw_to_canonical(const uint8_t* hw, uint8_t* canonical, int64_t M, int64_t K);
LYNX_API int lynx_meta_canonical_to_hw(const uint8_t* canonical, uint8_t* hw, int64_t M, int64_t K);

/* Profiling hook: when `event` (a cudaEvent_t passed as void*) is non-NULL,
 * lynx_linear records it on its stream between the sparsify pass and the GEMM,
 * so a caller can time the two kernels of one call separately with events
 * recorded before and after the call.  NULL (the default) turns it off.
 * While it is set, the GEMM no longer starts (programmatic launch) during the
 * tail of the sparsify pass, so a call takes slightly longer.
 * Process-wide; returns the previous event. */
LYNX_API void* lynx_profile_set_split_event(void* event);

/* Profiling hook: part 1 makes lynx_linear (and lynx_linear_act) enqueue only
 * its first kernel, the sparsify (or, on the dense path, LoRA-down) pass; part
 * 2 only what follows it (the GEMM, after a reset of its per-row-block state
 * words, and the split event, if set, between the two), on a workspace that
 * an earlier full call filled.  0 (the default) runs the whole layer.
 * Process-wide; returns the previous part (-1 for an invalid argument). */
LYNX_API int lynx_profile_set_part(int part);

/* Test hook (not for production use): when nonzero, kernels launched after
 * this call never load their inputs, so their bounded waits run out (about 2 s)
 * and lynx_check_error reports LYNX_ERR_DEVICE_TIMEOUT.  Returns the old value. */
LYNX_API int lynx_debug_set_stall(int enable);

#ifdef __cplusplus
}
#endif

#endif /* LYNX_H_ */
