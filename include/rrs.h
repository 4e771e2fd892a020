/*
 * rrs.h -- C ABI of the Rotated Runtime Smooth (RRS) W4A4 linear layer for
 * NVIDIA B200 (sm_100a).
 *
 * The method (web pages on "Rotated Runtime Smooth: Training-Free Activation
 * Smoother for accurate INT4 inference"):
 *   - activations X [M, K] are rotated online by a normalised Hadamard
 *     transform, the weights W [N, K] offline by the same transform
 *     (summary page, "Approach");
 *   - the channels of both are permuted by one fixed reorder index, which
 *     leaves Y = X W^T = sum_i X_i W_i^T unchanged (rebuttal page,
 *     "Description of the reorder process");
 *   - each group g of G consecutive reordered channels is divided by its
 *     runtime scale s_g = max |X'| over all tokens and channels of the group,
 *     computed at inference and never folded into the weights (summary page,
 *     "Approach"; rebuttal page, "Novelty": group-wise scales aligned with the
 *     hardware GEMM);
 *   - the smoothed activations are quantised per token to symmetric INT4
 *     (scale_t = amax_t / 7), the weights per output channel (scale_w =
 *     amax_n / 7, round-to-nearest), and
 *       Y[t][n] = (sum_g s_g * P_g[t][n]) * scale_t[t] * scale_w[n],
 *       P_g[t][n] = sum_{k in group g} qX[t][k] * qW[n][k]   (exact int32).
 *
 * Arithmetic contract (readings where the pages are silent):
 *   - Hadamard: fp32, radix-2 stages h = 1, 2, 4, ..., pair (j, j+h) ->
 *     (a + b, a - b); then one multiply by c_n = (float)(1/sqrt(n)).  n is the
 *     Hadamard block size; K = B * n gives a block-diagonal rotation; n = 1
 *     (or RRS_NO_ROTATE) means no rotation (plain Runtime Smooth).
 *   - reorder after rotation: X'[t][j] = X_rot[t][perm[j]].
 *   - smoothing is an IEEE fp32 division by s_g (s_g == 0 divides by 1).
 *   - codes q = clamp(rint(x / scale), -8, 7), round half to even; a scale of 0
 *     gives all-zero codes.
 *   - packing: byte i of a row = (q[2i] & 0xF) | (q[2i+1] & 0xF) << 4.
 *   - the integer stages (codes, s, scale_t, scale_w, P_g) are bit-exact
 *     functions of the inputs; Y is fp32 with the group sum accumulated in
 *     fp32 in group order.
 *
 * Layouts (all row-major, all device pointers unless stated otherwise):
 *   X        fp16  [M, K]            W      fp16 [N, K]
 *   perm     int32 [K]  (a permutation of 0..K-1)
 *   qX       uint8 [M, K/2]          qW     uint8 [N, K/2]
 *   s        fp32  [K/G]             scale_t fp32 [M]     scale_w fp32 [N]
 *   Y        fp32  [M, N]            P      int32 [K/G, M, N] (debug only)
 *
 * Ownership: the caller owns every buffer, including the workspace.  The
 * library allocates no device or host memory and never synchronises the host
 * except in rrs_check_workspace, rrs_check_perm and rrs_linear_from_host
 * (documented there).
 * Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 * and outputs are valid when the stream reaches that point.  Calls that share
 * output buffers or a workspace must be ordered on one stream.
 *
 * Errors: every entry point returns an rrs_status; rrs_last_error_string()
 * gives a thread-local description of the last failure.  Argument checks
 * happen on the host before anything is enqueued.  Kernels bound every wait
 * (about one second); a kernel that gives up sets an error word in the
 * workspace and returns, which rrs_check_workspace reports as
 * RRS_ERR_TIMEOUT.
 *
 * Limits of the CUDA path: K % 128 == 0, K <= 32768; G % 128 == 0 and
 * K % G == 0 (RRS_ERR_UNSUPPORTED otherwise); n a power of two <= 8192 with
 * K % n == 0; M, N >= 1; pointers to fp16/uint8/fp32 arrays 16-byte aligned.
 */
#ifndef RRS_H
#define RRS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the same type, spelled without CUDA headers). */
typedef struct CUstream_st *rrs_stream_t;

typedef enum {
    RRS_OK = 0,
    RRS_ERR_INVALID_ARG = 1, /* a null/misaligned pointer or an inconsistent size */
    RRS_ERR_UNSUPPORTED = 2, /* valid for the method, outside this path's limits */
    RRS_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
    RRS_ERR_TIMEOUT = 4,     /* a kernel gave up on a bounded wait */
    RRS_ERR_WORKSPACE = 5    /* workspace null or smaller than rrs_workspace_size */
} rrs_status;

/* flags */
#define RRS_NO_ROTATE 1u         /* identity instead of the Hadamard (plain Runtime Smooth) */
#define RRS_FORCE_UNIT_SCALES 2u /* s := 1 for every group (A4W4 per-channel scheme, no smoothing) */
#define RRS_WS_HOLDS_A8 4u       /* rrs_w4a4_gemm: the workspace already holds the activation operand
                                    that rrs_smooth_quant (or rrs_smooth_quant_scaled) wrote for this
                                    qX with the same RRS_W_EXPANDED bit (same ws, same stream,
                                    nothing in between); skips expanding qX again */
#define RRS_W_EXPANDED 8u        /* qW points at the weight codes one per byte in e4m3 form that
                                    rrs_expand_weights wrote ([N, K] bytes) instead of the packed
                                    INT4 codes, and the GEMM runs on the fp8 tensor-core path
                                    (rrs_w4a4_gemm, rrs_linear, rrs_linear_from_host, the debug
                                    partials).  Passed to rrs_smooth_quant / rrs_smooth_quant_scaled
                                    it makes them leave the e4m3 activation operand in the
                                    workspace (otherwise the int8 one of the packed path). */
#define RRS_Y_BF16 16u           /* rrs_w4a4_gemm, rrs_linear, rrs_linear_from_host: Y (and Y_host)
                                    hold bf16 [M, N] -- the fp32 result rounded to nearest even --
                                    instead of fp32; pass the buffer cast to float *.  The pages fix
                                    no output type; bf16 is the usual deployment type of Y. */
#define RRS_Y_SILU_MUL 32u       /* rrs_w4a4_gemm, rrs_linear, rrs_linear_from_host, fp8 path only
                                    (with RRS_W_EXPANDED): the layer is the fused gate/up projection
                                    of a gated MLP block with its weight rows interleaved (row 2f
                                    the gate row of feature f, row 2f+1 its up row; N even), and
                                    instead of Y the GEMM writes the down projection's input
                                    H fp16 [M, N/2], H[t][f] = fp16(silu(Y[t][2f]) * Y[t][2f+1])
                                    from the fp32 Y it would have stored, with rrs_silu_mul's
                                    arithmetic (same bits).  Pass H cast to float *.  Saves
                                    writing and reading the fp32 gate/up output. */
#define RRS_ONE_LAUNCH 64u       /* rrs_linear, rrs_linear_from_host: for M <= 16 with packed
                                    weights, always take the single-launch layer where the
                                    shape allows it.  Without it the single launch is taken
                                    only where it is the faster of the two forms: M <= 6, or
                                    N * K >= 2^27 (the weight stream then outweighs the
                                    fixed cost of the in-kernel activation phases). */

/* Bytes of workspace the calls below need for this problem.  Layout: a
 * 256-byte header (zero-fill it once before first use: it holds the kernels'
 * error word and the state of the activation kernel's grid-wide barrier, which
 * every completed call leaves zeroed again), then the activation codes that the
 * GEMM's tensor cores read (M*K bytes: int8, or e4m3 under RRS_W_EXPANDED),
 * then, when K is a multiple of 2048, a table of group maxima with one row of
 * K/128 floats per CTA of the activation kernel (at most 1024 rows).  For
 * M <= 16 and N > 0 the space after the operand is at least 16*M*N*4 bytes: the
 * packed-weight GEMM then splits k across CTAs and keeps its partial sums there
 * (the table is dead by then); and the space after the header also holds the
 * single-launch layer of rrs_linear (rotated rows M*K*4 bytes, a table of group
 * maxima of M*(K/1024)*(K/128) floats, and K/1024 chunk sums of M*N*4 bytes each,
 * every part 256-byte aligned).  rrs_w4a4_gemm alone needs only the first two
 * parts; given less room it simply does not split.  N = 0 sizes a workspace for
 * the activation calls alone.  One workspace must not be used by two calls in
 * flight at the same time.  A call that times out (RRS_ERR_TIMEOUT) may leave
 * the barrier state dirty: zero-fill the header before using the workspace
 * again. */
size_t rrs_workspace_size(int M, int N, int K, int G, int had_block, unsigned flags);

/* Offline weight path (summary page "Approach"; rebuttal page "Description of
 * the reorder process"): W' = reorder(rotate_n(W)), scale_w[r] = max_k |W'[r][k]| / 7,
 * qW = pack(clamp(rint(W' / scale_w), -8, 7)).  W fp16 [N, K] -> qW uint8
 * [N, K/2], scale_w fp32 [N].  Same n and perm as the activations. */
rrs_status rrs_prepare_weights(const void *W, int N, int K, int had_block, const int32_t *perm,
                               uint8_t *qW, float *scale_w, unsigned flags, rrs_stream_t stream);

/* Online activation path (summary page "Approach": rotate, reorder, divide
 * each group by its runtime max; per-token INT4 quantiser scale = amax / 7):
 * X fp16 [M, K] -> qX uint8 [M, K/2], s fp32 [K/G], scale_t fp32 [M].
 * s is computed from all M tokens (two passes over X).  Under
 * RRS_FORCE_UNIT_SCALES, s is written as 1. */
rrs_status rrs_smooth_quant(const void *X, int M, int K, int G, int had_block, const int32_t *perm,
                            uint8_t *qX, float *s, float *scale_t, void *ws, size_t ws_bytes,
                            unsigned flags, rrs_stream_t stream);

/* The two passes of rrs_smooth_quant as separate calls, for one batch whose
 * tokens are split across devices (or calls).  The runtime scale of a group is
 * the maximum over ALL tokens of the batch (summary page, "Approach": the
 * smoothing scales are computed at inference from the activations), and a
 * maximum of maxima is exact, so
 *     rrs_group_max on every shard -> elementwise MAX of the shards' s (for
 *     example an all-reduce with the MAX operation) -> rrs_smooth_quant_scaled
 *     on every shard with that s
 * gives, row for row, the same qX and scale_t bits (and the same s) as one
 * rrs_smooth_quant over the whole batch.
 *
 * rrs_group_max (pass A): s[g] = max over this call's M tokens and the channels
 * of group g of |X'|, fp32 [K/G] (0 for a group that is zero on every token).
 * Under RRS_FORCE_UNIT_SCALES it writes s = 1.  Same arguments, limits,
 * workspace (rrs_workspace_size(M, 0, K, G, had_block, flags) bytes) and errors
 * as rrs_smooth_quant. */
rrs_status rrs_group_max(const void *X, int M, int K, int G, int had_block, const int32_t *perm, float *s,
                         void *ws, size_t ws_bytes, unsigned flags, rrs_stream_t stream);

/* rrs_smooth_quant_scaled (pass B): qX and scale_t of this call's M tokens,
 * each group divided by the given s[g] (a zero s[g] divides by 1), exactly as
 * rrs_smooth_quant's second pass does.  s is an input, fp32 [K/G] device.
 * RRS_FORCE_UNIT_SCALES is refused (RRS_ERR_INVALID_ARG): pass s filled with 1.
 * With RRS_W_EXPANDED it also leaves the fp8 GEMM operand in the workspace,
 * like rrs_smooth_quant.  Otherwise as rrs_smooth_quant. */
rrs_status rrs_smooth_quant_scaled(const void *X, int M, int K, int G, int had_block, const int32_t *perm,
                                   const float *s, uint8_t *qX, float *scale_t, void *ws, size_t ws_bytes,
                                   unsigned flags, rrs_stream_t stream);

/* Group-scaled W4A4 GEMM (rebuttal page "Novelty": the smoothing scale is
 * applied group-wise to match the hardware GEMM): exact int32 P_g per group
 * on the tensor cores, Y = (sum_g s_g * P_g) * scale_t * scale_w in fp32.
 * flags: 0, or RRS_WS_HOLDS_A8 (see above).  Without it the packed qX is
 * first expanded into the workspace's int8 operand. */
rrs_status rrs_w4a4_gemm(const uint8_t *qX, const float *s, const float *scale_t, const uint8_t *qW,
                         const float *scale_w, int M, int N, int K, int G, float *Y, void *ws,
                         size_t ws_bytes, unsigned flags, rrs_stream_t stream);

/* rrs_smooth_quant followed by rrs_w4a4_gemm on one stream, no host sync.
 * qX, s and scale_t are caller-provided intermediate buffers (written as by
 * rrs_smooth_quant).  For M <= 16 tokens with packed weights (no
 * RRS_W_EXPANDED, no RRS_Y_SILU_MUL), N % 16 == 0, K % 1024 == 0, G dividing
 * 1024 and a workspace of rrs_workspace_size(M, N, ...) bytes, the whole layer
 * can run as one cooperative kernel instead (where it is faster, or always
 * under RRS_ONE_LAUNCH): the same codes, s and scale_t bit for
 * bit, and Y differing only in the order of its fp32 sums over 1024-channel
 * chunks (summed in chunk order).  Other shapes, or a smaller workspace, take the
 * two launches. */
rrs_status rrs_linear(const void *X, const uint8_t *qW, const float *scale_w, const int32_t *perm,
                      int M, int N, int K, int G, int had_block, uint8_t *qX, float *s,
                      float *scale_t, float *Y, void *ws, size_t ws_bytes, unsigned flags,
                      rrs_stream_t stream);

/* End-to-end variant for callers holding HOST buffers: copies X_host (fp16
 * [M, K], ideally pinned) to X_dev, runs rrs_linear, copies Y back into
 * Y_host (fp32 [M, N]) with cudaMemcpyAsync on `stream`, then synchronises
 * that stream.  All device buffers are caller-provided. */
rrs_status rrs_linear_from_host(const void *X_host, void *X_dev, const uint8_t *qW,
                                const float *scale_w, const int32_t *perm, int M, int N, int K,
                                int G, int had_block, uint8_t *qX, float *s, float *scale_t,
                                float *Y_dev, float *Y_host, void *ws, size_t ws_bytes,
                                unsigned flags, rrs_stream_t stream);

/* Debug: the exact per-group partial sums P [K/G, M, N] (int32) of the same
 * GEMM, written instead of Y.  For small problems only. */
rrs_status rrs_w4a4_gemm_debug_partials(const uint8_t *qX, const uint8_t *qW, int M, int N, int K,
                                        int G, int32_t *P, void *ws, size_t ws_bytes, unsigned flags,
                                        rrs_stream_t stream);

/* Weight operand of the fp8 tensor-core GEMM, written once per layer after
 * rrs_prepare_weights: qW8[n][k] = the INT4 code q of qW[n][k] as an e4m3 byte
 * (natural k order; every code in [-8, 7] is an e4m3 number exactly, and so is
 * every product of two codes, which the fp32 accumulators of the MMA sum
 * without rounding).  The pages have no counterpart: the INT4 codes are
 * unchanged, only stored one per byte in a form the fp8 MMA reads, so that the
 * per-group promotion of the GEMM is one fused multiply-add on an fp32 partial
 * sum.  It doubles the weight bytes (N * K instead of N * K / 2); pass
 * RRS_W_EXPANDED to use it.  qW packed [N, K/2] as rrs_prepare_weights writes it;
 * qW8 [N, K] bytes, device, caller-owned, 16-byte aligned.  K as for
 * rrs_w4a4_gemm.  Asynchronous on `stream`.  Errors: RRS_ERR_INVALID_ARG for a
 * null or misaligned pointer or N < 1; RRS_ERR_UNSUPPORTED for K % 128 != 0;
 * RRS_ERR_CUDA if the launch fails. */
rrs_status rrs_expand_weights(const uint8_t *qW, int N, int K, uint8_t *qW8, rrs_stream_t stream);

/* Gated-MLP step between two RRS linears (summary page "Key results": the method is
 * applied to every linear layer of the model, so the down projection's input is the
 * gated activation): H[m][f] = silu(GU[m][f]) * GU[m][F + f], silu(g) = g / (1 +
 * exp(-g)) in fp32, rounded to fp16 and saturated to +-65504.  GU fp32 [M, 2F], the
 * output of the fused gate/up projection whose weight rows are [W_gate; W_up]; H fp16
 * [M, F], the down projection's X.  Both device, caller-owned, 16-byte aligned.  The
 * pages fix no activation function; SiLU is that of the LLaMA models they evaluate.
 * Asynchronous on `stream`.  Errors: RRS_ERR_INVALID_ARG for a null or misaligned
 * pointer or M, F < 1; RRS_ERR_CUDA if the launch fails. */
rrs_status rrs_silu_mul(const float *GU, int M, int F, void *H, rrs_stream_t stream);

/* KV cache of the 4-4-4 setting (summary page, "Key results": weights,
 * activations and the KV cache in 4 bits).  Reading: every head vector of K or
 * V (length D) is rotated by the normalised Hadamard transform of size D (the
 * same fp32 stage order and c_D as the activations) and quantised to
 * symmetric INT4 with its own scale, scale = max |x_rot| / 7, code =
 * clamp(rint(x_rot / scale), -8, 7), no reorder and no runtime smoothing (the
 * runtime group scales belong to the linear layer's GEMM).  A query rotated by
 * the same transform gives the same attention scores (the transform is
 * orthogonal).  KV fp16 [T, H, D] (token, head, channel), q uint8 [T, H, D/2]
 * (low nibble = even channel), scale fp32 [T, H]; device, caller-owned,
 * 16-byte aligned.  D a power of two, 128 <= D <= 8192 on the CUDA path
 * (RRS_ERR_UNSUPPORTED otherwise); flags must be 0.  Asynchronous on `stream`;
 * no workspace. */
rrs_status rrs_kv_quant(const void *KV, int T, int H, int D, uint8_t *q, float *scale, unsigned flags,
                        rrs_stream_t stream);

/* The cached vectors back, in the rotated space: out fp16 [T, H, D] =
 * fp16(code * scale) (the product in fp32, then rounded to nearest even).
 * D a positive multiple of 8.  Asynchronous on `stream`. */
rrs_status rrs_kv_dequant(const uint8_t *q, const float *scale, int T, int H, int D, void *out,
                          rrs_stream_t stream);

/* Calibration statistic for the reorder index: cmax[k] = max_t |X_rot[t][k]|
 * (rotation only, no reorder).  cmax fp32 [K]. */
rrs_status rrs_channel_absmax(const void *X, int M, int K, int had_block, float *cmax,
                              unsigned flags, rrs_stream_t stream);

/* Host helper: perm = channels sorted by descending cmax_host, ties by lower
 * channel index.  Both arrays are HOST memory of length K. */
rrs_status rrs_perm_from_channel_max(const float *cmax_host, int K, int32_t *perm_host);

/* Synchronises `stream`, reads and clears the workspace error word.
 * Returns RRS_ERR_TIMEOUT if a kernel gave up on a bounded wait since the
 * last check, RRS_OK otherwise. */
rrs_status rrs_check_workspace(void *ws, rrs_stream_t stream);

/* Debug check of the reorder index (rebuttal page, "Description of the
 * reorder process": the reorder permutes channels).  The hot path trusts perm;
 * this entry checks that perm (device, int32 [K]) holds every value of
 * 0..K-1 exactly once.  Uses ws past its 256-byte header as scratch (needs
 * ws_bytes >= 256 + 16 + 4 * ceil(K / 32); any workspace sized by
 * rrs_workspace_size for this K is enough), then synchronises `stream` and
 * reads the result.  Returns RRS_OK, or RRS_ERR_INVALID_ARG naming the first
 * position whose value is out of range, else the smallest value no position
 * holds (which, with K in-range entries, means another value is repeated). */
rrs_status rrs_check_perm(const int32_t *perm, int K, void *ws, size_t ws_bytes, rrs_stream_t stream);

/* Fault-injection hook for tests: launches one kernel that waits on a
 * barrier nothing will release, with a wait limit of `limit_us`
 * microseconds (1..1000000).  The kernel records the timeout in the
 * workspace error word and returns; the context stays usable. */
rrs_status rrs_debug_wait_timeout(int limit_us, void *ws, size_t ws_bytes, rrs_stream_t stream);

/* Self-test hook for tests: q_fast[i] = a[i] / b[i] computed the way the
 * activation kernels divide (Markstein's correction from the correctly
 * rounded reciprocal of b, for b > 0), q_ieee[i] = the IEEE fp32 division.
 * All device arrays of length n. */
rrs_status rrs_debug_divide(const float *a, const float *b, int n, float *q_fast, float *q_ieee,
                            rrs_stream_t stream);

/* rrs_smooth_quant without a workspace argument, for callers that cannot
 * allocate device memory at call time: code running under an allocator it
 * does not own (a host framework or inference server that hands out only the
 * tensors it manages), code that must not allocate on its latency-critical
 * path, or code that cannot know a workspace size in advance.  There is no
 * counterpart on the pages; it computes exactly what rrs_smooth_quant
 * computes, with the same outputs and the same limits, plus one more:
 * M * K <= 1048576 (RRS_ERR_UNSUPPORTED above that).
 * The scratch is one fixed array in device memory that every GPU which loads
 * the library holds (about 5 MiB) until the process exits; this function calls
 * no cudaMalloc, cudaFree or allocating library routine.  The first call on a
 * device looks up that device's address of the array (cudaGetSymbolAddress,
 * with the device current), so make the first call on each device before any
 * stream capture.  All calls share the array: calls whose work overlaps on the
 * GPU (different streams, or different host threads without ordering) race on
 * it and must be serialised by the caller.  Each call clears the array's
 * error word; kernel timeouts are not reported through this entry point. */
rrs_status rrs_smooth_quant_noalloc(const void *X, int M, int K, int G, int had_block,
                                    const int32_t *perm, uint8_t *qX, float *s, float *scale_t,
                                    unsigned flags, rrs_stream_t stream);

/* Thread-local description of the last non-OK status returned on this thread. */
const char *rrs_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* RRS_H */
