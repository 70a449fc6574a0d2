/*
 * libfa2 -- exact FlashAttention-2 forward and backward for NVIDIA B200
 * (sm_100a), behind a plain C ABI.
 *
 * What the library computes
 * -------------------------
 * For every batch b and head h, with query rows i and key rows j in [0, N):
 *
 *     s_ij  = softmax_scale * <q_i, k_j> + bias_ij        (bias: ALiBi, below)
 *     s_ij  = -inf where the mask hides key j from query i
 *     P     = softmax over j of s (row by row)
 *     O     = P V,   LSE_i = log sum_j exp(s_ij)          (natural log)
 *
 * This is ordinary (exact) attention: the FlashAttention explainer
 * "AI基础 | Flash Attention" (yeyulingfeng.com) states in its opening that the
 * method changes how attention is computed on the GPU, not its result, and
 * the FlashAttention-2 abstract (arXiv 2307.08691) says "without
 * approximation".  The N x N score matrix is never written to device memory:
 * the forward pass streams key/value tiles through on-chip memory with an
 * online softmax (explainer, "Tiling" and "Online softmax" sections) and
 * keeps only the per-row log-sum-exp; the backward pass recomputes the
 * probabilities from Q, K and that statistic (explainer, "Backward pass").
 *
 * The options follow the call printed in the "FlashAttention v2" article
 * (wmrh.cn), §5.1 (API): dropout_p, softmax_scale, causal, window_size =
 * (left, right), alibi_slopes and deterministic.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors q, k, v, o, dout, dq, dk, dv are [B, N, H, d] with the d index
 *    contiguous (stride 1) and the other strides given in ELEMENTS by an
 *    fa2_strides value; every stride must be a multiple of 8 elements
 *    (16 bytes) for bf16 and of 4 elements for fp32, and every base pointer
 *    16-byte aligned.  lse and D are dense fp32 [B, H, N].
 *  - All pointers are DEVICE pointers, owned by the caller; the library
 *    allocates no device memory and keeps no state between calls except a
 *    small cache of device properties, the device status word read by
 *    fa2_device_status(), a table of 64 work-counter pairs per device and
 *    the scratch array of fa2_bwd_noalloc.  The first call that reaches a
 *    device looks up the device addresses of the last two
 *    (cudaGetSymbolAddress, with that device current); make that first
 *    call before any stream capture.
 *  - Work counters.  Calls whose work items differ in cost (the *_varlen
 *    and *_blocksparse calls, and backward calls with a causal mask over
 *    128 or more key blocks) take their items from a counter pair.  Each
 *    stream that makes such calls owns one pair: calls on one stream run in
 *    order and reuse it, calls on different streams never share one while
 *    both may run.  The pair is cleared on the call's stream before each
 *    launch, after the stream has been made to wait, on the GPU (an
 *    event), for the pair's last call to finish (free on the pair's own
 *    stream; it also covers a stream handle that is destroyed and reused
 *    while its last call still runs).  Up to 64 streams per device own a
 *    pair at a time; a further stream takes over the least recently used
 *    pair behind the same wait.  During stream
 *    capture no such wait can be recorded: a captured call keeps the pair
 *    of the capturing stream (a hand-over that would need a wait returns
 *    FA2_ERR_UNSUPPORTED), and the caller must not replay the graph while
 *    another call on the same pair runs (for instance the same graph on
 *    two streams at once).
 *  - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *    default stream); nothing is synchronised.
 *  - Every argument is checked before anything is launched.  An invalid
 *    argument returns FA2_ERR_INVALID_ARG and launches nothing; a valid but
 *    unimplemented combination returns FA2_ERR_UNSUPPORTED; a CUDA error at
 *    launch returns FA2_ERR_CUDA.
 *  - Supported shapes: d in {64, 128}; 1 <= N; B, H >= 1; the key/value
 *    sequence has the same length and head count as the queries.  Packed
 *    batches of sequences of different lengths have their own entry points
 *    (fa2_fwd_varlen, fa2_bwd_varlen) with a [total, H, d] layout.
 *  - dtype FA2_BF16: bf16 inputs/outputs, fp32 accumulation on the tensor
 *    cores.  dtype FA2_F32: fp32 inputs/outputs with full fp32 arithmetic
 *    (CUDA cores), for checks at 1e-4.
 */
#ifndef FA2_H_
#define FA2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA2_BF16 = 0,
  FA2_F32 = 1
} fa2_dtype;

typedef enum {
  FA2_OK = 0,
  FA2_ERR_INVALID_ARG = 1,     /* a pointer, shape, stride or option is invalid */
  FA2_ERR_UNSUPPORTED = 2,     /* valid, but not implemented (e.g. dropout_p != 0) */
  FA2_ERR_CUDA = 3,            /* a CUDA runtime/driver call failed */
  FA2_ERR_DEVICE_TIMEOUT = 4,  /* a kernel gave up a bounded wait or met malformed
                                  cu_seqlens (see fa2_device_status) */
  FA2_ERR_SCRATCH_LIMIT = 5    /* problem too large for fa2_bwd_noalloc's fixed scratch */
} fa2_status;

/* Element strides of a [B, N, H, d] tensor; the d stride is always 1. */
typedef struct {
  int64_t b;
  int64_t n;
  int64_t h;
} fa2_strides;

/*
 * Forward pass: O = softmax(scale * Q K^T + bias, masked) V and the per-row
 * natural-log log-sum-exp.
 *
 *   q, k, v       [B, N, H, d] inputs (dtype), strides sq, sk, sv.
 *   o             [B, N, H, d] output (dtype), strides so.  May not alias q/k/v.
 *   lse           [B, H, N] fp32 output, dense.
 *   softmax_scale <= 0 selects 1/sqrt(d) (the "softmax_scale=None" default).
 *   causal        nonzero: key j is visible to query i only if j <= i
 *                 (equivalent to window_right = 0).
 *   window_left, window_right
 *                 sliding window: key j is visible to query i only if
 *                 i - window_left <= j <= i + window_right (inclusive);
 *                 a negative value means unbounded on that side
 *                 ("window_size=(-1,-1)" is the default).
 *   alibi_slopes  NULL, or a device fp32 [H] array; adds -slope_h * |i - j|
 *                 to the scaled score (linear-bias attention).
 *   dropout_p     probability of zeroing each attention probability after
 *                 the softmax, 0 <= dropout_p < 255.5/256; kept ones are
 *                 scaled so the expected output is unchanged (see DROPOUT).
 *   dropout_seed  64-bit seed of the dropout mask (ignored when
 *                 dropout_p == 0).
 *
 * DROPOUT.  With t = round(256 * dropout_p), element (b, h, query i, key j)
 * is kept iff its random byte is >= t, and kept probabilities are multiplied
 * by 256 / (256 - t) (so the effective drop probability is t / 256).  The
 * random byte is byte (j mod 4), least significant first, of output word
 * (i mod 4) of Philox4x32-10 (Salmon et al., SC 2011) with counter
 * (j / 4, i / 4, h, b) and key (dropout_seed mod 2^32, dropout_seed / 2^32).
 * fa2_bwd with the same seed and dropout_p regenerates the same mask.  LSE
 * is always the log-sum-exp of the un-dropped scores.
 *
 * A query row that sees no key (impossible with the masks above, since the
 * diagonal is always visible) gets O = 0 and lse = -inf.  The result is
 * bitwise identical between runs with the same inputs and shapes.
 */
fa2_status fa2_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int N, int H, int d, fa2_dtype dtype,
                   fa2_strides sq, fa2_strides sk, fa2_strides sv, fa2_strides so,
                   float softmax_scale, int causal, int window_left, int window_right,
                   const float* alibi_slopes, float dropout_p, unsigned long long dropout_seed,
                   void* stream);

/*
 * Backward pre-processing: D[b, h, i] = sum_c dO[b, i, h, c] * O[b, i, h, c]
 * in fp32 (the row sums of dO o O that the softmax gradient needs).
 *
 * The backward pass keeps only per-row statistics of the forward and
 * rebuilds the scores on chip (explainer "AI基础 | Flash Attention",
 * "Backward pass"); with P the softmax, the gradient of the scores is
 * dS_ij = P_ij (dP_ij - D_i), dP = dO V^T, where D_i = sum_j P_ij dP_ij
 * equals sum_c dO_ic O_ic because O = P V.  This call computes D from O
 * and dO, so the backward kernels never form a row of dP in full before
 * they can use it.
 *
 *   o, dout  [B, N, H, d] (dtype), strides so, sdo.
 *   D        [B, H, N] fp32 output, dense.
 *
 * Unlike a common layout of this step, the call does not clear the fp32 dQ
 * accumulator: fa2_bwd clears its own workspace before it adds into it, so
 * the workspace's contents on entry never matter.
 */
fa2_status fa2_bwd_preprocess(const void* o, const void* dout, float* D,
                              int B, int N, int H, int d, fa2_dtype dtype,
                              fa2_strides so, fa2_strides sdo, void* stream);

/*
 * Bytes of device workspace fa2_bwd needs for these shapes: for bf16, an fp32
 * dQ accumulator (B * H * N * d floats) -- when deterministic, two of them
 * and, for each, one 32-bit counter per 32 query rows
 * (B * H * ceil(N / 128) * 4); nothing for fp32.
 * The caller allocates it; its contents on entry do not matter (the call
 * clears what it uses).  Returns 0 for invalid shapes.
 */
size_t fa2_bwd_workspace_size(int B, int N, int H, int d, fa2_dtype dtype, int deterministic);

/*
 * Backward pass: dQ, dK, dV of L = sum(O o dO) given the forward's lse and
 * the pre-processed D.  The probabilities are recomputed from q, k and lse
 * (explainer "AI基础 | Flash Attention", "Backward pass": the N x N matrices
 * are not stored; only the per-row statistics are, and the scores are
 * rebuilt block by block on chip).  The pages print no gradient formulas;
 * the ones computed are the textbook softmax and matrix-product gradients,
 * with c = softmax_scale:
 *     P = exp(c Q K^T + bias - LSE),  dV = P^T dO,  dP = dO V^T,
 *     dS = P o (dP - D),  dQ = c dS K,  dK = c dS^T Q.
 * Work is split over key blocks of every (batch, head) (FlashAttention-2
 * abstract, arXiv 2307.08691: parallelism across thread blocks within a
 * head); dQ partial sums of different key blocks are added in fp32.  The
 * `deterministic` option is the one of the call in the "FlashAttention v2"
 * article, §5.1-§5.2.
 *
 *   q, k, v, dout    [B, N, H, d] inputs (dtype) with strides sq, sk, sv, sdo.
 *   lse, D           [B, H, N] fp32 from fa2_fwd and fa2_bwd_preprocess.
 *   dq, dk, dv       [B, N, H, d] outputs (dtype) with strides sdq, sdk, sdv.
 *   workspace        device buffer of at least workspace_bytes >=
 *                    fa2_bwd_workspace_size(...) bytes, 256-byte aligned.
 *   softmax_scale, causal, window_left, window_right, alibi_slopes,
 *   dropout_p, dropout_seed
 *                    exactly as passed to fa2_fwd.
 *   deterministic    0: dQ partial sums from different key blocks are added
 *                    with fp32 reductions in whatever order they arrive
 *                    (fast, bits may differ between runs);
 *                    nonzero: dq, dk and dv are bitwise repeatable.  Under a
 *                    causal mask (window_right = 0) the partial sums of each
 *                    query block are added in a fixed order inside the same
 *                    kernel (even and odd key blocks into two accumulators,
 *                    each in descending key-block order, then the two added);
 *                    otherwise dQ comes from a second, ordered pass that
 *                    recomputes the scores.
 */
fa2_status fa2_bwd(const void* q, const void* k, const void* v, const void* dout,
                   const float* lse, const float* D, void* dq, void* dk, void* dv,
                   void* workspace, size_t workspace_bytes,
                   int B, int N, int H, int d, fa2_dtype dtype,
                   fa2_strides sq, fa2_strides sk, fa2_strides sv, fa2_strides sdo,
                   fa2_strides sdq, fa2_strides sdk, fa2_strides sdv,
                   float softmax_scale, int causal, int window_left, int window_right,
                   const float* alibi_slopes, float dropout_p, unsigned long long dropout_seed,
                   int deterministic, void* stream);

/*
 * Packed variable-length batches ("dynamic sequence support", named as
 * future work in §6 of the "FlashAttention v2" article): B independent
 * sequences of different lengths stored back to back, with no padding rows.
 *
 *   cu_seqlens    DEVICE int32 [B + 1]: sequence b owns tensor rows
 *                 [cu_seqlens[b], cu_seqlens[b + 1]); cu_seqlens[0] = 0,
 *                 non-decreasing, cu_seqlens[B] = total.  A length may be 0.
 *   max_seqlen    an upper bound on every length (>= 1); it sizes the grids,
 *                 so a tight bound wastes least.
 *   total         number of rows of every tensor (>= 0; 0 returns FA2_OK and
 *                 launches nothing).
 *   q, k, v, o, dout, dq, dk, dv
 *                 [total, H, d]; only the n (row) and h strides of each
 *                 fa2_strides value are used, with the alignment rules above.
 *   lse, D        dense fp32 [H, total] (row statistics of row r of head h at
 *                 h * total + r).  D comes from fa2_bwd_preprocess called with
 *                 B = 1, N = total on the same [total, H, d] tensors.
 *   workspace     fa2_bwd_workspace_size(1, total, H, d, dtype, deterministic)
 *                 bytes, 256-byte aligned.
 *
 * Every other argument means what it means for fa2_fwd / fa2_bwd.  Each
 * sequence is attended to on its own, as if it were the only one of a padded
 * call at batch index b: masks, ALiBi distances and the dropout counter use
 * positions 0 .. len_b - 1 inside the sequence, and the dropout counter's
 * batch field is the sequence index b.
 *
 * cu_seqlens lives on the device and is not read on the host.  Offsets
 * outside [0, total], decreasing offsets and lengths above max_seqlen are
 * clamped by the kernels (no access leaves the tensors) and recorded as code
 * 0xF10 in the device status word (fa2_device_status); the results of such
 * a call are unspecified.
 */
fa2_status fa2_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                          const int32_t* cu_seqlens, int B, int max_seqlen, int total,
                          int H, int d, fa2_dtype dtype,
                          fa2_strides sq, fa2_strides sk, fa2_strides sv, fa2_strides so,
                          float softmax_scale, int causal, int window_left, int window_right,
                          const float* alibi_slopes, float dropout_p,
                          unsigned long long dropout_seed, void* stream);

fa2_status fa2_bwd_varlen(const void* q, const void* k, const void* v, const void* dout,
                          const float* lse, const float* D, void* dq, void* dk, void* dv,
                          void* workspace, size_t workspace_bytes,
                          const int32_t* cu_seqlens, int B, int max_seqlen, int total,
                          int H, int d, fa2_dtype dtype,
                          fa2_strides sq, fa2_strides sk, fa2_strides sv, fa2_strides sdo,
                          fa2_strides sdq, fa2_strides sdk, fa2_strides sdv,
                          float softmax_scale, int causal, int window_left, int window_right,
                          const float* alibi_slopes, float dropout_p,
                          unsigned long long dropout_seed, int deterministic, void* stream);

/*
 * Block-sparse attention (named as future work in §6 of the "FlashAttention
 * v2" article): the padded calls above with a 128 x 128 block mask.  Key j is
 * hidden from query i unless byte
 *     block_mask[b * mask_stride_b + h * mask_stride_h + (i / 128) * nb + j / 128]
 * is nonzero, nb = ceil(N / 128), on top of the causal and window masks.
 *
 *   block_mask      DEVICE uint8 [B, H, nb, nb] (rows of nb bytes); owned by
 *                   the caller; read, never written.
 *   mask_stride_b, mask_stride_h
 *                   its batch and head strides in bytes, >= 0; 0 shares one
 *                   mask across the batch or across the heads.
 *
 * Every other argument means what it means for fa2_fwd / fa2_bwd (same
 * layouts, workspace size, dropout counter).  Blocks the mask hides are
 * neither loaded nor multiplied.  A query row that sees no key gets O = 0,
 * LSE = -inf and zero gradients.  The mask must be the same for the forward
 * and the backward call.
 */
fa2_status fa2_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int N, int H, int d, fa2_dtype dtype,
                               fa2_strides sq, fa2_strides sk, fa2_strides sv, fa2_strides so,
                               const uint8_t* block_mask, int64_t mask_stride_b,
                               int64_t mask_stride_h,
                               float softmax_scale, int causal, int window_left,
                               int window_right, const float* alibi_slopes, float dropout_p,
                               unsigned long long dropout_seed, void* stream);

fa2_status fa2_bwd_blocksparse(const void* q, const void* k, const void* v, const void* dout,
                               const float* lse, const float* D, void* dq, void* dk, void* dv,
                               void* workspace, size_t workspace_bytes,
                               int B, int N, int H, int d, fa2_dtype dtype,
                               fa2_strides sq, fa2_strides sk, fa2_strides sv, fa2_strides sdo,
                               fa2_strides sdq, fa2_strides sdk, fa2_strides sdv,
                               const uint8_t* block_mask, int64_t mask_stride_b,
                               int64_t mask_stride_h,
                               float softmax_scale, int causal, int window_left,
                               int window_right, const float* alibi_slopes, float dropout_p,
                               unsigned long long dropout_seed, int deterministic, void* stream);

/*
 * FP8 forward (the FlashAttention-3 page lists FP8 support as a further
 * speed-up; it gives no numerics, so this is the plain reading): q, k and v
 * are e4m3 (float8 e4m3fn: 1 sign, 4 exponent, 3 mantissa bits, max 448)
 * with per-tensor dequantisation factors, and the result is the attention of
 * the dequantised values q_descale * q, k_descale * k, v_descale * v.
 *
 *   q, k, v        [B, N, H, d] e4m3 bytes; strides in elements (= bytes),
 *                  multiples of 16; base pointers 16-byte aligned.
 *   o              [B, N, H, d] bf16 output, strides multiples of 8.
 *   lse            [B, H, N] fp32, as for fa2_fwd.
 *   q_descale, k_descale, v_descale
 *                  finite, > 0.
 *   d              128 only (FA2_ERR_UNSUPPORTED otherwise).
 *
 * Both products run on the tensor cores in e4m3 with fp32 accumulation: the
 * scores exactly (products of e4m3 values are exact in fp32), and P V with
 * the probabilities rounded to e4m3 (relative error <= 2^-4, or 2^-10
 * absolute below the normal range; the softmax statistics and LSE stay
 * fp32).  No dropout; the masks and ALiBi work as for fa2_fwd.
 */
fa2_status fa2_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int N, int H, int d,
                       fa2_strides sq, fa2_strides sk, fa2_strides sv, fa2_strides so,
                       float q_descale, float k_descale, float v_descale,
                       float softmax_scale, int causal, int window_left, int window_right,
                       const float* alibi_slopes, void* stream);

/*
 * fa2_bwd_noalloc: the bf16 backward pass without any caller-provided or
 * library-allocated workspace.  (No counterpart in the paper: this is an
 * interface convenience, not part of the method.)
 *
 * Some callers cannot allocate device memory at the point where they run
 * the backward pass: code inside a host framework that owns every byte of
 * device memory through its own pool and forbids cudaMalloc after start-up,
 * plugin interfaces that hand over inputs and outputs but no workspace, and
 * latency-critical loops where an allocation may block on the driver.  For
 * them this entry point takes the fp32 dQ accumulator from a fixed array
 * compiled into the library (FA2_NOALLOC_MAX_DQ_FLOATS floats, 16 MiB,
 * present on every GPU that loads the library until the process exits).
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments and results are those of fa2_bwd with dtype FA2_BF16,
 * deterministic = 0 (dQ partial sums added with fp32 reductions) and no
 * dropout (dropout_p != 0 returns FA2_ERR_UNSUPPORTED).  The caller still
 * provides q, k, v, dout, lse, D, dq, dk and dv.
 *
 *   Limit:   B * H * N * d must not exceed FA2_NOALLOC_MAX_DQ_FLOATS;
 *            larger problems return FA2_ERR_SCRATCH_LIMIT and launch
 *            nothing (use fa2_bwd with a workspace instead).
 *   Set-up:  the device address of the array is looked up
 *            (cudaGetSymbolAddress, with the device current) by the first
 *            call of any entry point that reaches the device; make that
 *            first call before any stream capture.
 *   Sharing: every call on a device uses the same array.  The accumulator
 *            is cleared at the start of each call, but two calls whose
 *            kernels overlap on the GPU (different streams, no ordering
 *            between them) race on it and give wrong gradients; order such
 *            calls on one stream or with events.
 */
#define FA2_NOALLOC_MAX_DQ_FLOATS (4u * 1024u * 1024u)
fa2_status fa2_bwd_noalloc(const void* q, const void* k, const void* v, const void* dout,
                           const float* lse, const float* D, void* dq, void* dk, void* dv,
                           int B, int N, int H, int d,
                           fa2_strides sq, fa2_strides sk, fa2_strides sv, fa2_strides sdo,
                           fa2_strides sdq, fa2_strides sdk, fa2_strides sdv,
                           float softmax_scale, int causal, int window_left, int window_right,
                           const float* alibi_slopes, float dropout_p, void* stream);

/* Human-readable name of a status code (static storage). */
const char* fa2_strerror(fa2_status status);

/*
 * Reads (and, if `clear` is nonzero, resets) the device status word of the
 * current device.  Synchronises the device.  *code receives 0 if no kernel
 * has given up a bounded wait or met malformed cu_seqlens (code 0xF10)
 * since the last clear, else the code of the first such event.  Returns
 * FA2_ERR_DEVICE_TIMEOUT when *code != 0, FA2_OK otherwise, FA2_ERR_CUDA on
 * a CUDA error.
 */
fa2_status fa2_device_status(int* code, int clear);

/*
 * Sets the time limit, in milliseconds, of every bounded wait inside the
 * kernels launched afterwards by this process (default 1000 ms).  Values
 * < 1 are rejected with FA2_ERR_INVALID_ARG.
 */
fa2_status fa2_set_wait_limit_ms(int ms);

/*
 * Test switch for the bounded-wait path (0 in normal use, the default).
 * With which = 1 every later forward launch of the tensor-core kernels, and
 * with which = 2 every later backward launch (the dK/dV kernel), has the
 * CTA that takes work item 0 (a query-tile pair, or a key block, of batch 0
 * and head 0; the first item that CTA takes) withhold one mbarrier arrive
 * on its first block, so that the MMA warp's wait for it runs out after the
 * limit set by fa2_set_wait_limit_ms.  That CTA then records the wait's
 * site code in the device status word, its other roles give up their own
 * waits through the CTA's abort flag, it waits (again with a limit) for the
 * copies and products it has in flight, frees its tensor memory and exits;
 * the other CTAs finish normally.  The outputs of such a call are unspecified;
 * fa2_device_status reports FA2_ERR_DEVICE_TIMEOUT.  Set 0 to switch it
 * off.  Returns FA2_ERR_INVALID_ARG for other values.
 */
fa2_status fa2_test_skip_arrive(int which);

/*
 * Number of kernels this library has launched in this process since it was
 * loaded (all devices, all entry points).  Lets a caller count the device
 * work of a region: read it before and after.
 */
uint64_t fa2_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* FA2_H_ */
