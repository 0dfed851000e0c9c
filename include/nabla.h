/*
 * nabla.h - C ABI of the NABLA block-sparse attention library for B200 (sm_100a).
 *
 * The library implements the data-parallel hot path of NABLA
 * ("∇NABLA: Neighborhood Adaptive Block-Level Attention", arXiv 2507.13546v1):
 *
 *   1. the adaptive mask builder of §3.1.2, Algorithm 1 "NABLA Sparse Mask
 *      Generation": average-pool Q and K over blocks of N = 64 tokens, form the
 *      reduced attention map softmax(Qa Ka^T / sqrt(D)) per head, sort each row,
 *      accumulate, keep the entries whose cumulative value reaches 1 - thr and
 *      restore the original order; optionally OR-ed (§3.1.3) with the
 *      sliding-tile (STA) window mask of §2.2;
 *   2. block-sparse attention over the kept 64 x 64 tiles: Eq. 4 of §2.2,
 *      softmax(Q K^T / sqrt(D) + M) V with M in {-inf, 0}, and its backward;
 *   3. around them: Eq. 1's projection Q = X W_Q, K = X W_K, V = X W_V with
 *      the block averaging fused into it, the §3.1.1 token reordering, the
 *      STA-only masks and block coordinates, a fixed-budget Top-k selection
 *      and a per-block fidelity check of the pooling proxy.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors Q, K, V, O, dO, dQ, dK, dV are dense, contiguous [B, H, S, D] in
 *   the dtype named by the shape (bf16 or fp32), in device memory, with a
 *   16-byte aligned base address.  S may be any value >= 1: the last 64-token
 *   block may be partial (its pooled mean averages its valid tokens and its
 *   missing keys are excluded from attention).
 * - nb = ceil(S / 64) blocks per sequence; W = ceil(nb / 32) bitmask words per
 *   mask row; npairs = ceil(nb / 2) query-block pairs per (b, h).
 * - Every pointer argument is a device pointer unless stated otherwise.  The
 *   caller owns every buffer, including the workspace; the library allocates no
 *   device memory and keeps no global device state, except the static scratch
 *   of nabla_build_mask_noalloc (below).
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *   stream).  A returned NABLA_OK means the arguments were valid and the work
 *   was enqueued; device-side failures (a bounded wait that ran out) are
 *   reported in the workspace status word, read with nabla_workspace_status().
 * - On any error the call enqueues nothing (argument errors) or stops enqueuing
 *   (launch errors), returns a status != NABLA_OK and records a message that
 *   nabla_last_error() returns in the calling thread.
 * - The builders, attention, projection, reorder and fidelity calls enqueue
 *   only kernel launches and memsets on `stream`, so a sequence of them can be
 *   captured into a CUDA graph and replayed; make one eager call of each on
 *   the device first (it loads the library's modules).  The status read-backs
 *   (nabla_workspace_status, nabla_build_mask_noalloc_status) copy to the host
 *   and synchronise, so they stay outside a capture.  No kernel accumulates
 *   with floating-point atomics: repeated calls on the same inputs give
 *   bit-identical results.
 */
#ifndef NABLA_H
#define NABLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define NABLA_API __attribute__((visibility("default")))
#else
#define NABLA_API
#endif

#define NABLA_ABI_VERSION 3
#define NABLA_BLOCK 64

typedef struct CUstream_st* nabla_stream_t; /* same type as cudaStream_t */

typedef enum {
  NABLA_OK = 0,
  NABLA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment, thr outside (0, 1] */
  NABLA_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement (e.g. D = 96) */
  NABLA_ERR_CUDA = 3,         /* a CUDA runtime call failed; message in nabla_last_error() */
  NABLA_ERR_TIMEOUT = 4,      /* device status only: a bounded wait inside a kernel ran out */
  NABLA_ERR_WORKSPACE = 5     /* workspace pointer null or smaller than nabla_workspace_size() */
} nabla_status;

typedef enum { NABLA_BF16 = 0, NABLA_FP32 = 1 } nabla_dtype;

/* Problem shape.  block must be 64 (N in Algorithm 1); D must be 64 or 128. */
typedef struct {
  int32_t B, H, S, D;
  int32_t block;
  int32_t dtype; /* nabla_dtype */
} nabla_shape;

/* Optional STA neighbourhood (§2.2, §3.1.3).  block_coords: device int32
 * [nb][3], the (t, y, x) tile coordinate of every 64-token block (shared by
 * all samples and heads).  Block j is visible from block i iff
 * |t_i - t_j| <= wT / 2, |y_i - y_j| <= wH / 2 and |x_i - x_j| <= wW / 2
 * (integer division; window centred on the query tile, cut at the grid edge).
 * Window sizes are in tiles and must be >= 1. */
typedef struct {
  const int32_t* block_coords;
  int32_t wT, wH, wW;
} nabla_sta;

/* Mask outputs (all device memory, written by the library).
 *   bits  uint32 [B, H, nb, W]: bit (j % 32) of word j / 32 of row i is set
 *         iff query block i attends to key block j.  Padding bits are zero.
 *   cnt   int32 [B, H, nb]: number of kept key blocks of each query block.
 *   idx   int32 [B, H, nb, nb]: row i holds its cnt[i] kept key-block indices
 *         in ascending order; entries past cnt[i] are not written.
 *   cnt_t, idx_t: the same lists transposed (per key block, the query blocks
 *         that attend to it, ascending).  Needed only by nabla_attn_bwd; may be
 *         NULL for forward-only use.
 *   work  int32 [B * H * npairs][2]: the forward scheduler's work list, one
 *         entry per pair of query blocks (2p, 2p + 1) of one (b, h):
 *         { (b * H + h) * npairs + p, number of key blocks in the union of the
 *         two rows }.  Entries are grouped by (b, h) in ascending order and
 *         sorted by descending cost inside a group. */
typedef struct {
  uint32_t* bits;
  int32_t* cnt;
  int32_t* idx;
  int32_t* cnt_t;
  int32_t* idx_t;
  int32_t* work;
} nabla_mask;

/* Bytes of device workspace the calls below need for `shape`.  want_bwd != 0
 * adds what nabla_attn_bwd needs.  Returns 0 for an invalid shape. */
NABLA_API size_t nabla_workspace_size(const nabla_shape* shape, int32_t want_bwd);

/* Mask builder: Algorithm 1 of §3.1.2 plus the STA union of §3.1.3.
 *   q, k   [B, H, S, D] in shape->dtype.
 *   thr    binarisation threshold, 0 < thr <= 1 (thr = 1 keeps every block).
 *          A row keeps block j iff the softmax mass of the entries ranked above
 *          j (larger values) is <= thr; this is the ascending cumulative-sum
 *          rule cvals >= 1 - thr of Algorithm 1 (entries tied with the cut-off
 *          value are all kept).
 *   sta    NULL or sta->block_coords NULL: no STA union.
 *   out    bits, cnt, idx, work are required; cnt_t/idx_t are filled if not NULL.
 * The pooled vectors are fp64 means of the inputs; the reduced scores use
 * them as tf32 hi / lo pairs accumulated in fp32, and entries whose fp32
 * values fall into the cut-off's 2^-7-wide bucket are ranked by fp64 logits. */
NABLA_API nabla_status nabla_build_mask(const nabla_shape* shape, const void* q, const void* k, float thr,
                              const nabla_sta* sta, const nabla_mask* out, void* workspace,
                              size_t workspace_bytes, nabla_stream_t stream);

/* Fixed-budget variant of the mask builder: the comparator the paper sets the
 * CDF rule against (Appendix C of the v2 paper, per its pith.science review: CDF
 * thresholding against a fixed Top-k at the same average block budget).
 * Identical pooling and reduced scores; every row then keeps its topk
 * largest entries of softmax(Qa Ka^T / sqrt(D)) instead of the CDF set (topk
 * >= 1, clipped to nb; entries with equal values ranked as the stable
 * ascending sort leaves them, the higher block index first; a row whose cut
 * falls inside more than 128 entries of one 2^-7-wide value bucket keeps every
 * entry tied in fp32 with the cut-off).  STA union, outputs, workspace and
 * errors as nabla_build_mask. */
NABLA_API nabla_status nabla_build_mask_topk(const nabla_shape* shape, const void* q, const void* k,
                                             int32_t topk, const nabla_sta* sta, const nabla_mask* out,
                                             void* workspace, size_t workspace_bytes, nabla_stream_t stream);

/* Mask builder that allocates nothing, for callers that cannot call
 * cudaMalloc when they build a mask (for instance a serving process that
 * reserved all device memory at start-up and allows no side allocation while
 * a request runs, or code that must not risk the device-wide synchronisation
 * an allocation can cause).  The paper has no counterpart: this is a packaging
 * variant of nabla_build_mask.
 *   Same arguments and results as nabla_build_mask, without the workspace: the
 *   builder's scratch (status word, pooled Qa / Ka, reduced logits) lives in a
 *   32 MiB static device array inside the library, held by every GPU that
 *   loads it until the process exits.  Shapes whose scratch exceeds it
 *   (B * H * (nb * (32 D + 4 nb) + 8) bytes plus about 2 KB must fit in 32 MiB,
 *   nb = ceil(S / 64)) are rejected with
 *   NABLA_ERR_UNSUPPORTED and a message naming both sizes.
 *   The first call on a device looks up the array's device address with that
 *   device current (cudaGetSymbolAddress) and caches it; make that first call
 *   before any stream capture.  CUDA loads the library's modules lazily, so
 *   that first call is also when the 32 MiB is committed on the device (and it
 *   may synchronise the device): make it, or a call of
 *   nabla_build_mask_noalloc_status, at start-up, before reserving the rest of
 *   the device memory or serving requests.  The caller still provides q, k and
 *   every mask output.  Argument checks and their messages are those of
 *   nabla_build_mask.
 *   All calls share the array and it keeps the last call's contents (the
 *   status word is cleared at the start of every call): calls whose GPU work
 *   overlaps race on it, so serialise them.  A bounded wait that ran out inside
 *   the builder (NABLA_ERR_TIMEOUT) is recorded in the array's status word, which
 *   nabla_build_mask_noalloc_status reads back (not nabla_workspace_status). */
NABLA_API nabla_status nabla_build_mask_noalloc(const nabla_shape* shape, const void* q,
                                                const void* k, float thr, const nabla_sta* sta,
                                                const nabla_mask* out, nabla_stream_t stream);

/* Reads the status word of nabla_build_mask_noalloc's static scratch on the
 * current device into *host_status (a host pointer): NABLA_OK, or
 * NABLA_ERR_TIMEOUT if a bounded wait of the most recent call on this device
 * ran out (its mask is then incomplete).  Copies on `stream` and synchronises
 * it, so call it after the build on the same stream.  Allocates nothing; the
 * paper has no counterpart.  Errors: NABLA_ERR_INVALID_ARG for a NULL
 * host_status, NABLA_ERR_CUDA if the copy fails. */
NABLA_API nabla_status nabla_build_mask_noalloc_status(int32_t* host_status, nabla_stream_t stream);

/* Eq. 1 (§2.1), Q = X W_Q, K = X W_K, V = X W_V, on the tensor cores, with the
 * block averaging of Algorithm 1 (§3.1.2) fused into the same kernel: while it
 * writes Q and K it also writes their 64-token block means, so that
 * nabla_build_mask_pooled builds the mask without reading Q and K again.
 *   shape  as for nabla_build_mask; dtype must be NABLA_BF16.  Head h of Q is
 *          columns h D .. h D + D - 1 of X W_Q (likewise K and V).
 *   C      hidden size: the columns of X and the rows of W_Q; >= 8 and a
 *          multiple of 8 (rows of 16-byte multiples), at most 1,048,576.
 *   x      device, [B, S, C] bf16, token-major hidden states, read only.
 *   wt     device, [3, H * D, C] bf16: W_Q^T, W_K^T, W_V^T, one row of C
 *          weights per output feature n = h D + d (the layout of a linear
 *          layer's weight), read only.
 *   q, k, v  device, [B, H, S, D] bf16, written: the fp32-accumulated products
 *          rounded to the nearest bf16 (ties to even).  They must not overlap
 *          x, wt, each other or the workspace.
 *   workspace, workspace_bytes  the mask builder's workspace (at least
 *          nabla_workspace_size(shape, 0) bytes, 256-byte aligned): receives
 *          the block means of the stored Q and K, the same values the
 *          builder's own pooling computes from them; its status word is
 *          cleared first and records NABLA_ERR_TIMEOUT if a bounded wait of
 *          the kernel ran out.
 * All pointers 16-byte aligned.  Asynchronous on `stream`; allocates nothing.
 * Errors: NABLA_ERR_INVALID_ARG for an invalid shape, a NULL or misaligned
 * pointer, a bad C, or q, k or v overlapping another buffer of the call;
 * NABLA_ERR_UNSUPPORTED for fp32 inputs, a block size, D or sequence length
 * this build does not handle, C above the limit or 3 H D above 2^31 - 1;
 * NABLA_ERR_WORKSPACE for a workspace that is too small or misaligned;
 * NABLA_ERR_CUDA if the launch fails. */
NABLA_API nabla_status nabla_qkv_project(const nabla_shape* shape, int32_t C, const void* x, const void* wt,
                                         void* q, void* k, void* v, void* workspace, size_t workspace_bytes,
                                         nabla_stream_t stream);

/* nabla_build_mask starting from the block means that nabla_qkv_project left
 * in the workspace: the reduced scores, selection, STA union and lists of
 * Algorithm 1 without reading Q and K.  thr, sta, out and the results as for
 * nabla_build_mask (bit-identical masks for the same Q and K).  The workspace
 * must be the one the projection wrote for this shape, on the same stream (or
 * ordered after it), with no other call using it in between; its status word
 * is not cleared, so a timeout of the projection stays visible to
 * nabla_workspace_status.  Allocates nothing.  Errors as nabla_build_mask. */
NABLA_API nabla_status nabla_build_mask_pooled(const nabla_shape* shape, float thr, const nabla_sta* sta,
                                               const nabla_mask* out, void* workspace, size_t workspace_bytes,
                                               nabla_stream_t stream);

/* Sliding-tile (STA) mask alone, without the NABLA selection: the STA
 * configurations of Table 1 (§4.1) and the neighbourhood mask of §2.2 (Eq. 5).
 *   sta    required: block_coords (device int32 [nb][3]) and the window, as in
 *          nabla_sta; query block i keeps key block j iff j lies in the window
 *          centred on i (every row keeps at least block i).  The same mask for
 *          every sample and head.
 *   out    bits, cnt, idx, work are required; cnt_t/idx_t are filled if not NULL.
 * Needs no workspace and allocates nothing.  Errors: NABLA_ERR_INVALID_ARG for
 * an invalid shape, a NULL sta or coordinate pointer, a window size < 1 or a
 * missing or misaligned output; NABLA_ERR_UNSUPPORTED for a block size, D or
 * sequence length this build does not handle (as nabla_build_mask);
 * NABLA_ERR_CUDA if a launch fails.  The
 * coordinates must name tiles of the grid the tokens were laid out on (for
 * instance the result of nabla_sta_block_coords); they are not range-checked. */
NABLA_API nabla_status nabla_build_sta_mask(const nabla_shape* shape, const nabla_sta* sta, const nabla_mask* out,
                                            nabla_stream_t stream);

/* Host helper: the STA tile coordinate of every 64-token block of a latent
 * video laid out in the token order of §3.1.1 (Figure 3: inside each frame the
 * P x P spatial patches follow in row-major patch order, each patch's tokens
 * contiguous; frames keep their time order), for the window test of §2.2 ("a
 * fixed 3D window ... centered on the query tile") used by nabla_build_mask
 * and nabla_build_sta_mask.
 *   T, H_lat, W_lat  latent frames and frame height / width in tokens (>= 1);
 *   P                patch side in tokens (>= 1; 8 in the paper, so a full
 *                    patch is one 64-token block);
 *   S                tokens in the sequence the mask is built for (>= 1):
 *                    T * H_lat * W_lat, or that count padded at the end; every
 *                    block must start inside the latent, i.e.
 *                    64 * (ceil(S / 64) - 1) < T * H_lat * W_lat;
 *   coords_host      HOST int32 [ceil(S / 64)][3], caller-owned, written with
 *                    (t, y / P, x / P) of each block's first token.
 * When H_lat or W_lat is not a multiple of P the pages are silent; the reading
 * used: an edge patch cut by the frame holds only its valid tokens (row-major)
 * as one run, so blocks there may straddle patches and take the tile of their
 * first token.  Then copy the array to the device for nabla_sta.block_coords.
 * Runs on the host only (no CUDA call).  Errors: NABLA_ERR_INVALID_ARG for a
 * NULL pointer, a size < 1, more than 2^31 - 1 latent tokens, or a block that
 * starts past the latent. */
NABLA_API nabla_status nabla_sta_block_coords(int32_t T, int32_t H_lat, int32_t W_lat, int32_t P, int32_t S,
                                              int32_t* coords_host);

/* Builds cnt, idx, work (and cnt_t, idx_t if not NULL) of `out` from a
 * caller-supplied bitmask `bits` [B, H, nb, W] (padding bits must be zero);
 * out->bits is ignored.  Lets attention run under any externally computed
 * block mask, e.g. a reference mask. */
NABLA_API nabla_status nabla_mask_from_bits(const nabla_shape* shape, const uint32_t* bits,
                                  const nabla_mask* out, void* workspace, size_t workspace_bytes,
                                  nabla_stream_t stream);

/* Block-sparse attention forward, Eq. 4 of §2.2 with M = -inf outside the kept
 * tiles of `mask` (bits, cnt, idx and work must all describe the same mask:
 * the bf16 path walks bits and work, the fp32 path cnt and idx) and outside
 * the sequence.
 *   o      [B, H, S, D] output, shape->dtype.
 *   o_res  NULL, or (bf16 only) [B, H, S, D] bf16, 16-byte aligned: the
 *          rounding residual of o, bf16(O - bf16(O)), for training.  With it
 *          the tensor cores also multiply V by the bf16 remainder of the
 *          softmax weights P (P itself enters the product in bf16), so that
 *          o + o_res carries the attention output to about 2^-16 relative
 *          instead of 2^-9; nabla_attn_bwd uses it for
 *          Delta = rowsum(dO * O), which rows with a nearly one-hot softmax
 *          need (there dS = P (dP - Delta) cancels).  Costs one more P V
 *          product per tile.  NABLA_ERR_INVALID_ARG for fp32 (no residual).
 *   lse    float [B, H, S]: natural-log log-sum-exp of the scaled logits
 *          (Q K^T / sqrt(D)) over the attended keys, needed by the backward.
 *          May be NULL.  A row with no kept block gets o = 0 (and o_res = 0),
 *          lse = -inf.
 * bf16 runs on the tensor cores (tcgen05, fp32 accumulation in TMEM); fp32 runs
 * in fp32 on the CUDA cores. */
NABLA_API nabla_status nabla_attn_fwd(const nabla_shape* shape, const void* q, const void* k, const void* v,
                            const nabla_mask* mask, void* o, void* o_res, float* lse, void* workspace,
                            size_t workspace_bytes, nabla_stream_t stream);

/* Backward of nabla_attn_fwd with the mask held constant (no gradient flows
 * into the mask builder).  o and lse are the forward's outputs, dout the
 * upstream gradient; o_res is NULL or the forward's o_res (bf16 only): with it
 * Delta = rowsum(dO * (o + o_res)), else rowsum(dO * o); mask needs bits, cnt, idx, cnt_t and idx_t, all of the
 * same mask (the bf16 path walks cnt / idx for dQ and bits / cnt_t for dK and
 * dV; the fp32 path the four lists).  Writes dq, dk, dv [B, H, S, D] in
 * shape->dtype.  The result is deterministic (no atomics). */
NABLA_API nabla_status nabla_attn_bwd(const nabla_shape* shape, const void* q, const void* k, const void* v,
                            const void* o, const void* o_res, const void* dout, const float* lse,
                            const nabla_mask* mask, void* dq, void* dk, void* dv, void* workspace,
                            size_t workspace_bytes, nabla_stream_t stream);

/* Per-block fidelity of a block mask (the check the pith.science review of the
 * v2 paper asks of Algorithm 1's pooling proxy: how much of dense attention's
 * token-level mass falls inside the retained blocks).
 * nabla_block_mass writes the true block mass of dense attention (§2.1,
 * Eq. 2-3, softmax over all S keys):
 *   mass[b, h, i, j] = mean over the valid query tokens s of block i of
 *                      sum over the keys t of block j of softmax_t(q_s . k_t / sqrt(D))
 *   mass   float [B, H, nb, nb], caller-allocated; every row sums to 1.
 *   q, k   [B, H, S, D] bf16 (tensor cores; fp32 inputs: NABLA_ERR_UNSUPPORTED).
 *   workspace  any device buffer of >= 256 bytes, 256-byte aligned (its status
 *          word reports a bounded wait that ran out, NABLA_ERR_TIMEOUT).
 * Two dense passes of S = Q K^T (4 S^2 D flops per (b, h)); no V. */
NABLA_API nabla_status nabla_block_mass(const nabla_shape* shape, const void* q, const void* k, float* mass,
                                        void* workspace, size_t workspace_bytes, nabla_stream_t stream);

/* Kept mass of every query block under a block mask:
 *   recall[b, h, i] = sum over the kept key blocks j of row i of mass[b, h, i, j]
 * mass from nabla_block_mass; bits [B, H, nb, W] as in nabla_mask (padding bits
 * zero); recall float [B, H, nb]. */
NABLA_API nabla_status nabla_mask_recall(const nabla_shape* shape, const float* mass, const uint32_t* bits,
                                         float* recall, nabla_stream_t stream);

/* Fractal token reordering of §3.1.1 (Figure 3) and its inverse: the
 * permutation a DiT applies to its token sequence at the input stage (and
 * inverts at the output stage) so that the tokens of every P x P spatial
 * patch of a latent frame form one contiguous run; frames keep their temporal
 * order.
 *   x, y      device arrays of B * T * H * W rows of row_bytes bytes each (the
 *             rows are moved, not interpreted: any element type, e.g. [B, S, C]
 *             activations with row_bytes = C * element size); 16-byte aligned;
 *             row_bytes a positive multiple of 16; y must not overlap x.
 *   T, H, W   latent frames and frame height and width in tokens (>= 1);
 *   P         patch side in tokens (>= 1; 8 in the paper, so a patch is one
 *             64-token block);
 *   inverse   0: x in raster order (t, y, x) -> y in fractal order;
 *             1: x in fractal order -> y in raster order.
 * Reading for frames whose H or W is not a multiple of P (the pages show full
 * patches only): an edge patch holds its valid tokens, row-major, as one run.
 * Memory-bound: every row is read once and written once. */
NABLA_API nabla_status nabla_fractal_reorder(const void* x, void* y, int32_t B, int32_t T, int32_t H,
                                             int32_t W, int32_t P, size_t row_bytes, int32_t inverse,
                                             nabla_stream_t stream);

/* Reads the device status word of `workspace` into *host_status (a host
 * pointer): NABLA_OK, or NABLA_ERR_TIMEOUT if a bounded wait inside a kernel of
 * the most recent call on this workspace ran out.  Synchronises `stream`. */
NABLA_API nabla_status nabla_workspace_status(const void* workspace, int32_t* host_status,
                                    nabla_stream_t stream);

/* Self-test of the bounded-wait path: launches one small kernel whose only
 * wait is on a barrier that nothing ever arrives on, so the wait runs out after
 * limit_ns nanoseconds (1 <= limit_ns <= 1e10) and the kernel records
 * NABLA_ERR_TIMEOUT in the status word of `workspace` (any device buffer of at
 * least 256 bytes, 256-byte aligned), as every pipelined kernel does when one
 * of its waits runs out.  Read the result with nabla_workspace_status(). */
NABLA_API nabla_status nabla_selftest_wait_timeout(void* workspace, uint64_t limit_ns,
                                                   nabla_stream_t stream);

/* Sets the time limit, in nanoseconds, of every bounded spin-wait in the
 * kernels launched after this call by the calling process (0 restores the
 * default of 2 s).  A wait that runs out makes its kernel stop cleanly and set
 * NABLA_ERR_TIMEOUT in the workspace status word. */
NABLA_API void nabla_set_wait_limit_ns(uint64_t ns);

/* Message of the last error recorded in the calling thread ("" if none). */
NABLA_API const char* nabla_last_error(void);

/* NABLA_ABI_VERSION of the loaded library. */
NABLA_API int32_t nabla_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NABLA_H */
