/*
 * fa.h - C ABI of the B200 (sm_100a) exact-attention library, libfa_sm100.so.
 *
 * The library computes exact scaled-dot-product attention
 *     O = softmax(scale * Q K^T [+ causal mask]) V
 * tile by tile with the online-softmax recurrence, so the N x N score matrix never
 * reaches device memory, and its gradient by recomputing the score tiles on chip.
 *
 * Sources of the operations (web pages on FlashAttention):
 *  - tiling and on-chip recomputation in the backward pass: "The Future of AI: How
 *    FlashAttention Revolutionizes Deep Learning", bullets "Tiling" and "Recomputation";
 *  - the online softmax (running max m, running sum l, rescaling of partial results
 *    when a block raises the max): "FlashAttention1" interview Q&A, question on how
 *    FlashAttention computes the softmax function, items 1-3; "Flash attention ... a deep
 *    dive", section "What is the mathematical aspect of softmax?" ("Intuition");
 *  - exactness (the blocked result equals standard attention): the same Q&A, question
 *    on the key algorithmic innovations; the deep-dive page, section "Algorithm behind
 *    the article";
 *  - attention dropout: named by the deep-dive page ("Quantitative Evidence"); the mask
 *    generator is Philox4x32-10 (see fa_fwd_dropout);
 *  - grouped- and multi-query attention and head dimensions up to 256: the
 *    FlashAttention-2 page, "FlashAttention-2: Enhanced Performance";
 *  - causal masking: the deep-dive page names masking among the memory-bound steps
 *    ("Quantitative Evidence"); this library uses the top-left causal mask, key j is
 *    visible to query i when j <= i;
 *  - local (sliding-window) attention: the "FlashAttention1" Q&A, question on scaling to
 *    very long sequences, item 4, proposes combining the method with local attention;
 *    neither page defines the window; this library's reading is the band
 *    i - left <= j <= i + right, and key blocks outside every row's band are skipped
 *    rather than masked;
 *  - block-sparse attention: the deep-dive page's closing paragraph names block-sparse
 *    FlashAttention; this library's reading is a per-head 0/1 mask over 128 x 128 blocks
 *    (see fa_fwd_blocksparse).
 *
 * Conventions shared by every entry point
 *  - Layout: Q, dQ, O, dO are [B, Hq, N, d]; K, V, dK, dV are [B, Hkv, N, d]; all
 *    contiguous bf16 (row of d elements, then N rows, then heads, then batch).  LSE is
 *    [B, Hq, N] fp32 (natural-log logsumexp of the scaled scores of each query row).
 *  - Query head h uses K/V head h / (Hq / Hkv) (contiguous groups).
 *  - Supported head dimensions: d in {64, 128, 256}.  Any 1 <= N <= 2^30 with
 *    B * Hq * N < 2^31.
 *  - Every pointer is a DEVICE pointer owned by the caller and must be 16-byte aligned.
 *    The library allocates no device memory except its 8-byte status words, which live
 *    in a file-scope __device__ variable.  Input buffers are read-only.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *    asynchronous with respect to the host; it returns after enqueueing kernels.
 *  - Argument errors are detected on the host before anything is launched; the outputs
 *    are then left untouched.  A launch failure returns FA_ERR_CUDA.
 *  - Device-side failures (a pipeline wait that exceeded its time limit) are recorded in
 *    the device status word and reported by fa_device_status().
 *  - The calls may be made from several host threads; the tensor-map encoder they share
 *    holds no state.
 */
#ifndef FA_SM100_H
#define FA_SM100_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
enum fa_status {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,    /* null pointer, non-positive size, non-finite/<=0 scale,
                                  causal not 0/1, window bound below -1 */
    FA_ERR_UNSUPPORTED = 2,    /* d not in {64, 128, 256}, or sizes beyond int32 index range */
    FA_ERR_GQA = 3,            /* Hq is not a multiple of Hkv */
    FA_ERR_ALIGN = 4,          /* a pointer is not 16-byte aligned */
    FA_ERR_WORKSPACE = 5,      /* workspace missing or smaller than fa_bwd_workspace_bytes() */
    FA_ERR_CUDA = 6,           /* CUDA runtime/driver error (no sm_100 device, launch failure) */
    FA_ERR_DEVICE_TIMEOUT = 7, /* a kernel's bounded pipeline wait expired (device watchdog) */
    FA_ERR_SCRATCH_LIMIT = 8,  /* fa_bwd_noalloc: problem needs more than FA_NOALLOC_SCRATCH_BYTES */
    FA_ERR_SEQLENS = 9         /* packed-sequence offsets inconsistent (found on the device) */
};

/*
 * Forward pass.
 *   q   [B, Hq,  N, d] bf16 in      k, v [B, Hkv, N, d] bf16 in
 *   o   [B, Hq,  N, d] bf16 out     lse  [B, Hq, N] fp32 out (natural log)
 *   causal: 0 or 1 (top-left mask, key j visible to query i iff j <= i)
 *   scale: softmax scale (> 0, finite), typically 1/sqrt(d), applied to Q K^T.
 * O and LSE are each written exactly once; rows are independent.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int Hq, int Hkv, int N, int d, int causal, float scale, void *stream);

/*
 * Forward pass of local (sliding-window) attention.  Arguments as fa_fwd, with the mask
 * given by two bounds instead of `causal`: key j is visible to query i iff
 *     i - window_left <= j <= i + window_right,
 * where a bound of -1 is unlimited on that side (values below -1 are FA_ERR_INVALID_ARG;
 * a bound >= N - 1 hides nothing and is treated as unlimited).  Every row sees at least
 * its own key, so every row's softmax is defined.  (-1, -1) is fa_fwd with causal = 0 and
 * (-1, 0) is fa_fwd with causal = 1, bit for bit.  Work is proportional to the number of
 * 128-key blocks that intersect each query tile's band.
 */
int fa_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse,
                  int B, int Hq, int Hkv, int N, int d, int window_left, int window_right,
                  float scale, void *stream);

/*
 * Forward pass over a batch of variable-length sequences packed along the token axis
 * (the "FlashAttention1" Q&A page names variable sequence lengths among the scaling
 * challenges, item 2; the packing and alignment below are this library's reading).
 *   q, o [total_q, Hq, d] bf16;  k, v [total_k, Hkv, d] bf16;  lse [total_q, Hq] fp32 out
 *   cu_seqlens_q, cu_seqlens_k: DEVICE int32 [B + 1] (4-byte aligned), nondecreasing row
 *        offsets: sequence b owns query rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 and key
 *        rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1 (the offsets need not start at 0).
 *   max_seqlen_q, max_seqlen_k: upper bounds on the per-sequence lengths (they size the
 *        launch); total_q, total_k: rows of the packed tensors (<= 2^29 each).
 * Query and key lengths may differ.  The key band is aligned to the END of both (bottom
 * right): with dlt = Lk - Lq, query i sees keys j with
 *     i + dlt - window_left <= j <= i + dlt + window_right,  0 <= j < Lk,
 * a bound of -1 being unlimited (causal: window_left = -1, window_right = 0; full
 * attention: both -1).  A query row that sees no key gets O = 0 and LSE = -inf.
 * Offsets that are decreasing, exceed total_q / total_k, or describe a sequence longer
 * than max_seqlen_q rows are reported on the device as FA_ERR_SEQLENS (fa_device_status);
 * the affected sequences are left unwritten.
 */
int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                  const int *cu_seqlens_q, const int *cu_seqlens_k, int B, int Hq, int Hkv,
                  int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                  int window_left, int window_right, float scale, void *stream);

/*
 * Forward pass with attention dropout.  The deep-dive page names dropout among the
 * memory-bound steps of standard attention ("Quantitative Evidence") without specifying
 * it; this library's reading: each probability P_ij of query head bh = b * Hq + h is kept
 * with probability 1 - p' and kept ones are scaled by 1 / (1 - p'):
 *     O_i = sum_j P_ij Z_ij / (1 - p') v_j,   LSE_i as without dropout,
 * where p' = thr / 2^16, thr = min(floor(dropout_p * 2^16), 2^16 - 1) (|p' - p| < 2^-16).
 * The keep mask Z is a pure function of (seed, bh, i, j): Philox4x32-10 (Salmon et al.,
 * SC 2011) with key (seed & 0xffffffff, seed >> 32) and counter (j / 8, i, bh, 0); its
 * four output words hold eight 16-bit values, value j % 8 being the low (even j) or high
 * (odd j) half of word (j % 8) / 2, and the element is kept iff that value is >= thr.
 * fa_bwd_dropout regenerates the same mask, so nothing N x N is stored.
 * Arguments as fa_fwd, plus dropout_p in [0, 1) (0 runs fa_fwd) and the 64-bit seed.
 * Dense layout; full or causal attention.
 */
int fa_fwd_dropout(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                   int Hq, int Hkv, int N, int d, int causal, float dropout_p,
                   unsigned long long seed, float scale, void *stream);

/*
 * Size in bytes of the fp32 scratch that fa_bwd needs: Delta_i = <dO_i, O_i> per query
 * row ([B, Hq, N] fp32) plus a dQ accumulator ([B, Hq, N, d] fp32), each padded to
 * 256 bytes.  Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d);

/*
 * Backward pass: gradients of <O, dO> with respect to Q, K and V.
 *   q, k, v, o, lse: as given to / produced by fa_fwd with the same sizes, causal, scale.
 *   dout [B, Hq, N, d] bf16 in (dL/dO)
 *   dq   [B, Hq, N, d] bf16 out;  dk, dv [B, Hkv, N, d] bf16 out (summed over the query
 *        heads that share each K/V head)
 *   workspace: device scratch of at least fa_bwd_workspace_bytes() bytes, 16-byte
 *        aligned; its contents on entry do not matter and on return are unspecified.
 * The score tiles are recomputed from Q, K and LSE (nothing N x N is stored).  At d = 256
 * the main kernel runs as clusters of two CTAs on two SMs (one forms P, the other dS; the
 * bf16 tiles cross through distributed shared memory), so dQ, dK and dV of this entry point
 * and of fa_bwd_window with a causal or unlimited band agree with the d = 256 paths of the
 * other entry points (packed, windowed, block-sparse, dropout) to rounding, not bit for bit.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
           const void *dout, void *dq, void *dk, void *dv, void *workspace,
           size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d, int causal,
           float scale, void *stream);

/* Scratch bytes fa_bwd_varlen needs: Delta ([total_q, Hq] fp32) and a dQ accumulator
 * ([total_q, Hq, d] fp32), each padded to 256 bytes.  0 for invalid sizes. */
size_t fa_bwd_varlen_workspace_bytes(int Hq, int total_q, int d);

/*
 * Backward pass of fa_fwd_varlen: arguments as fa_fwd_varlen plus dout [total_q, Hq, d],
 * dq [total_q, Hq, d], dk and dv [total_k, Hkv, d] (bf16; dK, dV summed over the query
 * heads of each K/V head) and a workspace of fa_bwd_varlen_workspace_bytes() bytes.  A key
 * that no query sees gets dK = dV = 0.  Offsets are checked as in the forward, with
 * max_seqlen_k bounding the key lengths.
 */
int fa_bwd_varlen(const void *q, const void *k, const void *v, const void *o, const float *lse,
                  const void *dout, void *dq, void *dk, void *dv, void *workspace,
                  size_t workspace_bytes, const int *cu_seqlens_q, const int *cu_seqlens_k, int B,
                  int Hq, int Hkv, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                  int d, int window_left, int window_right, float scale, void *stream);

/*
 * Backward pass of fa_fwd_dropout (same dropout_p and seed; O and LSE from it): arguments
 * as fa_bwd.  dV = sum_i P Z / (1 - p') dO, dS = P (Z dP / (1 - p') - Delta).
 */
int fa_bwd_dropout(const void *q, const void *k, const void *v, const void *o, const float *lse,
                   const void *dout, void *dq, void *dk, void *dv, void *workspace,
                   size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d, int causal,
                   float dropout_p, unsigned long long seed, float scale, void *stream);

/*
 * Backward pass of local attention: arguments as fa_bwd, with the window bounds of
 * fa_fwd_window in place of `causal`; q, k, v, o, lse must come from fa_fwd_window with
 * the same bounds.  Key blocks are visited only by the query blocks whose band meets them.
 */
int fa_bwd_window(const void *q, const void *k, const void *v, const void *o, const float *lse,
                  const void *dout, void *dq, void *dk, void *dv, void *workspace,
                  size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d, int window_left,
                  int window_right, float scale, void *stream);

/*
 * Block-sparse attention: the deep-dive page's closing paragraph names block-sparse
 * FlashAttention without defining it.  The library's reading: a 0/1 mask over the
 * 128 x 128 blocks of each query head's score matrix; key j is visible to query i iff
 * block_mask[b][h][i / 128][j / 128] != 0 (and, with causal = 1, j <= i).  Only enabled
 * blocks are loaded and multiplied; the others cost nothing.
 *   q, k, v, o, lse, B, Hq, Hkv, N, d, scale, stream: as fa_fwd (dense [B, H, N, d]).
 *   block_mask: DEVICE uint8 [B, Hq, nb, nb], nb = ceil(N / 128), row-major; any nonzero
 *        byte enables its block.  Read, never written; the caller keeps it alive until
 *        the call's kernels have run.  With causal = 1, blocks above the diagonal are
 *        ignored whatever their byte.
 * A row whose blocks are all disabled gets O = 0 and LSE = -inf.  Limits: nb <= 4096, and
 * (Hq / Hkv) * ceil(nb / 32) * 4 bytes of per-key-block bitmap for the backward within
 * its shared-memory budget (8192 bytes for d = 64 and 128, 1392 bytes for d = 256);
 * larger sizes return FA_ERR_UNSUPPORTED (checked by both calls, so a forward that runs
 * always has a backward).  A NULL mask or a causal flag other than 0/1 is
 * FA_ERR_INVALID_ARG.
 */
int fa_fwd_blocksparse(const void *q, const void *k, const void *v, void *o, float *lse,
                       const unsigned char *block_mask, int B, int Hq, int Hkv, int N, int d,
                       int causal, float scale, void *stream);

/*
 * Backward pass of fa_fwd_blocksparse (same mask and causal flag; O and LSE from it):
 * arguments as fa_bwd plus block_mask.  A key block is visited only by the query blocks
 * of the query heads that enable it; a key that no query sees gets dK = dV = 0, a query
 * that sees no key dQ = 0.
 */
int fa_bwd_blocksparse(const void *q, const void *k, const void *v, const void *o,
                       const float *lse, const void *dout, void *dq, void *dk, void *dv,
                       void *workspace, size_t workspace_bytes, const unsigned char *block_mask,
                       int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                       void *stream);

/*
 * Backward pass for callers that cannot allocate device memory.
 *
 * No counterpart on the pages: this is a library convenience.  Some callers are not
 * allowed to call cudaMalloc or a caching allocator at the point where they run the
 * backward pass - for example code running under a fixed, pre-reserved memory budget,
 * a real-time or latency-critical path where an allocation could block or fail, or a
 * framework hook that must not touch the allocator.  fa_bwd needs caller-provided
 * scratch; this variant takes none and instead uses one static device buffer of
 * FA_NOALLOC_SCRATCH_BYTES (64 MiB) compiled into the library.  That buffer exists on
 * every GPU that loads the library, for as long as the process lives.
 *
 * Arguments, layout and results are those of fa_bwd without `workspace` and
 * `workspace_bytes`.  The problem fits when fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) <=
 * FA_NOALLOC_SCRATCH_BYTES (for d = 128 about 130 000 query rows B*Hq*N); larger problems
 * return FA_ERR_SCRATCH_LIMIT before anything is launched.  No call allocates memory.
 *
 * The first call on a device (with that device current) looks up the buffer's device
 * address; make that first call before any stream capture.  A lookup that fails returns
 * FA_ERR_CUDA, leaves no error pending in the CUDA runtime and is retried by the next
 * call; once it has succeeded it is not repeated.  Every call on a device
 * shares the same buffer, which keeps the previous call's contents (the kernels
 * re-initialise what they need), so calls whose kernels overlap on the GPU - on different
 * streams without ordering between them - race on it: order them on one stream or with
 * events.
 */
#define FA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const float *lse,
                   const void *dout, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int N,
                   int d, int causal, float scale, void *stream);

/*
 * Decode: attention of Nq new query rows against a key/value cache of Nk rows.
 *
 * Source: the "FlashAttention1" Q&A page names incremental attention updates for
 * streaming inference (question on scaling to long sequences, item 8) and the combination
 * of partial results from different blocks by a reduction (question on the key
 * algorithmic innovations, item 3).  The pages give no decode algorithm; this is the
 * library's reading: the keys are split into `num_splits` ranges processed in parallel,
 * and the partial results (O_s normalised, LSE_s) are merged as
 *     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s.
 *
 *   q    [B, Hq, Nq, d] bf16 in        k, v [B, Hkv, Nk, d] bf16 in (the cache)
 *   o    [B, Hq, Nq, d] bf16 out       lse  [B, Hq, Nq] fp32 out (natural log)
 *   seqlens_k: DEVICE int32 [B] (4-byte aligned), valid keys per batch (the first
 *        seqlens_k[b] rows of the cache; values are clamped to [0, Nk]), or NULL for Nk.
 *   causal: 0 or 1; with 1 the Nq queries are the LAST Nq positions of the sequence
 *        (bottom-right alignment): query t sees keys j <= seqlens_k[b] - Nq + t.
 *   num_splits: 1 .. 1024 key ranges (fa_decode_num_splits gives the library's choice).
 *   workspace: device scratch of fa_decode_workspace_bytes() bytes, 16-byte aligned (may be
 *        NULL when that is 0, i.e. num_splits == 1).
 * Rows that see no key (seqlens_k[b] == 0, or causal with seqlens_k[b] < Nq) get O = 0 and
 * LSE = -inf.  Limits: (Hq / Hkv) * Nq <= 128 (<= 64 for d = 256) query rows per K/V head
 * (longer query blocks belong to fa_fwd), Nk <= 2^30, B * Hq * Nq < 2^31,
 * B * Hkv * Nk < 2^31; other sizes return FA_ERR_UNSUPPORTED.
 */
int fa_decode(const void *q, const void *k, const void *v, void *o, float *lse,
              const int *seqlens_k, void *workspace, size_t workspace_bytes, int B, int Hq,
              int Hkv, int Nq, int Nk, int d, int causal, int num_splits, float scale,
              void *stream);

/*
 * The library's split count for fa_decode: enough (b, K/V head, key range) units to fill
 * the current device's SMs once, with at least two 128-key blocks per range.  Returns 0
 * for sizes fa_decode rejects.
 */
int fa_decode_num_splits(int B, int Hq, int Hkv, int Nq, int Nk, int d);

/* Scratch bytes fa_decode needs for `num_splits` (0 when num_splits == 1 or invalid). */
size_t fa_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_splits);

/*
 * Merge of `num_parts` partial attention results over disjoint key sets (the reduction
 * that fa_decode uses, exposed for callers that compute the parts themselves, e.g. over
 * key ranges held by different devices):
 *   o_parts   [num_parts, rows, d] fp32 in (each part normalised by its own sum)
 *   lse_parts [num_parts, rows]    fp32 in (natural log; -inf for a part with no key)
 *   o [rows, d] bf16 out,  lse [rows] fp32 out
 * A row whose parts are all -inf gets O = 0 and LSE = -inf.  d in {64, 128, 256}.
 */
int fa_merge(const float *o_parts, const float *lse_parts, void *o, float *lse, int num_parts,
             int rows, int d, void *stream);

/*
 * Synchronises `stream`, returns the device status word of the current device
 * (FA_OK, FA_ERR_DEVICE_TIMEOUT or FA_ERR_SEQLENS) and clears it.  Returns FA_ERR_CUDA if the
 * synchronisation itself fails.
 */
int fa_device_status(void *stream);

/*
 * Kernel timing for benchmarks.  fa_kernel_timing(1) resets the counters and makes every
 * later fa_fwd / fa_bwd / fa_decode call (and their window, varlen, dropout and
 * block-sparse forms, and fa_bwd_noalloc) in this process record
 * a pair of CUDA events (created by the
 * library, no device memory) around its main attention kernel, on the call's stream;
 * fa_kernel_timing(0) stops recording.  fa_kernel_time_ms(which, &ms, &launches)
 * synchronises those events and returns the summed device time in milliseconds and the
 * number of launches recorded since the reset: which = 0 for the forward kernel, 1 for
 * the backward main kernel (the Delta and dQ-conversion kernels are not included), 2 for
 * the decode kernel (the merge kernel is not included).  At
 * most 4096 launches per kind are recorded; later ones are not counted.  Returns FA_OK,
 * FA_ERR_INVALID_ARG or FA_ERR_CUDA.  Not thread-safe.
 */
int fa_kernel_timing(int enable);
int fa_kernel_time_ms(int which, float *ms, int *launches);

/*
 * Forward tile scheduler for dense full and causal attention with d = 64 or 128 (fa_fwd,
 * fa_fwd_window with bands (-1, -1) / (-1, 0), fa_fwd_dropout).  The FlashAttention-2
 * page ("Better Parallelism") parallelises over batch x heads x query blocks; here a work
 * unit is two 128-row query tiles, numbered heaviest first under a causal mask.
 *   persistent = 1 (default): one CTA per SM walks the units, taking each next unit from a
 *       device counter (dynamic assignment), so one unit's epilogue overlaps the next
 *       unit's loads and first products.  The counter is one of 64 library-owned launch
 *       slots, taken in turn by successive launches and reset by each launch's last CTA;
 *       a launch captured in a CUDA graph keeps its slot, so replays of that graph must
 *       not run on the GPU at the same time as the launch that takes the same slot 64
 *       launches later.
 *   persistent = 0: one CTA per unit, started by the hardware in unit order.
 * The environment variable FA_FWD_PERSISTENT=0, read when the library loads, makes
 * one CTA per unit the starting choice.
 * Both compute bit-identical O and LSE.  Other variants (d = 256, other bands, packed
 * sequences, block masks) always use one CTA per unit.  Affects later calls of this
 * process; returns the previous setting, or FA_ERR_INVALID_ARG.  Not synchronised with
 * calls running on other host threads.
 */
int fa_set_fwd_scheduler(int persistent);
/* The current choice (1: persistent, 0: one CTA per unit). */
int fa_get_fwd_scheduler(void);

/*
 * Watchdog self-test: launches one thread that waits, with a limit of `limit_us`
 * microseconds (1 .. 10^7), on a pipeline barrier that nothing ever signals - the same
 * bounded-wait code every attention kernel uses.  The wait expires, the kernel records
 * FA_ERR_DEVICE_TIMEOUT in the device status word and returns normally, so a following
 * fa_device_status() reports the timeout and the CUDA context stays usable.  Returns
 * FA_OK once enqueued, FA_ERR_INVALID_ARG or FA_ERR_CUDA.
 */
int fa_watchdog_selftest(int limit_us, void *stream);

/* Static, human-readable text for a status code. */
const char *fa_status_string(int code);

/* Library ABI version (major * 100 + minor). */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H */
