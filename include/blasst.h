/*
 * blasst.h -- C ABI of libblasst.so: BLASST blocked attention with
 * softmax-threshold block skipping on NVIDIA B200 (sm_100a).
 *
 * The method (BLASST: "Dynamic BLocked Attention Sparsity via Softmax
 * Thresholding", arXiv:2512.12087):
 *   attention = softmax(Q K^T * scale) V  (xllm-io paper review, section 3,
 *   "core formulas"), computed FlashAttention-style over KV blocks in order
 *   with a running row max m.  A KV block j is skipped for a query tile when
 *   every row r of the tile that sees a key of the block satisfies
 *       m~_r(j) - max(m_r, m~_r(j)) < ln(lambda)
 *   where m~_r(j) is the row max of the block's scaled scores (same section,
 *   skip condition; gist.science (de) summary, section 2 "Kernidee").  A
 *   skipped block adds nothing to the row sum l or to O; its exp, its V load
 *   (decode) and its P.V product are not done (gist.science (de), section 2;
 *   fugumt abstract).  The first visited block of a tile is never skipped
 *   (nervesearch commentary, six-block figure).  lambda = 0 means dense.
 *
 * Conventions common to every entry point
 *   - Tensors are row-major and head-major: q [B, Hq, Lq, d], k [B, Hkv, Lk,
 *     *], v [B, Hkv, Lk, *], o [B, Hq, Lq, dv] in bf16 (raw 16-bit words),
 *     lse [B, Hq, Lq] fp32 natural-log logsumexp of the kept scores.  k and v
 *     rows hold k_row_stride / v_row_stride elements (default d / dv), so an
 *     MLA latent cache can pass the same buffer as k and v with dv < d.
 *   - Every pointer argument is a DEVICE pointer (except in the host-only
 *     functions marked so).  q, k, v, o must be 16-byte aligned; row strides
 *     must be multiples of 8 elements.  The caller owns every buffer; the
 *     library keeps no per-call state (TMA descriptors are built on the host
 *     for each call), and calls on different streams may run concurrently.
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only enqueues work on it and returns; results are ready when the stream
 *     is synchronised.
 *   - Causal masking is aligned bottom-right: query i may see keys
 *     0 .. i + (Lk - Lq).  causal requires Lq <= Lk.
 *   - lambda must be finite with 0 <= lambda < 1; scale must be > 0.
 *   - skip_mask (nullable) receives one bit per (query tile, KV block), 1 =
 *     skipped, as rows of W = ceil(n_blocks / 32) uint32 words: bit (j % 32)
 *     of word (j / 32) is block j.  Prefill: rows [B, Hq, ceil(Lq / 128)],
 *     128 queries per tile, blocks of 128 keys.  Decode: rows [B, Hkv, 1], the
 *     tile being all G = Hq/Hkv query heads x Lq queries of one KV head,
 *     blocks of 64 keys.  The library writes every word of the mask (blocks a
 *     tile never visits read 0).
 *   - skip_count (nullable) is one uint64 on the device: the library sets it
 *     to the number of skipped (tile, block) pairs of the call.  The
 *     denominator, visited pairs, comes from blasst_visited_pairs().
 *   - Errors: invalid arguments return BLASST_ERR_INVALID / _UNSUPPORTED /
 *     _WORKSPACE before anything is enqueued; a failed CUDA call returns
 *     BLASST_ERR_CUDA (text via blasst_last_error()).  Device-side bounded
 *     waits that time out write a nonzero code into opts->status_word (when
 *     given) and make the kernel return early; the host sees it after
 *     synchronising.  No C++ exception crosses this interface.
 */
#ifndef BLASST_H
#define BLASST_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BLASST_API __attribute__((visibility("default")))
#else
#define BLASST_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BLASST_OK = 0,
    BLASST_ERR_INVALID = 1,     /* bad pointer, shape, scale or lambda */
    BLASST_ERR_UNSUPPORTED = 2, /* valid in principle, not built (e.g. head dim) */
    BLASST_ERR_WORKSPACE = 3,   /* caller's workspace too small */
    BLASST_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
    BLASST_ERR_TIMEOUT = 5      /* device status word: a bounded wait expired */
} blasst_status;

/* Optional arguments; pass NULL for all defaults.  struct_size must be
 * sizeof(blasst_opts) as compiled by the caller (ABI versioning): fields past
 * struct_size are treated as zero. */
typedef struct blasst_opts {
    size_t struct_size;
    int dv;                    /* value head dim; 0 -> d.  MLA: d = 576, dv = 512 */
    int block_n;               /* 0, or the fixed block size (128 prefill, 64 decode) */
    int num_splits;            /* decode: KV chunks per sequence; 0 -> 16 (d = 128) or 2
                                  (MLA, d = 576); -1 -> adaptive for d = 128
                                  (blasst_decode_pick_splits_rows with the tile's rows
                                  G * Lq and this device's SM count; MLA rejects it
                                  with BLASST_ERR_INVALID) */
    int mode;                  /* blasst_calibrate only: 0 = prefill tiling, 1 = decode tiling */
    long long k_row_stride;    /* elements between consecutive keys; 0 -> d */
    long long v_row_stride;    /* elements between consecutive values; 0 -> dv */
    void *workspace;           /* decode partials; NULL -> stream-ordered cudaMallocAsync */
    size_t workspace_bytes;
    float *gaps_out;           /* device, per (tile, block) pair: max over rows of
                                  m~ - max(m, m~) in natural-log units; +inf on a
                                  tile's (split's) first block, NaN if not visited */
    unsigned int *status_word; /* device word the caller zeroes; the library ORs in
                                  a nonzero code when a bounded wait expires */
    int seed_splits;           /* decode only (d = 128 tiles of any width, and MLA):
                                  nonzero seeds the running
                                  max of every split after the first with the row
                                  maxima of block 0, and such a split has no forced
                                  first block.  Block 0 enters those splits only
                                  through the comparison (one extra 64-key Q.K^T per
                                  split); it lifts the cap that restarting the max
                                  puts on sparsity.  Not a rule of the paper: a
                                  restatement of its single-pass rule (block 0's
                                  maxima are part of the running max) for split-KV.
                                  Other paths return BLASST_ERR_UNSUPPORTED. */
} blasst_opts;

/*
 * Prefill: Lq queries attend to Lk keys per sequence, query tiles of 128
 * rows of one query head, KV blocks of 128 keys, kv head = hq / (Hq / Hkv).
 * d = dv = 128 only.  QK^T is computed for every visited block; the skip
 * decision then omits exp and the P.V tensor-core product of skipped blocks
 * (xllm-io paper review, section 3 "prefill kernel optimisation").
 */
BLASST_API blasst_status blasst_prefill(const void *q, const void *k, const void *v, void *o, float *lse,
                             int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, float lambda,
                             int causal, uint32_t *skip_mask, unsigned long long *skip_count,
                             void *stream, const blasst_opts *opts);

/*
 * Decode: the G = Hq/Hkv query heads x Lq queries of one KV head form the
 * tile (G * Lq <= 128; up to 16 rows on mma.sync, 17 to 128 rows -- MQA with
 * many heads, large GQA groups -- on tcgen05 with the tile in tensor memory),
 * KV blocks of 64 keys, split-KV over num_splits
 * contiguous chunks of ceil(n_blocks / num_splits) blocks.  Each split is an
 * independent online-softmax pass (running max restarts, its first block is
 * kept); the skip decision for a block is taken after its K block is read and
 * before any load of its V block, V is loaded only for kept blocks (xllm-io
 * paper review, section 3 "decode kernel optimisation"), then a combine step
 * merges the splits exactly on lse.  d = dv = 128 (GQA/MQA).
 * Workspace: blasst_decode_workspace_bytes() bytes, 256-byte aligned.
 */
BLASST_API blasst_status blasst_decode(const void *q, const void *k, const void *v, void *o, float *lse,
                            int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, float lambda,
                            int causal, uint32_t *skip_mask, unsigned long long *skip_count,
                            void *stream, const blasst_opts *opts);

/*
 * Decode over an FP8 (e4m3, OCP "E4M3FN": bias 7, no infinities) KV cache.
 * Not on the pages: a storage format that halves the bytes of K and V, which
 * decode reads from HBM once per step.  Experimental: on B200 this kernel is
 * bound by the conversion of the bytes to f16, not by HBM, and runs slower
 * than blasst_decode over a bf16 cache; what it saves is the cache's memory.  The cache holds K = k_scale * k8 and
 * V = v_scale * v8 (per-tensor scales, finite and > 0); the arithmetic is
 * exactly blasst_decode's on those dequantized values (same tile, 64-key
 * blocks, splits, skip rule, combine), with one difference in rounding: the
 * products run in f16 (e4m3 -> f16 is exact; q is re-rounded from bf16 to
 * f16, which is exact for |q| in f16's normal range, 6.1e-5 .. 65504; P is
 * rounded to f16 before P.V).
 *
 * k8, v8  [B, Hkv, Lk, 128] bytes (e4m3), 16-byte aligned, dense rows.
 * q, o, lse, skip_mask, skip_count, stream and opts (num_splits, workspace,
 * status_word, seed_splits) as blasst_decode.  d = 128 and G * Lq <= 16 only
 * (BLASST_ERR_UNSUPPORTED otherwise); non-finite or non-positive scales are
 * BLASST_ERR_INVALID.
 */
BLASST_API blasst_status blasst_decode_fp8(const void *q, const void *k8, const void *v8, void *o, float *lse,
                                           int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                                           float k_scale, float v_scale, float lambda, int causal,
                                           uint32_t *skip_mask, unsigned long long *skip_count, void *stream,
                                           const blasst_opts *opts);

/*
 * Decode over a paged, ragged KV cache.  Not on the pages as such: they report
 * the method integrated into serving frameworks (xllm-io paper review,
 * overview table; gist.science (de), section 1), whose caches are paged.  Per
 * sequence the arithmetic is exactly blasst_decode's (same tile, 64-key blocks,
 * num_splits chunks of that sequence's own blocks, lse combine, skip rule).
 *
 * k_pages, v_pages  [num_pages, Hkv, 64, d] bf16, dense: one 64-key page of one
 *                   KV head is 64 x d contiguous elements.  d = dv = 128.
 * block_table       device int32 [B, max_pages]: sequence b's block i lives in
 *                   page block_table[b * max_pages + i].
 * seq_lens          device int32 [B]: keys of sequence b, 0 .. max_pages * 64.
 *                   Causal decode needs Lq <= seq_lens[b] (rows that see no key
 *                   give O = 0 and lse = -inf).
 * q, o, lse, skip_mask ([B, Hkv, W], W = ceil(max_pages / 32) words; blocks past
 * a sequence's end are 0), skip_count, stream and opts (num_splits, workspace,
 * status_word, seed_splits) as blasst_decode.  Argument errors return before
 * any launch.  The device arrays are read by the kernel: a page index outside
 * [0, num_pages) or a length outside [0, max_pages * 64] is not checked on the
 * host; the kernel then reads zeros for that page (or clamps the length) and
 * ORs 2 into *opts->status_word when given.
 */
BLASST_API blasst_status blasst_decode_paged(const void *q, const void *k_pages, const void *v_pages, void *o,
                                             float *lse, const int *block_table, const int *seq_lens, int B, int Hq,
                                             int Hkv, int Lq, int max_pages, int num_pages, int d, float scale,
                                             float lambda, int causal, uint32_t *skip_mask,
                                             unsigned long long *skip_count, void *stream, const blasst_opts *opts);

/*
 * Attention backward with the forward's skip mask held fixed (prefill tiling:
 * query tiles of 128 rows of one query head, KV blocks of 128 keys, d = dv =
 * 128).  The pages describe an optional sparsity-aware training in which the
 * forward skips blocks and the skipped blocks receive no gradient (xllm-io
 * paper review, section 3, "training procedure").  With the mask fixed the
 * forward is plain masked softmax attention over the kept pairs, and this
 * call returns its exact gradient up to rounding:
 *   P = exp(scale*QK^T - lse) on kept, visible scores (0 elsewhere),
 *   dV = P^T dO, dP = dO V^T, D = rowsum(dO * O), dS = P * (dP - D),
 *   dQ = scale * dS K, dK = scale * dS^T Q  (dK, dV summed over the G query
 *   heads of each KV head).
 *
 * q, k, v, o, lse  the forward's inputs and outputs (o, lse as blasst_prefill
 *                  wrote them); dout [B, Hq, Lq, 128] bf16, the gradient of o.
 * dq [B, Hq, Lq, 128], dk, dv [B, Hkv, Lk, 128]: bf16 outputs, fully written.
 * skip_mask        the forward's mask (layout as above; blocks a tile never
 *                  visits must read 0), or NULL: nothing skipped.
 * causal           as in the forward.
 * opts             workspace (>= blasst_backward_workspace_bytes() bytes,
 *                  256-byte aligned; NULL -> stream-ordered cudaMallocAsync)
 *                  and status_word; dv, strides and block_n must be defaults.
 * Rounding: P and dS enter the tensor-core products as bf16, accumulation is
 * fp32, dQ is accumulated across key blocks in an fp32 workspace by atomic
 * adds (so the order of those additions, and the last bits of dq, can vary
 * from run to run; dk and dv are deterministic).
 */
BLASST_API blasst_status blasst_prefill_backward(const void *q, const void *k, const void *v, const void *o,
                                                 const float *lse, const void *dout, void *dq, void *dk, void *dv,
                                                 int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                                                 int causal, const uint32_t *skip_mask, void *stream,
                                                 const blasst_opts *opts);
/* Workspace of blasst_prefill_backward: an fp32 dQ accumulator and two fp32
 * rows per query, padded to whole 128-row tiles.  0 for invalid sizes. */
BLASST_API size_t blasst_backward_workspace_bytes(int B, int Hq, int Lq);

/*
 * Calibration pass: the decision part of prefill (opts->mode = 0) or decode
 * (mode = 1) only -- QK^T, block row maxima, running max, gaps -- without
 * exp, P.V or V traffic.  v, o and lse may be NULL and are not touched.
 * Writes opts->gaps_out (required) and, for the given lambda, skip_mask and
 * skip_count exactly as the matching attention call would.  One pass serves
 * every lambda: a skipped block never raises the running max, so a pair is
 * skipped at lambda iff its gap < ln(lambda) (xllm-io paper review, section 3,
 * "calibration module": one forward pass).
 */
BLASST_API blasst_status blasst_calibrate(const void *q, const void *k, const void *v, void *o, float *lse,
                               int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale, float lambda,
                               int causal, uint32_t *skip_mask, unsigned long long *skip_count,
                               void *stream, const blasst_opts *opts);

/*
 * HOST-ONLY.  Least-squares fit of ln(lambda_i * L_i) = ln(alpha) + beta * s_i
 * over n >= 2 points: the calibration model lambda * L = alpha * exp(beta * s)
 * (xllm-io paper review, section 3, "calibration model").  Host arrays.
 */
BLASST_API blasst_status blasst_calibrate_fit(const double *L, const double *lambda, const double *sparsity, int n,
                                   double *alpha, double *beta);

/*
 * HOST-ONLY.  From n gaps of one calibration pass (host copy of gaps_out),
 * the lambda whose sparsity (skipped / visited pairs) is closest to
 * target_sparsity, and the sparsity it reaches.  NaN entries are not visited,
 * +inf entries are first blocks (visited, never skipped).
 */
BLASST_API blasst_status blasst_calibrate_threshold(const float *gaps, long long n, double target_sparsity,
                                         double *lambda_out, double *achieved_out);

/*
 * Decode that allocates nothing.  The paper has no counterpart: this is a
 * deployment variant of blasst_decode for callers that cannot allocate device
 * memory while they run -- e.g. an engine that reserves (nearly) all device
 * memory for its own pool up front, so any further cudaMalloc/cudaMallocAsync
 * fails or fragments it, or a latency-critical loop where an allocation or a
 * free could stall the device.  Same arguments, results and errors as
 * blasst_decode, except:
 *   - the split partials live in one fixed device array owned by the library
 *     (BLASST_NOALLOC_SCRATCH_BYTES per GPU, held from library load until
 *     process exit); opts->workspace must be NULL;
 *   - calls needing more than BLASST_NOALLOC_SCRATCH_BYTES of partials
 *     (blasst_decode_workspace_bytes) return BLASST_ERR_WORKSPACE with the
 *     sizes in blasst_last_error();
 *   - the first call on each device (in each CUDA context) looks up the
 *     array's device address (cudaGetSymbolAddress, which loads the module
 *     on that device) and caches it for later calls in that context; make
 *     that first call before any stream capture.  The cached address does
 *     not survive cudaDeviceReset: after a reset of a device, do not call
 *     this function on that device again in the same process;
 *   - every call on a device shares the one array and it keeps the last
 *     call's contents (nothing in it needs clearing: each call writes every
 *     partial it reads), so calls that may overlap on the GPU -- on different
 *     streams or from different host threads -- race: serialise them.
 * num_splits (0, positive or -1) and dv are resolved exactly as blasst_decode
 * resolves them before the size check.  It calls no cudaMalloc,
 * cudaMallocAsync, cudaFree or other allocating routine.
 */
#define BLASST_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
BLASST_API blasst_status blasst_decode_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                                               int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                                               float lambda, int causal, uint32_t *skip_mask,
                                               unsigned long long *skip_count, void *stream,
                                               const blasst_opts *opts);

/* Bytes of decode workspace for these sizes (num_splits 0 -> 16, dv 0 -> 128). */
/* Host only.  The split count that num_splits = -1 selects for a decode of B
 * sequences x Hkv KV heads over Lk keys on a device with num_sms SMs: about
 * 16 CTAs per SM over the call (ceil(16 * num_sms / (B * Hkv))), but at least
 * 32 blocks of 64 keys per split, and at most 64 splits; 1 for short caches.
 * Not on the pages (split-KV is not); it follows a measured sweep on B200:
 * batch 32 x 8 KV heads at 32K keys is as fast at 8-16 splits as at any count
 * and loses reachable sparsity past 16, while batch 1 needs 16-32 to fill the
 * device.  A decode that used -1 is reproduced by passing this count
 * explicitly (the skip mask depends on the split count).  Size a caller
 * workspace with it too.  Invalid sizes return 1. */
BLASST_API int blasst_decode_pick_splits(int B, int Hkv, int Lk, int num_sms);

/* Host only.  The split count that num_splits = -1 selects for a tile of rows
 * = G * Lq query rows: blasst_decode_pick_splits for tiles of up to 16 rows;
 * for wider tiles (the tcgen05 kernel, two CTAs per SM) floor(4 * num_sms /
 * (B * Hkv)) -- the most splits that keep the grid within two full waves of
 * two CTAs per SM -- under the same cap (at least 32 blocks of 64 keys per
 * split, at most 64) and at least 1.  Measured on B200 for 128 query heads on
 * one KV head, batch 64, 32K keys (dense ms): 8 splits 0.214, 9 splits 0.208
 * (this rule), 10 splits 0.253, 12 splits 0.233, 16 splits 0.237; past two
 * waves the last one runs partly empty.  Invalid sizes return 1. */
BLASST_API int blasst_decode_pick_splits_rows(int B, int Hkv, int rows, int Lk, int num_sms);

BLASST_API size_t blasst_decode_workspace_bytes(int B, int Hq, int Lq, int dv, int num_splits);

/* Number of visited (tile, block) pairs: the sparsity denominator.
 * is_decode selects the decode tiling; -1 on invalid sizes. */
BLASST_API long long blasst_visited_pairs(int B, int Hq, int Hkv, int Lq, int Lk, int causal, int is_decode,
                               const blasst_opts *opts);

/* Static text for a status code. */
BLASST_API const char *blasst_status_string(blasst_status s);

/* Text of the last CUDA failure seen by this thread ("" if none). */
BLASST_API const char *blasst_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BLASST_H */
