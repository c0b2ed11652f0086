/*
 * rf.h -- C ABI of librf, the B200 (sm_100a) RainFusion v2 block-sparse
 * video attention path.
 *
 * The path (one call each, all asynchronous on the caller's stream):
 *   rf_rearrange          (t,h,w) token permutation with suffix promotion, for
 *                         Q, K and V in one launch; also writes the 128-row
 *                         block means of Q and K into the workspace.
 *   rf_pool_select        per-query-block ranking of key blocks by block-mean
 *                         scores; writes selectIdx / selectNum.
 *   rf_block_sparse_attn  Softmax(scale * Q K^T) V over the selected blocks,
 *                         fp32 softmax, tcgen05 tensor cores.
 *   rf_inverse_rearrange  scatter of the output back to the original order.
 *   rf_forward            the four steps above in one call.
 *
 * Sources (the web pages the method is described on):
 *   [UG]  "RainFusion Attention" user guide (vllm-omni docs): opening
 *         paragraphs, "Configuration", "Geometry handling".
 *   [PR]  xllm pull request "feat: add RainFusion sparse attention for
 *         wan2.2" (#1867): change summary (rearrange, inverse, QKV in one
 *         call, round-trip check).
 *   [API] CANN "aclnnRainFusionAttention" API page: "Formula", the two-phase
 *         call (workspace size, then execute), and the constraints list.
 *   [ABS] RainFusion2.0 abstract: block means as representative tokens,
 *         spatiotemporal token permutation, first-frame sink.
 *   [MX]  "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
 *         Quantization for MXFP4 Attention", abstract: MXFP4 attention, UOS
 *         scaling boundary Qmax = 7.25, PNQ.
 *
 * Conventions (all entry points):
 *   - Every pointer named q, k, v, *_r, o, select_idx, select_num or ws is a
 *     DEVICE pointer owned by the caller; the library never frees or keeps it
 *     beyond the call.  The library owns only the host-side plan.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     enqueue work and return; they do not synchronise (except
 *     rf_check_device_status).
 *   - The return value reports host-side validation and launch errors.  A
 *     call that returns an error enqueued nothing.
 *   - Device-side problems (an out-of-range selectIdx entry, an expired
 *     bounded wait) never trap: the kernel records them in the workspace
 *     status words and skips the offending work; rf_check_device_status
 *     reports them as RF_ERR_DEVICE_FAULT.
 *   - Only sm_100 devices are accepted (RF_ERR_UNSUPPORTED_DEVICE
 *     otherwise), as [UG] "Requirements" has the NPU backend raise on any
 *     other platform.
 *
 * Tensor layouts ([API] "Formula": TND and BNSD):
 *   BNSD: Q [B, N1, L, D], K/V [B, N2, L, D], every batch element has the
 *         same geometry (one rf_seq_geom_t).
 *   TND:  Q [T, N1, D], K/V [T, N2, D]; sequences are packed back to back
 *         along T in the order given to rf_plan_create.
 *   All tensors are contiguous, dtype bf16 or fp16 (Q, K and V share it,
 *   [API] constraints), D in {64, 128}.  Original row order of a sequence:
 *   [text/condition prefix (prefix_len rows) | video in raster (t, y, x)].
 *   Rearranged order: [prefix | promoted video rows | sparse video rows in
 *   8x8-tile order], i.e. Lp = prefix_len + promoted dense rows, then
 *   nb = S / 128 sparse blocks.
 */
#ifndef RF_H_
#define RF_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RF_API __attribute__((visibility("default")))
#else
#define RF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* rf_stream_t; /* == cudaStream_t */

typedef enum {
  RF_OK = 0,
  RF_ERR_INVALID_ARG = 1,         /* an argument breaks a documented constraint */
  RF_ERR_UNSUPPORTED_DEVICE = 2,  /* no CUDA device, or not sm_100 */
  RF_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < rf_plan_info().workspace_bytes */
  RF_ERR_CUDA = 4,                /* a CUDA runtime / driver call failed */
  RF_ERR_DEVICE_FAULT = 5,        /* a kernel recorded a bad index or an expired wait */
  RF_ERR_UNSUPPORTED = 6          /* allowed by the pages but not built here */
} rf_status_t;

typedef enum { RF_LAYOUT_BNSD = 0, RF_LAYOUT_TND = 1 } rf_layout_t;
typedef enum { RF_BF16 = 0, RF_FP16 = 1 } rf_dtype_t;

/* How rf_pool_select obtains the block means of Q and K. */
typedef enum {
  RF_POOL_FROM_WS = 0,   /* use the means rf_rearrange wrote into this same workspace */
  RF_POOL_RECOMPUTE = 1  /* recompute them from q_r / k_r first */
} rf_pool_mode_t;

/* Token order of the aligned video tokens in the rearranged sequence.
 *   RF_ORDER_TILE       8x8 spatial tiles of one frame in (frame, tile row,
 *                       tile column, row, column) order: a 128-row block is
 *                       two adjacent tiles of one frame ([UG] opening
 *                       paragraph and "Geometry handling": (t, h, w) order).
 *   RF_ORDER_FRAME_PAIR the frame-pairing variant of [PR] (change summary:
 *                       frame-pairing approach, first frame before the rest):
 *                       frame 0 in tile order, then frames (1,2), (3,4), ...
 *                       cube by cube, a cube being the same 8x8 tile of both
 *                       frames (128 rows: frame in pair, row, column), then
 *                       an unpaired last frame in tile order.
 * Both orders give the same counts (sparse rows, promoted rows, blocks,
 * sinks); only the order of the aligned tokens differs. */
typedef enum { RF_ORDER_TILE = 0, RF_ORDER_FRAME_PAIR = 1 } rf_token_order_t;
/* One sequence: text/condition prefix length and video latent grid
 * ([UG] "Geometry handling").  t, h, w >= 0; prefix_len >= 0; length > 0. */
typedef struct {
  int32_t prefix_len;
  int32_t t, h, w;
} rf_seq_geom_t;

/* Sizes derived by rf_plan_create (phase one of the two-phase call, [API]). */
typedef struct {
  int64_t rows_total;      /* rows per head: BNSD B*L, TND T */
  int64_t t_qblk;          /* total query blocks over all sequences ([API] selectIdx dim 0) */
  int64_t max_kv_blocks;   /* selectIdx dim 2 = max over sequences of n_pb_kv + nb_kv (n_pb + nb
                            * with 128-row key blocks) */
  int64_t workspace_bytes; /* device workspace every call below needs */
  int64_t pooled_blocks;   /* total sparse blocks over sequences (block means per head) */
  int64_t kept_flops_upper;/* 4*D*rows_q*rows_kv over the maximal selection (for reporting) */
  int64_t ws_pooled_q;     /* byte offset in ws of the Q block means, fp32 [n1][pooled_blocks][d] */
  int64_t ws_pooled_k;     /* byte offset in ws of the K block means, fp32 [n2][pooled_k_blocks][d] */
  int32_t n_seqs;          /* sequences (BNSD: batch elements) */
  int32_t n1, n2, d;
  int32_t precision;       /* rf_precision_t of the plan */
  int32_t token_order;     /* rf_token_order_t of the plan */
  /* RF_PRECISION_MIX and RF_PRECISION_FP8 (else -1): byte offsets in ws of the
   * E4M3 copies of Q' and K' (uint8, same layout and strides as q_r / k_r with
   * one byte per element) and of their scales (fp32 [n1][t_qblk] and
   * [n2][t_qblk], indexed by global query-block number).  RF_PRECISION_MXFP4 at
   * head dim 128 uses ws_q8 and ws_k8 for its E4M3-carried MXFP4 values and has
   * no scales (ws_q_scale = ws_k_scale = -1). */
  int64_t ws_q8, ws_k8, ws_q_scale, ws_k_scale;
  /* RF_PRECISION_MXFP4 at head dim 64 only (else -1): byte offsets in ws of
   * the MXFP4-rounded copies of Q', K' (the inputs' 16-bit type) and V' (always
   * f16), each with the layout and strides of q_r / k_r / v_r. */
  int64_t ws_q_mx, ws_k_mx, ws_v_mx;
  /* RF_PRECISION_FP8 only (else -1): byte offsets in ws of the E4M3 codes of V'
   * and of their exponents.  The codes are stored transposed per block, uint8
   * [n2][t_qblk][d][128]: for head h and global block t, column c of the block
   * holds its 128 keys contiguously (rows past a partial block's end are 0).
   * The exponents are int32 [n2][t_qblk]: the codes of block t of head h
   * represent code * 2^exp. ws_q8 .. ws_k_scale are as for RF_PRECISION_MIX.
   * RF_PRECISION_MXFP4 at head dim 128 stores its E4M3-carried V' in ws_v8 in
   * the same transposed layout, with no exponents (ws_v_exp = -1). */
  int64_t ws_v8, ws_v_exp;
  /* key block means per key/value head: pooled_blocks, or 2 * pooled_blocks
   * with blockShape 128 x 64 (the means of the 64-row key blocks) */
  int64_t pooled_k_blocks;
} rf_plan_info_t;

/* Per-sequence geometry under suffix promotion ([UG] "Geometry handling"). */
typedef struct {
  int64_t row_offset;  /* first row of the sequence along the row axis (TND T; BNSD 0) */
  int64_t length;      /* L = prefix_len + t*h*w */
  int64_t lp;          /* dense prefix rows after promotion */
  int64_t sparse;      /* S = 128 * nb */
  int64_t promoted;    /* video rows moved into the dense prefix */
  int32_t n_pb;        /* prefix blocks = ceil(lp / 128); the last may be partial */
  int32_t nb;          /* sparse video blocks */
  int32_t ns;          /* first-frame sink blocks */
  int32_t k;           /* ranked key blocks kept per sparse query block */
  int32_t qblk_offset; /* first global query block of this sequence */
  int32_t dense;       /* 1: the sequence runs dense (nb < 32, [UG]) */
  /* Key-side counts of the selection.  128-row key blocks: n_pb, nb, ns, k.
   * 64-row key blocks (blockShape 128 x 64): ceil(lp / 64) prefix key blocks,
   * 2 * nb sparse key blocks, min(nb_kv, ceil(h8 * w8 / 64)) first-frame sinks
   * and k_kv = ceil((1 - sparsity) * nb_kv) ranked blocks kept (nb_kv if dense). */
  int32_t n_pb_kv, nb_kv, ns_kv, k_kv;
} rf_seq_info_t;

typedef struct rf_plan rf_plan_t;

/* Phase one: validate the problem and derive every size.  Host only; no
 * device is touched, so it also works on a machine without a GPU.
 *   seqs/n_seqs : sequences.  BNSD requires n_seqs == 1 (batch gives the count);
 *                 TND requires batch == 1 and 1 <= n_seqs <= 32.
 *   batch       : BNSD batch size B (1..32).
 *   n1, n2      : query and key/value heads, n1 % n2 == 0 ([API] GQA constraint).
 *   d           : head dim, 64 or 128 (others: RF_ERR_UNSUPPORTED).
 *   sparsity    : finite, in [0, 1] ([UG] "Configuration"); 0 keeps every block.
 *   block_q, block_kv : [API] blockShape; must be > 0.  Built: 128 x 128, and
 *                 128 x 64 (query blocks of 128 rows, key/value blocks of 64
 *                 rows: ceil(lp / 64) prefix key blocks from row 0, the last
 *                 possibly partial, then 2 * nb from row lp; native precision
 *                 only).  With 128 x 64, selectIdx entries and max_kv_blocks
 *                 count 64-row key blocks, and the selection step ranks them
 *                 (see rf_pool_select).  Others: RF_ERR_UNSUPPORTED.
 *   out         : receives the plan; free with rf_plan_destroy.
 * Errors: RF_ERR_INVALID_ARG for a broken constraint (out untouched). */
RF_API rf_status_t rf_plan_create(const rf_seq_geom_t* seqs, int32_t n_seqs, int32_t batch,
                           int32_t n1, int32_t n2, int32_t d, rf_layout_t layout,
                           rf_dtype_t dtype, double sparsity, int32_t block_q,
                           int32_t block_kv, rf_plan_t** out);

/* Kernel precision ([UG] "Configuration": precision "bf16" | "fp8" | "mix").
 *   RF_PRECISION_NATIVE  Q K^T and P V in the inputs' 16-bit type (the pages'
 *                        "bf16"; fp16 inputs stay fp16).
 *   RF_PRECISION_MIX     Q K^T on FP8 E4M3 copies of Q' and K' with one fp32
 *                        scale per (head, 128-row block); P V stays 16-bit.
 *                        rf_rearrange writes the E4M3 copies and scales into the
 *                        workspace (amax = max |x| over the block's valid rows,
 *                        inv = 448 / amax, codes = E4M3(x * inv) rounded to
 *                        nearest even with saturation, scale = amax / 448; an
 *                        all-zero block has inv = scale = 1), and
 *                        rf_block_sparse_attn multiplies each S tile by
 *                        scale_q * scale_k.  Head dim 128 only.
 *   RF_PRECISION_FP8     FP8 E4M3 for P V as well.  Q' and K' as in
 *                        RF_PRECISION_MIX.  V' is quantized per (head, 128-row
 *                        block) on a power-of-two scale: exp = the smallest
 *                        integer with amax <= 448 * 2^exp (-127 for an all-zero
 *                        block), codes = E4M3(v * 2^-exp) rounded to nearest
 *                        even with saturation (the scaling is exact).  The
 *                        softmax probabilities of key block j enter the P V
 *                        product as E4M3 values of P * 2^(exp_j - exp_max),
 *                        exp_max the largest V exponent among the row's selected
 *                        blocks (so every code stays below 448); the row sum is
 *                        taken from the unrounded probabilities, and the output
 *                        is multiplied back by 2^exp_max.  Both products run on
 *                        the FP8 tensor cores (kind::f8f6f4).  Head dim 128 only,
 *                        blockShape 128 x 128.
 * The pages name the three modes and nothing more; the E4M3 format, the block
 * granularity and the scale rules above are this library's reading.
 *   RF_PRECISION_MXFP4   MXFP4 attention with Universal Optimal Scaling and
 *                        Pre-Normalization Quantization ([MX] "MXAttention",
 *                        abstract).  Every operand of both products is MXFP4:
 *                        E2M1 elements (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
 *                        nearest, ties to the even code, saturating) sharing a
 *                        power-of-two scale 2^e per group of 32, e the smallest
 *                        integer with amax <= 7.25 * 2^e (UOS, Qmax = 7.25).
 *                        Groups run along each product's reduction axis: Q and K
 *                        rows in groups of 32 columns; V columns and P rows in
 *                        groups of 32 keys counted from the first row of each
 *                        key block.  rf_rearrange (or rf_quantize_mx) writes the
 *                        rounded Q', K', V' into the workspace.  The softmax
 *                        takes the exponentials against an integer running
 *                        maximum (log2 units), rounds each group of 32 of them to
 *                        MXFP4 the same way, and sums the rounded values into the
 *                        row sum, so the weights that multiply V' sum to one
 *                        exactly.  Head dim 128: the rounded values are stored as
 *                        E4M3 codes (an MXFP4 value c * 2^e is an E4M3 value for
 *                        -8 <= e <= 6; outside that range it rounds to the
 *                        nearest E4M3 value, saturating at 448), Q' and K' in
 *                        their layouts, V' transposed per block as for
 *                        RF_PRECISION_FP8; P enters
 *                        P V as E4M3 of the rounded values times 2^8 and the
 *                        output is multiplied by 2^-8; both products run on the
 *                        FP8 tensor cores (kind::f8f6f4) with unit scales.  Head
 *                        dim 64: exact 16-bit copies (V' as f16; values that
 *                        would round past 65504 saturate there) on the 16-bit
 *                        tensor cores, P V in f16. */
typedef enum {
  RF_PRECISION_NATIVE = 0,
  RF_PRECISION_MIX = 1,
  RF_PRECISION_FP8 = 2,
  RF_PRECISION_MXFP4 = 3
} rf_precision_t;
/* Options of rf_plan_create_ex; zero-initialised means the defaults. */
typedef struct {
  int32_t token_order;  /* rf_token_order_t, default RF_ORDER_TILE */
  int32_t precision;    /* rf_precision_t, default RF_PRECISION_NATIVE */
  int32_t reserved[6];  /* must be zero */
} rf_plan_options_t;
/* rf_plan_create with options (rf_plan_create is rf_plan_create_ex with
 * options == NULL, i.e. tile order and native precision).  Every other
 * argument and error as rf_plan_create; an unknown option value or a non-zero
 * reserved field is RF_ERR_INVALID_ARG; RF_PRECISION_MIX or RF_PRECISION_FP8
 * with d != 128 is RF_ERR_UNSUPPORTED.  RF_PRECISION_MXFP4 takes d 64 or 128.  Every later call on the plan
 * (rearrange, pooling, selection, attention, inverse, rf_plan_permutation)
 * follows the plan's options. */
RF_API rf_status_t rf_plan_create_ex(const rf_seq_geom_t* seqs, int32_t n_seqs, int32_t batch,
                                     int32_t n1, int32_t n2, int32_t d, rf_layout_t layout,
                                     rf_dtype_t dtype, double sparsity, int32_t block_q,
                                     int32_t block_kv, const rf_plan_options_t* options,
                                     rf_plan_t** out);
/* Sizes of a plan (host only). */
RF_API rf_status_t rf_plan_info(const rf_plan_t* plan, rf_plan_info_t* out);

/* Geometry of sequence `seq` (0 <= seq < n_seqs; host only). */
RF_API rf_status_t rf_plan_seq_info(const rf_plan_t* plan, int32_t seq, rf_seq_info_t* out);

/* Step 1 ([UG] opening paragraph and "Geometry handling"; [PR] rearrange with
 * QKV in one call; [ABS] spatiotemporal token permutation).
 * q, k, v     : inputs in original order (layout above).
 * q_r,k_r,v_r : outputs, same shapes, rows permuted within each sequence.
 *               Must not alias the inputs.
 * ws          : workspace of at least workspace_bytes; receives the fp32
 *               block means of the sparse blocks of Q and K (the fused
 *               pooling of [UG] opening paragraph / [ABS] insight 1) and, with
 *               precision "mix", the E4M3 copies of Q' and K' and their scales;
 *               with precision "mxfp4", the MXFP4 copies of Q', K' and V'.
 * Bit-exact copy; deterministic. */
RF_API rf_status_t rf_rearrange(const rf_plan_t* plan, const void* q, const void* k, const void* v,
                         void* q_r, void* k_r, void* v_r, void* ws, size_t ws_bytes,
                         rf_stream_t stream);

/* Precision "mix" only: the E4M3 copies of already-rearranged q_r and k_r and
 * their scales, written into ws exactly as rf_rearrange writes them (see
 * rf_precision_t).  rf_rearrange already does this in the same pass; this call
 * is for callers that produce q_r / k_r themselves.  RF_ERR_INVALID_ARG for a
 * plan with another precision. */
RF_API rf_status_t rf_quantize_qk(const rf_plan_t* plan, const void* q_r, const void* k_r, void* ws,
                                  size_t ws_bytes, rf_stream_t stream);
/* Precision "mxfp4": write the MXFP4-rounded copies of q_r, k_r and v_r into
 * ws (offsets ws_q_mx, ws_k_mx, ws_v_mx of rf_plan_info_t; the rounding rule
 * is stated at RF_PRECISION_MXFP4).  rf_rearrange already does this in the same
 * pass; this call is for callers that produce q_r / k_r / v_r themselves.
 * Inputs 16-byte aligned, non-null.  RF_ERR_INVALID_ARG for a plan with another
 * precision. */
RF_API rf_status_t rf_quantize_mx(const rf_plan_t* plan, const void* q_r, const void* k_r,
                                  const void* v_r, void* ws, size_t ws_bytes, rf_stream_t stream);
/* Every quantized copy the plan's precision needs, written into ws from
 * already-rearranged q_r, k_r, v_r exactly as rf_rearrange writes them in its
 * own pass (see rf_precision_t): "mix" the E4M3 Q' and K' with their scales
 * (v_r may be NULL); "fp8" those and the transposed E4M3 V' with its
 * exponents; "mxfp4" the MXFP4-rounded Q', K', V'.  For callers that produce
 * q_r / k_r / v_r themselves.  Inputs 16-byte aligned and non-null (v_r except
 * for "mix").  RF_ERR_INVALID_ARG for a native plan. */
RF_API rf_status_t rf_quantize(const rf_plan_t* plan, const void* q_r, const void* k_r,
                               const void* v_r, void* ws, size_t ws_bytes, rf_stream_t stream);
/* Steps 2-3 ([UG] opening paragraphs and "Configuration"; [API] selectIdx and
 * selectNum constraints).
 * q_r, k_r    : rearranged Q and K (read only when pool_mode == RF_POOL_RECOMPUTE;
 *               may be NULL otherwise).
 * select_idx  : int32 [t_qblk, n1, max_kv_blocks]; per row the kept key blocks of
 *               the query block's own sequence, ascending, prefix blocks first,
 *               padded with -1 ([API]).
 * select_num  : int32 [t_qblk, n1], the number of valid entries per row.
 * Selection: prefix and first-frame query blocks keep everything; other
 * video query blocks keep every prefix block, the first-frame sink blocks,
 * and the k key blocks with the highest block-mean dot product (ties: lower
 * block index), k = ceil((1 - sparsity) * nb).  Sequences with nb < 32 are
 * dense.  With blockShape 128 x 64 the key blocks hold 64 rows ([API]
 * "Formula": blocks of blockShapeX x blockShapeY): the 128-row query block
 * means are ranked against 64-row key block means, and the prefix, sink and
 * kept counts are rf_seq_info_t's n_pb_kv, ns_kv and k_kv.  Deterministic
 * (fp32 scores, no atomics). */
RF_API rf_status_t rf_pool_select(const rf_plan_t* plan, const void* q_r, const void* k_r,
                           int32_t* select_idx, int32_t* select_num, void* ws,
                           size_t ws_bytes, rf_pool_mode_t pool_mode, rf_stream_t stream);

/* Steps 2-3 without any device allocation by the caller or the library.
 * The pages have no counterpart: this entry point exists for callers that
 * cannot allocate device memory -- code running inside a host framework whose
 * device memory belongs to the framework's own allocator (a plugin cannot
 * cudaMalloc behind its back), or code on a latency-critical path where a
 * cudaMalloc, which may synchronise the device, is not acceptable.
 * Same result as rf_pool_select(..., RF_POOL_RECOMPUTE): the block means are
 * recomputed from q_r and k_r (both required, 16-byte aligned), then ranked.
 * Scratch: one static device array of 32 MiB inside librf.  It is set up on
 * the first call on each device (with that device current), which loads it
 * onto that GPU, where it stays until the process exits; make that first call
 * before any stream capture.  The device address found at that set-up is
 * kept for the life of the process: after cudaDeviceReset (or anything else
 * that replaces the device's primary context) this entry point must not be
 * called again on that device.  Size limit: the selection part of the plan's
 * workspace layout must fit in 32 MiB -- that is the offset of the first
 * quantized region (rf_plan_info().ws_q8 for a precision "mix" plan,
 * ws_q_mx for a precision "mxfp4" plan), otherwise workspace_bytes; larger
 * problems are rejected with RF_ERR_INVALID_ARG before any device work.
 * Every call on a device shares the array: calls that overlap on the GPU
 * (other streams, other threads) race and must be serialised by the caller.
 * Calls no cudaMalloc, cudaFree or other allocating routine. */
RF_API rf_status_t rf_pool_select_noalloc(const rf_plan_t* plan, const void* q_r, const void* k_r,
                                          int32_t* select_idx, int32_t* select_num,
                                          rf_stream_t stream);

/* Step 4 ([API] "Formula": Softmax(scale * Q K^T + atten_mask) V, restricted to
 * the key blocks of selectIdx; no user mask is consumed, the only masked keys
 * are rows past the dense prefix in its last, partial block).
 * q_r,k_r,v_r : rearranged inputs; o_r : output, same shape as q_r (may not alias).
 * select_idx, select_num : as written by rf_pool_select (any valid selection is
 *               accepted: entries in [0, n_pb + nb) of the row's sequence; the
 *               first select_num entries are used; out-of-range entries are
 *               skipped and flagged in ws).  With blockShape 128 x 64 the
 *               entries are 64-row key blocks in [0, ceil(lp / 64) + 2 * nb);
 *               the kernel pairs consecutive entries into 128-key tiles (the
 *               partial last prefix block never opens a pair), so listing both
 *               halves of a 128-row block gives that block's tile.
 * scale       : > 0 and finite (typically 1/sqrt(D)).
 * inner_precise : 0 = fp32 softmax ([API]: 1 = fp16 softmax is not allowed with
 *               bf16 and is not built here: RF_ERR_UNSUPPORTED).
 * Precision "mix": Q K^T reads the E4M3 copies of Q' and K' and their scales in
 *               ws (written by rf_rearrange or rf_quantize_qk on this ws), not
 *               q_r / k_r; P V reads v_r as usual.
 * Precision "mxfp4": both products read the MXFP4 copies in ws (written by
 *               rf_rearrange or rf_quantize_mx on this ws), not q_r / k_r / v_r.
 * Deterministic: no split-K, no atomics. */
RF_API rf_status_t rf_block_sparse_attn(const rf_plan_t* plan, const void* q_r, const void* k_r,
                                 const void* v_r, const int32_t* select_idx,
                                 const int32_t* select_num, float scale,
                                 int32_t inner_precise, void* o_r, void* ws, size_t ws_bytes,
                                 rf_stream_t stream);

/* Step 5 ([PR] inverse rearrange): o[orig(r)] = o_r[r] for every row r.
 * o_r : [.., N1 heads ..] in rearranged order; o : same shape, original order. */
RF_API rf_status_t rf_inverse_rearrange(const rf_plan_t* plan, const void* o_r, void* o,
                                 rf_stream_t stream);

/* The whole path: rf_rearrange, rf_pool_select (RF_POOL_FROM_WS),
 * rf_block_sparse_attn (inner_precise 0) and rf_inverse_rearrange.
 * q_r, k_r, v_r, o_r, select_idx, select_num are caller-provided intermediates. */
RF_API rf_status_t rf_forward(const rf_plan_t* plan, const void* q, const void* k, const void* v,
                       void* q_r, void* k_r, void* v_r, int32_t* select_idx,
                       int32_t* select_num, float scale, void* o_r, void* o, void* ws,
                       size_t ws_bytes, rf_stream_t stream);

/* The token permutation of sequence `seq` (host only, no device needed):
 * src_rows[r] = original row (within the sequence) of rearranged row r, for
 * r < length.  n must equal rf_seq_info_t.length.  This is the same index
 * arithmetic the kernels run ([UG] "Geometry handling"). */
RF_API rf_status_t rf_plan_permutation(const rf_plan_t* plan, int32_t seq, int64_t* src_rows, int64_t n);

/* Reads and clears the device status words in ws.  Synchronises `stream`.
 * [API] constraints: selectIdx entries must be valid block indices or -1, and
 * the call returns a status code; a CUDA kernel cannot return one, so the
 * kernels record what they skipped and this call reports it.  It also stands
 * in for a memory checker on the kernels' own bounds (they check every
 * selectIdx entry themselves and record, rather than fault).
 * flags_out (may be NULL) receives the raw words: [0] out-of-range selectIdx
 * entries seen, [1] expired bounded waits.  Returns RF_ERR_DEVICE_FAULT if
 * either is non-zero.  ws is the caller's device workspace; nothing else is
 * read or written. */
RF_API rf_status_t rf_check_device_status(const rf_plan_t* plan, void* ws, uint32_t* flags_out,
                                   rf_stream_t stream);

/* Self-test of the attention kernel's two exponential paths (the pages have no
 * counterpart; this exists so the polynomial can be checked on the device):
 * y_poly[i] = the FMA-pipe polynomial 2^x[i], y_mufu[i] = ex2.approx(x[i]),
 * for n float32 device values.  Asynchronous on `stream`. */
RF_API rf_status_t rf_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int64_t n,
                                    rf_stream_t stream);

/* Self-test of the failure path of the kernels' bounded waits (the pages have
 * no counterpart): one thread waits on a barrier that nothing completes, gives
 * up after the same limit as every wait in rf_block_sparse_attn (1 s), and
 * records the expiry in ws's status words as an attention CTA would (bit 31
 * of the expired-wait word).  The next rf_check_device_status reports
 * RF_ERR_DEVICE_FAULT and clears the words; the CUDA context stays usable.
 * Takes about one second of device time; asynchronous on `stream`. */
RF_API rf_status_t rf_selftest_expired_wait(const rf_plan_t* plan, void* ws, size_t ws_bytes,
                                            rf_stream_t stream);
/* Frees a plan (NULL is a no-op).  [API]: the second phase of the two-phase
 * call releases what the first made; here the plan is the only thing the
 * library owns (host memory), so this is all that is freed. */
RF_API void rf_plan_destroy(rf_plan_t* plan);

/* Static description of a status code (the [API] page's return codes are
 * named aclnnStatus values; these are this library's).  The string is owned by
 * the library and never freed. */
RF_API const char* rf_status_string(rf_status_t status);

/* Detail of the last error returned on the calling thread ("" if none; every
 * entry point clears it first).  The pages have no counterpart: aclnn reports
 * its detail through the CANN log instead.  The string is owned by the
 * library and valid until the next call on the same thread. */
RF_API const char* rf_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* RF_H_ */
