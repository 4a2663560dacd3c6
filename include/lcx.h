/*
 * lcx.h -- C ABI of the long-context RoPE + causal attention prefill library
 * (liblcx.so, sm_100a).
 *
 * Three calls make up the hot path (lcx_attn_fwd_split and lcx_attn_merge
 * add split-KV evaluation for decode-sized problems):
 *   lcx_rope_table  per-pair RoPE frequencies theta'_i and the attention scale
 *                   for plain RoPE, Position Interpolation, NTK-aware base
 *                   scaling and YaRN (NTK-by-parts ramp + 0.1 ln s + 1).
 *   lcx_apply_rope  the memory-bound rotate-pairs pass over a Q or K tensor.
 *   lcx_attn_fwd    blockwise online-softmax causal attention prefill that
 *                   rotates Q/K tiles on chip, with GQA, an optional sliding
 *                   window and attention sinks.
 *
 * Sources (page title, section):
 *   [LC]  "Long Context: RoPE / YaRN / NTK / MLA" (mathieu0905.github.io):
 *         2.1-2.4 RoPE and rope_attention, 4.2 PI, 5.2 NTK-aware base,
 *         6.2-6.6 YaRN, 10.1 sliding window, 10.2 attention sinks.
 *   [B83] "8.3 长上下文技术" (paper.xwysyy.cn llm-fullstack-book): 8.3.1-8.3.3
 *         frequencies, PI, NTK-aware, NTK-by-parts, YaRN recipe; 8.3.4
 *         FlashAttention tiling and online softmax.
 *
 * Conventions shared by every call:
 *   - Ownership: the caller owns every buffer.  The library allocates no device
 *     memory, keeps no state besides a per-thread last-error string, and never
 *     synchronises a stream.  Device work is enqueued on `stream` (a
 *     cudaStream_t passed as void*; NULL = the legacy default stream).
 *   - Tensors are [B, H, L, D] with element strides given per dimension; the
 *     last dimension must be contiguous (stride 1).  Pointers and strides must
 *     keep every row 16-byte aligned.
 *   - Every tensor, workspace and status pointer is device memory of the
 *     current device, unless a call says otherwise (lcx_rope_table works on
 *     host arrays).  The library does not query a pointer's kind, so a host
 *     pointer reaches the kernel that reads it; the Python binding refuses
 *     host tensors before the call.
 *   - Errors: argument problems are detected on the host before any device
 *     work and return LCX_ERR_INVALID_ARG (malformed) or LCX_ERR_UNSUPPORTED
 *     (well-formed but outside what the kernels implement).  A failed launch
 *     returns LCX_ERR_CUDA.  lcx_last_error() describes the last failure on
 *     the calling thread.  Device-side watchdog expiries are reported through
 *     the optional device status word of lcx_attn_fwd.
 *   - Thread safety: every call is reentrant.
 */
#ifndef LCX_H
#define LCX_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LCX_VERSION 102

#if defined(__GNUC__)
#define LCX_API __attribute__((visibility("default")))
#else
#define LCX_API
#endif

typedef enum {
    LCX_OK = 0,
    LCX_ERR_INVALID_ARG = 1,
    LCX_ERR_UNSUPPORTED = 2,
    LCX_ERR_CUDA = 3,
    LCX_ERR_TIMEOUT = 4
} lcx_status;

/* Frequency-scaling modes ([LC] 2.3, 4.2, 5.2, 6.2, 7.3; [B83] 8.3.2-8.3.3).
 * NONE leaves vectors unrotated (theta' = 0) and is meant for testing. */
typedef enum {
    LCX_ROPE_NONE = 0,
    LCX_ROPE_PLAIN = 1,   /* theta'_i = b^(-2i/D)                              */
    LCX_ROPE_PI = 2,      /* theta'_i = theta_i / s  (positions m -> m/s)      */
    LCX_ROPE_NTK = 3,     /* theta'_i = (b s^(D/(D-2)))^(-2i/D)                */
    LCX_ROPE_YARN = 4,    /* theta'_i = theta_i ((1-g_i)/s + g_i), g_i = clip((r_i-alpha)/(beta-alpha),0,1),
                             r_i = L_train theta_i / (2 pi); mscale = 0.1 ln s + 1 (s > 1) */
    LCX_ROPE_DYNAMIC_NTK = 5, /* NTK-aware base with s = seq_len / L_train when
                             seq_len > L_train, plain RoPE otherwise ("AI Day 9:
                             长上下文技术", RoPE extension list, Dynamic NTK)     */
    LCX_ROPE_FACTORS = 6  /* theta'_i = theta_i / lambda_i with caller-supplied
                             per-pair factors ([LC] 7.3 LongRoPE); the optional
                             short table applies while seq_len <= L_train ([LC] 7.4) */
} lcx_rope_mode;

/* Which dimensions form a rotated pair ([LC] 2.4): HALF pairs (i, i + D/2)
 * (HuggingFace halves), INTERLEAVED pairs (2i, 2i + 1) (adjacent, [LC] 2.1). */
typedef enum { LCX_PAIR_HALF = 0, LCX_PAIR_INTERLEAVED = 1 } lcx_pairing;

typedef enum { LCX_BF16 = 0, LCX_F32 = 1 } lcx_dtype;

typedef struct {
    int32_t mode;              /* lcx_rope_mode                                  */
    int32_t head_dim;          /* D: even, 2..512                                */
    int32_t pairing;           /* lcx_pairing                                    */
    int32_t reserved;          /* must be 0                                      */
    double base;               /* b > 1 (10000 in the pages)                     */
    double scale;              /* s = L_new / L_train > 0 (PI, NTK, YARN)        */
    int64_t original_max_pos;  /* L_train > 0 (YARN)                             */
    double alpha;              /* YARN ramp lower bound in turns (default 1)     */
    double beta;               /* YARN ramp upper bound in turns (default 32)    */
    int64_t seq_len;           /* DYNAMIC_NTK, FACTORS: the actual context length.
                                  lcx_rope_table needs it > 0; lcx_apply_rope and
                                  lcx_attn_fwd use their own length when it is 0
                                  (pos_offset + L, resp. L)                       */
    const double *factors;     /* FACTORS: HOST array of head_dim/2 factors > 0  */
    const double *factors_short; /* FACTORS: optional HOST table of head_dim/2
                                  factors used while seq_len <= original_max_pos */
} lcx_rope_params;

/*
 * lcx_rope_table -- the per-pair frequencies of a mode, rounded once from fp64
 * to fp32 (nearest even), and the attention scale sqrt(1/t).
 *   Defines: [LC] 2.4 (theta_i = b^(-2i/D)), 4.2 (PI), 5.2 (NTK-aware base),
 *            6.2 (NTK-by-parts ramp), 6.3/6.6 (sqrt(1/t) = 0.1 ln s + 1);
 *            [B83] 8.3.3 five-step YaRN recipe.
 *   inv_freq: HOST array of head_dim/2 floats, written on success.
 *   mscale  : HOST float, written on success (1 unless YARN with s > 1).
 *   Host-only; touches no GPU.  Returns LCX_OK or LCX_ERR_INVALID_ARG.
 */
LCX_API lcx_status lcx_rope_table(const lcx_rope_params *params, float *inv_freq, float *mscale);

/*
 * lcx_apply_rope -- rotate every pair of x by m * theta'_i and multiply by
 * mscale: (x_p, x_q) -> ms (x_p cos - x_q sin, x_p sin + x_q cos), with
 * m = pos_offset + l for sequence index l.
 *   Defines: [LC] 2.2 (rotation matrix), 2.4 apply_rope, 6.4 (mscale folded
 *            into cos/sin); [B83] 8.3.3 step 4-5.
 *   x, y      : DEVICE pointers to [B, H, L, D] tensors of `dtype`; y may equal
 *               x (in place; then the strides must match).  16-byte aligned.
 *   x_strides : element strides of x for (B, H, L, D); D's stride must be 1.
 *   y_strides : element strides of y, or NULL for "same as x".
 *   Angles are evaluated from the exact product m * theta'_i (fp64), so the
 *   result is accurate for positions up to 2^31.
 *   Supported: head_dim % 16 == 0, head_dim <= 512, strides multiples of 16
 *   bytes.  Enqueued on `stream`; returns before the work completes.
 */
LCX_API lcx_status lcx_apply_rope(const lcx_rope_params *params, const void *x, void *y, int32_t dtype,
                          int64_t B, int64_t H, int64_t L, const int64_t *x_strides,
                          const int64_t *y_strides, int64_t pos_offset, void *stream);

/* lcx_attn_args.flags */
#define LCX_ATTN_PREROTATED 1u  /* q and k already hold rotated vectors (e.g. from
                                   lcx_apply_rope with the same params, mscale
                                   included): skip the on-chip rotation and the
                                   mscale^2 factor on the logits.             */
#define LCX_ATTN_SPLIT_QK 2u    /* split mode: hold each rotated q' and k' as an
                                   fp16 part h = f16(x') plus the residual
                                   r = x' - h and form QK^T as
                                   qh.kh (fp16 tensor cores) + [e5m2(qh) |
                                   e5m2(qr)].[e5m2(kr) | e5m2(kh)] (one e5m2
                                   product over 2 D, about one fp16 product's
                                   time), with P and V in fp16 for PV,
                                   so the logits are accurate to ~2^-15
                                   relative instead of bf16's 2^-9 (needed when
                                   the logits are large, e.g. outlier-heavy
                                   activations); twice the tensor-core time
                                   of plain QK^T.  The rotated values must lie
                                   inside fp16's range (|x'| < 65504)        */
#define LCX_ATTN_PREROTATED_K 4u /* k alone already holds rotated vectors (a KV
                                   cache filled by lcx_apply_rope with the same
                                   params, mscale included); q is rotated on
                                   chip.  Ignored when LCX_ATTN_PREROTATED is set */
#define LCX_ATTN_TEST_STALL 0x80000000u /* test hook for the watchdog: the loader
                                   issues no copies, so every wait of the
                                   kernel expires after watchdog_ms and the
                                   status word receives LCX_ERR_TIMEOUT; o is
                                   left unwritten.  Never set in production.  */

typedef struct {
    const void *q;             /* DEVICE [B, Hq, L, D]                            */
    const void *k;             /* DEVICE [B, Hkv, Lk, D] ([.., D - d_R] with k_rope) */
    const void *v;             /* DEVICE [B, Hkv, Lk, Dv]                         */
    void *o;                   /* DEVICE [B, Hq, L, Dv], same dtype as q          */
    float *lse;                /* DEVICE [B, Hq, L] fp32 natural-log sum-exp of the
                                  scaled logits, or NULL                          */
    int32_t *dev_status;       /* DEVICE int32 or NULL: set to LCX_ERR_TIMEOUT by a
                                  kernel whose bounded wait expired; never cleared.
                                  After an expiry o and lse are undefined (the call
                                  still returns LCX_OK: the expiry happens on the
                                  device after the call returned), so callers that
                                  must detect it pass this word and read it      */
    int32_t dtype;             /* lcx_dtype of q, k, v, o                         */
    int32_t causal;            /* 1 = key j visible to query i only if j <= i    */
    int64_t B, Hq, Hkv, L, D;  /* Hq % Hkv == 0; D = query/key head dim           */
    int64_t q_strides[4], k_strides[4], v_strides[4], o_strides[4];  /* elements  */
    lcx_rope_params rope;      /* head_dim = D (every dim rotated) or, partial
                                  rotary, the number of LAST dims rotated      */
    int64_t window;            /* W > 0: key j visible only if i - j < W (W counts
                                  the query itself); 0 = no window.  Needs causal */
    int64_t sinks;             /* S: keys j < S stay visible to every i >= j when
                                  a window is set; 0 = none                       */
    float softmax_scale;       /* logit scale; 0 -> 1/sqrt(D)                     */
    uint32_t flags;            /* LCX_ATTN_* bits                                 */
    int32_t watchdog_ms;       /* wall-clock limit of every device wait, 1..60000;
                                  0 -> 2000 ms                                    */
    int32_t reserved0;         /* must be 0                                       */
    int64_t Lk;                /* key / value rows; 0 -> L (prefill)              */
    int64_t q_offset;          /* position of query row 0: query i sits at
                                  q_offset + i, key j at position j.  Chunked
                                  prefill and decode pass the chunk's start
                                  (decode: Lk - L).  With causal masking
                                  q_offset + L <= Lk (every query sees its own
                                  key); 0 for plain prefill                      */
    int64_t Dv;                /* value / output head dim; 0 -> D                 */
    const void *k_rope;        /* DEVICE [B, 1, Lk, rope.head_dim] or NULL: the
                                  rotary key part shared by every head (decoupled
                                  RoPE).  When set, k holds only the first
                                  D - rope.head_dim columns of each key       */
    int64_t k_rope_strides[4]; /* elements; the head stride is not used        */
    void *k_rot;               /* DEVICE scratch or NULL.  When set, and the keys
                                  would be rotated on chip (no PREROTATED flags),
                                  the rotated keys are written once into it by
                                  the rotate pass of lcx_apply_rope (mscale
                                  included) and the attention kernel reads them
                                  from there: one rotation per key instead of
                                  one per key tile and CTA.  Every dim rotated,
                                  no k_rope: contiguous [B, Hkv, Lk, D] of
                                  dtype; in the split-QK^T mode with bf16
                                  operands the keys' fp16 parts ([B, Hkv, Lk,
                                  D] fp16) followed by their 8-bit cross parts
                                  ([B, Hkv, Lk, 2 D] bytes: e5m2 of the
                                  residual, then of the fp16 part) and by the
                                  values in fp16 ([B, Hkv, Lk, D]).  With
                                  k_rope: the shared rotary key, contiguous
                                  [B, 1, Lk, rope.head_dim].  16-byte aligned.
                                  Ignored otherwise (partial rotary without
                                  k_rope)                                        */
    int64_t k_rot_bytes;       /* bytes at k_rot: >= B*Hkv*Lk*D*element size,
                                  three times that for split-QK^T with bf16, or
                                  B*Lk*rope.head_dim*element size with k_rope */
} lcx_attn_args;

/*
 * lcx_attn_fwd -- o_i = sum_j softmax_j(c <q'_i, k'_j>) v_j over the visible
 * keys, q' and k' the RoPE-rotated vectors times mscale, c = softmax_scale;
 * query head h reads kv head h / (Hq / Hkv) (GQA).
 *   Defines: [LC] 2.4 rope_attention (rotate, QK^T / sqrt(d), mask, softmax,
 *            times V), 6.3-6.4 (temperature via mscale on q and k), 10.1
 *            sliding window, 10.2 sinks; [B83] 8.3.4 (blockwise tiling with an
 *            exact online softmax), 8.3.3 (YaRN attention scaling).
 *   Positions: query i at p_i = q_offset + i, key j at j (prefill: q_offset = 0,
 *   Lk = L).  Visibility: j <= p_i if causal; with W > 0 also p_i - j < W or
 *   j < S.  Chunked prefill / decode ([LC] 10.3, position offsets) passes the
 *   new queries with the whole key cache; a StreamingLLM cache (sink entries
 *   then the recent window, keys stored un-rotated) passes its entries in that
 *   order, so every key is re-rotated on chip at its logical position (its
 *   index in the cache) on every call.  Rows with no visible key get o = 0 and
 *   lse = -inf.
 *   Decoupled RoPE ([LC] 9.5, 9.7, A.1): with rope.head_dim = d_R < D only the
 *   last d_R dims of q and k are rotated (by a d_R-dim RoPE; mscale multiplies
 *   the rotated parts only, as the scaled cos/sin do), the first D - d_R are
 *   used as they are, and the default scale 1/sqrt(D) is 1/sqrt(d_h + d_R).
 *   k_rope supplies the rotated key part once for all heads.
 *   Arithmetic: q', k' rounded to bf16 on chip (split mode: an fp16 part
 *   and e5m2 cross parts, see LCX_ATTN_SPLIT_QK), QK^T and PV on tensor cores
 *   with fp32 accumulation, P rounded to bf16 for PV (split mode: P and V in
 *   fp16), softmax statistics in
 *   fp32, o rounded once to the output dtype.  fp32 inputs at D = 64 keep
 *   32-bit operands: q', k', v and P rounded to tf32 (10-bit mantissa) for
 *   tf32 tensor-core products; at D = 128 (and in the split mode) fp32 inputs
 *   are rounded to the 16-bit operands above.
 *   Supported (D, Dv, rope.head_dim): (64, 64, 64), (128, 128, 128) with bf16
 *   or fp32 and either QK^T mode; (128, 128, 64) and (192, 128, 64) with bf16
 *   and plain QK^T.  Pointers 16-byte aligned, strides multiples of 16 bytes,
 *   D's stride 1.  Enqueued on `stream`.
 */
LCX_API lcx_status lcx_attn_fwd(const lcx_attn_args *args, void *stream);

/*
 * lcx_attn_fwd_split -- lcx_attn_fwd evaluated as num_splits partial
 * attentions, each over a consecutive stretch of a query block's key tiles
 * (split-KV), combined by the merge of lcx_attn_merge.  It runs num_splits
 * times more CTAs, which fills the GPU when there are few query blocks
 * (decode, short chunks against a long cache); the result equals
 * lcx_attn_fwd's up to rounding (the partial outputs are fp32).
 *   Defines: [B83] 8.3.4 (online softmax), 8.3.5 step 3 (a KV block's partial
 *            output folded in by rescaling with its softmax statistics).
 *   num_splits     : 1..256; 1 is lcx_attn_fwd and uses no workspace.  Splits
 *                    beyond a query block's tile count are empty and cost a
 *                    CTA each.
 *   workspace      : DEVICE buffer, 256-byte aligned, of at least
 *                    lcx_attn_split_workspace_bytes(B, Hq, L, D, num_splits)
 *                    bytes.  Owned by the caller; its contents on entry are
 *                    ignored and overwritten; two calls in flight at the same
 *                    time must not share it.
 *   Enqueues two kernels on `stream` (attention, then merge; the merge is a
 *   programmatic dependent launch that waits for the attention kernel before
 *   reading its results).  With bf16 operands, D = Dv = rope.head_dim = 128,
 *   no k_rope and at most 16 queries per kv group (G L <= 16, e.g. a decode
 *   step), and in the split-QK^T mode only with args.k_rot (keys split by the
 *   rotate pass), the attention kernel is the transposed-score decode kernel
 *   (one CTA per batch, kv group and split; keys along the tensor-memory
 *   lanes, the group's queries along its columns).  Errors as for lcx_attn_fwd; a short
 *   workspace is LCX_ERR_INVALID_ARG.
 */
LCX_API lcx_status lcx_attn_fwd_split(const lcx_attn_args *args, int32_t num_splits,
                                      void *workspace, int64_t workspace_bytes, void *stream);

/* Workspace bytes lcx_attn_fwd_split needs: room for two partial results
 * per split, [2 num_splits, B, Hq, L, D] fp32 partial outputs (D here: the
 * output head dim, args.Dv or args.D when Dv is 0) then [2 num_splits, B, Hq,
 * L] fp32 partial LSEs, each block rounded up to 256 bytes.  (Launches whose
 * query tiles are head-packed -- few queries per head, as in decode -- give
 * each of a split's two query tiles every other key tile and so write two
 * partial results per split; the others use the first num_splits.)  0 when
 * num_splits == 1; -1 for invalid sizes (D not 64/128, num_splits outside
 * 1..256, or more than 2^40 query rows). */
LCX_API int64_t lcx_attn_split_workspace_bytes(int64_t B, int64_t Hq, int64_t L, int64_t D,
                                               int32_t num_splits);

/*
 * lcx_attn_merge -- combine n_parts partial attention results of the same
 * query rows over disjoint key sets: with m = max_s lse_s and
 * w_s = exp(lse_s - m), o = sum_s w_s o_s / sum_s w_s and
 * lse = m + ln sum_s w_s.  Parts with lse_s = -inf (no key) weigh nothing; a
 * row with no non-empty part gets o = 0, lse = -inf.
 *   Defines: [B83] 8.3.4 (online softmax rescaling), 8.3.5 step 3 (Ring
 *            Attention: partial outputs combined by their statistics).
 *   o_parts  : DEVICE fp32 [n_parts, B, Hq, L, D], contiguous, 16-byte
 *              aligned; row r of part s normalised over that part's keys.
 *   lse_parts: DEVICE fp32 [n_parts, B, Hq, L], contiguous (natural log).
 *   o        : DEVICE [B, Hq, L, D] of `dtype`, element strides o_strides
 *              (D's stride 1, others multiples of 16 bytes), 16-byte aligned.
 *   lse      : DEVICE fp32 [B, Hq, L] contiguous, or NULL.
 *   Supported: D in {64, 128}, n_parts 1..4096.  Enqueued on `stream`.
 */
LCX_API lcx_status lcx_attn_merge(const float *o_parts, const float *lse_parts, int32_t n_parts,
                                  int64_t B, int64_t Hq, int64_t L, int64_t D, void *o,
                                  int32_t dtype, const int64_t *o_strides, float *lse,
                                  void *stream);

/* Size of the static device scratch of lcx_attn_fwd_split_static (32 MiB). */
#define LCX_STATIC_SCRATCH_BYTES (32 * 1024 * 1024)

/*
 * lcx_attn_fwd_split_static -- lcx_attn_fwd_split with the library's own
 * static device scratch in place of a caller workspace: the call allocates
 * nothing (no cudaMalloc, no caller buffer besides the tensors of `args`).
 * The pages describe no counterpart of this call; it exists for callers that
 * have no device allocator at hand.
 *   Scratch : one static __device__ array of LCX_STATIC_SCRATCH_BYTES per
 *             CUDA context (256-byte aligned).  Every call looks up the
 *             current context's copy with cudaGetSymbolAddress (a checked
 *             call; failure is LCX_ERR_CUDA), so a context that was destroyed
 *             and created again (cudaDeviceReset) is never handed a stale
 *             address.  The first call in a context is the set-up: under lazy
 *             module loading the CUDA runtime loads the library's module, and
 *             with it the array, at that lookup; make that first call before
 *             capturing the stream into a graph.  Later calls allocate
 *             nothing.  Nothing in the array must start at zero (every
 *             partial row the merge reads is written earlier in the same
 *             call), so it is never cleared.
 *   Limit   : requests whose lcx_attn_split_workspace_bytes exceeds
 *             LCX_STATIC_SCRATCH_BYTES return LCX_ERR_UNSUPPORTED before any
 *             device work.
 *   Races   : every call on a device shares the one array, so two calls whose
 *             executions overlap (different streams, or threads without
 *             ordering) corrupt each other's partial results; order them.
 *   Watchdog: if a bounded device wait expires (args.watchdog_ms), o and lse
 *             are undefined -- the merge may read partial rows that an
 *             earlier call left in the array.  Pass args.dev_status to learn
 *             of it.
 *   Otherwise as lcx_attn_fwd_split (num_splits 1..256; 1 uses no scratch).
 */
LCX_API lcx_status lcx_attn_fwd_split_static(const lcx_attn_args *args, int32_t num_splits,
                                             void *stream);

/* Static description of a status code. */
LCX_API const char *lcx_status_string(lcx_status status);

/* Description of the last failure on the calling thread ("" if none). */
LCX_API const char *lcx_last_error(void);

/* LCX_VERSION of the built library. */
LCX_API int32_t lcx_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LCX_H */
