/*
 * kvq.h -- C ABI of libkvq, a B200 (sm_100a) library for rotated INT2
 * KV caches: rotate -> quantize -> append, and decode attention over the
 * packed cache.
 *
 * The method (pages on the subject):
 *   "Output-Aware Rotation for INT2 KV-Cache Quantization" (OptR), section
 *   "Key Details": every head owns an orthogonal rotation that is applied to
 *   the cache before INT2 quantization and removed after the attention
 *   computation; section "Why It Matters": the attention kernel itself is
 *   unchanged.  "RotateKV: Accurate and Robust 2-Bit KV Cache Quantization for
 *   LLMs via Outlier-Aware Adaptive Rotations", abstract: (i) channel
 *   reordering followed by a fast Walsh-Hadamard transform, (iii) attention
 *   sinks protected from 2-bit quantization.  "KVLinC : KV Cache Quantization
 *   with Hadamard Rotation and Linear Correction", abstract: Hadamard rotation
 *   of the values.  The rotation itself is learned or chosen offline and is an
 *   input here.
 *
 * Conventions
 *   - head_dim is 128; quantization groups are 32 consecutive elements of
 *     head_dim (4 per row); each group stores an fp16 scale s and fp16 zero z.
 *   - fp16 values cross the ABI as uint16_t bit patterns (IEEE binary16).
 *   - Row-vector convention: x_rot = x . R with R row-major, R[i][j] at
 *     R + i*128 + j.  FWHT mode: y[i] = x[perm[i]], x_rot = FWHT(y)/sqrt(128),
 *     FWHT in Sylvester order, H[i][j] = (-1)^popcount(i & j).
 *   - Every pointer argument except the descriptor itself and kvq_get_status's
 *     host_out is DEVICE memory owned by the caller.  The library never
 *     allocates or frees memory and keeps no state between calls (it caches
 *     per-device attributes only).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Compute
 *     calls are asynchronous on it; argument errors are reported before any
 *     launch and nothing is launched then.  The kernels use programmatic
 *     dependent launch: the rotation inputs (R_k, R_v, perm) may be read
 *     while the kernel enqueued just before the call is still finishing, so
 *     they must not be written by that kernel when it is itself launched
 *     with programmatic dependent launch (a kernel launched the ordinary way
 *     has completed by then; a libkvq append writes none of them).  Every
 *     other input is read only after the preceding work in the stream
 *     completed.
 *   - Device-detected errors never trap: they OR a bit into cache->status[0]
 *     (see KVQ_DEV_*) and the affected work is skipped.
 *
 * Quantizer (exact IEEE fp32, no contraction), per group of 32 values x:
 *   mn = min x, mx = max x
 *   s  = fp16_rn((mx - mn) / 3)          z = fp16_rn(mn)    (zeros stored +0)
 *   inv = (s == 0) ? 0 : fp32(1 / s)
 *   c  = clamp(rint_even(fp32(fp32(x - z) * inv)), 0, 3)
 *   dequantised value: c * s + z
 * Logical packing: the code of element j is byte (j % 32), bits 2*(j/32).
 *
 * Cache layout.  One cache holds B sequences x Hkv KV heads; each (b, h)
 * "unit" owns capacity/16 blocks of 16 tokens, 1536 bytes each:
 *   blocks + ((b*Hkv + h) * (capacity/16) + p/16) * 1536   for position p.
 * A paged cache (kvq_cache_desc.block_table set) keeps the same 1536-byte
 * blocks in a pool of num_blocks x Hkv blocks and finds position p of
 * sequence b through the table:
 *   blocks + (block_table[b*(capacity/16) + p/16] * Hkv + h) * 1536.
 * Inside a block, with tau = p % 16, r = tau % 8, th = tau / 8,
 * pair q = tau / 2, side = tau % 2 (all offsets in bytes):
 *   K codes  [0,512)     logical 32-bit word wi (bytes 4wi..4wi+3 of the
 *                        token's 32 code bytes) at 16*(4r + wi%4) + 4*(2th + wi/4)
 *   V codes  [512,1024)  logical 16-bit piece w (bytes 2w, 2w+1) at
 *                        512 + 16*(4*(w%8) + q%4) + 4*(2*(q/4) + w/8) + 2*side
 *   K meta   [1024,1280) group g: fp16 s then fp16 z at 1024 + 8*(4r + g) + 4*th
 *   V meta   [1280,1536) group g: fp16 s then fp16 z at 1280 + 8*(4r + g) + 4*th
 * This order is the operand order of the decode kernel's tensor-core
 * fragments, so one warp reads each 512-byte region as 32 x 16 contiguous
 * bytes.  The 96 bytes per token-head (3 bits per element) are the whole
 * cache read of a decode step.
 * Sinks (RotateKV abstract, item (iii): attention sinks are protected from
 *   2-bit quantization) are kept as fp16 rotated rows in
 *   k_sink / v_sink [B][Hkv][sink_fp16][128], in one of two ways:
 *   - leading sinks (sink_pos == NULL): positions p < sink_fp16 of every
 *     sequence, row p; their block slots are zeroed;
 *   - identified sinks (sink_pos != NULL): the positions that
 *     kvq_identify_sinks picked because their activations are massive
 *     (same item: massive activations single out the sinks), listed in
 *     ascending order in sink_pos[b][0 .. sink_count[b]); the one at list
 *     index j is row j.  Its block slot holds zero codes, V meta
 *     {0, 0} and K meta {s, z} = {0x7E00 (a quiet NaN), 0} in every group:
 *     the marker that keeps the INT2 path from scoring the position.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, mode/pointer mismatch */
    KVQ_ERR_UNSUPPORTED = 2,  /* head_dim != 128, group != 32, misalignment   */
    KVQ_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed          */
    KVQ_ERR_CAPACITY = 4,     /* reserved: capacity errors are device-side     */
    KVQ_ERR_WORKSPACE = 5     /* decode workspace too small                    */
} kvq_status;

typedef enum {
    KVQ_ROT_DENSE = 0,        /* per-head dense 128x128 orthogonal R (OptR)     */
    KVQ_ROT_PERM_FWHT = 1     /* per-head channel permutation + FWHT (RotateKV) */
} kvq_rot_mode;

/* Bits ORed into *status by device code. */
#define KVQ_DEV_CAPACITY 1    /* append would exceed capacity: sequence skipped */
#define KVQ_DEV_BAD_LEN 2     /* seq_lens[b] < 0 (append) or not in [1, capacity]
                                 (decode): skipped, decode output row is 0      */
#define KVQ_DEV_TIMEOUT 4     /* a bounded pipeline wait gave up: output invalid */
#define KVQ_DEV_BAD_TABLE 8   /* paged cache: a block-table entry outside
                                 [0, num_blocks): the append skips that store,
                                 the decode reads pool block 0 instead (output
                                 invalid)                                       */

typedef struct {
    int32_t B;                /* sequences                                      */
    int32_t Hkv;              /* KV heads                                       */
    int32_t head_dim;         /* must be 128                                    */
    int32_t group;            /* must be 32                                     */
    int32_t capacity;         /* tokens per sequence, multiple of 16            */
    int32_t sink_fp16;        /* leading positions kept in fp16 (0..64)         */
    void *blocks;             /* [B][Hkv][capacity/16][1536] bytes (paged:
                                 [num_blocks][Hkv][1536]), 16-B aligned          */
    uint16_t *k_sink;         /* [B][Hkv][sink_fp16][128] fp16, or NULL if 0     */
    uint16_t *v_sink;         /* same                                           */
    int32_t *status;          /* two device words, 8-B aligned: [0] sticky error
                                 bits (KVQ_DEV_*); [1] the library's append
                                 completion counter.  Zero both once before
                                 first use; [1] is zero again after every
                                 append.                                        */
    const int32_t *block_table; /* NULL: the contiguous layout above.  Otherwise
                                 a paged cache: int32 [B][capacity/16] device
                                 array, 4-B aligned; logical block lb of
                                 sequence b (positions 16lb..16lb+15) lives in
                                 pool block n = block_table[b*(capacity/16) + lb],
                                 whose KV head h is the 1536-byte block at
                                 blocks + (n*Hkv + h)*1536.  Entries of blocks a
                                 call touches must be in [0, num_blocks);
                                 several sequences may not share a block.      */
    int32_t num_blocks;       /* paged: pool blocks (blocks holds
                                 num_blocks*Hkv*1536 bytes); ignored otherwise */
    int32_t *sink_pos;        /* NULL: leading sinks.  Otherwise identified
                                 sinks: int32 [B][sink_fp16], ascending
                                 positions (sink_fp16 >= 1); written by
                                 kvq_identify_sinks, read by the append and the
                                 decode.  4-B aligned.                         */
    int32_t *sink_count;      /* identified sinks: int32 [B], entries of
                                 sink_pos in use (0..sink_fp16); zero it with
                                 the cache.  Ignored when sink_pos is NULL.    */
} kvq_cache_desc;

/* Bytes of the blocks array for a cache of this shape (0 on bad arguments). */
KVQ_API size_t kvq_cache_bytes(int32_t B, int32_t Hkv, int32_t capacity);

/*
 * Rotate, quantize and append T tokens to every sequence.
 *   K, V      fp16 [B][T][Hkv][128] (post-RoPE keys, values), 16-B aligned.
 *   mode      KVQ_ROT_DENSE: R_k, R_v fp32 [Hkv][128][128] required, perm ignored.
 *             KVQ_ROT_PERM_FWHT: perm int32 [2][Hkv][128] required (plane 0
 *             keys, plane 1 values; each row a permutation of 0..127),
 *             R_k / R_v ignored.
 *   seq_lens  int32 [B]: in = current length, out = length + T.  Positions
 *             seq_lens[b] .. seq_lens[b]+T-1 are written.  If that exceeds
 *             capacity (or seq_lens[b] < 0) the sequence is left untouched
 *             and a KVQ_DEV_* bit is set.
 * Rotation: OptR page "Key Details"; RotateKV abstract item (i); KVLinC
 * abstract.  Sinks: RotateKV abstract item (iii).
 */
KVQ_API kvq_status kvq_rotate_quantize_append(const uint16_t *K, const uint16_t *V, int32_t T,
                                      kvq_rot_mode mode, const float *R_k, const float *R_v,
                                      const int32_t *perm, const kvq_cache_desc *cache,
                                      int32_t *seq_lens, void *stream);

/*
 * Pick the attention sinks among the next T positions of every sequence by
 * their activation magnitude (RotateKV abstract, item (iii)); call it just
 * before the kvq_rotate_quantize_append of the same T tokens, with the same
 * seq_lens (it does not change them).
 *   act       fp32 [B][T]: the caller's activation magnitude of each new token
 *             (for instance the largest |hidden-state| entry of the token at
 *             this layer's input; the library only compares it).
 *   tau       threshold: token t of sequence b is a sink when
 *             act[b*T + t] >= tau (NaN compares false) and the sequence has a
 *             free sink row; rows are taken in position order, so the first
 *             sink_fp16 such positions of a sequence are kept.
 *   cache     needs sink_pos / sink_count (identified sinks).
 *   seq_lens  int32 [B] device, the lengths before the append.  A sequence
 *             the append would skip (seq_lens[b] < 0 or seq_lens[b] + T >
 *             capacity) is skipped here too.
 * Appends the picked positions to sink_pos[b] and raises sink_count[b].
 * Errors: KVQ_ERR_INVALID_ARG for null pointers, T < 1, or a cache without
 * sink_pos; nothing is launched then.
 */
KVQ_API kvq_status kvq_identify_sinks(const float *act, int32_t T, float tau,
                                      const kvq_cache_desc *cache, const int32_t *seq_lens,
                                      void *stream);

/* Workspace bytes needed by kvq_decode_attention for these sizes on a GPU
 * with sm_count SMs (0 on bad arguments). */
KVQ_API size_t kvq_decode_workspace_size(int32_t B, int32_t Hq, int32_t Hkv, int32_t max_ctx,
                                 int32_t sm_count);

/*
 * Decode attention of one query per query head over the packed cache.
 *   Q         fp16 [B][Hq][128]; query head hq reads KV head hq / (Hq/Hkv).
 *   mode, R_k, R_v, perm   the rotations used at append time.
 *   seq_lens  int32 [B] device: context length of each sequence (>= 1).
 *   sink_fp16 must equal cache->sink_fp16.
 *   max_ctx   host upper bound of seq_lens (sizes the work split).
 *   workspace >= kvq_decode_workspace_size(B, Hq, Hkv, max_ctx, SMs) bytes,
 *             256-B aligned; contents need not be initialised.
 *   out       fp16 [B][Hq][128].
 * Computes q_rot = q . R_k, s_t = q_rot . k_t / sqrt(128) over the dequantised
 * rotated keys (sinks in fp16), softmax, o_rot = sum p_t v_t and
 * out = o_rot . R_v^T: the rotation is removed after attention (OptR page,
 * "Key Details"); the attention itself is the standard one ("Why It Matters").
 */
KVQ_API kvq_status kvq_decode_attention(const uint16_t *Q, int32_t Hq, const kvq_cache_desc *cache,
                                kvq_rot_mode mode, const float *R_k, const float *R_v,
                                const int32_t *perm, const int32_t *seq_lens,
                                int32_t sink_fp16, int32_t max_ctx, void *workspace,
                                size_t ws_bytes, uint16_t *out, void *stream);

/* Same as kvq_decode_attention; in addition records the caller's CUDA events
 * ev_begin / ev_end (cudaEvent_t, either may be NULL) on `stream` immediately
 * before and after the kernel that streams the packed cache, so a caller can
 * time that kernel alone. */
KVQ_API kvq_status kvq_decode_attention_timed(const uint16_t *Q, int32_t Hq,
                                              const kvq_cache_desc *cache, kvq_rot_mode mode,
                                              const float *R_k, const float *R_v,
                                              const int32_t *perm, const int32_t *seq_lens,
                                              int32_t sink_fp16, int32_t max_ctx, void *workspace,
                                              size_t ws_bytes, uint16_t *out, void *stream,
                                              void *ev_begin, void *ev_end);

/* Size of the fixed device array that kvq_decode_attention_noalloc uses as
 * its workspace (4 MiB).  Decode shapes whose workspace
 * (kvq_decode_workspace_size) exceeds it are rejected. */
#define KVQ_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * kvq_decode_attention without a workspace argument, for callers that cannot
 * allocate device memory (a serving loop whose device memory is fixed at
 * start-up, a plugin inside a framework that owns every allocation).  The
 * pages describe no such entry point; it is a deployment convenience with no
 * counterpart in the method.
 *   Same arguments and results as kvq_decode_attention, minus workspace /
 *   ws_bytes.  The workspace is a fixed KVQ_NOALLOC_SCRATCH_BYTES array in
 *   the library's own device memory, held by every GPU that loads the
 *   library until the process exits; nothing is allocated or freed.
 *   Errors: KVQ_ERR_WORKSPACE if the shape needs more than the fixed array
 *   (checked on the host before any launch), otherwise as
 *   kvq_decode_attention.
 *   The first call on each device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   All calls share the array: calls that may overlap on the GPU (other
 *   streams, other host threads) race and must be serialised by the caller.
 */
KVQ_API kvq_status kvq_decode_attention_noalloc(const uint16_t *Q, int32_t Hq,
                                                const kvq_cache_desc *cache, kvq_rot_mode mode,
                                                const float *R_k, const float *R_v,
                                                const int32_t *perm, const int32_t *seq_lens,
                                                int32_t sink_fp16, int32_t max_ctx, uint16_t *out,
                                                void *stream);

/* Read (and leave set) the device status word: synchronises `stream`.
 * host_out is a host pointer. */
KVQ_API kvq_status kvq_get_status(const kvq_cache_desc *cache, void *stream, int32_t *host_out);

/* Clear both device status words (asynchronous on `stream`); do not call it
 * while an append may be in flight. */
KVQ_API kvq_status kvq_clear_status(const kvq_cache_desc *cache, void *stream);

/*
 * Test exports: the same device code as the hot path, with fp32 outputs.
 * kvq_debug_rotate_f32: X fp16 [N][128] rows, all rotated by one head's
 *   rotation (R fp32 [128][128] in dense mode, perm int32 [128] in FWHT mode)
 *   -> Xrot fp32 [N][128].  `variant` selects the append kernel whose
 *   rotation is exercised: 0 = the small-batch kernels (CUDA cores), 1 = the
 *   bulk kernel on the tcgen05 tensor cores, used by appends with 16-byte
 *   aligned K and V of T new rows per sequence over B sequences when, in
 *   dense mode (R split into fp16 hi + lo), T >= 32 or T >= 8 with
 *   B*T >= 256, and in FWHT mode (the product with the permuted +-1
 *   Hadamard matrix, scaled by 1/sqrt(128) in fp32), T >= 128 or T >= 32
 *   with B*T >= 1024.  Other values: KVQ_ERR_INVALID_ARG.
 * kvq_debug_quantize_f32: Xrot fp32 [N][128] -> codes [N][32] in the logical
 *   packing, meta [N][4] as {s, z} fp16 pairs (uint16 [N][4][2]).
 */
KVQ_API kvq_status kvq_debug_rotate_f32(const uint16_t *X, int32_t N, kvq_rot_mode mode,
                                const float *R, const int32_t *perm, int32_t variant,
                                float *Xrot, void *stream);
KVQ_API kvq_status kvq_debug_quantize_f32(const float *Xrot, int32_t N, uint8_t *codes,
                                  uint16_t *meta, void *stream);

/*
 * Test export for the failure path of the kernels' bounded waits (device
 * errors are reported in a status word, never by a trap).  One thread runs
 * the decode ring protocol on two slots: a real 1536-byte bulk copy of `src`
 * into slot 0, and a wait on slot 1, which nothing ever fills, that gives up
 * after poll_limit polls (each poll may sleep up to about 20 us).  It then
 * ORs KVQ_DEV_TIMEOUT into *status and drains the ring with the same routine
 * an aborted decode CTA runs before it returns, so that no copy still
 * targets its shared memory.
 *   src     device, 1536 bytes, 16-byte aligned.
 *   status  device int32 word (e.g. a cache's status).
 *   result  device int32 [3]: [0] = 1 if the wait gave up, [1] = stages the
 *           drain could not see land (0 expected), [2] = sum of the 1536
 *           bytes as copied into shared memory.
 * Errors: null pointers or poll_limit 0 -> KVQ_ERR_INVALID_ARG; misaligned
 * pointers -> KVQ_ERR_UNSUPPORTED.  No page counterpart: library plumbing.
 */
KVQ_API kvq_status kvq_debug_wait_timeout(const void *src, uint32_t poll_limit, int32_t *status,
                                          int32_t *result, void *stream);

/* Options of kvq_decode_attention_ex. */
#define KVQ_DECODE_OUT_ROTATED 1u  /* out = o_rot: the caller applies R_v^T (or the inverse
                                      permutation + FWHT) itself, e.g. folded into W_O */

/*
 * Decode with q_len new tokens per sequence (multi-query / speculative
 * decode) and options.  The q_len tokens are the last ones already appended:
 * query i (0 <= i < q_len) of a sequence of length L is the token at
 * position L - q_len + i and attends to positions [0, L - q_len + i], i.e.
 * causally among the new tokens; each is the standard attention of
 * kvq_decode_attention (OptR page, "Why It Matters") over its own prefix.
 *   Q        fp16 [B][Hq][q_len][128]; out fp16 [B][Hq][q_len][128].
 *   q_len    1..8 with (Hq / Hkv) * q_len in {1, 2, 4, 8}.
 *   flags    0 or KVQ_DECODE_OUT_ROTATED.
 *   workspace >= kvq_decode_workspace_size(B, Hq * q_len, Hkv, max_ctx, SMs).
 *   max_ctx  >= q_len.
 * Other arguments and errors as kvq_decode_attention.  A sequence with
 * seq_lens[b] < q_len gets zero rows for the queries that would start
 * before position 0 and sets KVQ_DEV_BAD_LEN.  q_len = 1 with flags = 0 is
 * exactly kvq_decode_attention.
 */
KVQ_API kvq_status kvq_decode_attention_ex(const uint16_t *Q, int32_t Hq, int32_t q_len,
                                   uint32_t flags, const kvq_cache_desc *cache,
                                   kvq_rot_mode mode, const float *R_k, const float *R_v,
                                   const int32_t *perm, const int32_t *seq_lens,
                                   int32_t sink_fp16, int32_t max_ctx, void *workspace,
                                   size_t ws_bytes, uint16_t *out, void *stream);

/*
 * Decode with KVLinC key correction adapters ("KVLinC : KV Cache
 * Quantization with Hadamard Rotation and Linear Correction", abstract:
 * lightweight linear correction adapters compensate for the errors that the
 * quantized keys introduce; with the values Hadamard-rotated and the keys
 * unrotated - dense mode with R_k = I, R_v = H/sqrt(128) - this is KVLinC's
 * configuration).  The page gives no formula; the library's reading: a
 * rank-r linear map of every dequantised INT2 key in the model's
 * (unrotated) basis,
 *     k~ = k^ + (k^ . U) . V^T,
 * scored as q . k~ / sqrt(128); fp16 sink keys (no quantization error) are
 * scored as stored.  The map is folded into the query once per call
 * (q . k~ = k^ . (q + (q . V) . U^T)), so the streaming over the cache is
 * that of kvq_decode_attention_ex.
 *   U_k, V_k  device fp32 [Hkv][128][rank], row-major, caller-owned.
 *   rank      1..128.
 * Other arguments, layouts and errors as kvq_decode_attention_ex.  Null
 * U_k / V_k or rank outside [1, 128] -> KVQ_ERR_INVALID_ARG; U_k or V_k not
 * 4-byte aligned -> KVQ_ERR_UNSUPPORTED.
 */
KVQ_API kvq_status kvq_decode_attention_adapter(const uint16_t *Q, int32_t Hq, int32_t q_len,
                                        uint32_t flags, const kvq_cache_desc *cache,
                                        kvq_rot_mode mode, const float *R_k, const float *R_v,
                                        const int32_t *perm, const float *U_k, const float *V_k,
                                        int32_t rank, const int32_t *seq_lens,
                                        int32_t sink_fp16, int32_t max_ctx, void *workspace,
                                        size_t ws_bytes, uint16_t *out, void *stream);

/*
 * Pre-RoPE grouped-head key rotation (RotateKV abstract, item (ii): the
 * outlier-aware rotation applied to the keys before RoPE and across heads).
 * The keys of group_heads (gh) consecutive KV heads form one row of
 * n = 128*gh channels, which is reordered and Hadamard-transformed:
 *   x_rot = FWHT_n(x[perm_group]) / sqrt(n),
 * and head j of the group stores channels 128j .. 128j+127 of x_rot in its
 * cache unit (the same block format).  Values are rotated per head as in
 * KVQ_ROT_PERM_FWHT.  RoPE is the rotate-half form: channel c < 64 pairs with
 * c + 64 and turns by t * base^(-2c/128) at position t (0-based).
 *   perm   int32 [2][Hkv*128]: plane 0 holds the Hkv/gh key permutations of n
 *          entries (group q at perm + q*n, each a permutation of 0..n-1),
 *          plane 1 one value permutation of 0..127 per head (at
 *          perm + Hkv*128 + h*128).  16-B aligned.
 *   gh     1, 2, 4 or 8, dividing Hkv.
 * Sinks, leading or identified (kvq_identify_sinks before the append), keep
 * the key as given (fp16, pre-RoPE, unrotated) and the rotated value in their
 * fp16 rows; the decode turns a sink key by RoPE at the sink's position.
 * Paged caches are fine.
 */
/* Append T tokens: K fp16 [B][T][Hkv][128] PRE-RoPE keys, V fp16 values
 * (same layout), 16-B aligned; seq_lens as in kvq_rotate_quantize_append. */
KVQ_API kvq_status kvq_prerope_append(const uint16_t *K, const uint16_t *V, int32_t T,
                                      int32_t group_heads, const int32_t *perm,
                                      const kvq_cache_desc *cache, int32_t *seq_lens,
                                      void *stream);
/* Workspace bytes of kvq_prerope_decode for these sizes (0 on bad arguments). */
KVQ_API size_t kvq_prerope_workspace_size(int32_t B, int32_t Hq, int32_t Hkv,
                                          int32_t group_heads, int32_t max_ctx,
                                          int32_t sm_count);
/* Decode one query per query head over a pre-RoPE cache.
 *   Q     fp16 [B][Hq][128] POST-RoPE queries (the model's own q at the new
 *         position); query head hq reads KV head hq / (Hq/Hkv).
 *   (Hq/Hkv) * group_heads <= 8.
 * For every position t < seq_lens[b]: k_t = RoPE_t(head slice of the inverse
 * group rotation of the dequantised keys), s_t = q . k_t / sqrt(128),
 * softmax, o_rot = sum p_t v_t over the rotated values, out = o_rot rotated
 * back (FWHT + value permutation).  Other arguments and errors as
 * kvq_decode_attention; KVQ_ERR_UNSUPPORTED for a shape outside the limits
 * above. */
KVQ_API kvq_status kvq_prerope_decode(const uint16_t *Q, int32_t Hq, const kvq_cache_desc *cache,
                                      int32_t group_heads, const int32_t *perm, float rope_base,
                                      const int32_t *seq_lens, int32_t max_ctx, void *workspace,
                                      size_t ws_bytes, uint16_t *out, void *stream);
/* Test export: the pre-RoPE append's key rotation with fp32 output.
 * X fp16 [N][128*gh] group rows, perm int32 [128*gh] -> Xrot fp32 [N][128*gh]. */
KVQ_API kvq_status kvq_debug_rotate_group_f32(const uint16_t *X, int32_t N, int32_t group_heads,
                                              const int32_t *perm, float *Xrot, void *stream);

/*
 * One serving step in one call: kvq_rotate_quantize_append of the step's T
 * new tokens, then kvq_decode_attention of one query per query head over the
 * updated cache (seq_lens, updated by the append on the device, are the
 * decode's lengths).  Arguments as in those two calls; all argument checks
 * run before anything is launched; an error leaves nothing enqueued.
 */
KVQ_API kvq_status kvq_append_decode(const uint16_t *K, const uint16_t *V, int32_t T,
                                     const uint16_t *Q, int32_t Hq, const kvq_cache_desc *cache,
                                     kvq_rot_mode mode, const float *R_k, const float *R_v,
                                     const int32_t *perm, int32_t *seq_lens, int32_t max_ctx,
                                     void *workspace, size_t ws_bytes, uint16_t *out,
                                     void *stream);

/*
 * The serving step with host buffers: the step's new K, V rows and queries
 * are in host memory, and so is the output.  Inside one call: the
 * host-to-device copies of K, V and Q into the staging part of the
 * workspace (one copy when V_host starts where K_host ends and Q_host where
 * V_host ends, else three), kvq_append_decode on them, and one
 * device-to-host copy of the output,
 * all asynchronous on `stream` (host memory should be pinned for the copies
 * to overlap; pageable memory works, synchronously).  Synchronise the
 * stream before reading out_host.
 *   K_host, V_host  fp16 [B][T][Hkv][128];  Q_host, out_host fp16 [B][Hq][128].
 *   workspace       device, >= kvq_step_workspace_size(B, T, Hq, Hkv, max_ctx,
 *                   SMs) bytes, 256-B aligned.
 * Other arguments and errors as kvq_append_decode.
 */
KVQ_API size_t kvq_step_workspace_size(int32_t B, int32_t T, int32_t Hq, int32_t Hkv,
                                       int32_t max_ctx, int32_t sm_count);
KVQ_API kvq_status kvq_append_decode_host(const uint16_t *K_host, const uint16_t *V_host,
                                          int32_t T, const uint16_t *Q_host, int32_t Hq,
                                          const kvq_cache_desc *cache, kvq_rot_mode mode,
                                          const float *R_k, const float *R_v,
                                          const int32_t *perm, int32_t *seq_lens,
                                          int32_t max_ctx, void *workspace, size_t ws_bytes,
                                          uint16_t *out_host, void *stream);

/* Short text for a status code (static storage). */
KVQ_API const char *kvq_status_string(kvq_status s);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
