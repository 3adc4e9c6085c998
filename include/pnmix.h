/*
 * pnmix.h -- C ABI of the PN-Mix mixed-precision KV-cache library for B200 (sm_100a).
 *
 * What the library computes
 * -------------------------
 * The method is PN-Mix ("PN-Mix: Pair-Norm Guided Mixed-Precision Key Cache
 * Quantization for Efficient Long-Output LLM Inference", abstract): RoPE
 * channel pairs whose query pair-norm x key pair-norm product is large carry
 * most of the attention-logit error under low-bit key quantization, so those
 * pairs get more bits.  The salient pairs are chosen once at prefill and kept
 * for the whole decode.  Values are quantized per token (the per-token value
 * scheme of "MixKVQ: Query-Aware Mixed-Precision KV Cache Quantization for
 * Long-Context Reasoning", abstract and "Innovation" list; the KIVI-style
 * per-channel-key / per-token-value split recorded in the PM-KVQ review,
 * "key_machinery").
 *
 * The five calls of the path, in call order:
 *   pnmix_select_pairs    -- prefill: score the 64 RoPE pairs per KV head, keep the top k
 *   pnmix_quantize_keys   -- prefill: per-channel 32-token groups, salient pairs at b_hi bits
 *   pnmix_quantize_values -- prefill: per-token 32-channel groups at b_v bits
 *   pnmix_append          -- decode: write one new K/V row, quantize every full 32-token group
 *   pnmix_decode_attention-- decode: split-K attention over the packed cache + bf16 residual
 *   (pnmix_decode_attention_multi: the same for several new tokens per sequence, causal)
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - All tensor pointers are DEVICE pointers unless a comment says otherwise.
 *    bf16 tensors are passed as `const uint16_t*` holding the raw bf16 bits.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call only enqueues work on that stream; no call synchronises, allocates
 *    or frees device memory.  The caller owns every buffer.
 *  - Arguments are validated on the host before anything is enqueued.  A call
 *    that returns anything but PNMIX_OK has enqueued nothing, except
 *    PNMIX_ERR_CUDA, which reports a launch error from the CUDA runtime.
 *  - Conditions only the device can see (a full cache on append, a bounded wait
 *    that ran out) set bits in the cache's device error word; read it with
 *    pnmix_read_error.  No kernel traps or asserts.
 *  - A cache's device state (lengths, permutation, records) is valid only once
 *    pnmix_cache_reset has run on it, and is kept valid by these calls alone: the
 *    caller orders every call after the work it depends on (the zero fill and reset
 *    of the cache memory included) when it uses more than one stream.  The decode
 *    kernels take the lengths as they find them; append and shrink clamp them to
 *    [0, capacity], and the quantizers mask permutation entries to a channel index.
 *  - head_dim is 128; rows of K, V and Q are 128 contiguous bf16 values.
 *
 * Numerical contract
 * ------------------
 * Quantization (codes, fp16 scales and zero points, packing, pair indices) is
 * computed in IEEE fp32 round-to-nearest-even in the op order below, with no
 * FMA contraction, and is bit-exact with the reference definition:
 *   pair p in [0,64) is channels (p, p+64) (half-split RoPE pairing);
 *   key norm     K_p = sqrt(max_t (k_{t,p}^2 + k_{t,p+64}^2)) over all L prefill tokens;
 *   query norm   Q_p = (sum over heads h of the group, then tokens of the window,
 *                       of sqrt(q_{h,t,p}^2 + q_{h,t,p+64}^2)) / (G * W');
 *   score        s_p = Q_p * K_p (or the statistic cfg->saliency_score names, see
 *                PNMIX_SCORE_*), top k by (s desc, p asc);
 *   quantizer    mn, mx over the group; s16 = fp16(fl(mx - mn) / (2^b - 1));
 *                z16 = fp16(mn); code = clamp(rint((x - z) / s), 0, 2^b - 1)
 *                with s, z the fp32 values of s16, z16; all codes 0 when s16 == 0.
 * Attention is  out_h = sum_t softmax_t(q_h . k^_t * scale) v^_t  over every
 * cached token (over a causal prefix in pnmix_decode_attention_multi), with
 * k^ = code*s + z for packed tokens and the bf16 value for residual tokens; it is
 * accumulated in fp32 and returned in fp32.
 *
 * Packed cache layout (the contract the oracle and the kernels share)
 * ------------------------------------------------------------------
 * The cache of one sequence b and KV head h is a run of fixed-size GROUP
 * RECORDS, one per 32 tokens, followed (logically) by a bf16 residual window of
 * the newest len % 32 tokens.  Group g of (b, h) lives at
 *     records + ((b * n_kv_heads + h) * (capacity_tokens / 32) + g) * record_bytes.
 *
 * Key positions.  Within (b, h) the 128 key channels are put in POSITION order:
 * first the 2k salient channels {p, p+64 : p salient} ascending, then the other
 * channels ascending.  perm[j] is the channel at position j.  Positions
 * [0, 2k) use b_hi bits, positions [2k, 128) use b_lo bits.  Position slice
 * sigma = j / 16 (8 slices; 2k is a multiple of 16).
 *
 * Lane coordinates.  Everything below is indexed by a 32-lane coordinate
 * L = 4*gq + tq (gq = L >> 2 in [0,8), tq = L & 3 in [0,4)), the fragment
 * ownership of a 16x8x16 matrix-multiply-accumulate tile.
 *
 * Record, in this order (all offsets are multiples of 128 bytes):
 *  1. Key codes, KC = 128 * (WH + WL) bytes, WH = (2k/16) * b_hi / 2,
 *     WL = ((128-2k)/16) * b_lo / 2 words per lane.
 *     A key SLOT is (slice sigma, c in {0,1}, u in {0..3}); it names the two
 *     positions P0 = 16*sigma + 2*tq + 8*c and P1 = P0 + 1 of token
 *     tau = gq + 8*u.  Within the hi block (slices [0, 2k/16)) the lane-local
 *     slot number is n = (sigma*8 + c*4 + u); within the lo block it is
 *     n = ((sigma - 2k/16)*8 + c*4 + u).  With m = 16 / b slots per 32-bit word,
 *     the slot sits in lane-local word n / m (counted from 0 for the hi block and
 *     from WH for the lo block), at position r = n % m: the code of (tau, P0) at
 *     bits [b*r, b*r + b) and the code of (tau, P1) at bits [16 + b*r, 16 + b*r + b).
 *     Lane-local word w of lane L is stored at byte offset (w * 32 + L) * 4.
 *  2. Key scales, 128 fp16 (256 B): the scale of position
 *     j = 16*sigma + 8*e + 2*tq + v  (e, v in {0,1}) is fp16 element
 *     ((tq * 4 + sigma / 2) * 4 + 2 * e + sigma % 2) * 2 + v, so the 16 bytes of one
 *     (tq, slice pair) hold the pairs (even slice e=0, odd slice e=0, even slice e=1,
 *     odd slice e=1).
 *  3. Key zero points, 128 fp16 (256 B), same order as 2.
 *  4. Value codes, 1024 B, b_v = 2 bits.  A value SLOT is (m in {0..7},
 *     r in {0,1}, p in {0..3}); it names channel 16*m + gq + 8*r and the token
 *     pair (2*tq + 8*p, 2*tq + 8*p + 1).  The slot is word m of lane L at
 *     position q = r*4 + p: the code of the first token at bits [2q, 2q+2), of the
 *     second at bits [16 + 2q, 16 + 2q + 2).  Word m of lane L is stored at
 *     byte offset ((m >> 2) * 32 + L) * 16 + (m & 3) * 4.
 *  5. Value scales, 64 fp16x2 (256 B): element (tp * 4 + jg) is the pair
 *     (scale of token 2*tp, scale of token 2*tp+1) of channel group jg
 *     (channels [32*jg, 32*jg + 32)), tp in [0,16).
 *  6. Value zero points, 64 fp16x2 (256 B): the pair (zero of token 2*tp, zero of
 *     token 2*tp+1) of channel group jg is element
 *     ((tp % 4) * 4 + jg) * 4 + (tp / 8) + 2 * ((tp / 4) % 2),
 *     so the 16 bytes of one (tp % 4, jg) hold tp, tp + 8, tp + 4, tp + 12 in that order.
 * record_bytes = KC + 2048 (3200 B at b_hi=4, b_lo=2, k=8, i.e. 100 B/token).
 *
 * Other regions of the cache (all carved out of one caller-owned buffer by
 * pnmix_cache_init): residual K and V bf16 [B][Hkv][32][128] (slot = token % 32),
 * len int32 [B], pair_idx uint8 [B][Hkv][64] (first k entries, ascending),
 * pair_mask uint64 [B][Hkv] (bit p set iff pair p is salient), perm uint8
 * [B][Hkv][128], pair_scores fp32 [B][Hkv][64] (s_p of the last
 * pnmix_select_pairs), scratch and the error word.
 */
#ifndef PNMIX_H
#define PNMIX_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PNMIX_API __attribute__((visibility("default")))
#else
#define PNMIX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PNMIX_OK = 0,
  PNMIX_ERR_INVALID_ARG = 1,  /* null pointer, negative size, inconsistent shapes */
  PNMIX_ERR_UNSUPPORTED = 2,  /* a configuration outside the supported set below */
  PNMIX_ERR_CAPACITY = 3,     /* the request does not fit the cache or the workspace */
  PNMIX_ERR_CUDA = 4,         /* the CUDA runtime reported an error for a launch */
  PNMIX_ERR_ALIGNMENT = 5,    /* a pointer is not aligned as required */
  PNMIX_ERR_DEVICE = 6        /* pnmix_read_error found a non-zero device error word */
} pnmix_status;

/* Device error word bits (pnmix_read_error). */
#define PNMIX_DEVERR_APPEND_FULL 0x1u  /* pnmix_append found len == capacity_tokens */
#define PNMIX_DEVERR_TIMEOUT 0x2u      /* a bounded wait for staged cache data ran out in a
                                          decode call (its output is then invalid); see
                                          pnmix_debug_decode_stall */

/*
 * Method parameters.  Supported set:
 *   head_dim 128; group_tokens 32; residual_tokens 32; value_group 32; value_bits 2;
 *   (key_bits_hi, key_bits_lo) in {(4,2), (2,1)};
 *   n_salient_pairs k in {0, 8, 16, 32, 64} with WH and WL (see the layout) whole
 *     numbers, i.e. every k for (4,2) and k in {0, 16, 32, 64} for (2,1);
 *   G = n_q_heads / n_kv_heads in [1, 8];
 *   saliency_window W in [1, 1024];
 *   saliency_score in {0, 1, 2} (PNMIX_SCORE_*);
 *   n_pruned_pairs in [0, 63]; n_pruned_slices in [0, 8]; not both non-zero;
 *   decode_kernel in {0, 1, 2, 3, 4} (PNMIX_DECODE_*).
 * softmax_scale <= 0 selects 1/sqrt(head_dim).
 *
 * Dynamic query-channel pruning (n_pruned_pairs > 0; the query-channel pruning of the
 * "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches" abstract, applied
 * to RoPE pairs): in every decode call each query row drops the n_pruned_pairs pairs with
 * the smallest squared pair norm fl(fl(q_p^2) + fl(q_{p+64}^2)), never pair 0 (the
 * abstract's channel-0 protection), the higher pair index first among equal norms.  A
 * dropped pair contributes nothing to that row's logits (its query channels count as
 * zero).  The packed records are still read whole; what changes is the arithmetic.
 *
 * Key-slice pruning (n_pruned_slices > 0; the same abstract's query-channel pruning taken
 * at the granularity the records store keys in): in every decode call, per (sequence, KV
 * head) unit and for all query rows that attend it together,
 * the n_pruned_slices position slices of the low-precision block (sigma in [2k/16, 8)) with
 * the least energy  E_sigma = sum over rows v of sum over the slice's 16 positions j of
 * q_v[perm[j]]^2  are dropped: rows in order, positions in order, every square and partial
 * sum rounded to fp32; slices holding channel 0 or 64 are never dropped (channel-0
 * protection); the higher slice goes first among equal energies; when fewer slices are
 * candidates, all of them are dropped.  A dropped slice's channels count as zero in every
 * row's query (packed and residual tokens alike).  The records are still read whole: at
 * b_lo = 2 a dropped slice is one 128-byte row of each record, and leaving those rows
 * unread (one copy per run of kept rows) or skipping their products (a branch per slice in
 * the unrolled group loop) measured slower on B200 than reading and multiplying them.
 * Not available in pnmix_decode_attention_two (its two parts order positions differently).
 */
typedef struct {
  int32_t head_dim;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t group_tokens;
  int32_t residual_tokens;
  int32_t key_bits_hi;
  int32_t key_bits_lo;
  int32_t n_salient_pairs;
  int32_t value_bits;
  int32_t value_group;
  int32_t saliency_window;
  float softmax_scale;
  int32_t saliency_score;   /* statistic that ranks the pairs, PNMIX_SCORE_* (0 = PN-Mix) */
  int32_t n_pruned_pairs;   /* decode: query pairs each query row drops, 0..63 (0 = none) */
  int32_t decode_kernel;    /* decode: which kernel runs, PNMIX_DECODE_* (0 = automatic) */
  int32_t n_pruned_slices;  /* decode: low-precision key slices each unit drops, 0..8 (0 = none) */
} pnmix_config;

/*
 * Decode kernels (cfg->decode_kernel).  All give the result of the numerical contract
 * above; they differ in speed.  The choice is part of the configuration, so it costs no
 * host work per call.
 *   PNMIX_DECODE_AUTO   the faster tensor-core kernel for the shape (one role per warp for
 *                       up to 4 query rows per KV head, warp pairs up to 8, warps of 8 rows
 *                       up to 32, PNMIX_DECODE_TC from 33 rows on).
 *   PNMIX_DECODE_SIMT   CUDA cores only (a baseline): one query per sequence and no query
 *                       pruning (PNMIX_ERR_UNSUPPORTED otherwise).
 *   PNMIX_DECODE_MMA    tensor cores, every warp scores and accumulates its own groups.
 *   PNMIX_DECODE_PAIRS  tensor cores, a key-side and a value-side warp per group stream.
 *   PNMIX_DECODE_TC     5th-generation tensor cores (tcgen05, accumulators in TMEM): each
 *                       group's keys and values dequantized once into shared memory for all
 *                       of a unit's query rows (up to 128); its cost per group hardly depends
 *                       on the rows, so it is the multi-token kernel.  Keys and values whose
 *                       32-token group range exceeds 65504 are outside its domain (c * s must
 *                       be a finite fp16).
 */
#define PNMIX_DECODE_AUTO 0
#define PNMIX_DECODE_SIMT 1
#define PNMIX_DECODE_MMA 2
#define PNMIX_DECODE_PAIRS 3
#define PNMIX_DECODE_TC 4

/*
 * Pair statistics pnmix_select_pairs can rank by (all per (b, kv head), fp32, one
 * rounding per operation; K_p and Q_p as defined at pnmix_select_pairs):
 *   PNMIX_SCORE_PNMIX        s_p = Q_p * K_p, the PN-Mix pair-norm product (default).
 *   PNMIX_SCORE_KEY_ONLY     s_p = K_p: key statistics alone, the channel-saliency
 *                            estimate of the earlier mixed-precision methods that the
 *                            PN-Mix abstract compares against.
 *   PNMIX_SCORE_RANGE_QUERY  s_p = Q_p * sqrt(r_p^2 + r_{p+64}^2), r_c = max_t k - min_t k
 *                            of channel c over the L rows: quantization difficulty (the
 *                            range the min-max code must span) times query relevance, the
 *                            two factors named by the MixKVQ abstract.  The page gives no
 *                            formula; this is its plainest pair-level reading.
 */
#define PNMIX_SCORE_PNMIX 0
#define PNMIX_SCORE_KEY_ONLY 1
#define PNMIX_SCORE_RANGE_QUERY 2

/* Device pointers into one caller-owned buffer; filled by pnmix_cache_init. */
typedef struct {
  int32_t batch;
  int32_t capacity_tokens;   /* multiple of 32 */
  int32_t n_kv_heads;
  int32_t record_bytes;
  uint8_t* records;          /* [B][Hkv][capacity/32][record_bytes] */
  uint16_t* k_resid;         /* bf16 [B][Hkv][32][128] */
  uint16_t* v_resid;         /* bf16 [B][Hkv][32][128] */
  int32_t* len;              /* [B] tokens held (packed + residual) */
  uint8_t* pair_idx;         /* [B][Hkv][64] */
  uint64_t* pair_mask;       /* [B][Hkv] */
  uint8_t* perm;             /* [B][Hkv][128] */
  float* pair_scores;        /* [B][Hkv][64] */
  uint32_t* scratch;         /* library-internal counters and reduction space */
  uint32_t* error;           /* device error word */
  void* base;
  size_t total_bytes;
} pnmix_cache;

/* Bytes of one group record (layout item list above); 0 if unsupported. */
PNMIX_API size_t pnmix_record_bytes(const pnmix_config* cfg);

/*
 * Bytes a cache of `batch` sequences and `capacity_tokens` tokens each needs.
 * capacity_tokens must be a positive multiple of 32.  Host-only.
 */
PNMIX_API pnmix_status pnmix_cache_bytes(const pnmix_config* cfg, int batch, int capacity_tokens,
                               size_t* total_bytes);

/*
 * Carve the regions of a cache out of `device_base` (>= pnmix_cache_bytes bytes,
 * 256-byte aligned) and fill *out.  Host-only: touches no device memory.  The
 * buffer must be zero-filled before the first pnmix call that uses it
 * (pnmix_cache_reset does that).
 */
PNMIX_API pnmix_status pnmix_cache_init(const pnmix_config* cfg, int batch, int capacity_tokens,
                              void* device_base, size_t bytes, pnmix_cache* out);

/* Zero the whole cache buffer on `stream` (lengths 0, no salient pairs, no error). */
PNMIX_API pnmix_status pnmix_cache_reset(const pnmix_cache* cache, void* stream);

/*
 * Prefill step 1 (PN-Mix abstract: salient pairs are picked once at prefill from
 * the query-key pair-norm product).  For every (b, kv head h):
 *   K_p = sqrt(max over the first L rows of k of k_p^2 + k_{p+64}^2), Q_p = the mean
 *   over the n_window rows of q_window of the G query heads h*G .. h*G+G-1 of
 *   sqrt(q_p^2 + q_{p+64}^2) (heads outer, rows inner), s_p = Q_p * K_p (or the
 *   statistic cfg->saliency_score names); the k = n_salient_pairs pairs with the
 *   largest s_p (ties to the lower p) become salient.
 * q_window: bf16 [B][Hq][n_window][128] -- the LAST n_window prefill queries, after RoPE.
 * k:        bf16 [B][Hkv][ld_tokens][128], rows [0, L) used, after RoPE.
 * n_window must equal min(L, saliency_window); 1 <= L <= ld_tokens.
 * Writes pair_idx, pair_mask, perm and pair_scores of every (b, h).
 */
PNMIX_API pnmix_status pnmix_select_pairs(const pnmix_config* cfg, const uint16_t* q_window, int n_window,
                                const uint16_t* k, int L, int ld_tokens, pnmix_cache* cache,
                                void* stream);

/*
 * Prefill step 2 (mixed-precision per-channel keys; PN-Mix abstract).  Quantizes
 * tokens [0, 32*floor(L/32)) of k into the key part of group records 0..,
 * copies the last L % 32 rows into the K residual and sets len[b] = L.
 * Uses the salient set written by pnmix_select_pairs.  L <= capacity_tokens.
 */
PNMIX_API pnmix_status pnmix_quantize_keys(const pnmix_config* cfg, const uint16_t* k, int L, int ld_tokens,
                                 pnmix_cache* cache, void* stream);

/*
 * Prefill step 3 (per-token values; MixKVQ abstract).  Same token split as
 * pnmix_quantize_keys, into the value part of the records and the V residual;
 * sets len[b] = L.
 */
PNMIX_API pnmix_status pnmix_quantize_values(const pnmix_config* cfg, const uint16_t* v, int L, int ld_tokens,
                                   pnmix_cache* cache, void* stream);

/*
 * Decode step 1 (streaming append; PN-Mix abstract: the prefill choice of
 * salient pairs is reused for the whole decode).  k_new, v_new: bf16 [B][Hkv][128].
 * For every b: the row goes to residual slot len[b] % 32; when that slot is 31
 * the 32 residual rows are quantized into group record len[b] / 32 with the
 * prefill's salient pairs; then len[b] += 1.  A sequence whose len[b] equals
 * capacity_tokens is left unchanged and PNMIX_DEVERR_APPEND_FULL is raised.
 */
PNMIX_API pnmix_status pnmix_append(const pnmix_config* cfg, const uint16_t* k_new, const uint16_t* v_new,
                          pnmix_cache* cache, void* stream);

/*
 * Workspace bytes pnmix_decode_attention needs for `batch` sequences whose
 * lengths are at most max_context.  The workspace must be zero-filled before its
 * first use; every call leaves it ready for the next one.
 */
PNMIX_API size_t pnmix_workspace_bytes(const pnmix_config* cfg, int batch, int max_context);

/*
 * Decode step 2 (attention over the quantized cache).  q: bf16 [B][Hq][128]
 * (after RoPE); out: fp32 [B][Hq][128].  Attends over all len[b] cached tokens
 * (the query's own K/V must have been appended first if it is to be included).
 * max_context is an upper bound on len[b] used to size the split-K grid; the
 * result does not depend on it.  A sequence with len[b] == 0 gets zeros.
 */
PNMIX_API pnmix_status pnmix_decode_attention(const pnmix_config* cfg, const uint16_t* q,
                                    const pnmix_cache* cache, int max_context, float* out,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * One decode step in one call: pnmix_append of k_new, v_new (bf16 [B][Hkv][128]) followed
 * by pnmix_decode_attention of q (bf16 [B][Hq][128]) over the cache that includes the new
 * token; out fp32 [B][Hq][128].  The result, the cache contents and the error bits are
 * those of the two calls in sequence.  With the one-role tensor-core kernel (the automatic
 * choice for up to 4 query heads per KV head, or PNMIX_DECODE_MMA) the append runs inside
 * the decode launch: the CTA that attends over a unit's residual window stores the new row
 * there, on a step that completes a 32-token group the CTA owning that group quantizes it
 * (the same quantizers, bit-exact) and stores its record, and the launch's last CTA
 * advances len[].  Other kernels take an append launch first.  max_context bounds the
 * lengths after the append; workspace as for pnmix_decode_attention.  Errors as for
 * pnmix_decode_attention and pnmix_append.
 */
PNMIX_API pnmix_status pnmix_append_decode(const pnmix_config* cfg, const uint16_t* k_new, const uint16_t* v_new,
                                           const uint16_t* q, pnmix_cache* cache, int max_context, float* out,
                                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Workspace bytes pnmix_decode_attention_multi needs for n_queries queries per
 * sequence (n_queries = 1 gives pnmix_workspace_bytes); 0 if unsupported.
 */
PNMIX_API size_t pnmix_workspace_bytes_multi(const pnmix_config* cfg, int batch, int max_context,
                                             int n_queries);

/*
 * Decode attention of T = n_queries new tokens per sequence at once (a speculative
 * verify or chunked decode step), after all T of their K/V rows were appended with
 * pnmix_append.  q: bf16 [B][T][Hq][128] (after RoPE); out: fp32 [B][T][Hq][128].
 * Query j (0-based) of sequence b attends causally over the first len[b] - T + 1 + j
 * cached tokens: the cache before the step plus the new tokens up to its own.  The
 * pages have no such call; it is the multi-token neighbour of pnmix_decode_attention
 * (T = 1 gives the same result).  Requires 1 <= T and G * T <= 128 with the automatic
 * choice or PNMIX_DECODE_TC, G * T <= 64 with the other kernels (PNMIX_ERR_UNSUPPORTED
 * otherwise; PNMIX_DECODE_SIMT takes T = 1 only).  Up to 8 query rows per KV head (G * T)
 * run on the single-query kernels; 9 to 32 rows on a kernel whose warps each hold 8 rows
 * and share one staging of the packed records, and from 33 rows on the tcgen05 kernel
 * (PNMIX_DECODE_TC, one row per tensor-memory lane), so the cache is read once for all T
 * queries.  A query that sees no
 * token gets zeros.  Workspace from pnmix_workspace_bytes_multi with the same T.
 */
PNMIX_API pnmix_status pnmix_decode_attention_multi(const pnmix_config* cfg, const uint16_t* q,
                                                    int n_queries, const pnmix_cache* cache,
                                                    int max_context, float* out, void* workspace,
                                                    size_t workspace_bytes, void* stream);

/*
 * Shrink the salient key positions of a cache from b_hi to b_lo = b_hi / 2 bits (the
 * equivalent right shift of the PM-KVQ review page, "key_machinery": the bit-width
 * shrinking step of its progressive quantization).
 *   cfg  the configuration src was built with (key_bits_hi = 2 * key_bits_lo, which holds
 *        for both supported pairs, and n_salient_pairs > 0).
 *   src  a cache of cfg; read only.
 *   dst  a cache of the same batch and capacity laid out for cfg with n_salient_pairs = 0
 *        (pnmix_cache_init with that config), in memory that does not overlap src's.
 * Every full group record of src is written to dst with all positions at b_lo bits in the
 * SAME position order: for positions [0, 2k) the code X becomes
 * ((2^(2b) - 2^b + 1) * (X + 2^(b-1))) >> 3b with b = b_lo, which is round(X / (2^b + 1)),
 * and the scale becomes fp16(fl(s * (2^b + 1))); zero points, the other positions, the value
 * part, the residual window, len, perm and pair_scores are copied, and pair_idx and
 * pair_mask cleared.  Decode dst with the n_salient_pairs = 0 config.  One launch on
 * `stream`, asynchronous.  Errors: INVALID_ARG for null pointers, a dst of another shape
 * or layout, or overlapping caches; UNSUPPORTED for k = 0 or a configuration outside the
 * supported set; CUDA for a launch failure.
 */
PNMIX_API pnmix_status pnmix_shrink_keys(const pnmix_config* cfg, const pnmix_cache* src, pnmix_cache* dst,
                                         void* stream);

/*
 * Token-level two-precision mixing, prefill side ("SemKV: Semantic Mixed-Precision KV
 * Cache Quantization Guided by the Quality Cliff for Long-Context LLM Inference",
 * abstract: tokens ranked by a model-internal score take one of two adjacent precisions).
 * The unit of assignment is a 32-token group.  Per (sequence b, KV head h), with
 * ng = L / 32 full groups and n_hi = floor(ng * hi_percent / 100):
 *   qbar[c]  = (sum over the G heads of h and the window tokens of q_window[c]) / (G * W'),
 *              heads outer, tokens inner, fp32;
 *   score[g] = max over the tokens t of group g of sum_c qbar[c] * k[t][c] (channels in
 *              order; every product and sum one fp32 rounding; first maximum kept);
 *   route[g] = 1 for the n_hi best-ranked groups (score descending, ties: lower g), else 0;
 *   dest[g]  = the number of groups before g with the same route.
 * Group g's 32 K and V rows are copied to rows [32 dest[g], 32 dest[g] + 32) of the high
 * part (route 1) or the low part (route 0); the L mod 32 tail rows end the low part.
 *   cfg, batch    the configuration and batch of the caches the parts will fill (only its
 *                 head counts and saliency_window are read here).
 *   q_window      bf16 [batch][Hq][n_window][128], n_window = min(L, saliency_window), as
 *                 for pnmix_select_pairs.
 *   k, v          bf16 [batch][Hkv][ld_tokens][128], tokens [0, L) read.
 *   hi_percent    0..100.
 *   scores        fp32 [batch][Hkv][ng], route uint8 [batch][Hkv][ng], dest int32
 *                 [batch][Hkv][ng]: written (may be NULL when ng = 0).
 *   k_hi, v_hi    bf16 [batch][Hkv][L_hi][128], L_hi = 32 n_hi (NULL allowed if L_hi = 0).
 *   k_lo, v_lo    bf16 [batch][Hkv][L_lo][128], L_lo = L - L_hi (NULL allowed if L_lo = 0).
 * A mixed cache is then two caches: pnmix_select_pairs of each on the full k (its own
 * n_salient_pairs), and pnmix_quantize_keys / _values of each part with L_hi / L_lo.
 * Two launches on `stream`; the ranking costs ng^2 comparisons per (b, h).  Errors:
 * INVALID_ARG (null pointers, L < 1, ld_tokens < L, n_window, hi_percent outside 0..100,
 * query heads not a multiple of KV heads), UNSUPPORTED (a configuration outside the
 * supported set), ALIGNMENT (bf16 pointers not 16-byte aligned), CUDA.
 */
PNMIX_API pnmix_status pnmix_split_groups(const pnmix_config* cfg, int batch, const uint16_t* q_window,
                                          int n_window, const uint16_t* k, const uint16_t* v, int L,
                                          int ld_tokens, int hi_percent, float* scores, uint8_t* route,
                                          int32_t* dest, uint16_t* k_hi, uint16_t* v_hi, uint16_t* k_lo,
                                          uint16_t* v_lo, void* stream);

/*
 * pnmix_decode_attention without a caller-provided workspace.  The pages have no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory (a plugin whose host runtime owns all device memory, or an interface
 * with no slot for a workspace pointer).  Same arguments, validation and result as
 * pnmix_decode_attention minus the workspace: the split-K scratch comes from a
 * 4 MiB array inside the library image, held on every device that loads the
 * library until the process exits.  A call whose pnmix_workspace_bytes exceeds
 * 4 MiB returns PNMIX_ERR_CAPACITY, and every rejected call enqueues nothing.
 * Every call on a device shares that array and first clears the words of it that
 * must start at zero (a memset on `stream`), so calls that overlap on the GPU race
 * and must be serialised by the caller.  The array's address is looked up on every
 * call for the current device, which `stream` must belong to; the first call on a
 * device also loads the library's device code there, so make it before any stream
 * capture.  Allocates nothing.
 */
PNMIX_API pnmix_status pnmix_decode_attention_noalloc(const pnmix_config* cfg, const uint16_t* q,
                                                      const pnmix_cache* cache, int max_context,
                                                      float* out, void* stream);

/*
 * Decode attention over a cache held in two parts (SemKV abstract, "SemKV: Semantic
 * Mixed-Precision KV Cache Quantization Guided by the Quality Cliff for Long-Context LLM
 * Inference": every token is kept, at one of two adjacent precisions).  Part a and part b
 * are two caches of the same batch and head layout holding disjoint token sets, e.g. the
 * high and the low precision parts that pnmix_split_groups prepares; each is read with its
 * own configuration (cfg_a / cfg_b: bit widths and salient pairs may differ).  The result
 * is the attention of every query row over the union of both parts' tokens:
 *     out = sum over the tokens of both parts of softmax(q . k^ * scale) v^,
 * computed as two decode launches: part a's normalised output and log-sum-exp go to the
 * workspace, and part b's combine merges them with its own,
 *     out = (2^(La - M) oa + 2^(Lb - M) ob) / (2^(La - M) + 2^(Lb - M)),  M = max(La, Lb)
 * (log2-domain log-sum-exps; a part that holds no token of a sequence weighs nothing, and
 * a sequence with no token in either part gets zeros).  q bf16 [B][Hq][128], out fp32
 * [B][Hq][128].  max_context_a / _b bound the lengths of each part as in
 * pnmix_decode_attention.  Workspace: pnmix_workspace_bytes_two bytes, 256-byte aligned,
 * zero-filled before first use; it is left ready for the next call.  Errors as for
 * pnmix_decode_attention, INVALID_ARG when the parts' batch or head counts differ, and
 * UNSUPPORTED when either configuration asks for key-slice pruning.
 */
PNMIX_API size_t pnmix_workspace_bytes_two(const pnmix_config* cfg_a, const pnmix_config* cfg_b, int batch,
                                           int max_context_a, int max_context_b);
PNMIX_API pnmix_status pnmix_decode_attention_two(const pnmix_config* cfg_a, const pnmix_cache* cache_a,
                                                  int max_context_a, const pnmix_config* cfg_b,
                                                  const pnmix_cache* cache_b, int max_context_b,
                                                  const uint16_t* q, float* out, void* workspace,
                                                  size_t workspace_bytes, void* stream);

/*
 * Test hook of the bounded staging wait; the pages have no counterpart.  Runs
 * pnmix_decode_attention (same arguments and validation) with two changes: the
 * packed records of unit skip_unit (= b * n_kv_heads + h, in [0, batch * n_kv_heads))
 * are never staged, and every staging wait gives up after wait_rounds (>= 1) rounds of
 * mbarrier try_wait.  The waits for that unit's records therefore run out: the kernel
 * sets PNMIX_DEVERR_TIMEOUT in the cache's error word, lets every copy it issued land,
 * and returns.  The output of the call is then invalid; the cache, the workspace and
 * the CUDA context stay usable.  Needs a tensor-core decode kernel (PNMIX_ERR_UNSUPPORTED
 * with PNMIX_DECODE_SIMT, which stages nothing).
 */
PNMIX_API pnmix_status pnmix_debug_decode_stall(const pnmix_config* cfg, const uint16_t* q,
                                                const pnmix_cache* cache, int max_context, float* out,
                                                void* workspace, size_t workspace_bytes, int skip_unit,
                                                uint32_t wait_rounds, void* stream);

/* Synchronously read (and, if clear != 0, zero) the device error word.  Host pointer out. */
PNMIX_API pnmix_status pnmix_read_error(const pnmix_cache* cache, int clear, uint32_t* host_error);

/* Static string for a status code. */
PNMIX_API const char* pnmix_status_string(pnmix_status status);

/* Library version, e.g. "pnmix 0.1". */
PNMIX_API const char* pnmix_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PNMIX_H */
