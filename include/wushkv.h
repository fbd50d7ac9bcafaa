/*
 * wushkv.h -- C ABI of libwushkv.so: the online hot path of WUSH-KV
 * ("WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms",
 * arXiv 2609.38121) on NVIDIA B200 (sm_100a).
 *
 * Method facts this library implements (sources are the summary pages of the
 * paper; page titles and sections are named at each call below):
 *   - every KV head owns an invertible d x d key transform T_k applied after
 *     RoPE (k' = T_k k, one d x d product per new token), and queries use its
 *     inverse transpose (q' = T_k^{-T} q) so that q'.k' = q.k;
 *   - values arrive already transformed (the value transform is folded into
 *     W_V and W_O offline), so the cache stores them as given;
 *   - keys and values are quantised per token to 2, 3 or 4 bits with QuEST
 *     INT (RMS-based scale, bin-centre reconstruction) or a percentile-clipped
 *     affine quantiser, and bit-packed;
 *   - the first `sink` tokens and the latest `recent` tokens stay in fp16;
 *     the recent window is flushed to the packed cache `chunk` tokens at a
 *     time;
 *   - decoding is grouped-query attention over the packed cache plus the
 *     fp16 windows.
 *
 * Conventions shared by every call:
 *   - Pointers named *_dev are device pointers; *_host are host pointers.
 *     The library borrows them for the duration of the call (asynchronous
 *     calls: until the work on `stream` completes).  It never allocates
 *     device memory: the caller allocates the cache buffer
 *     (wushkv_cache_bytes) and every input and output.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Compute calls are asynchronous on it.
 *   - Argument errors are detected on the host before any launch and
 *     returned synchronously; nothing is written in that case.  CUDA launch
 *     errors return WUSHKV_ECUDA.  Errors found inside kernels set a sticky
 *     device status word read by wushkv_device_status.
 *   - head_dim is 128.  KV head of query head h is floor(h / G), G =
 *     n_q_heads / n_kv_heads (contiguous groups).
 *   - One cache object holds one layer for `batch` sequences.  wushkv_append
 *     adds n_tok tokens to every sequence; wushkv_append_varlen adds a
 *     per-sequence count, and wushkv_reset_sequence empties one sequence, so
 *     sequences may hold different numbers of tokens (the window policy
 *     applies to each sequence on its own).  With num_pages > 0 the packed
 *     region is paged through a caller-owned page table
 *     (wushkv_set_page_table).
 *   - A "unit" is one (sequence b, KV head h); unit index u = b*n_kv_heads+h.
 */
#ifndef WUSHKV_H
#define WUSHKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WUSHKV_API __attribute__((visibility("default")))
#else
#define WUSHKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WUSHKV_OK = 0,
  WUSHKV_EINVAL = 1,        /* bad argument (NULL pointer, mismatched bits, ...) */
  WUSHKV_ECAPACITY = 2,     /* append would exceed max_ctx; nothing written   */
  WUSHKV_EUNSUPPORTED = 3,  /* valid but not built (head_dim != 128, ...)     */
  WUSHKV_ECUDA = 4          /* a CUDA runtime call failed                     */
} wushkv_status;

typedef enum { WUSHKV_QUEST_INT = 0, WUSHKV_AFFINE_PCTCLIP = 1 } wushkv_quantizer;

/* Bits of the sticky device status word (wushkv_device_status).  A kernel
 * that detects one of these conditions skips the offending access, sets the
 * bit and finishes; the call's results are then not to be trusted.
 *   WUSHKV_DEV_RANGE:   a packed token index beyond the cache's capacity.
 *   WUSHKV_DEV_SPLITS:  a decode split partial beyond the workspace.
 *   WUSHKV_DEV_TIMEOUT: an asynchronous copy did not complete within the
 *                       wait limit (about a second by default). */
enum { WUSHKV_DEV_RANGE = 1, WUSHKV_DEV_SPLITS = 2, WUSHKV_DEV_TIMEOUT = 4 };
typedef enum { WUSHKV_F16 = 0, WUSHKV_BF16 = 1, WUSHKV_F32 = 2 } wushkv_dtype;

/* Cache configuration (one layer).
 *   batch, n_kv_heads, n_q_heads: GQA shape; n_q_heads % n_kv_heads == 0 and
 *     G = n_q_heads / n_kv_heads in {1, 2, 4, 8}.
 *   head_dim: must be 128.
 *   max_ctx: tokens per sequence the cache can hold (>= 1).
 *   bits: 2, 3 or 4.  quantizer: wushkv_quantizer.
 *   sink, recent, chunk: window sizes (summary page "WUSH-KV：数据自适应变换的
 *     KV Cache 低比特量化", sections 工作参考价值 and 方法关键点: 64, 256 and
 *     8 or 16).  sink % 4 == 0, chunk % 4 == 0, chunk >= 4, recent >= 0.
 *   quest_alpha: QuEST clip ratio (clip range +-alpha * RMS); 0 selects the
 *     Gaussian-MSE-optimal default for `bits` (wushkv_default_quest_alpha).
 *     Must satisfy 0 < alpha <= 2^(bits-1).
 *   clip_lo_rank, clip_hi_rank: affine quantiser order statistics (1-indexed
 *     ranks among the 128 values; default 2 and 127).  Supported:
 *     1 <= lo <= 8, 121 <= hi <= 128.
 */
typedef struct {
  int32_t batch, n_kv_heads, n_q_heads, head_dim, max_ctx, bits;
  int32_t quantizer;
  int32_t sink, recent, chunk;
  double quest_alpha;
  int32_t clip_lo_rank, clip_hi_rank;
  int32_t num_pages;   /* 0: dense packed region; > 0: paged (see wushkv_set_page_table) */
} wushkv_config;

typedef struct wushkv_cache wushkv_cache; /* opaque host handle */

/* Byte layout of a cache buffer (offsets from the buffer base).  Exposed so
 * that callers can checkpoint, inspect or move the cache.
 *   Packed region (at offset 0): per unit, packed_capacity / 64 block
 *     records of block_stride bytes, unit u's at u * unit_stride.  A record
 *     holds 64 consecutive packed tokens as [K plane 0][K plane 1][V plane 0]
 *     [V plane 1][K meta][V meta] (plane 1 only for 3-bit), so that one bulk
 *     copy fetches everything the decode needs for those tokens.
 *     k_plane_off[p], v_plane_off[p], k_meta_off and v_meta_off are the
 *     offsets of these parts in unit 0's block 0; block b of unit u adds
 *     u * unit_stride + b * block_stride.  Within a record, 2-bit K quad
 *     b * 16 + q sits at 128 * q; at 3 and 4 bits the K row of packed token
 *     b * 64 + i sits at 16 * w * pos(i) with the row swizzle
 *     pos(i) = (i & 56) | ((i & 7) ^ ((i >> 3) & 3)) (spreads the decode's
 *     shared-memory reads over all banks); V quads b * 16 + q at 64 * w * q,
 *     meta entries at meta_bytes * i.
 * Formats:
 *   planes: 2-bit codes -> one 2-bit plane, 4-bit -> one 4-bit plane, 3-bit
 *     -> a 2-bit plane of (code & 3) and a 1-bit plane of (code >> 2).  A
 *     plane of width w packs 8/w fields per byte; field s of byte beta of a
 *     little-endian 32-bit word is at bit 8*beta + w*s.
 *   K, 2 bits (4-token quads, 128 bytes per quad): word omega holds dims
 *     4*omega + beta at byte beta and token 4*quad + f at field f; with
 *     omega = 8ks + 4h + c it sits at word 4*((2c + ks/2) xor (quad mod 2))
 *     + 2*(ks mod 2) + h of the quad (the decode's score fragment of m-tile
 *     f is the word masked to field f).
 *   K, 3 and 4 bits (token rows, 16*w bytes per token per plane): c in 0..3,
 *     h in 0..1, ks in 0..3, beta in 0..3, rho = 4h + ks: word c*w +
 *     rho/(8/w), field rho % (8/w), dim 32ks + 4c + 16h + beta.
 *   V (4-token quads, 64*w bytes per quad per plane): r in 0..7, rho in
 *     0..15 (mt = rho/2, rh = rho%2), beta in 0..3: unit word j = rho/(8/w),
 *     field rho % (8/w), dim 16mt + r + 8rh, token 4*quad + beta.  Row unit
 *     r sits at position pos = (r + 2*(quad mod 4)) mod 8 of its quad: word
 *     2w*pos + j for w <= 2; for w = 4 word 4pos + j (j < 4) or
 *     32 + 4pos + j - 4 (j >= 4).  (This spreads a warp's reads of a quad
 *     over all shared-memory banks.)
 *   meta: per token, fp16 delta (QuEST, 2 bytes) or fp16 (scale, lo) pair
 *     (affine, 4 bytes); K and V separately.
 *   sink, ring: fp16 [unit][slot][128]; ring slot of post-sink token t is
 *     (t - sink) mod (recent + chunk).
 * Guard bands: the packed region, sink K, sink V, ring K, ring V and the
 *   workspace are each followed by WUSHKV_GUARD_BYTES bytes set to
 *   WUSHKV_GUARD_FILL at creation, which no kernel writes (a test that finds
 *   them changed has found an out-of-bounds write). */
#define WUSHKV_GUARD_BYTES 256
#define WUSHKV_GUARD_FILL 0xA5
typedef struct {
  int32_t n_planes;
  int32_t plane_bits[2];
  int32_t packed_capacity;          /* token slots per unit in the packed region */
  uint64_t k_plane_off[2], v_plane_off[2];   /* parts of unit 0's block 0 */
  uint64_t k_meta_off, v_meta_off;
  uint32_t meta_bytes;              /* per token: 2 (QuEST) or 4 (affine) */
  uint64_t unit_stride;             /* bytes per unit of the packed region */
  uint64_t block_stride;            /* bytes per block record */
  uint64_t sink_k_off, sink_v_off, sink_unit_stride;
  uint64_t ring_k_off, ring_v_off, ring_unit_stride;
  int32_t ring_slots;               /* recent + chunk */
  uint64_t workspace_off, workspace_bytes;
  uint64_t status_off;
  uint64_t total_bytes;
  int32_t num_pages;                /* paged caches: pages in the pool (else 0) */
  uint64_t page_bytes;              /* paged caches: n_kv_heads * block_stride */
} wushkv_layout;

/* Bytes of device memory a cache with this configuration needs (0 if the
 * configuration is invalid).  Includes the split-K decode workspace and the
 * device status word. */
WUSHKV_API size_t wushkv_cache_bytes(const wushkv_config* cfg);

/* Create a cache over caller-allocated device memory `dev_mem` of `bytes`
 * bytes (>= wushkv_cache_bytes(cfg), 256-byte aligned).  Zeroes the buffer
 * asynchronously on `stream`.  On success *out receives a host handle that
 * owns only host metadata (free it with wushkv_cache_destroy; the device
 * buffer stays the caller's).  Errors: EINVAL, EUNSUPPORTED, ECUDA. */
WUSHKV_API wushkv_status wushkv_cache_create(const wushkv_config* cfg, void* dev_mem, size_t bytes,
                                  void* stream, wushkv_cache** out);
WUSHKV_API wushkv_status wushkv_cache_destroy(wushkv_cache* cache);

/* Fill *out with the byte layout of this cache. */
WUSHKV_API wushkv_status wushkv_cache_layout(const wushkv_cache* cache, wushkv_layout* out);

/* Token counts of sequence 0: total, sink, packed, recent (host-side
 * bookkeeping, no synchronisation).  Any pointer may be NULL. */
WUSHKV_API wushkv_status wushkv_cache_tokens(const wushkv_cache* cache, int64_t* n_tokens, int64_t* n_sink,
                                  int64_t* n_packed, int64_t* n_recent);

/* Token counts of sequence seq (0 <= seq < batch), as wushkv_cache_tokens.
 * Sequences may hold different numbers of tokens (wushkv_append_varlen,
 * wushkv_reset_sequence); the window policy applies to each on its own. */
WUSHKV_API wushkv_status wushkv_sequence_tokens(const wushkv_cache* cache, int32_t seq, int64_t* n_tokens,
                                                int64_t* n_sink, int64_t* n_packed, int64_t* n_recent);

/* Empty sequence seq (its count drops to 0; its slots are reused by later
 * appends), e.g. when a serving loop gives the batch slot to a new request.
 * Host bookkeeping only: nothing is launched. */
WUSHKV_API wushkv_status wushkv_reset_sequence(wushkv_cache* cache, int32_t seq);

/* Paged caches (config num_pages > 0).  The packed tokens of a sequence live
 * in 64-token blocks scattered over a pool of num_pages pages; a page holds
 * the block records of all n_kv_heads heads of one block (page_bytes =
 * n_kv_heads * block_stride, page p at byte p * page_bytes of the packed
 * region; one spare page follows the pool).  The caller owns the page
 * table, as a serving engine's cache manager does:
 *   page_table_dev: [batch][max_pages_per_seq] int32 device array; entry
 *     [b][i] is the page of block i (packed tokens 64i .. 64i + 63) of
 *     sequence b.  It must map every block an append writes or a decode
 *     reads (blocks 0 .. ceil(n_packed_after / 64) - 1 of each sequence)
 *     before that call runs, and distinct sequences must not share a page.
 *     A page id outside [0, num_pages) is redirected to the spare page and
 *     reported as WUSHKV_DEV_RANGE.
 *   max_pages_per_seq >= packed_capacity / 64 (EINVAL otherwise).
 * The pointer is borrowed until the cache is destroyed or the table is
 * replaced.  Sink and recent windows stay in the dense per-sequence regions.
 * EINVAL on a dense cache. */
WUSHKV_API wushkv_status wushkv_set_page_table(wushkv_cache* cache, const int32_t* page_table_dev,
                                               int32_t max_pages_per_seq);

/* Append n_tok tokens to every sequence.
 *   Source: summary page "WUSH-KV：数据自适应变换的 KV Cache 低比特量化",
 *   方法关键点 (key transform after RoPE, one d x d product per new token;
 *   quantiser choice; sink/recent windows with chunked flush).
 *   k_rope_dev: [batch][n_tok][n_kv_heads][128] post-RoPE keys, dtype in_dtype.
 *   v_dev:      [batch][n_tok][n_kv_heads][128] values (already in the
 *               transformed value space), dtype in_dtype.
 *   T_k_dev:    [n_kv_heads][128][128] fp32 row-major, k'_i = sum_j T[i][j] k_j,
 *               16-byte aligned (EINVAL otherwise); NULL means the keys are
 *               already transformed (no product).
 *   bits, quantizer: must equal the cache's configuration (EINVAL otherwise).
 * Every key and value is rounded once to fp16; tokens landing in the sink or
 * recent window are stored as those fp16 values, tokens that the window
 * policy sends to the packed cache are quantised from them.  The resulting
 * state depends only on the token count, not on how appends were batched.
 * ECAPACITY if n_tokens + n_tok > max_ctx (nothing written). */
WUSHKV_API wushkv_status wushkv_append(wushkv_cache* cache, const void* k_rope_dev, const void* v_dev,
                            int32_t in_dtype, const float* T_k_dev, int32_t n_tok, int32_t bits,
                            int32_t quantizer, void* stream);

/* Append a different number of tokens to each sequence.
 *   Source: as wushkv_append; the window policy of the summary page
 *   (sink, recent, chunked flush) applies to each sequence on its own.
 *   k_rope_dev, v_dev: [sum_b n_new[b]][n_kv_heads][128] in_dtype, the
 *     tokens of sequence 0, then those of sequence 1, ... (no padding).
 *   n_new_host: [batch] host array of new-token counts (0 = sequence
 *     unchanged).
 *   Other arguments and results as wushkv_append; ECAPACITY (nothing
 *   written) if any sequence would exceed max_ctx.  With equal counts on
 *   sequences of equal length this is wushkv_append; otherwise each
 *   sequence's tokens go through their own launches. */
WUSHKV_API wushkv_status wushkv_append_varlen(wushkv_cache* cache, const void* k_rope_dev, const void* v_dev,
                                              int32_t in_dtype, const float* T_k_dev, const int32_t* n_new_host,
                                              int32_t bits, int32_t quantizer, void* stream);

/* q' = T_k^{-T} q for every query head, with the transform of its KV group.
 *   Source: same page, 方法关键点 and 工作参考价值 (one d x d product per
 *   query; inverse transpose keeps q'.k' = q.k).
 *   q_dev:        [batch][n_q_heads][128], dtype q_dtype.
 *   T_k_invT_dev: [n_kv_heads][128][128] fp32 row-major, q'_i = sum_j M[i][j] q_j,
 *                 16-byte aligned (EINVAL otherwise).
 *   q_out_dev:    [batch][n_q_heads][128] fp32 (kept fp32 for the decode).
 * G = n_q_heads / n_kv_heads must be 1, 2, 4, 8 or 16 (EUNSUPPORTED otherwise). */
WUSHKV_API wushkv_status wushkv_query_transform(const void* q_dev, int32_t q_dtype, const float* T_k_invT_dev,
                                     float* q_out_dev, int32_t batch, int32_t n_q_heads,
                                     int32_t n_kv_heads, void* stream);

/* Chunked-prefill attention: the queries of the last n_q tokens of every
 * sequence attend causally to the cache.
 *   Source: not on the pages (they describe decoding); the decode's rules
 *   apply (summary page "WUSH-KV：数据自适应变换的 KV Cache 低比特量化",
 *   方法关键点: keys through T_k after RoPE, queries through T_k^{-T}).  The
 *   chunk's tokens have been appended first (wushkv_append); the query of
 *   token p = n - n_q + i attends to tokens 0 .. p as the cache holds them
 *   (fp16 sink and recent rows, dequantised packed tokens).
 *   q_prime_dev: [batch][n_q][n_q_heads][128] fp32 transformed queries
 *                (wushkv_query_transform with batch * n_q rows), 16-byte
 *                aligned (EINVAL otherwise).
 *   out_dev:     [batch][n_q][n_q_heads][128] fp32, 16-byte aligned.
 *   n_q: 1 .. tokens per sequence (EINVAL otherwise); scale as wushkv_decode.
 * Every sequence must hold the same number of tokens (EUNSUPPORTED
 * otherwise); dense and paged caches; at most 65535 (sequence, KV head)
 * units.  Reads the cache only (no workspace), so it may run concurrently
 * with other readers of the cache. */
WUSHKV_API wushkv_status wushkv_prefill_attention(const float* q_prime_dev, const wushkv_cache* cache,
                                                  float* out_dev, int32_t n_q, float scale, void* stream);

/* GQA decode attention of one query per query head over the whole cache.
 *   Source: review "[논문리뷰] WUSH-KV ..." (secrett2633), Key Terms (GQA);
 *   dequantisation happens inside the score and PV loops.
 *   q_prime_dev: [batch][n_q_heads][128] fp32 transformed queries, 16-byte
 *                aligned (EINVAL otherwise; read as float4).
 *   out_dev:     [batch][n_q_heads][128] fp32 = softmax(scale q'.k'^T) v
 *                in the transformed value space; 16-byte aligned (EINVAL otherwise).
 *   scale: softmax scale; 0 selects 1/sqrt(128).
 * Each sequence attends to its own tokens: sequences of different lengths
 * are decoded in the same launch (up to 1024 sequences when their lengths
 * differ, else EUNSUPPORTED); the output rows of a sequence without tokens
 * are left unchanged.
 * Uses the cache's workspace region for split-K partials; calls on the same
 * cache must therefore be stream-ordered.  EINVAL if every sequence is
 * empty, or the cache is paged and has no page table. */
WUSHKV_API wushkv_status wushkv_decode(const float* q_prime_dev, const wushkv_cache* cache, float* out_dev,
                            float scale, void* stream);

/* One decode step: append one token to every sequence (wushkv_append with
 * n_tok = 1), transform the step's queries (wushkv_query_transform into
 * q_prime_dev) and decode them (wushkv_decode), in stream order.
 *   Source: the three calls above; the pages describe the step as append
 *   with the key transform, the query-side transform and attention over the
 *   packed cache plus the fp16 windows (summary page 方法关键点).
 *   k_rope_dev, v_dev: [batch][1][n_kv_heads][128], dtype in_dtype.
 *   T_k_dev: as wushkv_append.  q_dev: [batch][n_q_heads][128], dtype
 *   q_dtype.  T_k_invT_dev: as wushkv_query_transform.  q_prime_dev:
 *   [batch][n_q_heads][128] fp32, receives q' (16-byte aligned).  out_dev,
 *   scale: as wushkv_decode.
 * When the append needs a single append launch (every one-token append
 * whose flush does not reach the new token, i.e. recent >= 1) the append
 * and the query transform share one launch, so a step is two launches.
 * Results are identical to the three separate calls.  Errors as those
 * calls; on an argument error nothing is launched and the cache is
 * unchanged. */
WUSHKV_API wushkv_status wushkv_decode_step(wushkv_cache* cache, const void* k_rope_dev, const void* v_dev,
                                            int32_t in_dtype, const float* T_k_dev, const void* q_dev,
                                            int32_t q_dtype, const float* T_k_invT_dev, float* q_prime_dev,
                                            float* out_dev, float scale, void* stream);

/* Decode for callers that cannot allocate device memory.  The paper has no
 * counterpart: this is a deployment convenience around wushkv_decode.
 * Some callers cannot call cudaMalloc when they decode -- code running inside
 * a host application's allocator hook, plug-ins whose host owns every device
 * allocation, or serving engines that forbid allocation after start-up.
 * This entry point takes the same inputs and writes the same output as
 * wushkv_decode, but keeps its split-K partials and arrival counters in a
 * fixed 8 MiB array inside the library (a file-scope __device__ array that
 * every GPU which loads the library holds until the process exits) instead of
 * the cache buffer's workspace.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *   - The first call on each device looks up the array's device address
 *     (with that device current).  Under lazy module loading that lookup
 *     can load the library's device code and allocate the array, so make
 *     the first call on each device during start-up, where allocation is
 *     still allowed, and before any stream capture.
 *   - All calls share the one array, which keeps the previous call's
 *     contents; each call zeroes its arrival counters first.  Calls that
 *     overlap on the GPU (other streams, threads or caches) race: issue
 *     them one after another.
 *   - WUSHKV_ECAPACITY, with nothing launched, when this call's partials
 *     (units x splits x G x 528 bytes) exceed 8 MiB minus 256 KiB of
 *     counters, or the cache has more than 65536 units.
 * Other errors as wushkv_decode. */
WUSHKV_API wushkv_status wushkv_decode_noalloc(const float* q_prime_dev, const wushkv_cache* cache,
                                               float* out_dev, float scale, void* stream);

/* Copy tokens [tok0, tok0 + ntok) of unit (seq, head), K (kv = 0) or V
 * (kv = 1), to host memory.  Synchronous (waits for the device).
 *   codes_host: [ntok][128] uint8, unpacked codes (0 for window tokens); or NULL.
 *   meta_host:  [ntok][2] uint16 fp16 bits: (delta, 0) for QuEST, (scale, lo)
 *               for affine (0 for window tokens); or NULL.
 *   fp16_host:  [ntok][128] uint16 fp16 bits of window tokens (0 for packed
 *               tokens); or NULL.
 *   kinds_host: [ntok] int8: 0 sink, 1 packed, 2 recent; or NULL. */
WUSHKV_API wushkv_status wushkv_export(const wushkv_cache* cache, int32_t seq, int32_t head, int32_t kv,
                            int32_t tok0, int32_t ntok, uint8_t* codes_host, uint16_t* meta_host,
                            uint16_t* fp16_host, int8_t* kinds_host);

/* Read (and with clear != 0, reset) the sticky device status word;
 * synchronises the device.  0 means no kernel reported an error; otherwise
 * an OR of the WUSHKV_DEV_* bits. */
WUSHKV_API wushkv_status wushkv_device_status(const wushkv_cache* cache, int32_t clear, int32_t* out);

/* Failure injection, for tests of the timeout path without a GPU fault.
 * With polls > 0, every decode launched afterwards (from any thread) makes
 * each warp's first copy wait on a barrier that nothing completes, giving
 * up after `polls` polls.  The warp then takes its real timeout path: it
 * records WUSHKV_DEV_TIMEOUT in the cache's status word, waits (at the full
 * limit, about a second) for the copies it has in flight, and contributes
 * nothing more; the call returns normally, its output is not meaningful,
 * and later decodes are unaffected.  polls = 0 turns the injection off.
 * Not part of the method: the paper has no counterpart. */
WUSHKV_API void wushkv_inject_decode_timeout(uint32_t polls);

/* Gaussian-MSE-optimal QuEST clip ratio for 2, 3 or 4 bits (0 otherwise). */
WUSHKV_API double wushkv_default_quest_alpha(int32_t bits);

/* Static description of a status code. */
WUSHKV_API const char* wushkv_strerror(int32_t status);

#ifdef __cplusplus
}
#endif
#endif /* WUSHKV_H */
