/*
 * tq.h -- C ABI of libtq: TurboQuant-style compressed KV cache and decode
 * attention over it, for NVIDIA B200 (sm_100a).
 *
 * What the library computes (web pages on the subject; sections as titled):
 *  - "TurboQuant" summary, de.news.hada.io topic 27867, section "Funktionsweise
 *    von TurboQuant": a vector is randomly rotated, each coordinate goes
 *    through a standard scalar quantiser, and the residual error is encoded
 *    with 1-bit QJL; section "QJL: Eine 1-Bit-Methode ohne Overhead": a
 *    Johnson-Lindenstrauss projection reduced to sign bits and an estimator
 *    that pairs a full-precision query with those bits; the discussion
 *    thread: Lloyd-Max boundaries and reconstruction values after rotation.
 *  - "Monarch v3: NES-inspiriertes KV-Paging", openclawradar.com, sections
 *    "Wie es funktioniert" and "Vereinfachte Decode-Schleife": recent tokens
 *    stay at full precision in a hot window, older ones are compressed into a
 *    cold region, and each decode step scores hot and cold tokens and takes
 *    one softmax over them.
 *  - The same summary, section "Leistung bei der Vektorsuche": the codec also
 *    serves inner-product vector search (top-k).
 *
 * Conventions for every call:
 *  - Device pointers are CUDA device addresses on the device that was current
 *    when the context was created; host pointers are marked "host".
 *  - Streams are cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls that take a stream only enqueue work and never synchronise.
 *  - Argument errors are found on the host, before any launch, and return
 *    TQ_ERR_INVALID_ARG (or TQ_ERR_UNSUPPORTED for valid but unimplemented
 *    shapes).  A failed launch returns TQ_ERR_CUDA.  Errors found on the
 *    device (a page id outside the pool, a length beyond capacity, a wait
 *    that timed out) are recorded in the context's device error word, the
 *    offending work is skipped, and tq_get_error() reports the first one.
 *  - The library allocates device memory only in tq_init_codebook (its
 *    constant tables and error word) and frees it in tq_destroy.  All other
 *    buffers (page pool, page tables, lengths, hot window, outputs,
 *    workspace) are owned by the caller.
 *  - No C++ exception crosses this boundary.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Version of the cold-page storage format (tq_page_bytes).  2: pages with
 * values in 16-token blocks with bit-sliced key planes. */
#define TQ_LAYOUT_VERSION 2
/* Token slots per cold page. */
#define TQ_PAGE_TOKENS 128

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,
  TQ_ERR_UNSUPPORTED = 2,
  TQ_ERR_CUDA = 3,
  TQ_ERR_OOM = 4,
  TQ_ERR_CAPACITY = 5, /* device: a sequence outgrew its page table or pool */
  TQ_ERR_TIMEOUT = 6,  /* device: a bounded wait on a copy ran out */
  TQ_ERR_RANGE = 7     /* device, range-checked build (libtq_debug.so) only: a
                          computed index fell outside its array; the access
                          was skipped */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_F16 = 1, TQ_BF16 = 2 } tq_dtype;

/* Codec configuration.  Supported: head_dim 64 or 128, key_bits 2 (1-bit
 * magnitude index + sign), qjl_dim == head_dim, value_bits 4 (3-bit
 * magnitude index + sign), page_tokens 128.  seed selects the rotation and
 * the QJL matrix. */
typedef struct {
  int head_dim;
  int key_bits;
  int qjl_dim;
  int value_bits;
  int page_tokens;
  uint64_t seed;
} tq_config;

typedef struct tq_ctx tq_ctx; /* opaque; immutable after creation */

/*
 * Host-only generation of the codec tables ("Funktionsweise von TurboQuant"
 * and its discussion), no device needed.  All outputs are host arrays:
 *  rot   [d*d]  row-major Haar rotation Pi (x_rot = Pi x), fp32.  Pi is the Q
 *               factor of the QR factorisation of a d x d matrix of standard
 *               normal draws (SplitMix64 stream seeded 2*seed, 53-bit
 *               uniforms, Box-Muller with both outputs, filled row by row),
 *               with the signs of its columns chosen so that diag(R) > 0.
 *  qjl   [m*d]  QJL matrix S, row-major: standard normal draws of stream
 *               2*seed+1, each rounded to the nearest fp16 value.
 *  key_c [2^(key_bits-1)], key_t [2^(key_bits-1)-1]: positive Lloyd-Max
 *               levels and boundaries for one coordinate of a uniform point
 *               on the unit sphere of R^d (levels are +-key_c), fp32.
 *  val_c, val_t: the same at value_bits.
 * Any output may be NULL.  Cost: a fraction of a second (fp64 solves).
 */
TQ_API tq_status tq_generate_params(const tq_config* cfg, float* rot, float* qjl, float* key_c,
                             float* key_t, float* val_c, float* val_t);

/* Generate the tables (as tq_generate_params) and upload them to the current
 * device.  *out receives the context; release it with tq_destroy. */
TQ_API tq_status tq_init_codebook(const tq_config* cfg, tq_ctx** out);

/* Copy the context's tables to host arrays (same layouts as
 * tq_generate_params; NULL outputs are skipped). */
TQ_API tq_status tq_get_params(const tq_ctx* ctx, float* rot, float* qjl, float* key_c, float* key_t,
                        float* val_c, float* val_t);

/*
 * Bytes of one cold page (TQ_PAGE_TOKENS token slots).  with_values = 1: key
 * and value records (15104 B at d=128, 7936 B at d=64); 0: keys only, as used
 * by a search database (6656 B, 3584 B).  Format version TQ_LAYOUT_VERSION.
 * Multi-byte fields are little endian; fp16 fields are IEEE binary16.  A key
 * record is a 2-bit code per coordinate (sign s, magnitude index u of the
 * level +-key_c[u]), a QJL sign bit per sketch index (1: (S r)_i < 0), the
 * norm n and the residual norm gamma; a value record is a 4-bit code per
 * coordinate, s << 3 | u (level +-val_c[u]), and the value norm.  Coordinates
 * are those of the rotated domain (x_rot = Pi x).
 *
 * Pages with values: 8 blocks of 16 token slots (slot = 16 kb + t), each
 * 12 d + 2 m + 96 bytes (m = qjl_dim):
 *   KH  at 0            key plane H, 2 d bytes
 *   KL  at 2 d          key plane L, 2 d bytes
 *   QS  at 4 d          QJL sign plane, 2 m bytes
 *   VC  at 4 d + 2 m    value codes, 8 d bytes
 *   NK  at 12 d + 2 m   per token t, at + 4 t: fp16 n, then fp16 gamma
 *   VN  at 12 d + 2m + 64   per token t, at + 2 t: fp16 value norm
 * The key code of a coordinate is the index 2 H + L of its level in ascending
 * order (-c1, -c0, +c0, +c1): H = 1 - s, L = s XOR u.  In a plane (KH and KL
 * over coordinates j < d, QS over sketch indices j < m) the bit of token t is
 * bit t mod 8 of the byte at
 *     16 (4 (j / 32) + (j / 4) mod 4) + 4 (2 ((j / 16) mod 2) + t / 8) + j mod 4,
 * so a 32-bit word holds 4 consecutive indices x 8 tokens.  In VC, the byte
 * of coordinate j for the token pair (2q, 2q + 1) of the block holds the even
 * token's code in its low nibble and sits at
 *     (i / 4) 512 + (4 g + c) 16 + (i mod 4) 4 + jh + 2 th,
 * i = j / 16, g = j mod 8, jh = (j mod 16) / 8, c = q mod 4, th = q / 4 (the
 * word at (4 g + c) 16 + (i mod 4) 4 holds coordinates (g, g + 8) x token
 * pairs (c, c + 4)).
 *
 * Keys-only pages: sections in this order, each starting on a 16-byte
 * boundary:
 *   KC  key codes        128 x d/4 B
 *   QS  QJL sign bits    128 x m/8 B
 *   KN  key norm n       128 x fp16
 *   KG  residual norm    128 x fp16
 * Key code word w (u32, w < d/16) of a token holds coordinates
 * j = 16w + 8h + 2i + e (h, e in {0,1}, i < 4) with the sign bit at
 * 16h + 15 - 4i - e and the magnitude bit at 16h + 13 - 4i - e.  QJL word w
 * (w < m/32) holds sketch index 32w + 16h + r (r < 16) at bit 16h + 15 - r.
 */
TQ_API size_t tq_page_bytes(const tq_ctx* ctx, int with_values);

/* Input flag for tq_compress_append: k and v already hold Pi x in fp32 (the
 * rotation folded into the projection that produced them). */
#define TQ_INPUT_ROTATED 1

/*
 * Compress n_new new tokens per (batch, kv head) and append them to the cold
 * pages ("Funktionsweise von TurboQuant"; eviction from the hot window into
 * the cold region as in Monarch's "Wie es funktioniert").
 *  k, v        device, [B, Hkv, n_new, d], dtype `dtype` (F16 or BF16; F32
 *              only with TQ_INPUT_ROTATED).  v = NULL writes keys-only pages.
 *  page_pool   device, 16-byte aligned, pool_pages pages of
 *              tq_page_bytes(ctx, v != NULL) bytes each.
 *  page_table  device int32 [B, Hkv, max_pages]: pool page of each logical
 *              page; token position t of (b, h) lives in page
 *              page_table[b, h, t / 128], slot t % 128.
 *  cold_len    device int32 [B]: tokens already stored per sequence (equal
 *              for all kv heads).  The new tokens take positions
 *              cold_len[b] .. cold_len[b] + n_new - 1; cold_len is advanced by
 *              n_new on the stream after the writes.
 * Per vector: n = fp16(|x|); codes from x_rot = Pi x against thresholds
 * fp32(n * t_k); keys also store gamma = fp16(|x_rot/n - c_hat|) and the
 * signs of S (x_rot/n - c_hat).  Device errors: a position beyond
 * max_pages*128 or a page id outside [0, pool_pages) -> TQ_ERR_CAPACITY and
 * that token is not written.
 */
TQ_API tq_status tq_compress_append(const tq_ctx* ctx, const void* k, const void* v, tq_dtype dtype,
                             int flags, int B, int Hkv, int n_new, uint8_t* page_pool,
                             int64_t pool_pages, const int32_t* page_table, int max_pages,
                             int32_t* cold_len, void* stream);

/* Workspace bytes tq_decode_attention needs for these maxima. */
TQ_API size_t tq_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_pages, int W_max);

/*
 * One decode step of attention over a hot fp16 window and cold compressed
 * pages, one softmax over both ("Vereinfachte Decode-Schleife"; the cold
 * scores use the QJL estimator of "QJL: Eine 1-Bit-Methode ohne Overhead"):
 *   cold score  n * (<Pi q, c_hat> + sqrt(pi/2)/m * gamma * <S Pi q, 1 - 2 bits>) * scale
 *   cold value  n_v * Pi^T c_hat_v
 *   hot score   <q, k> * scale, hot value v (exact)
 *  q          device [B, Hq, d], q_dtype F32, F16 or BF16.  Query head h
 *             attends with kv head h / (Hq / Hkv).
 *  scale      softmax scale; 0 selects 1/sqrt(d).
 *  k_hot, v_hot device fp16 [B, Hkv, W_max, d]; hot_len device int32 [B]
 *             (0 <= hot_len <= W_max).  May be NULL when W_max == 0.
 *  page_pool, pool_pages, page_table, max_pages, cold_len: as in
 *             tq_compress_append (values pages); cold_len is only read.
 *  out        device fp32 [B, Hq, d]; a sequence with no tokens gets zeros.
 *  workspace  device, ws_bytes >= tq_workspace_bytes(ctx, B, Hq, Hkv,
 *             max_pages, W_max), 256-byte aligned; contents are scratch.
 * Supported: Hq % Hkv == 0 with Hq / Hkv in {1, 2, 4, 8}.
 */
TQ_API tq_status tq_decode_attention(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                              int Hkv, float scale, const void* k_hot, const void* v_hot,
                              int W_max, const int32_t* hot_len, const uint8_t* page_pool,
                              int64_t pool_pages, const int32_t* page_table, int max_pages,
                              const int32_t* cold_len, float* out, void* workspace,
                              size_t ws_bytes, void* stream);

/*
 * tq_decode_attention with Monarch's threshold gate and a ring-buffer hot
 * window ("Vereinfachte Decode-Schleife": the cold pages are decompressed and
 * scored only if max(scores_hot) < threshold).
 *  threshold  per query head h of sequence b, the gate is open when
 *             max_t <q_h, k_t> < threshold, the maximum taken over the hot
 *             tokens of h's kv head in fp32 on the raw dot products (no
 *             softmax scale), -inf when there are none.  An open head
 *             attends to hot and cold tokens exactly as tq_decode_attention;
 *             a shut head to its hot tokens alone (zeros if it has none).
 *             +INFINITY opens every head; NaN is rejected.  Where the
 *             maximum lies within fp32 rounding of the threshold the decision
 *             may go either way; cold_used reports the one taken.
 *  cold_used  device int32 [B, Hq] out: the gate's decision per head, 1 when
 *             the head attends to its cold tokens (whether or not it has
 *             any), else 0.  May be NULL.
 *  hot_start  device int32 [B], or NULL for 0: the hot window of sequence b
 *             is a ring of W_max slots whose logical token i
 *             (0 <= i < hot_len[b]) sits in slot (hot_start[b] + i) mod
 *             W_max.  Attention does not depend on token order, so the ring
 *             only saves the caller from shifting the window when it evicts
 *             its oldest tokens.  A start outside [0, W_max) is a device
 *             error (TQ_ERR_CAPACITY) and reads as 0.
 * The other arguments, the workspace size and the results are those of
 * tq_decode_attention.  When every head of a (batch, kv head) group is shut,
 * the group's cold pages are not read at all.
 */
TQ_API tq_status tq_decode_attention_gated(const tq_ctx* ctx, const void* q, tq_dtype q_dtype,
                                           int B, int Hq, int Hkv, float scale,
                                           const void* k_hot, const void* v_hot, int W_max,
                                           const int32_t* hot_start, const int32_t* hot_len,
                                           const uint8_t* page_pool, int64_t pool_pages,
                                           const int32_t* page_table, int max_pages,
                                           const int32_t* cold_len, float threshold,
                                           int32_t* cold_used, float* out, void* workspace,
                                           size_t ws_bytes, void* stream);
/* Workspace bytes tq_monarch_step needs. */
TQ_API size_t tq_monarch_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_pages,
                                         int W_max, int evict_block);
/*
 * One decode step of Monarch's hot/cold cache ("Monarch v3: NES-inspiriertes
 * KV-Paging", sections "Wie es funktioniert" and "Vereinfachte
 * Decode-Schleife"), all on the stream, nothing on the host:
 *  1. append  k_new, v_new (device fp16 [B, Hkv, d], both NULL to skip): the
 *             token joins the hot ring of every kv head at slot
 *             (hot_start[b] + hot_len[b]) mod W_max and hot_len[b] grows by
 *             one.  A full ring (hot_len == W_max) is a device error
 *             (TQ_ERR_CAPACITY) and the token is dropped.
 *  2. attend  tq_decode_attention_gated over the ring (with the new token)
 *             and the cold pages, threshold and cold_used as there.
 *  3. evict   every sequence whose hot window now holds at least
 *             window + evict_block tokens has its oldest evict_block hot
 *             tokens compressed (tq_compress_append from fp16) and appended to
 *             its cold pages; hot_start advances by evict_block (mod W_max),
 *             hot_len shrinks and cold_len grows by it.  evict_block = 1 is
 *             the loop as written (evict whenever the window is exceeded);
 *             larger blocks keep between window and window + evict_block - 1
 *             tokens hot and compress a block at a time.
 *  k_hot, v_hot  device fp16 [B, Hkv, W_max, d], read and written.
 *  hot_start, hot_len, cold_len  device int32 [B], read and written.
 *  page_pool, pool_pages, page_table, max_pages  values pages, as in
 *             tq_compress_append.
 *  workspace  device, 256-byte aligned, ws_bytes >=
 *             tq_monarch_workspace_bytes(ctx, B, Hq, Hkv, max_pages, W_max,
 *             evict_block).
 * Requires window >= 0, evict_block >= 1 and window + evict_block <= W_max
 * (the ring never overflows while hot_len < window + evict_block holds
 * before a step).
 */
TQ_API tq_status tq_monarch_step(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B, int Hq,
                                 int Hkv, float scale, const void* k_new, const void* v_new,
                                 void* k_hot, void* v_hot, int W_max, int32_t* hot_start,
                                 int32_t* hot_len, uint8_t* page_pool, int64_t pool_pages,
                                 const int32_t* page_table, int max_pages, int32_t* cold_len,
                                 float threshold, int window, int evict_block,
                                 int32_t* cold_used, float* out, void* workspace,
                                 size_t ws_bytes, void* stream);
/*
 * Monarch's attention-weighted promotion with stickiness ("Monarch v3", section
 * "Wie es funktioniert": tokens with high attention move back to the hot
 * region, with a sticking mechanism against thrashing; section "Vereinfachte
 * Decode-Schleife": cold tokens read in a step move to the hot region for the
 * next step; section "Wie man es ausprobiert": thresholds 0.15 and 3).
 * After a step's attention, a cold position's weight is its largest softmax
 * probability over the query heads of its sequence that read the cold tier.
 * A weight >= threshold counts the step, a smaller one resets the count (the
 * count is of consecutive steps).  A position whose count reaches sticky
 * moves back: its decompressed key and value -- n Pi^T c_hat (the QJL
 * residual term is an estimator, not a vector) and n_v Pi^T c_hat_v, rounded
 * to fp16 -- become the newest hot tokens of every kv head of the sequence
 * (ring slots (hot_start + hot_len) mod W_max, hot_len grows), its cold slot
 * is masked (the attention skips it from then on), its count returns to 0.
 * At most max_per_step positions move per sequence and step, in increasing
 * position order, and never more than leave one ring slot free for the next
 * step's token; positions left over keep their counts.  Eviction follows.
 *  threshold     > 0, finite (weights are at most 1)
 *  sticky        >= 1
 *  max_per_step  1 .. TQ_PROMOTE_MAX_PER_STEP
 *  cold_mask     device uint32 [B][max_pages * 4]: bit p % 32 of word p / 32
 *                set = position p moved back; zero before the first step
 *  counts        device uint8 [B][max_pages * 128]: consecutive counted
 *                steps per position; zero before the first step
 *  logits        device fp32 scratch [B][Hq][max_pages * 128]
 */
#define TQ_PROMOTE_MAX_PER_STEP 64
typedef struct {
  float threshold;
  int sticky;
  int max_per_step;
  uint32_t* cold_mask;
  uint8_t* counts;
  float* logits;
} tq_promotion;

/* tq_monarch_step with promotion (promo NULL: exactly tq_monarch_step), the
 * moves taking place between the attention and the eviction.  Same
 * workspace. */
TQ_API tq_status tq_monarch_step_promote(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B,
                                         int Hq, int Hkv, float scale, const void* k_new,
                                         const void* v_new, void* k_hot, void* v_hot, int W_max,
                                         int32_t* hot_start, int32_t* hot_len,
                                         uint8_t* page_pool, int64_t pool_pages,
                                         const int32_t* page_table, int max_pages,
                                         int32_t* cold_len, float threshold, int window,
                                         int evict_block, const tq_promotion* promo,
                                         int32_t* cold_used, float* out, void* workspace,
                                         size_t ws_bytes, void* stream);
/* Largest decode workspace tq_decode_attention_noalloc can serve (8 MiB). */
#define TQ_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * tq_decode_attention without a caller-provided workspace and without any
 * device allocation.  The pages on the subject have no counterpart of this
 * call: it exists for callers that are not allowed to allocate device
 * memory -- for example a plugin inside an inference runtime that owns the
 * whole device-memory budget, or a serving loop that must never block on the
 * allocator -- and therefore cannot provide the workspace buffer.
 *
 * Arguments and results are those of tq_decode_attention, minus workspace
 * and ws_bytes.  The scratch space is one fixed array of
 * TQ_NOALLOC_SCRATCH_BYTES bytes that the library keeps in device memory on
 * every GPU that loads it, until the process exits.  A problem whose
 * workspace (tq_workspace_bytes) exceeds that size is rejected with
 * TQ_ERR_CAPACITY before any launch.
 *  - The first call on a device looks up the array's device address (a
 *    synchronous runtime call, once per device and CUDA context: after a
 *    device reset the next call looks it up again); make that first call
 *    before any stream capture.  The context's device must be the current
 *    device.
 *  - All calls share the one array and it keeps the last call's contents
 *    (nothing in it needs to start at zero).  Calls that overlap on the GPU,
 *    from different streams or threads, race on it: serialise them.
 */
TQ_API tq_status tq_decode_attention_noalloc(const tq_ctx* ctx, const void* q, tq_dtype q_dtype,
                                             int B, int Hq, int Hkv, float scale,
                                             const void* k_hot, const void* v_hot, int W_max,
                                             const int32_t* hot_len, const uint8_t* page_pool,
                                             int64_t pool_pages, const int32_t* page_table,
                                             int max_pages, const int32_t* cold_len, float* out,
                                             void* stream);

/* Workspace bytes tq_score_topk needs. */
TQ_API size_t tq_topk_workspace_bytes(const tq_ctx* ctx, int Q, int64_t N, int k);

/*
 * Compressed inner-product search ("Leistung bei der Vektorsuche"): the
 * estimated inner product of every query with every database vector (the
 * cold score above with scale 1), then the k best per query, ties to the
 * lower id.
 *  queries   device fp32 [Q, d].
 *  db_pages  device keys-only pages; vector i sits in page i / 128, slot
 *            i % 128 (pages written by tq_compress_append with v = NULL).
 *  out_ids   device int32 [Q, k]; out_scores device fp32 [Q, k], best first.
 *            When N < k the tail holds id -1 and score -inf.
 *  workspace device, ws_bytes >= tq_topk_workspace_bytes(ctx, Q, N, k).
 * Supported: 1 <= k <= 32.
 */
TQ_API tq_status tq_score_topk(const tq_ctx* ctx, const float* queries, int Q, const uint8_t* db_pages,
                        int64_t N, int k, int32_t* out_ids, float* out_scores, void* workspace,
                        size_t ws_bytes, void* stream);

/* Workspace bytes tq_tensor_cache_step needs. */
TQ_API size_t tq_tensor_cache_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int W);
/*
 * One decode step of Tensor Cache's two-level state ("Tensor Cache:
 * Eviction-conditioned Associative Memory for Transformers", section
 * "Methodik: Tensor Cache (TC)"):
 *  L1  an fp16 ring of the last W tokens per (batch, kv head), attended with
 *      exact softmax (scale as tq_decode_attention);
 *  L2  a d x d fp32 matrix A per (batch, kv head), written only by the ring's
 *      evictions: A <- lambda A + eta (k (x) v), i.e. A[i][j] += eta k_i v_j
 *      after scaling by lambda;
 *  read r = q A (r_j = sum_i q_i A[i][j], q unscaled) with the A of the query
 *      head's kv head; output y = y_local + sigmoid(g) r.
 * Order: the step's token (k_new, v_new: device fp16 [B, Hkv, d]) enters the
 * ring; when the ring already holds W tokens, the token it overwrites (the
 * oldest) is first written into A.  Then attention over the ring and the read
 * of A, so every token is in exactly one level.
 *  k_ring, v_ring  device fp16 [B, Hkv, W, d]; ring_start, ring_len device
 *                  int32 [B] (logical token i at slot (start + i) mod W),
 *                  updated on the device.
 *  A               device fp32 [B, Hkv, d, d], updated in place.
 *  lambda, eta     device fp32 [Hkv]; gate device fp32 [Hq] (g before the
 *                  sigmoid).
 *  out             device fp32 [B, Hq, d].
 * A ring length outside [0, W] or start outside [0, W) is a device error
 * (TQ_ERR_CAPACITY); that sequence's state restarts empty.
 */
TQ_API tq_status tq_tensor_cache_step(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B,
                                      int Hq, int Hkv, float scale, const void* k_new,
                                      const void* v_new, void* k_ring, void* v_ring, int W,
                                      int32_t* ring_start, int32_t* ring_len, float* A,
                                      const float* lambda, const float* eta, const float* gate,
                                      float* out, void* workspace, size_t ws_bytes, void* stream);
/*
 * Self-Indexing KV cache, index and compressed-domain scores ("Self-Indexing
 * KVCache", section "Methodologie: Self-Indexing KVCache", items 1-3).
 * tq_self_index_build, per (batch, kv head) over its T keys:
 *  k          device fp16 [B, Hkv, T, d], 16-byte aligned.
 *  mu         device fp32 [B, Hkv, d] out: the channel mean (fp32 sum / T).
 *  codes      device uint8 [B, Hkv, T, d/4] out, 16-byte aligned: for group
 *             g (coordinates 4g .. 4g+3) bit i set where k - mu is positive
 *             in coordinate 4g + i (zero is not).
 *  centroids  device fp32 [B, Hkv, d/4, 16, 4] out, 16-byte aligned: the
 *             mean of the centred subvectors with each index (zero vector for
 *             an index no token has).  Summed with float atomics: the
 *             summation order is not fixed.
 * tq_self_index_scores: for every query head and token, the sum over groups
 * of <q_g, centroid[g][code]> (a 16-entry table per group), i.e. the dot
 * product of q with the token's centred reconstruction.
 *  q          device [B, Hq, d] (F32, F16 or BF16); head h reads kv head
 *             h / (Hq / Hkv).
 *  scores     device fp32 [B, Hq, T] out.
 */
TQ_API tq_status tq_self_index_build(const tq_ctx* ctx, const void* k, int B, int Hkv, int T,
                                     float* mu, uint8_t* codes, float* centroids, void* stream);
TQ_API tq_status tq_self_index_scores(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B,
                                      int Hq, int Hkv, int T, const uint8_t* codes,
                                      const float* centroids, float* scores, void* stream);
/*
 * Top-k retrieval and sparse attention of the Self-Indexing form ("Self-
 * Indexing KVCache", Methodologie items 3 and 4): per query head the top_k
 * positions after the first n_sink tokens by LUT score, then exact softmax
 * attention over the n_sink sink tokens and those positions with the stored
 * full-precision keys and values.  k_eff = min(top_k, max(T - n_sink, 0)).
 * tq_self_index_select:
 *  scores   device fp32 [rows, T] (rows = B * Hq).  A NaN score ranks below
 *           every number, -inf included.
 *  picked   device int32 [rows, top_k] out: the k_eff best positions in
 *           [n_sink, T), in increasing position order; equal scores (and NaN
 *           scores among themselves) go to the lower position (-0.0 equals
 *           +0.0); entries k_eff.. are -1.
 * tq_self_index_attend:
 *  q        device [B, Hq, d] (F32, F16 or BF16); head h reads kv head
 *           h / (Hq / Hkv).
 *  keys, values  device fp16 [B, Hkv, T, d], 16-byte aligned.
 *  picked   device int32 [B * Hq, top_k] as tq_self_index_select writes it;
 *           the first k_eff entries are read.  An entry outside [0, T) is
 *           skipped and recorded as TQ_ERR_INVALID_ARG on the context.
 *  scale    softmax scale; 0 selects 1/sqrt(d); negative, NaN or infinite
 *           is TQ_ERR_INVALID_ARG.
 *  out      device fp32 [B, Hq, d] out: sum_j softmax_j(scale <q, k_j>) v_j
 *           over j in [0, min(n_sink, T)) and the picked positions; zero
 *           when T = 0.
 */
TQ_API tq_status tq_self_index_select(const tq_ctx* ctx, const float* scores, int rows, int T,
                                      int n_sink, int top_k, int32_t* picked, void* stream);
TQ_API tq_status tq_self_index_attend(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int B,
                                      int Hq, int Hkv, int T, const void* keys,
                                      const void* values, const int32_t* picked, int n_sink,
                                      int top_k, float scale, float* out, void* stream);
/*
 * Stage-1 quantiser variants on rotated vectors, for comparing distortion
 * ("Funktionsweise von TurboQuant": a standard per-coordinate quantiser after
 * the rotation; "PolarQuant: Ein neuer Winkel auf Kompression": coordinate
 * pairs to polar form, radii paired again recursively until one radius and a
 * set of angles remain, angles quantised on fixed grids).  Neither variant
 * carries the QJL sketch.
 *  TQ_STAGE1_MSE    bits1 = b in 2..4 (bits2 unused): per coordinate the
 *                   sign and a (b-1)-bit Lloyd-Max magnitude index of
 *                   x_rot / n (levels of one coordinate of a uniform point on
 *                   the sphere, as the key and value codebooks), decided as
 *                   |x_rot,j| >= fp32(n * t_k); n = fp16(|x_rot|).  Code of
 *                   coordinate j = sign << (b-1) | index, in bits
 *                   [b j, b j + b) of a little-endian bit stream.
 *  TQ_STAGE1_POLAR  bits1 = b1 in 2..5, bits2 = b2 in 1..3: level 1 pairs
 *                   coordinates (2i, 2i+1), angle in [0, 2 pi) on 2^b1 equal
 *                   bins (reconstructed at the bin centre); level l >= 2 pairs
 *                   the radii of blocks of k = 2^(l-1) coordinates, angle
 *                   atan(r_o / r_e) in [0, pi/2] with the 2^b2-level Lloyd-Max
 *                   codebook of its density, proportional to sin^(k-1)(2 phi);
 *                   the final radius is stored as fp16 in norms.  Radii are
 *                   sqrtf(fmaf(u, u, v * v)) in fp32; a level-1 pair is turned
 *                   into the first quadrant by exact swaps and negations and
 *                   its bin counts the boundaries with v >= u * fp32(tan); a
 *                   higher level counts r_o >= r_e * fp32(tan(boundary)) when
 *                   r_o > 0; a zero pair has angle 0.  Codes: level 1 (b1 bits
 *                   per pair, pair order), then level 2, 3, ... (b2 bits per
 *                   node, node order), one little-endian bit stream.
 *  x_rot   device fp32 [N, d] rotated vectors, 16-byte aligned.
 *  codes   device uint8 [N, tq_stage1_code_bytes(...)], 4-byte aligned (a
 *          record is a whole number of 32-bit words); norms device fp16 [N].
 *  x_hat   device fp32 [N, d] reconstruction in the rotated domain, 16-byte
 *          aligned.
 * Unsupported bit counts give TQ_ERR_UNSUPPORTED (and a code size of 0).
 */
typedef enum { TQ_STAGE1_MSE = 0, TQ_STAGE1_POLAR = 1 } tq_stage1_kind;
TQ_API size_t tq_stage1_code_bytes(const tq_ctx* ctx, int kind, int bits1, int bits2);
TQ_API tq_status tq_stage1_encode(const tq_ctx* ctx, int kind, int bits1, int bits2,
                                  const float* x_rot, int64_t N, uint8_t* codes,
                                  uint16_t* norms, void* stream);
TQ_API tq_status tq_stage1_decode(const tq_ctx* ctx, int kind, int bits1, int bits2,
                                  const uint8_t* codes, const uint16_t* norms, int64_t N,
                                  float* x_hat, void* stream);
/* Profiling hook: when ev_start / ev_stop (cudaEvent_t, passed as void*) are
 * set, the next calls of tq_decode_attention, tq_compress_append and
 * tq_score_topk record ev_start on their stream right before the launch of
 * their main kernel (the split-K attention, the compress, the scorer) and
 * ev_stop right after it, so a caller can time that kernel alone.  NULL, NULL
 * switches it off.  Not thread-safe: set it only while no other thread uses
 * the context. */
TQ_API tq_status tq_set_profile_events(tq_ctx* ctx, void* ev_start, void* ev_stop);

/* Testing aid for the bounded device waits (no counterpart on the pages).
 * With skip_unit >= 0, the next decode calls (tq_decode_attention and its
 * gated, Monarch and no-allocation forms) arm the copy of cold work unit
 * skip_unit (64 tokens; units are numbered over all (batch, kv head)
 * segments in order) without issuing it, so the wait for that unit can never
 * complete; every wait of the attention kernel gives up after limit_ns
 * nanoseconds (0: the default of 2 s).  The warp that owns the unit records
 * TQ_ERR_TIMEOUT, lets its other copies land and returns; the call's outputs
 * are then undefined, the context stays usable.  skip_unit = -1, limit_ns = 0
 * restores normal operation.  Not thread-safe: set it only while no other
 * thread uses the context. */
TQ_API tq_status tq_set_wait_test(tq_ctx* ctx, int skip_unit, uint64_t limit_ns);

/* Read and clear the context's device error word.  Synchronises with the
 * device; call it after the work of interest has completed. */
TQ_API tq_status tq_get_error(const tq_ctx* ctx);

TQ_API const char* tq_status_string(tq_status s);

TQ_API void tq_destroy(tq_ctx* ctx);

#ifdef __cplusplus
}
#endif
#endif /* TQ_H */
