/*
 * star_attention.h -- C ABI of libstar, the B200 (sm_100a) Star Attention
 * two-phase attention hot path for one GPU.
 *
 * Sources (page title, then section):
 *  [P2] "Star Attention: Efficient LLM Inference over Long Sequences"
 *       (paper-graph-ui analysis page), section 3.4 "Detailed, Sentence-Based
 *       Technical Breakdown": "Phase 1: Context Encoding with Anchor Blocks"
 *       Steps 1-5 and "Phase 2: Query Encoding and Token Generation with
 *       Distributed Softmax" Steps 3, 5 and 7 with the partition identity.
 *  [P3] "NVIDIA/Star-Attention" (README mirror), "Two Phases of Star
 *       Attention": Phase 1 and Phase 2 bullets.
 *
 * The pages' "hosts" are logical context blocks on one device: block i's KV
 * lives in its own cache segment, the query region (query and generated
 * tokens) is one more segment, and the distributed softmax of phase 2 runs
 * on-chip.
 *
 * Conventions for every call below
 *  - All tensor pointers are DEVICE pointers owned by the caller, except the
 *    cache segments, which belong to the star_cache.  Tensors are dense,
 *    row-major, 16-byte aligned; bf16 is IEEE bfloat16 (uint16 bits).
 *  - Q/K/V are already rotated (RoPE applied by the caller).  Because the
 *    anchor keeps its original positions ([P2] Phase 1 Step 2), the anchor's
 *    keys and values are rows 0..b_a-1 of the context K/V: no copy is made.
 *  - Grouped-query attention: q head h reads kv head h / (Hq / Hkv).
 *  - LSE values are natural-log log-sum-exp of the SCALED logits
 *    (scale * q.k), float32.
 *  - Every compute call is asynchronous on `stream` (a cudaStream_t passed
 *    as void*, NULL = legacy default stream).  Calls on one cache must be
 *    issued in order from one host thread on one stream.
 *  - No call allocates device memory except star_cache_create.
 *  - Return value: STAR_OK (0) or a negative STAR_E* code; shape and argument
 *    errors are caught on the host before anything is launched and leave the
 *    cache unchanged.  star_last_error() gives a one-line description of the
 *    last failure in the calling thread.
 */
#ifndef STAR_ATTENTION_H
#define STAR_ATTENTION_H

#if defined(__GNUC__)
#define STAR_API __attribute__((visibility("default")))
#else
#define STAR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define STAR_OK            0
#define STAR_EINVAL       -1   /* bad shape, ratio, b_a > b, null or misaligned pointer */
#define STAR_ENOSPC       -2   /* query region full (q_cap reached)                      */
#define STAR_ECUDA        -3   /* CUDA runtime / launch error                            */
#define STAR_EUNSUPPORTED -4   /* head_dim not 64/128, device not sm_100, > 191 blocks   */
#define STAR_ENOMEM       -5   /* cudaMalloc failed in star_cache_create                 */

/* Problem statement of one attention layer ([P2] Phase 1 Step 1, Phase 2
 * Step 3).  B sequences with identical shapes and independent caches. */
typedef struct {
  int B;            /* batch, >= 1                                          */
  int Hq;           /* query heads, a multiple of Hkv                       */
  int Hkv;          /* key/value heads                                      */
  int D;            /* head dim: 64 or 128                                  */
  long long L;      /* context length, >= 1                                 */
  int block;        /* block size b >= 1; n = ceil(L / b) blocks, n <= 191 */
  int anchor;       /* anchor size b_a, 0 <= b_a <= b (0 = no anchor)       */
  int q_cap;        /* query-region capacity: query tokens + decode steps   */
  float scale;      /* softmax scale; <= 0 selects 1/sqrt(D)                */
  int kv_fp8;       /* 1: the cache also keeps an FP8 (E4M3) copy of every
                       cached K/V row (context and query region), which
                       star_decode_step streams instead of the bf16 rows
                       (about half the bytes); 0: bf16 only.  D = 64 or
                       128.  Quantisation
                       (no counterpart in the pages, which call KV
                       quantisation orthogonal): per cached row of one kv
                       head, s = max|x| / 448 (1 if max|x| <= 1e-30), codes
                       = e4m3_rn(x * (1/s)) in float32, value = code * s.   */
} star_params;

/* Opaque KV cache: n context segments + 1 query-region segment, the segment
 * table and the phase-2 scratch (partials and merge tickets). */
typedef struct star_cache star_cache;

/* Allocates the cache for `p` on the current CUDA device (cudaMalloc).
 * Layout in HBM: context segment i holds K (then V) as [B][Hkv][len_i][D]
 * bf16, len_i = min(b, L - i*b), segments back to back; the query region is
 * [B][Hkv][q_cap][D] for K and for V.  *out is NULL on failure.
 * STAR_ENOMEM when the allocation fails; with the environment variable
 * STAR_FAULT_INJECT=alloc it fails on purpose (a test hook for that path). */
STAR_API int star_cache_create(const star_params* p, star_cache** out);

/* Frees everything the cache owns (synchronises the device first).  NULL is
 * accepted. */
STAR_API int star_cache_destroy(star_cache* c);

/* FP8 copy of segment `seg` (kv_fp8 caches only): E4M3 codes of K and V and
 * their per-row float32 scales, device pointers.  Context segment seg < n:
 * [B][Hkv][len][D] bytes and [B][Hkv][len] scales; seg = n, the query
 * region: [B][Hkv][q_cap][D] and [B][Hkv][q_cap] (rows in use as for
 * star_cache_segment).  STAR_EINVAL if the cache has no FP8 copy. */
STAR_API int star_cache_segment_fp8(const star_cache* c, int seg, void** k8, void** v8,
                                    float** k_scale, float** v_scale);

/* Reads and clears the cache's device error word (synchronous: waits for
 * the work already queued on the device).  *flag is non-zero if a kernel
 * gave up a bounded wait on one of its own pipeline barriers since the last
 * call -- outputs of that call are then invalid.  Kernels never trap. */
STAR_API int star_cache_device_error(star_cache* c, int* flag);

/* Canary check (a stand-in for a memory checker, which this pool does not
 * run): the cache's one allocation holds, after each of its parts (context
 * K, context V, query-region K and V, partials, tickets, error word, work
 * lists, the FP8 copies), a 4 KB guard filled with 0xA5 bytes when the cache
 * is made.  Synchronous: waits for all work on the device (every stream),
 * then *first_bad = -1 if every
 * guard is intact, else the index of the first overwritten one (in the order
 * above); star_last_error() then names the part it follows. */
STAR_API int star_cache_check_guards(star_cache* c, int* first_bad);

/* Number of segments: n context segments followed by the query region. */
STAR_API int star_cache_num_segments(const star_cache* c);

/* Segment table entry `seg` (0..n-1 context, n = query region): device
 * pointers to its K and V ([B][Hkv][cap][D] bf16), the first context token
 * it holds (`start`; L for the query region), the rows in use (`len`) and the
 * rows reserved (`cap`).  Any output pointer may be NULL. */
STAR_API int star_cache_segment(const star_cache* c, int seg, void** k, void** v,
                       long long* start, long long* len, long long* cap);

/* Empties the query region (length 0) so a new query can reuse the context
 * cache.  Nothing is launched. */
STAR_API int star_cache_reset_query(star_cache* c);

/* Phase 1 -- context encoding ([P2] Phase 1 Steps 1-5; [P3] Phase 1).
 * Q [B][Hq][L][D], K, V [B][Hkv][L][D] bf16 in; O [B][Hq][L][D] bf16 and
 * LSE [B][Hq][L] float32 out.  Token t of block i sees tokens j <= t of its
 * own block and, when i >= 1, the whole anchor [0, b_a).  Writes the cache:
 * segment i receives K/V rows of block i only (anchor KV discarded, every
 * context token cached exactly once), and with kv_fp8 also their FP8 copy.
 * Empties the query region. */
STAR_API int star_ctx_encode(star_cache* c, const void* Q, const void* K, const void* V,
                    void* O, float* LSE, void* stream);

/* Debug form of star_ctx_encode ([P2] Phase 1 Steps 1-5): the same encode,
 * cache, O and LSE, and also O32 [B][Hq][L][D] float32, every output row
 * before its bf16 rounding (O is bit for bit the round-to-nearest-even of
 * O32).  For tests and inspection: with very short blocks or anchors a row
 * averages a handful of values, and the bf16 rounding of O alone can then be
 * most of an absolute error bar.  Errors as star_ctx_encode, plus STAR_EINVAL
 * for a NULL O32. */
STAR_API int star_ctx_encode_fp32(star_cache* c, const void* Q, const void* K, const void* V,
                                  void* O, float* LSE, float* O32, void* stream);

/* RoPE front end ("Star Attention", Phase 1 Step 2: every token keeps its
 * position ID; anchor tokens keep theirs).  Rotary embedding of
 * x [B][H][L][D] bf16 into y (y == x allowed): each adjacent pair
 * (x_2k, x_2k+1) of row t turns by p_t * theta^(-2k/D), p_t = pos[t] when
 * pos (device, int32 [L]) is given, else pos0 + t.  Angles are formed and
 * reduced in double, rotated in float32, rounded once to bf16.  D = 64 or
 * 128 (else STAR_EUNSUPPORTED); theta > 1; B <= 65535; positions >= 0. */
STAR_API int star_rope(int B, int H, long long L, int D, double theta, const int* pos,
                       long long pos0, const void* x, void* y, void* stream);

/* Phase 1 from and to HOST memory ([P2] Phase 1 Steps 1-5): star_ctx_encode
 * with the host->device copies of Q, K, V and the device->host copies of O,
 * LSE overlapped with the encoding.  The blocks are encoded in order 0..n-1,
 * each in one or more units of (batch x kv head) ranges; a unit's rows are
 * copied in on one copy stream while earlier units compute, and its O / LSE
 * rows are copied out on another while later units compute (block 0's units
 * come first, since every later block reads its anchor rows).
 *   hQ, hK, hV   host inputs, same layout as star_ctx_encode's Q, K, V
 *   hO, hLSE     host outputs, same layout as O, LSE
 *   Q, K, V, O, LSE  device buffers of the same shapes (caller-owned,
 *                16-byte aligned): the staging copies, left holding the
 *                inputs and outputs
 * Host buffers should be page-locked (cudaHostAlloc, or a pinned tensor):
 * with pageable memory the copies are still correct but not overlapped.
 * Results are identical, bit for bit, to star_ctx_encode on the same inputs.
 * Asynchronous on `stream`: work already on `stream` finishes before the
 * device buffers are written, and `stream` reaches completion only after the
 * host outputs are written.  The first call creates two copy streams and
 * their events (kept until star_cache_destroy). */
STAR_API int star_ctx_encode_host(star_cache* c, const void* hQ, const void* hK, const void* hV,
                                  void* hO, float* hLSE, void* Q, void* K, void* V, void* O,
                                  float* LSE, void* stream);

/* Anchor keys of blocks 1..n-1 under a position-ID variant ("Star
 * Attention", Section 4.1, Table 4): Ka[i-1] = the anchor rows 0..b_a-1 of
 * K (un-rotated, [B][Hkv][L][D] bf16) rotated at the IDs block i gives its
 * anchor -- mode 0: 0..b_a-1 (first block, the method); 1: i*b - b_a ..
 * i*b - 1 (the positions just before block i); 2: pos[(i-1)*b_a + j]
 * (device int32 [n-1][b_a], e.g. random draws from [0, i*b)).
 * Ka: [n-1][B][Hkv][b_a][D] bf16, caller-owned.  Nothing to do when n = 1
 * or b_a = 0. */
STAR_API int star_anchor_keys(const star_cache* c, int mode, const int* pos, double theta,
                              const void* K, void* Ka, void* stream);

/* Phase 1 of blocks that follow an anchor held outside this context ([P2]
 * Phase 1 Steps 3-4, one host's blocks when the context is spread over
 * several GPUs: every host but the first receives the anchor and encodes
 * each of its blocks behind it).  Every block i of this cache -- block 0
 * included -- attends to the anchor rows Ka, Va [B][Hkv][b_a][D] bf16
 * (the longer context's rows 0..b_a-1, already rotated at their positions)
 * with no mask, and to its own rows causally.  Q, K, V, O, LSE and the cache
 * as star_ctx_encode; the anchor rows are only read.  With b_a = 0 the
 * blocks are plain causal blocks (star_ctx_encode) and Ka, Va may be NULL. */
STAR_API int star_ctx_encode_after_anchor(star_cache* c, const void* Q, const void* K, const void* V,
                                          const void* Ka, const void* Va, void* O, float* LSE,
                                          void* stream);

/* Phase 1 as star_ctx_encode, except that block i >= 1 attends to the
 * anchor keys Ka[i-1] (from star_anchor_keys) instead of K rows
 * 0..b_a-1; the anchor's values are V rows 0..b_a-1 as before.  Q and K are
 * the rotated inputs (star_rope at positions 0..L-1); Ka = NULL is
 * star_ctx_encode.  The cache receives the rotated K rows of each block. */
STAR_API int star_ctx_encode_anchored(star_cache* c, const void* Q, const void* K, const void* V,
                                      const void* Ka, void* O, float* LSE, void* stream);

/* Phase 2 -- query prefill ([P2] Phase 2 Steps 3, 5, 7).  Appends K, V
 * [B][Hkv][lq][D] bf16 to the query region, then every query row r of
 * Q [B][Hq][lq][D] attends to all context segments and to query-region rows
 * 0..len0+r (len0 = rows present before the call), computing per-partition
 * (A_h, s_h) partials and merging them on-chip.  O [B][Hq][lq][D] bf16, LSE
 * [B][Hq][lq] float32.  STAR_ENOSPC if len0 + lq > q_cap. */
STAR_API int star_query_prefill(star_cache* c, int lq, const void* Q, const void* K,
                       const void* V, void* O, float* LSE, void* stream);

/* Debug form of star_query_prefill ([P2] Phase 2 Steps 3 and 5, one partial
 * per partition): the same append, O and LSE, computed with exactly one
 * partial per context segment and one for the query region, and returned:
 *   Ah  [n+1][B][Hq][lq][D] float32, sh [n+1][B][Hq][lq] float32 (required):
 *       part h < n is (A_h, s_h) of context segment h, part n that of the
 *       query region (rows 0..len0+r for row r); s_h is the natural-log LSE
 *       of the scaled logits, A_h the normalised local output;
 *   O32 [B][Hq][lq][D] float32 (optional, NULL = none): the merged rows
 *       before the bf16 rounding of O.
 * n = star_cache_num_segments(c) - 1.  With lq = 1 this is a generation step
 * (append, then attend to every row, itself included) on the bf16 cache.
 * Slower than star_query_prefill (one CTA per segment); for tests and
 * inspection.  Errors as star_query_prefill, plus STAR_EINVAL for a NULL Ah
 * or sh. */
STAR_API int star_query_prefill_partials(star_cache* c, int lq, const void* Q, const void* K,
                                         const void* V, void* O, float* LSE, float* Ah, float* sh,
                                         float* O32, void* stream);

/* Phase 2 -- one generation step ([P2] Phase 2 Step 7).  Appends k, v
 * [B][Hkv][1][D] to the query region, then q [B][Hq][1][D] attends to every
 * context token and every query-region row (itself included): split-KV
 * partials merged on-chip.  o [B][Hq][1][D] bf16, lse [B][Hq] float32.
 * With kv_fp8 every cached row is read from the FP8 copy (dequantised on
 * chip, fp16 MMA: q is rounded to fp16, so its magnitude must stay within
 * fp16 range); the step's own new token enters exactly (bf16), and its FP8
 * copy is written for the steps after it.  STAR_ENOSPC if the query region is full. */
STAR_API int star_decode_step(star_cache* c, const void* q, const void* k, const void* v,
                     void* o, float* lse, void* stream);

/* Phase-2 partial over part of the cache ([P2] Phase 2 Steps 2-4: every host
 * attends the broadcast query to its own blocks and returns its local A_h
 * and s_h), for a caller that spreads the context blocks over several GPUs
 * and merges the hosts' partials itself (star_lse_merge).  Rows Q
 * [B][Hq][lq][D] bf16 attend to the context segments [first_seg, first_seg +
 * n_seg) and, when with_query = 1, to the query region after K, V
 * [B][Hkv][lq][D] are appended to it (causal, as star_query_prefill; lq = 1
 * is a generation step).  With with_query = 0 the query region is neither
 * read nor written and K, V may be NULL.  Outputs, float32: A [B][Hq][lq][D]
 * the normalised local attention output, s [B][Hq][lq] its natural-log LSE
 * of the scaled logits (A = 0, s = -inf for a row that sees no key).
 * 1 <= lq <= q_cap.  STAR_ENOSPC if with_query and the region is full.
 * lq = 1 over segments that reach the last one runs the split-KV decode
 * kernel (as star_decode_step over those rows: on a kv_fp8 cache it reads
 * the E4M3 copy of the cached rows, the token exact); other calls run the
 * prefill tile kernel on a span plan of the range, on the bf16 rows. */
STAR_API int star_partial_attend(star_cache* c, int first_seg, int n_seg, int with_query, int lq,
                                 const void* Q, const void* K, const void* V, float* A, float* s,
                                 void* stream);

/* Debug form of star_decode_step ([P2] Phase 2 Steps 3 and 5): the same
 * step, append, o and lse, and the decode kernel's own partials.  The cached
 * rows of every (batch, kv head) -- context tokens 0..L-1, then query-region
 * rows at L + r -- are split over the kernel's CTAs; each piece one CTA folds
 * is one part:
 *   Ah [P][G][D], sh [P][G] float32: the part's local output A_h (normalised)
 *       and s_h (natural-log LSE of the scaled logits) for the G q heads of
 *       its kv head;
 *   spans [P][3]: (b*Hkv + kv head, first row, end row) of the part, host
 *       memory, written before the call returns.
 * The step's own new token is one more part the kernel folds in at the merge
 * (s = scale * q.k, A = v); it is not listed.  P is written to *n_parts;
 * STAR_EINVAL (nothing launched) when P > max_parts.  For tests and
 * inspection: slower than star_decode_step by the copies. */
STAR_API int star_decode_step_partials(star_cache* c, const void* q, const void* k, const void* v,
                                       void* o, float* lse, float* Ah, float* sh, long long* spans,
                                       int max_parts, int* n_parts, void* stream);

/* Phase 2 merge of P partials ([P2] Phase 2 Step 5; [P3] s_global, A_global):
 * A [P][R][D], s [P][R] float32 (s_h as natural-log LSE, -inf = empty part)
 * -> out_A [R][D] = sum_h exp(s_h - s) A_h, out_s [R] = s = log sum_h
 * exp(s_h).  Rows whose parts are all empty give 0 and -inf.  P >= 1,
 * R >= 0, 1 <= D <= 1024.  out_* must not alias the inputs. */
STAR_API int star_lse_merge(int P, long long R, int D, const float* A, const float* s,
                   float* out_A, float* out_s, void* stream);

/* The same merge with the output rounded once to bf16 (nearest even): out_O
 * [R][D] bf16, out_s [R] float32 -- the last step on the query host when the
 * partials come from several GPUs ([P2] Phase 2 Steps 4-5). */
STAR_API int star_lse_merge_bf16(int P, long long R, int D, const float* A, const float* s,
                                 void* out_O, float* out_s, void* stream);

/* Host-only introspection of the query prefill's work split (no device is
 * touched; for tests and capacity planning).  The prefill cuts the key rows of
 * each (batch, kv head) -- context tokens 0..L-1, then query-region rows from
 * L on -- into spans, one CTA per (span, batch x kv head, 256-row pair of
 * packed query rows):
 *   star_plan_prefill: the spans a call with `lq` query rows on a region of
 *     len0 rows would use on a GPU of `num_sms` SMs -- context segments
 *     [first_seg, first_seg + n_seg) and, with with_query, the region (as
 *     star_partial_attend; star_query_prefill is the full range with the
 *     region), or with per_segment the debug form's one span per segment and
 *     one for the region.  spans[2k], spans[2k+1] = [x0, x1) of span k;
 *     *n_spans = their count (STAR_EINVAL if it exceeds max_spans).
 *   star_prefill_span_tiles: the 128-key tiles of span [x0, x1) of (batch x
 *     kv head) bg: tiles[4t..4t+3] = (first row in the TMA map read, 1 if
 *     that map is the query region's, keys in the tile, the region row of its
 *     first key); tiles never cross a context segment's end.
 * Arguments as star_cache_create's params otherwise. */
STAR_API int star_plan_prefill(const star_params* p, int num_sms, int lq, long long len0, int first_seg,
                               int n_seg, int with_query, int per_segment, int max_spans, int* n_spans,
                               int* spans);
STAR_API int star_prefill_span_tiles(const star_params* p, long long x0, long long x1, int bg, int max_tiles,
                                     int* n_tiles, int* tiles);

/* Self-test of the failure path every pipelined kernel here uses: one CTA
 * waits, with the kernels' bounded mbarrier wait limited to `polls` polls
 * (1..2^22; the kernels use 2^22), on a barrier nothing completes, so the
 * wait must run out; the kernel then sets its error word and returns.
 * Synchronous (waits for `stream`): *gave_up = 1 when the wait gave up, the
 * expected outcome.  The context stays usable.  STAR_EINVAL for a NULL
 * gave_up or polls out of range. */
STAR_API int star_selftest_wait_timeout(unsigned polls, int* gave_up, void* stream);

/* Decode step that allocates nothing (the pages have no counterpart: this is
 * an integration entry point).  For callers that cannot call cudaMalloc on
 * their serving path -- a runtime that hands out all device memory from its
 * own pool, or one that forbids the CUDA allocator while it serves -- the KV
 * cache is the caller's memory and the split-KV scratch (partials, merge
 * tickets, error word) lives in one static device array of the library,
 * 4.3 MiB, present on every GPU that loads the library until the process
 * exits.  Same arithmetic and kernel as star_decode_step.
 *   p          layer parameters, as for star_cache_create (scale <= 0: 1/sqrt(D));
 *              kv_fp8 must be 0 (bf16 context only)
 *   q_len      query-region rows in use before this step; this call writes
 *              row q_len of q_k / q_v with k / v
 *   ctx_k/v    context cache, the layout star_cache_create uses: segment i
 *              as [B][Hkv][len_i][D] bf16, segments back to back
 *   q_k/v      query region [B][Hkv][q_cap][D] bf16
 *   q, k, v, o, lse   as for star_decode_step
 * Limits: B*Hkv*G*D*(ceil(SMs/(B*Hkv)) + 3) <= 1048576 and B*Hkv <= 1024,
 * else STAR_EINVAL.  The first call on a device looks up the array's device
 * address (make it before any stream capture).  Every call shares the one
 * array, so calls that overlap on the GPU (other streams, other threads) race;
 * each call clears the merge tickets it needs.  A kernel that gives up one of
 * its bounded pipeline waits sets the array's error word and returns early
 * (o and lse of that call are then invalid); the word is not cleared by later
 * calls: read it with star_noalloc_device_error. */
STAR_API int star_decode_step_noalloc(const star_params* p, long long q_len,
                                      const void* ctx_k, const void* ctx_v, void* q_k, void* q_v,
                                      const void* q, const void* k, const void* v,
                                      void* o, float* lse, void* stream);

/* Error word of star_decode_step_noalloc's static scratch on the current
 * device (no counterpart in the pages, like the entry point it serves):
 * waits for the work queued on `stream`, then *flag = non-zero if any
 * no-alloc decode step since the last read gave up a bounded wait (its o and
 * lse are invalid).  Clears the word and the merge tickets when it was set.
 * Allocates nothing.  STAR_EINVAL for a NULL flag. */
STAR_API int star_noalloc_device_error(int* flag, void* stream);

/* Description of the last error in this thread ("" if none). */
STAR_API const char* star_last_error(void);

/* Library version string. */
STAR_API const char* star_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STAR_ATTENTION_H */
