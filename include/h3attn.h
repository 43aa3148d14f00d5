/*
 * h3attn — biased, block-routed attention over MiniMax-H3's packed sequence
 * [text | image-ref | audio | guide video | output video], on one B200
 * (sm_100a).  Plain C ABI: pointers and sizes only.
 *
 * Operation (sources are web pages, cited by title and section):
 *
 *  Routing — "H3 SLA Attention" node page, "How it works": Q and K are
 *  mean-pooled per 64-row block ("pooled centroids"), every video query block
 *  is scored against every video key block with one small pooled matmul, and
 *  only the top (1 - sparsity_ratio) fraction of those key blocks is attended.
 *  Its inputs table: protect_audio always attends the blocks overlapping text,
 *  conditioning and audio rows; block_size 64.  "Per-layer attention config
 *  LoRAs", "Experimental: audio/text protection": prefix keys stay exact
 *  (sink_keys "prefix") and audio queries stay fully exact (sink_queries
 *  "audio").  "H3 sparse-attention breakpoints", "Results at a glance": the
 *  kept fraction counts the available video key/value tiles only.
 *
 *  Attention — "Flash Partitions for H3 native temporal alignment", section 1
 *  "What receives the temporal bias?": for an output-video query and a
 *  guide-video key,
 *     dt = |t_q - t_k|,
 *     penalty(dt) = min(strength * (max(dt - window, 0) / falloff)^2, cap),
 *     score = q.k / sqrt(head_dim) - penalty(dt);
 *  every other pair keeps score = q.k / sqrt(head_dim).  Defaults: strength
 *  2.0, window 0.20 s, falloff 0.25 s, cap 6.0 (same page; also "TARA :
 *  alignement temporel natif ...", "La règle temporelle").  The output is the
 *  exact softmax-weighted sum of V over the attended keys; LSE is the
 *  natural-log normaliser (same page, section 4).
 *
 * Readings where the pages are silent: pooled score = Qp.Kp / sqrt(d), per
 * head; k = clamp(ceil((1 - s) * nV - 1e-9), 1, nV); ties go to the lower
 * block index; a key block is forced and a query block is dense iff it holds
 * any non-video row; dropped blocks leave the softmax; routing ignores the
 * penalty, which is applied exactly on the routed output -> guide pairs.
 *
 * Conventions for every call:
 *  - Q, K, V, O are bf16 (passed as uint16_t bit patterns), layout
 *    [H][S][d], contiguous, row-major, on the device; base addresses 16-byte
 *    aligned.  seg is uint8 [S] and times is float32 [S] (seconds, 4-byte
 *    aligned), on the device; times are read only for guide/output rows.
 *    Integer and float32 arrays (kv_sel, lse, times) need 4-byte alignment.
 *  - The caller owns every buffer; the library allocates no memory.
 *  - All device work is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).  Only h3attn_check synchronises.
 *  - Return value 0 on success, a negative H3ATTN_E* code otherwise.  On a
 *    host-side error nothing is launched and outputs are untouched.  Device-
 *    side failures (a bounded wait that ran out, a corrupt routed list) are
 *    recorded in the workspace status word and reported by h3attn_check.
 *  - No call prints, aborts or throws.
 */
#ifndef H3ATTN_H
#define H3ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define H3ATTN_API __attribute__((visibility("default")))
#else
#define H3ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define H3ATTN_OK 0
#define H3ATTN_EINVAL (-1)       /* bad argument: null pointer, bad size, bad value */
#define H3ATTN_EUNSUPPORTED (-2) /* d not 64/128, block not 64, video rows not a suffix, S too large */
#define H3ATTN_EALIGN (-3)       /* a base address is misaligned (16 bytes for tensors, 4 for int32/float32 arrays) */
#define H3ATTN_ECUDA (-4)        /* a CUDA runtime/driver call or launch failed */
#define H3ATTN_ETIMEOUT (-5)     /* a bounded device-side wait gave up */
#define H3ATTN_EWORKSPACE (-6)   /* workspace missing or too small */
#define H3ATTN_EDATA (-7)        /* device found a corrupt routed list (index out of range) */

/* Segment ids of the packed sequence. */
enum {
  H3ATTN_SEG_TEXT = 0,
  H3ATTN_SEG_IMAGE_REF = 1,
  H3ATTN_SEG_AUDIO = 2,
  H3ATTN_SEG_GUIDE = 3,
  H3ATTN_SEG_OUTPUT = 4
};

/* Temporal penalty controls ("Flash Partitions ...", section 1).
 * strength >= 0, window >= 0, falloff > 0, cap >= 0, all finite.
 * strength == 0 or cap == 0 removes the penalty (same page, section 4). */
typedef struct {
  float strength;
  float window;  /* seconds */
  float falloff; /* seconds */
  float cap;
} h3attn_penalty;

/* Block plan of one packed sequence.  Plain data, caller-owned, filled by
 * h3attn_plan_init (host only, no CUDA call).
 *  n_blocks          ceil(S / block)
 *  prefix_rows       rows before the first video row (video rows are a suffix)
 *  first_video_block first block whose rows are all video = ceil(prefix_rows / block)
 *  n_forced          = first_video_block: key blocks always attended, and
 *                    query blocks attended densely (they hold a non-video row)
 *  n_video_blocks    n_blocks - first_video_block (nV)
 *  k                 routed video key blocks per video query block:
 *                    ceil((1 - sparsity) nV), at least 1 (a product within
 *                    1e-9 above an integer counts as that integer) */
typedef struct {
  int32_t H, S, d, block;
  double sparsity;
  int32_t n_blocks, prefix_rows, first_video_block, n_forced, n_video_blocks, k;
} h3attn_plan;

/* Fill *plan from the host copy of seg[S].  block must be 64; d 64 or 128;
 * 0 <= sparsity < 1; rows with seg 3/4 (video) must form a contiguous suffix
 * of the sequence ("Flash Partitions ...", section 7: contiguous video rows).
 * A sequence without video rows is accepted (no routing; everything dense). */
H3ATTN_API int h3attn_plan_init(h3attn_plan* plan, int H, int S, int d, int block, double sparsity,
                     const uint8_t* seg_host);

/* Bytes of device workspace a plan needs for h3attn_route and h3attn_forward
 * (status word; the attention scratch: per-block key descriptors, per-key
 * guide times and a bitmap of the key blocks that need per-key handling,
 * about 0.5 MB at S = 116,883; the query-block pair table of a routed
 * forward, 4 bytes per head and 128-row tile of video query blocks, about
 * 0.2 MB at S = 116,883, H = 56; and the routing scratch: three-part bf16
 * pooled Q and K of the video blocks, six d-long parts per row, and the fp32
 * pooled-score matrix, about 1.2 GB at S = 116,883, H = 56, d = 128).
 * The caller allocates it once, zero-filled (the first 256 bytes hold the
 * status word that h3attn_check reads and clears). */
H3ATTN_API size_t h3attn_workspace_bytes(const h3attn_plan* plan);

/* Block mean-pool of one tensor ("H3 SLA Attention", pooled centroids):
 * out[h][b - first_block][c] = mean over the valid rows r of block b
 * (rows [b*64, min(S, b*64+64))) of x[h][r][c], accumulated in fp32.
 * x: bf16 [H][S][d] device; out: float32 [H][n_out][d] device;
 * blocks [first_block, first_block + n_out) must lie in [0, n_blocks). */
H3ATTN_API int h3attn_pool(const h3attn_plan* plan, const uint16_t* x, int first_block, int n_out, float* out,
                void* stream);

/* Routing (pool + pooled score + top-k).  For every head h and video query
 * block i (block first_video_block + i):
 *   kv_sel[h][i][0..k) = the k video key blocks j with the highest
 *   Qp[h][i].Kp[h][j] / sqrt(d), ties to the lower block, listed as absolute
 *   block indices in ascending order.  Qp, Kp are fp32 block means; the dot
 *   products run on the tensor cores over three-part bf16 splits of them
 *   (x = h + m + l, the 24 significant bits of the fp32 mean; the six
 *   products of parts down to relative order 2^-16, each exact, accumulated
 *   in fp32: the dropped ones are below 2^-24 of the product).
 * q, k: bf16 [H][S][d] device; kv_sel: int32 [H][n_video_blocks][k] device.
 * ws: workspace of at least h3attn_workspace_bytes(plan) bytes. */
H3ATTN_API int h3attn_route(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, int32_t* kv_sel,
                 void* ws, size_t ws_bytes, void* stream);

/* Routing with no workspace and no allocation.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory when they route (a framework that owns all device memory
 * through its own pool, a loop that must not pay cudaMalloc's implicit
 * synchronisation, a host with a fixed memory budget).
 * Same result as h3attn_route.  Its scratch (the three-part bf16 pooled
 * centroids of Q and K and the fp32 score matrix) is a fixed 64 MiB array
 * inside the library that every GPU loading the library holds until the
 * process exits; its first 256 bytes are the status word of these calls, and
 * problems needing more than the remaining 64 MiB - 256 bytes, i.e. with
 * 24 * H * n_video_blocks * d + 16 * H * n_video_blocks * ceil(n_video_blocks / 4)
 * bytes above that, are rejected with H3ATTN_EWORKSPACE.  Every call overwrites
 * all the scratch it reads, so nothing needs clearing between calls; calls
 * that overlap on the GPU (other streams, other threads) share the array and
 * race.  A bounded device-side wait that gives up is recorded in the status
 * word, not returned: call h3attn_route_static_check to read it.  The array's
 * device address is looked up on the first call with a device current, and
 * again when that device's current context has changed (for instance after
 * cudaDeviceReset); make that first call before any stream capture.
 * Allocates nothing and calls no allocating routine. */
H3ATTN_API int h3attn_route_static(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, int32_t* kv_sel,
                                   void* stream);

/* Synchronise `stream`, then return and clear the status word of the
 * h3attn_route_static calls made on the current device: H3ATTN_OK, or
 * H3ATTN_ETIMEOUT when a bounded device-side wait of one of them gave up (its
 * kv_sel is then not valid); H3ATTN_ECUDA if the stream reports an error.
 * Allocates nothing. */
H3ATTN_API int h3attn_route_static_check(void* stream);

/* Exact attention over the routed tiles with the temporal penalty.
 * Each query row attends: all keys if its block is a forced (non-video)
 * block or kv_sel is NULL; otherwise the forced key blocks plus the routed
 * blocks kv_sel[h][qblock - first_video_block][0..k).  pen NULL = no penalty.
 * o: bf16 [H][S][d] device (rounded to nearest even); lse: float32 [H][S]
 * device natural-log normaliser, or NULL.
 * Routed indices outside [first_video_block, n_blocks) are ignored and flagged
 * (H3ATTN_EDATA from h3attn_check).
 * ws: the workspace (h3attn_workspace_bytes(plan) bytes always suffices); a
 * call with kv_sel NULL reads and writes only its status word and attention
 * scratch, a routed call also the pair table that follows them.  The routed
 * call pairs its video query blocks into 128-row tiles by the overlap of their
 * routed lists (groups of 32 consecutive blocks, greedy largest overlap first);
 * the pairing affects only the speed, not which keys a row attends. */
H3ATTN_API int h3attn_forward(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const uint8_t* seg, const float* times, const h3attn_penalty* pen,
                   const int32_t* kv_sel, uint16_t* o, float* lse, void* ws, size_t ws_bytes,
                   void* stream);

/* The whole call from host memory: routing (when the plan routes) and
 * attention for every head, with the host<->device copies overlapped with the
 * kernels.  Every step of the path is independent per head ("H3 SLA
 * Attention", "How it works": routing per head; the attention is per head),
 * so the heads go in chunks of chunk_heads: chunk c's Q/K/V copy in on
 * copy_in_stream, its routing and attention run on `stream` once they have
 * landed, and its O (and LSE) copy out on copy_out_stream, while chunk c+1 is
 * already copying in.
 *  q_host, k_host, v_host: bf16 [H][S][d]; o_host: bf16 [H][S][d];
 *  seg_host: uint8 [S]; times_host: float32 [S] (may be NULL when pen is NULL);
 *  lse_host: float32 [H][S] or NULL -- host memory, page-locked for the copies
 *  to overlap (pageable memory works but serialises).
 *  q, k, v, o: device buffers of the same shapes; seg, times: device [S];
 *  kv_sel: device int32 [H][n_video_blocks][k] (may be NULL when the plan does
 *  not route); lse: device float32 [H][S], NULL exactly when lse_host is.
 *  ws: as for h3attn_route / h3attn_forward (h3attn_workspace_bytes(plan)).
 *  Results: o_host / lse_host as h3attn_forward would give; they are complete
 *  when `stream` reaches the point where this call returns (the call makes
 *  `stream` wait for the last copy out).  The copies start only after the work
 *  already queued on `stream`, so back-to-back calls on the same buffers do
 *  not overlap one another.  Three distinct streams give the
 *  overlap; the same stream three times gives the same results in sequence.
 *  Errors as for h3attn_route / h3attn_forward, checked before each chunk's
 *  launches; chunk_heads must lie in [1, H]. */
H3ATTN_API int h3attn_attend_host(const h3attn_plan* plan, const uint16_t* q_host, const uint16_t* k_host,
                                  const uint16_t* v_host, const uint8_t* seg_host, const float* times_host,
                                  const h3attn_penalty* pen, uint16_t* o_host, float* lse_host, uint16_t* q,
                                  uint16_t* k, uint16_t* v, uint8_t* seg, float* times, int32_t* kv_sel, uint16_t* o,
                                  float* lse, void* ws, size_t ws_bytes, int chunk_heads, void* stream,
                                  void* copy_in_stream, void* copy_out_stream);

/* Pooled tail term ("H3 SLA Attention", inputs table, tail_correction):
 * instead of dropping the video key blocks a query block's top-k left out,
 * fold them in as one pooled term, scored from the pooled centroids routing
 * computed.  For video query block i of head h (dropped set D_i, n_j valid
 * rows of block j, Qp/Kp/Vp block means):
 *     Lt_i = log sum_{j in D_i} n_j exp(Qp_i . Kp_j / sqrt(d)),
 *     Ot_i = sum_{j in D_i} n_j exp(Qp_i . Kp_j / sqrt(d) - Lt_i) Vp_j,
 * no temporal penalty (routing sees none); each row of block i then merges
 * (Ot_i, Lt_i) with its routed result (o, lse) as one more partition of weight
 * 1 (the merge of h3attn_merge), in place.  Rows of dense (prefix) query
 * blocks are unchanged.  The dot products are the fp32-accurate pooled scores
 * routing computed; the weights n_j exp(...) and Vp are rounded to bf16 for the
 * tensor-core sum (fp32 accumulation).
 * Contract: call after h3attn_route(plan, q, k, kv_sel, ws, ...) and
 * h3attn_forward(plan, ..., kv_sel, o, lse, ws, ...) with the same plan, ws
 * and kv_sel, before anything else reuses ws (this call reads the pooled
 * scores h3attn_route left in it).  v: bf16 [H][S][d] device; kv_sel as for
 * h3attn_forward; o, lse: that call's outputs (lse not NULL), updated in
 * place; tail_ws: device scratch of h3attn_tail_workspace_bytes(plan) bytes
 * (about 0.43 GB at S = 116,883, H = 56, d = 128; no zeroing needed).
 * Routed indices outside the video blocks are ignored. */
H3ATTN_API size_t h3attn_tail_workspace_bytes(const h3attn_plan* plan);
H3ATTN_API int h3attn_tail_correct(const h3attn_plan* plan, const uint16_t* v, const int32_t* kv_sel, uint16_t* o,
                                   float* lse, void* ws, size_t ws_bytes, void* tail_ws, size_t tail_ws_bytes,
                                   void* stream);

/* Int8 QK ("H3 SLA Attention", inputs table, use_int8_qk: Q and K quantised
 * to int8 per token with a dynamic scale before the QK dot product on the
 * selected blocks; PV stays at full precision).
 *
 * h3attn_quantize_qk: per row x (d values) of Q and of K,
 *   a = max|x|,  s = a / 127,  code = clamp(rint(x * (127 / a)), -127, 127),
 * in fp32 with round-to-nearest-even (ties to even); a zero row gets s = 0 and
 * zero codes.  q, k: bf16 [H][S][d] device, 16-byte aligned.  qk8_ws: device
 * scratch of h3attn_qk8_workspace_bytes(plan) bytes, 16-byte aligned (about
 * 1.7 GB at S = 116,883, H = 56, d = 128), laid out as int8 codes of Q
 * [H][S][d], int8 codes of K [H][S][d], float32 scales of Q [H][64 n_blocks],
 * float32 scales of K [H][64 n_blocks], each part starting on a 256-byte
 * boundary (scale rows S .. 64 n_blocks - 1 hold 0); every call rewrites it.
 *
 * h3attn_forward_qk8: h3attn_quantize_qk, then the attention of
 * h3attn_forward with the score of (query i, key j) taken as
 * s_q,i s_k,j (sum over d of the codes' products) / sqrt(d), accumulated exactly
 * in int32 on the tensor cores; penalty, softmax and PV (bf16 V) unchanged.
 * d must be 128 (H3ATTN_EUNSUPPORTED otherwise).  Other arguments, outputs and
 * workspace as for h3attn_forward.  The result differs from h3attn_forward's
 * by the quantisation (about 1 % relative on Gaussian inputs, the scale the
 * page reports for int8 attention). */
H3ATTN_API size_t h3attn_qk8_workspace_bytes(const h3attn_plan* plan);
H3ATTN_API int h3attn_quantize_qk(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, void* qk8_ws,
                                  size_t qk8_ws_bytes, void* stream);
H3ATTN_API int h3attn_forward_qk8(const h3attn_plan* plan, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                  const uint8_t* seg, const float* times, const h3attn_penalty* pen,
                                  const int32_t* kv_sel, uint16_t* o, float* lse, void* ws, size_t ws_bytes,
                                  void* qk8_ws, size_t qk8_ws_bytes, void* stream);

/* Merge of normalised partition results ("Flash Partitions for H3 native
 * temporal alignment", section 4 "Why log-sum-exp is necessary"): partition i
 * is an attention output O_i over some key set (normalised by its own sum)
 * with its natural-log normaliser L_i -- h3attn_forward's o and lse -- and a
 * non-negative multiplier w_i of its probabilities, given as log_w[i] (-inf
 * for w_i = 0; log_w NULL: every w_i = 1).  Per (head, row):
 *     adjusted_L_i = L_i + log w_i,  L = logsumexp_i adjusted_L_i,
 *     O = sum_i exp(adjusted_L_i - L) O_i    (fp32, rounded to bf16 RNE),
 * which for disjoint key sets equals the attention over their union with
 * each set's probabilities scaled by its w_i.  A row whose adjusted
 * normalisers are all -inf gets O = 0 and L = -inf.
 *  n_parts in [1, 8]; o_parts / lse_parts: host arrays of n_parts device
 *  pointers to bf16 [H][S][d] (16-byte aligned) and float32 [H][S]; log_w:
 *  host array of n_parts floats (no NaN, no +inf) or NULL; o: bf16 [H][S][d]
 *  device, 16-byte aligned (may be o_parts[0]); lse: float32 [H][S] device or
 *  NULL. */
H3ATTN_API int h3attn_merge(int n_parts, const uint16_t* const* o_parts, const float* const* lse_parts,
                            const float* log_w, int H, int S, int d, uint16_t* o, float* lse, void* stream);

/* Dense biased attention (every query attends every key; the penalty on
 * output -> guide pairs): h3attn_forward with a dense plan and kv_sel NULL.
 * Needs h3attn_dense_workspace_bytes(S) bytes of zero-filled workspace (the
 * status word and the attention scratch). */
H3ATTN_API size_t h3attn_dense_workspace_bytes(int S);
H3ATTN_API int h3attn_dense_biased(int H, int S, int d, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const uint8_t* seg, const float* times, const h3attn_penalty* pen, uint16_t* o,
                        float* lse, void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, then return and clear the device-side status word
 * of ws: H3ATTN_OK, H3ATTN_ETIMEOUT or H3ATTN_EDATA; H3ATTN_ECUDA if the
 * stream reports an error. */
H3ATTN_API int h3attn_check(void* ws, void* stream);

/* Test and diagnostics only: bound every device-side wait of the attention
 * kernels launched by later calls (h3attn_forward, h3attn_dense_biased,
 * h3attn_forward_qk8, h3attn_attend_host) to `polls` unsuccessful polls of its
 * barrier; 0 restores the default (no poll bound).  The time bound of 2 s per
 * wait always applies, and the waits that drain a give-up (for the kernel's
 * own TMA loads and MMAs already in flight) are bounded by time only, so a
 * kernel that gives up still lets its own copies complete before it exits.
 * A wait that runs out records H3ATTN_ETIMEOUT in the workspace status word
 * (h3attn_check reports and clears it) and the outputs of that call are not
 * valid.  Process-wide; not synchronised with calls already launched. */
H3ATTN_API int h3attn_set_wait_polls(uint32_t polls);

/* Self-test of the bounded-wait mechanism: launches one block that waits on
 * an mbarrier nothing arrives at, with a limit of `polls` polls, and records
 * H3ATTN_ETIMEOUT in the status word when it gives up.  No other work. */
H3ATTN_API int h3attn_selftest_timeout(void* ws, uint32_t polls, void* stream);

/* Static description of a status code (never NULL). */
H3ATTN_API const char* h3attn_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* H3ATTN_H */
