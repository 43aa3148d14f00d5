/*
 * ORACLE — test infrastructure only.
 *
 * A plain, slow, double-precision CPU statement of what the biased, routed
 * attention call over MiniMax-H3's packed sequence computes.  Only the tests,
 * the smoke check and the CPU-baseline leg of the benchmark may load it.  It
 * shares no code, header or table with the CUDA library: it does not include
 * the library's header and re-states every constant it needs.
 *
 * Sources (web pages; cited by title and section):
 *  [FP]  "Flash Partitions for H3 native temporal alignment"
 *        §1 "What receives the temporal bias?" (edge rule, penalty, score),
 *        §3 "Decompose the same rule into positive contributions",
 *        §4 "Why log-sum-exp is necessary" (partition merge).
 *  [SLA] "H3 SLA Attention" node page, "How it works" (pooled matmul, top
 *        1 - sparsity_ratio) and its inputs table (sparsity_ratio,
 *        block_size, protect_audio).
 *  [CFG] "Per-layer attention config LoRAs",
 *        "Experimental: audio/text protection"
 *        (sink_keys "prefix", sink_queries "audio"; 64-token query blocks).
 *  [BRK] "H3 sparse-attention breakpoints: FL2VA, Ref2VA, and Turbo",
 *        "Results at a glance" (what "10 %" of video KV means).
 *  [WIKI] "TARA : alignement temporel natif pour les références MiniMax H3",
 *        "La règle temporelle" (same rule and defaults).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - logit scale 1/sqrt(d), natural-log softmax [FP §1];
 *  - only output-video queries x guide-video keys are penalised [FP §1];
 *  - dt = |t_q - t_k| from per-row times;
 *  - pooled centroid = mean of the block's valid rows; pooled score =
 *    Qp . Kp / sqrt(d); routing is per head;
 *  - k = clamp(ceil((1 - s) * nV - 1e-9), 1, nV);
 *  - ties in the pooled score go to the lower block index;
 *  - a key block is forced (always attended) and a query block is dense iff
 *    it overlaps any non-video row; every other block is a video block;
 *  - dropped blocks leave the softmax (no pooled tail term);
 *  - routing ignores the penalty; the exact penalty applies on the routed
 *    output -> guide pairs;
 *  - int8 QK: per-row scale max|x| / 127 and codes rint(x * (127 / max|x|)),
 *    in fp32 with ties to even.
 *
 * Segment ids: 0 text, 1 image-ref, 2 audio, 3 guide video, 4 output video.
 * bf16 inputs are passed as their 16-bit patterns and widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define SEG_GUIDE 3
#define SEG_OUTPUT 4

static inline int is_video(uint8_t s) { return s == SEG_GUIDE || s == SEG_OUTPUT; }

static inline double bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* [FP §1], [WIKI]: penalty(dt) = min(strength * (max(dt - window, 0) / falloff)^2, cap). */
double oracle_penalty(double dt, double strength, double window, double falloff, double cap) {
    double excess = dt - window;
    if (excess < 0.0) excess = 0.0;
    double r = excess / falloff;
    double p = strength * r * r;
    return p < cap ? p : cap;
}

/* [SLA] top (1 - sparsity_ratio) fraction of the video key blocks; [BRK] the
 * fraction counts video KV tiles only.  Reading: round up, at least one. */
int oracle_k(int n_video_blocks, double sparsity) {
    double want = ceil((1.0 - sparsity) * (double)n_video_blocks - 1e-9);
    int k = (int)want;
    if (k < 1) k = 1;
    if (k > n_video_blocks) k = n_video_blocks;
    return k;
}

/* Block classes ([SLA] protect_audio: "blocks overlapping" text/cond/audio;
 * [CFG] sink_keys "prefix", sink_queries "audio").  nonvideo[b] = 1 iff block
 * b (rows [b*B, min(S,(b+1)*B))) holds a non-video row.  Returns the number of
 * blocks ceil(S/B). */
int oracle_block_classes(int S, int B, const uint8_t *seg, uint8_t *nonvideo) {
    int nkb = (S + B - 1) / B;
    for (int b = 0; b < nkb; ++b) {
        int lo = b * B, hi = lo + B < S ? lo + B : S;
        uint8_t nv = 0;
        for (int r = lo; r < hi; ++r)
            if (!is_video(seg[r])) nv = 1;
        nonvideo[b] = nv;
    }
    return nkb;
}

/* Per-head mean of every block's valid rows ([SLA] "pooled centroids").
 * x: bf16 [H][S][d]; out: [H][nKB][d]. */
void oracle_pool(int H, int S, int d, int B, const uint16_t *x, double *out) {
    int nkb = (S + B - 1) / B;
#pragma omp parallel for schedule(static)
    for (long hb = 0; hb < (long)H * nkb; ++hb) {
        int h = (int)(hb / nkb), b = (int)(hb % nkb);
        int lo = b * B, hi = lo + B < S ? lo + B : S;
        double *o = out + (size_t)hb * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int r = lo; r < hi; ++r) {
            const uint16_t *row = x + ((size_t)h * S + r) * d;
            for (int c = 0; c < d; ++c) o[c] += bf16_to_f64(row[c]);
        }
        for (int c = 0; c < d; ++c) o[c] /= (double)(hi - lo);
    }
}

typedef struct {
    double score;
    int32_t block;
} scored_block;

/* score descending, then block index ascending */
static int by_score_then_index(const void *a, const void *b) {
    const scored_block *x = (const scored_block *)a, *y = (const scored_block *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->block > y->block) - (x->block < y->block);
}

static int ascending_i32(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Block-sparse routing ([SLA] "How it works"): for every head and video query
 * block i, score every video key block j with the pooled product
 * Qp[i] . Kp[j] / sqrt(d), keep the k best (ties -> lower j), list them in
 * ascending block order.
 *
 * sel: int32 [H][nV][k] (absolute block indices).  Optional outputs (NULL to
 * skip): scores [H][nV][nV] (video q-block x video kv-block, both in
 * ascending block order) and kth [H][nV] (the k-th best score).
 * Returns k, or -1 if there is no video block.
 */
int oracle_route(int H, int S, int d, int B, double sparsity, const uint8_t *seg,
                 const uint16_t *q, const uint16_t *k, int32_t *sel, double *scores,
                 double *kth) {
    int nkb = (S + B - 1) / B;
    uint8_t *nonvideo = (uint8_t *)malloc((size_t)nkb);
    oracle_block_classes(S, B, seg, nonvideo);
    int nv = 0;
    for (int b = 0; b < nkb; ++b) nv += !nonvideo[b];
    if (nv == 0) {
        free(nonvideo);
        return -1;
    }
    int32_t *vid = (int32_t *)malloc(sizeof(int32_t) * (size_t)nv);
    for (int b = 0, i = 0; b < nkb; ++b)
        if (!nonvideo[b]) vid[i++] = b;
    int kk = oracle_k(nv, sparsity);

    double *qp = (double *)malloc(sizeof(double) * (size_t)H * nkb * d);
    double *kp = (double *)malloc(sizeof(double) * (size_t)H * nkb * d);
    oracle_pool(H, S, d, B, q, qp);
    oracle_pool(H, S, d, B, k, kp);
    double inv_sqrt_d = 1.0 / sqrt((double)d);

#pragma omp parallel
    {
        scored_block *cand = (scored_block *)malloc(sizeof(scored_block) * (size_t)nv);
#pragma omp for schedule(dynamic, 4)
        for (long hi = 0; hi < (long)H * nv; ++hi) {
            int h = (int)(hi / nv), i = (int)(hi % nv);
            const double *a = qp + ((size_t)h * nkb + vid[i]) * d;
            for (int j = 0; j < nv; ++j) {
                const double *bvec = kp + ((size_t)h * nkb + vid[j]) * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += a[c] * bvec[c];
                cand[j].score = dot * inv_sqrt_d;
                cand[j].block = vid[j];
                if (scores) scores[(size_t)hi * nv + j] = cand[j].score;
            }
            qsort(cand, (size_t)nv, sizeof(scored_block), by_score_then_index);
            if (kth) kth[hi] = cand[kk - 1].score;
            int32_t *dst = sel + (size_t)hi * kk;
            for (int t = 0; t < kk; ++t) dst[t] = cand[t].block;
            qsort(dst, (size_t)kk, sizeof(int32_t), ascending_i32);
        }
        free(cand);
    }
    free(qp);
    free(kp);
    free(vid);
    free(nonvideo);
    return kk;
}

/*
 * The key blocks a query row attends.  Dense when sel is NULL or the row's
 * block is non-video; otherwise the forced (non-video) blocks plus the routed
 * list of the row's video query block.  Writes a 0/1 flag per block.
 */
static void attended_blocks(int nkb, const uint8_t *nonvideo, const int32_t *vid_index,
                            const int32_t *sel, int kk, int H, int nv, int h, int qblock,
                            uint8_t *use) {
    if (sel == NULL || nonvideo[qblock]) {
        for (int b = 0; b < nkb; ++b) use[b] = 1;
        return;
    }
    for (int b = 0; b < nkb; ++b) use[b] = nonvideo[b];
    const int32_t *lst = sel + ((size_t)h * nv + vid_index[qblock]) * kk;
    for (int t = 0; t < kk; ++t) use[lst[t]] = 1;
    (void)H;
}

/* score of one (query row, key row) pair, before any penalty: q.k / sqrt(d) */
static inline double raw_score(const uint16_t *qr, const uint16_t *kr, int d, double inv_sqrt_d) {
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += bf16_to_f64(qr[c]) * bf16_to_f64(kr[c]);
    return dot * inv_sqrt_d;
}

/* Int8 QK operands of the quantised score (oracle_attend_qk8); NULL for the exact one. */
typedef struct {
    const int8_t *q8, *k8;  /* codes [H][S][d] */
    const float *sq, *sk;   /* scales [H][S] */
} qk8_operands;

/* the quantised score s_q s_k (sum_c cq_c ck_c) / sqrt(d); the integer sum is exact */
static inline double qk8_score(const qk8_operands *o, size_t qi, size_t kj, int d, double inv_sqrt_d) {
    const int8_t *qr = o->q8 + qi * d, *kr = o->k8 + kj * d;
    long dot = 0;
    for (int c = 0; c < d; ++c) dot += (long)qr[c] * (long)kr[c];
    return (double)dot * (double)o->sq[qi] * (double)o->sk[kj] * inv_sqrt_d;
}

/*
 * Direct definition ([FP §1], [WIKI]).  For each requested (head, row):
 *   x_j = q.k_j / sqrt(d) - p_j over the attended keys j,
 *   p_j = penalty(|t_q - t_j|) if seg_q = output and seg_j = guide, else 0,
 *   O = sum_j exp(x_j - m) v_j / sum_j exp(x_j - m),  LSE = m + ln sum_j exp(x_j - m).
 * pen: {strength, window, falloff, cap} or NULL (no penalty).
 * sel/kk: routed lists from a routing call, or NULL for dense attention.
 * out_o: [n][d]; out_lse: [n].
 */
static void attend_core(int H, int S, int d, int B, const uint8_t *seg, const float *times,
                        const double *pen, const int32_t *sel, int kk, const uint16_t *q,
                        const uint16_t *k, const uint16_t *v, const qk8_operands *qk8, int n,
                        const int32_t *heads, const int32_t *rows, double *out_o, double *out_lse) {
    int nkb = (S + B - 1) / B;
    uint8_t *nonvideo = (uint8_t *)malloc((size_t)nkb);
    oracle_block_classes(S, B, seg, nonvideo);
    int32_t *vid_index = (int32_t *)malloc(sizeof(int32_t) * (size_t)nkb);
    int nv = 0;
    for (int b = 0; b < nkb; ++b) vid_index[b] = nonvideo[b] ? -1 : nv++;
    double inv_sqrt_d = 1.0 / sqrt((double)d);

#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)S);
        uint8_t *use = (uint8_t *)malloc((size_t)nkb);
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < n; ++t) {
            int h = heads[t], i = rows[t];
            attended_blocks(nkb, nonvideo, vid_index, sel, kk, H, nv, h, i / B, use);
            const uint16_t *qr = q != NULL ? q + ((size_t)h * S + i) * d : NULL;
            int biased_row = pen != NULL && seg[i] == SEG_OUTPUT;
            double m = -INFINITY;
            for (int j = 0; j < S; ++j) {
                if (!use[j / B]) continue;
                double s = qk8 != NULL ? qk8_score(qk8, (size_t)h * S + i, (size_t)h * S + j, d, inv_sqrt_d)
                                       : raw_score(qr, k + ((size_t)h * S + j) * d, d, inv_sqrt_d);
                if (biased_row && seg[j] == SEG_GUIDE) {
                    double dt = fabs((double)times[i] - (double)times[j]);
                    s -= oracle_penalty(dt, pen[0], pen[1], pen[2], pen[3]);
                }
                x[j] = s;
                if (s > m) m = s;
            }
            double l = 0.0;
            double *o = out_o + (size_t)t * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int j = 0; j < S; ++j) {
                if (!use[j / B]) continue;
                double w = exp(x[j] - m);
                l += w;
                const uint16_t *vr = v + ((size_t)h * S + j) * d;
                for (int c = 0; c < d; ++c) o[c] += w * bf16_to_f64(vr[c]);
            }
            for (int c = 0; c < d; ++c) o[c] /= l;
            out_lse[t] = m + log(l);
        }
        free(x);
        free(use);
    }
    free(vid_index);
    free(nonvideo);
}

void oracle_attend(int H, int S, int d, int B, const uint8_t *seg, const float *times,
                   const double *pen, const int32_t *sel, int kk, const uint16_t *q,
                   const uint16_t *k, const uint16_t *v, int n, const int32_t *heads,
                   const int32_t *rows, double *out_o, double *out_lse) {
    attend_core(H, S, d, B, seg, times, pen, sel, kk, q, k, v, NULL, n, heads, rows, out_o, out_lse);
}

/* ---- int8 QK ([SLA] inputs table, use_int8_qk) ----
 *
 * Q and K are quantised to int8 per token with a dynamic scale before the
 * QK dot product; PV stays at the inputs' precision.  Per row x of d values:
 *   a = max_c |x_c|,  s = a / 127,  code_c = clamp(rint(x_c * (127 / a)), -127, 127);
 *   a row of zeros gets s = 0 and zero codes.
 * The page fixes no arithmetic for this; the two quotients and the product
 * are taken in fp32 with round-to-nearest-even (rint: ties to even), so that
 * a code is decided the same way wherever the rule is evaluated.  The score
 * of (query i, key j) becomes s_q,i s_k,j (sum_c code_q,c code_k,c) / sqrt(d);
 * everything after it (penalty, softmax, PV) is unchanged.
 */
static inline float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

void oracle_quantize_rows(long n_rows, int d, const uint16_t *x, int8_t *codes, float *scales) {
    for (long r = 0; r < n_rows; ++r) {
        const uint16_t *xr = x + (size_t)r * d;
        int8_t *cr = codes + (size_t)r * d;
        float a = 0.0f;
        for (int c = 0; c < d; ++c) {
            float m = fabsf(bf16_to_f32(xr[c]));
            if (m > a) a = m;
        }
        if (a == 0.0f) {
            scales[r] = 0.0f;
            for (int c = 0; c < d; ++c) cr[c] = 0;
            continue;
        }
        scales[r] = a / 127.0f;
        float inv = 127.0f / a;
        for (int c = 0; c < d; ++c) {
            float t = rintf(bf16_to_f32(xr[c]) * inv);
            if (t != t) t = 0.0f; /* 0 * inf when 127 / a overflows (a tiny subnormal max) */
            if (t > 127.0f) t = 127.0f;
            if (t < -127.0f) t = -127.0f;
            cr[c] = (int8_t)t;
        }
    }
}

/*
 * As oracle_attend, with the int8 QK score above: q8/k8 are the codes and
 * sq/sk the scales of Q and K ([H][S][d] and [H][S], from oracle_quantize_rows);
 * v stays bf16.
 */
void oracle_attend_qk8(int H, int S, int d, int B, const uint8_t *seg, const float *times,
                       const double *pen, const int32_t *sel, int kk, const int8_t *q8,
                       const float *sq, const int8_t *k8, const float *sk, const uint16_t *v,
                       int n, const int32_t *heads, const int32_t *rows, double *out_o,
                       double *out_lse) {
    qk8_operands o = {q8, k8, sq, sk};
    attend_core(H, S, d, B, seg, times, pen, sel, kk, NULL, NULL, v, &o, n, heads, rows, out_o, out_lse);
}

/* ---- Flash-Partitions evaluation of the same rule ([FP §3], [FP §4]) ---- */

typedef struct {
    double time;
    int32_t key;
} timed_key;

static int by_time(const void *a, const void *b) {
    const timed_key *x = (const timed_key *)a, *y = (const timed_key *)b;
    if (x->time < y->time) return -1;
    if (x->time > y->time) return 1;
    return (x->key > y->key) - (x->key < y->key);
}

/* Normalised softmax attention over one key partition: fills o[d] and returns
 * its natural-log normaliser L = ln sum exp(x_j) over the partition (unbiased
 * scores: the partition weight carries the penalty). */
static double partition_attend(const uint16_t *qr, const uint16_t *kbase, const uint16_t *vbase,
                               int d, double inv_sqrt_d, const int32_t *keys, int nkeys,
                               double *x, double *o) {
    double m = -INFINITY;
    for (int t = 0; t < nkeys; ++t) {
        x[t] = raw_score(qr, kbase + (size_t)keys[t] * d, d, inv_sqrt_d);
        if (x[t] > m) m = x[t];
    }
    double l = 0.0;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int t = 0; t < nkeys; ++t) {
        double w = exp(x[t] - m);
        l += w;
        const uint16_t *vr = vbase + (size_t)keys[t] * d;
        for (int c = 0; c < d; ++c) o[c] += w * bf16_to_f64(vr[c]);
    }
    for (int c = 0; c < d; ++c) o[c] /= l;
    return m + log(l);
}

static inline double logaddexp(double a, double b) {
    if (a == -INFINITY) return b;
    if (b == -INFINITY) return a;
    double hi = a > b ? a : b, lo = a > b ? b : a;
    return hi + log1p(exp(lo - hi));
}

/*
 * Same outputs as oracle_attend, reached by the partition algorithm: since
 * 0 <= p <= cap, exp(-p) = exp(-cap) + [exp(-p) - exp(-cap)] with both terms
 * non-negative ([FP §3]).  For a penalised (output-video) query the attended
 * keys split into
 *   N: non-guide keys, weight 1;
 *   G: all guide keys, weight exp(-cap);
 *   C_tau: guide keys with time tau where p(|t_q - tau|) < cap, weight
 *          exp(-p) - exp(-cap) = exp(-cap) * expm1(cap - p);
 * each partition is attended on its own (O_i, L_i) and the results merged by
 * adjusted_L_i = L_i + log w_i, L = logsumexp_i adjusted_L_i,
 * O = sum_i exp(adjusted_L_i - L) O_i ([FP §4]), with successive logaddexp.
 * Any other query is one partition of weight 1.
 */
void oracle_attend_partitions(int H, int S, int d, int B, const uint8_t *seg,
                              const float *times, const double *pen, const int32_t *sel,
                              int kk, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              int n, const int32_t *heads, const int32_t *rows,
                              double *out_o, double *out_lse) {
    int nkb = (S + B - 1) / B;
    uint8_t *nonvideo = (uint8_t *)malloc((size_t)nkb);
    oracle_block_classes(S, B, seg, nonvideo);
    int32_t *vid_index = (int32_t *)malloc(sizeof(int32_t) * (size_t)nkb);
    int nv = 0;
    for (int b = 0; b < nkb; ++b) vid_index[b] = nonvideo[b] ? -1 : nv++;
    double inv_sqrt_d = 1.0 / sqrt((double)d);

#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)S);
        uint8_t *use = (uint8_t *)malloc((size_t)nkb);
        int32_t *part = (int32_t *)malloc(sizeof(int32_t) * (size_t)S);
        int32_t *plain = (int32_t *)malloc(sizeof(int32_t) * (size_t)S);
        timed_key *guide = (timed_key *)malloc(sizeof(timed_key) * (size_t)S);
        double *op = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < n; ++t) {
            int h = heads[t], i = rows[t];
            attended_blocks(nkb, nonvideo, vid_index, sel, kk, H, nv, h, i / B, use);
            const uint16_t *qr = q + ((size_t)h * S + i) * d;
            const uint16_t *kb = k + (size_t)h * S * d;
            const uint16_t *vb = v + (size_t)h * S * d;
            double *o = out_o + (size_t)t * d;
            int biased_row = pen != NULL && seg[i] == SEG_OUTPUT && pen[0] != 0.0 && pen[3] != 0.0;
            int np = 0, ng = 0;
            for (int j = 0; j < S; ++j) {
                if (!use[j / B]) continue;
                if (biased_row && seg[j] == SEG_GUIDE) {
                    guide[ng].time = (double)times[j];
                    guide[ng].key = j;
                    ++ng;
                } else {
                    plain[np++] = j;
                }
            }
            double L = -INFINITY;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            /* merge one normalised partition result (op, adjusted_L) into (o, L) */
#define MERGE(adjL)                                                        \
    do {                                                                   \
        double newL = logaddexp(L, (adjL));                                \
        double a = exp(L - newL), bw = exp((adjL) - newL);                 \
        for (int c = 0; c < d; ++c) o[c] = a * o[c] + bw * op[c];          \
        L = newL;                                                          \
    } while (0)
            if (np > 0) {
                double Li = partition_attend(qr, kb, vb, d, inv_sqrt_d, plain, np, x, op);
                MERGE(Li); /* weight 1: log 1 = 0 */
            }
            if (ng > 0) {
                double cap = pen[3];
                for (int g = 0; g < ng; ++g) part[g] = guide[g].key;
                double Li = partition_attend(qr, kb, vb, d, inv_sqrt_d, part, ng, x, op);
                MERGE(Li - cap); /* weight exp(-cap) */
                qsort(guide, (size_t)ng, sizeof(timed_key), by_time);
                for (int g0 = 0; g0 < ng;) {
                    int g1 = g0;
                    while (g1 < ng && guide[g1].time == guide[g0].time) ++g1;
                    double dt = fabs((double)times[i] - guide[g0].time);
                    double p = oracle_penalty(dt, pen[0], pen[1], pen[2], cap);
                    if (p < cap) {
                        /* w = exp(-p) - exp(-cap) = exp(-cap) * expm1(cap - p) > 0 */
                        double logw = -cap + log(expm1(cap - p));
                        for (int g = g0; g < g1; ++g) part[g - g0] = guide[g].key;
                        double Lc = partition_attend(qr, kb, vb, d, inv_sqrt_d, part, g1 - g0, x, op);
                        MERGE(Lc + logw);
                    }
                    g0 = g1;
                }
            }
#undef MERGE
            out_lse[t] = L;
        }
        free(x);
        free(use);
        free(part);
        free(plain);
        free(guide);
        free(op);
    }
    free(vid_index);
    free(nonvideo);
}

/*
 * Merge of normalised partition results ([FP §4] "Why log-sum-exp is
 * necessary"): partition i has output O_i (already divided by its own
 * normaliser), natural-log normaliser L_i and a non-negative multiplier w_i
 * given as log_w[i] (-inf for w_i = 0; log_w NULL means every w_i = 1).
 *     adjusted_L_i = L_i + log w_i
 *     L            = logsumexp_i adjusted_L_i
 *     O            = sum_i exp(adjusted_L_i - L) O_i
 * A row whose adjusted normalisers are all -inf gets O = 0 and L = -inf.
 * o_parts [n_parts][rows][d], lse_parts [n_parts][rows]; o [rows][d], lse [rows].
 */
void oracle_merge(int n_parts, long rows, int d, const double *o_parts, const double *lse_parts,
                  const double *log_w, double *o, double *lse) {
    for (long r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int i = 0; i < n_parts; ++i) {
            double a = lse_parts[(long)i * rows + r] + (log_w ? log_w[i] : 0.0);
            if (a > m) m = a;
        }
        double *orow = o + r * d;
        for (int c = 0; c < d; ++c) orow[c] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double s = 0.0;
        for (int i = 0; i < n_parts; ++i) s += exp(lse_parts[(long)i * rows + r] + (log_w ? log_w[i] : 0.0) - m);
        double L = m + log(s);
        for (int i = 0; i < n_parts; ++i) {
            double w = exp(lse_parts[(long)i * rows + r] + (log_w ? log_w[i] : 0.0) - L);
            const double *oi = o_parts + ((long)i * rows + r) * d;
            for (int c = 0; c < d; ++c) orow[c] += w * oi[c];
        }
        lse[r] = L;
    }
}

/*
 * Pooled tail term ("H3 SLA Attention", inputs table, tail_correction):
 * instead of dropping the video key blocks top-k left out, one pooled term
 * stands in for all of them, scored from the pooled centroids the selection
 * already uses.  Reading (the page gives no formula): for video query block i
 * of head h, with D_i the video key blocks not in its routed list, n_j the
 * valid rows of block j and Qp, Kp, Vp the block means,
 *     Lt_i = log sum_{j in D_i} n_j exp(Qp_i . Kp_j / sqrt(d)),
 *     Ot_i = sum_{j in D_i} n_j exp(Qp_i . Kp_j / sqrt(d) - Lt_i) Vp_j,
 * i.e. each dropped block counts as n_j keys at its pooled score with its mean
 * value, without the temporal penalty (routing does not see it either).  Each
 * row of block i then merges (Ot_i, Lt_i) with its exact routed attention as a
 * partition of weight 1 (oracle_merge).  D_i empty: Lt_i = -inf.
 * sel [H][nV][k] absolute block ids; lt [H][nV]; ot [H][nV][d].
 */
void oracle_tail(int H, int S, int d, int B, const uint8_t *seg, const uint16_t *q, const uint16_t *k,
                 const uint16_t *v, const int32_t *sel, int kk, double *lt, double *ot) {
    int nkb = (S + B - 1) / B;
    uint8_t *nonvideo = (uint8_t *)calloc((size_t)nkb, 1);
    oracle_block_classes(S, B, seg, nonvideo);
    int fvb = 0;
    while (fvb < nkb && nonvideo[fvb]) ++fvb;
    int nv = nkb - fvb;
    double *qp = (double *)malloc(sizeof(double) * (size_t)H * nkb * d);
    double *kp = (double *)malloc(sizeof(double) * (size_t)H * nkb * d);
    double *vp = (double *)malloc(sizeof(double) * (size_t)H * nkb * d);
    oracle_pool(H, S, d, B, q, qp);
    oracle_pool(H, S, d, B, k, kp);
    oracle_pool(H, S, d, B, v, vp);
    double inv_sqrt_d = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic)
    for (long hi = 0; hi < (long)H * nv; ++hi) {
        int h = (int)(hi / nv), i = (int)(hi % nv);
        uint8_t *kept = (uint8_t *)calloc((size_t)nkb, 1);
        for (int t = 0; t < kk; ++t) kept[sel[(size_t)hi * kk + t]] = 1;
        const double *qrow = qp + ((size_t)h * nkb + fvb + i) * d;
        double m = -INFINITY;
        double *x = (double *)malloc(sizeof(double) * (size_t)nkb);
        for (int j = fvb; j < nkb; ++j) {
            x[j] = -INFINITY;
            if (kept[j]) continue;
            const double *krow = kp + ((size_t)h * nkb + j) * d;
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += qrow[c] * krow[c];
            int nj = (j + 1) * B <= S ? B : S - j * B;
            x[j] = s * inv_sqrt_d + log((double)nj);
            if (x[j] > m) m = x[j];
        }
        double *o = ot + (size_t)hi * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (m == -INFINITY) {
            lt[hi] = -INFINITY;
        } else {
            double sum = 0.0;
            for (int j = fvb; j < nkb; ++j)
                if (x[j] > -INFINITY) sum += exp(x[j] - m);
            double L = m + log(sum);
            for (int j = fvb; j < nkb; ++j) {
                if (x[j] == -INFINITY) continue;
                double w = exp(x[j] - L);
                const double *vrow = vp + ((size_t)h * nkb + j) * d;
                for (int c = 0; c < d; ++c) o[c] += w * vrow[c];
            }
            lt[hi] = L;
        }
        free(x);
        free(kept);
    }
    free(qp);
    free(kp);
    free(vp);
    free(nonvideo);
}
