/*
 * dsa_oracle.c -- plain, slow, fp64 CPU oracle for the DeepSeek Sparse Attention
 * (DSA) forward path: lightning indexer -> causal top-k -> sparse MLA (MQA mode).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code, header,
 * table or helper with the CUDA path, and it never sees a value produced there
 * except the fp32 score array handed to the top-k check (the same array the GPU
 * top-k receives).
 *
 * Sources (web pages on the subject, cited by page title and section):
 *  [R]  "DeepSeek-V3.2 技术报告摘要" (summary of the DeepSeek-V3.2 tech report),
 *       §1 "关键设计: DeepSeek Sparse Attention (DSA)":
 *         ① Lightning Indexer: I_{t,s} = sum_{j=1..H_I} w^I_{t,j} * ReLU(q^I_{t,j} . k^I_s)
 *            over the preceding tokens s of query t; FP8-capable.
 *         ② Fine-grained token selection: keep the top-k index scores per query and
 *            run full attention only over those k tokens.
 *         "基于 MLA 的实现": DSA runs in MLA's MQA mode; every latent KV entry is
 *            shared by all query heads.
 *  [M]  "Model techniques map -- DeepSeek-V3.2", feature "Indexer-selected sparse
 *       attention": topk = min(index_topk, #scores), indices returned as int32.
 *       Feature "Multi-head latent attention": latent = 512 (KV-LoRA) + 64 (RoPE).
 *  [D]  "DeepSeek-V3.2" (miles docs), §1 Model Introduction: 128 heads of
 *       128 NoPE + 64 RoPE dims, indexer 64 heads x 128, index_topk = 2048.
 *
 * Readings taken where the pages are silent (each is restated in the design notes):
 *  - "preceding tokens" includes the query token itself: keys s <= pos(t).
 *  - Ragged batches: the queries of sequence b are its LAST len_q(b) tokens, so
 *    pos(t) = len_k(b) - len_q(b) + (t - cu_q[b]).
 *  - Top-k: k_eff = min(k, pos(t)+1); order by (score desc, index asc); -0.0 == +0.0;
 *    unused slots are -1.
 *  - Sparse attention: z_i = scale * q . kv[idx_i] over all d_qk dims, softmax over
 *    the valid listed indices (0 <= idx <= pos(t)), value = first d_v dims of the
 *    latent, lse = natural-log log-sum-exp of z.  A listed index counts once per
 *    occurrence.  A row with no valid index gives o = 0 and lse = -inf.
 *  - FP8 indexer: q = e4m3(q8) * q_scale[t], k = e4m3(k8) * k_scale[s] (per token), or
 *    with block scales (128-element blocks as in the checkpoint format of "DeepSeek-V3.2"
 *    (miles docs) §1; a block of q_I is one head of one token, a block of k_I one token):
 *    q = e4m3(q8) * q_scale[t,j], k = e4m3(k8) * k_scale[s], the scales given as ue8m0
 *    bytes (8-bit exponents, value 2^(e - 127)).
 *  - Paged caches ("DeepSeek-V3.2" (miles docs) §5.3: the KV cache is paged, 64 tokens per
 *    page): when a block table is set, key position s of sequence b is the row
 *    table[b * max_pages + s / page_size] * page_size + s % page_size of the key arrays
 *    (k, k8 and k_scale, kv); otherwise it is the row cu_k[b] + s.
 *
 * Every function here runs the definition directly, one output element at a time,
 * with OpenMP over query rows.  No blocking, fusion or reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* --- ragged-batch bookkeeping (reading stated above) ----------------------- */

/* Block table of the paged layout (NULL: packed rows), set by dsa_oracle_set_pages. */
static const int32_t *g_table = NULL;
static int g_max_pages = 0, g_page = 0;

void dsa_oracle_set_pages(const int32_t *table, int max_pages, int page_size) {
    g_table = table;
    g_max_pages = max_pages;
    g_page = page_size;
}

/* For global query row t, find its sequence b, key-row base and position. */
static int row_info(int64_t t, int batch, const int32_t *cu_q, const int32_t *cu_k,
                    int64_t *kbase, int64_t *len_k, int64_t *pos, int64_t *seq) {
    for (int b = 0; b < batch; ++b) {
        if (t >= cu_q[b] && t < cu_q[b + 1]) {
            int64_t lq = (int64_t)cu_q[b + 1] - cu_q[b];
            int64_t lk = (int64_t)cu_k[b + 1] - cu_k[b];
            *kbase = cu_k[b];
            *len_k = lk;
            *pos = lk - lq + (t - cu_q[b]);
            *seq = b;
            return 1;
        }
    }
    return 0;
}

/* Row of the key arrays that holds key position s of sequence b. */
static int64_t key_row(int64_t b, int64_t kbase, int64_t s) {
    if (g_table == NULL) return kbase + s;
    return (int64_t)g_table[b * g_max_pages + s / g_page] * g_page + s % g_page;
}

int dsa_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* --- ① lightning indexer ---------------------------------------------------- */

/*
 * Index scores for the query rows listed in `rows` [R] (section ① of [R]):
 *     I[t,s] = sum_{j<H} w[t,j] * max(0, sum_{d<D} q[t,j,d] * k[kbase+s, d])
 * for 0 <= s <= pos(t); every other entry of the output row is -INFINITY.
 *   q_rows : [n_rows, H, D] -- the query vectors of the listed rows, in order
 *   w_rows : [n_rows, H]
 *   k      : [total_k, D]  -- all key rows of all sequences
 *   out    : [n_rows, ld]  (ld >= len_k of every listed row's sequence)
 */
void dsa_oracle_indexer(int n_rows, const int64_t *rows, const double *q_rows,
                        const double *w_rows, const double *k, int H, int D,
                        int batch, const int32_t *cu_q, const int32_t *cu_k,
                        double *out, int64_t ld) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        int64_t kbase = 0, len_k = 0, pos = -1, seq = 0;
        double *orow = out + (int64_t)r * ld;
        for (int64_t s = 0; s < ld; ++s) orow[s] = -INFINITY;
        if (!row_info(rows[r], batch, cu_q, cu_k, &kbase, &len_k, &pos, &seq)) continue;
        const double *qr = q_rows + (int64_t)r * H * D;
        const double *wr = w_rows + (int64_t)r * H;
        for (int64_t s = 0; s <= pos && s < len_k; ++s) {
            const double *ks = k + key_row(seq, kbase, s) * D;
            double score = 0.0;
            for (int j = 0; j < H; ++j) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += qr[(int64_t)j * D + d] * ks[d];
                double relu = dot > 0.0 ? dot : 0.0;
                score += wr[j] * relu;
            }
            orow[s] = score;
        }
    }
}

/*
 * e4m3 (OCP FP8, "fn" variant: 1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits, no infinities, S.1111.111 = NaN) decoded from its bit fields.
 */
double dsa_oracle_e4m3_value(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, 1 - 7);          /* subnormal: 0.m x 2^-6 */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);    /* normal: 1.m x 2^(e-7) */
    return sign ? -v : v;
}

/* ue8m0 (an 8-bit unsigned exponent, no sign or mantissa): 2^(e - 127); 0xFF is NaN. */
double dsa_oracle_ue8m0_value(uint8_t code) {
    if (code == 0xFF) return NAN;
    return ldexp(1.0, (int)code - 127);
}

/*
 * FP8 indexer (section ① of [R], "supports FP8"): the same sum as
 * dsa_oracle_indexer with q[t,j,d] = e4m3(q8) * q_scale and
 * k[s,d] = e4m3(k8) * k_scale[s], decoded here in fp64.  The q scale is per token
 * (qs_per_head = 0: qs_rows [n_rows]) or per (token, head) block (qs_per_head = 1:
 * qs_rows [n_rows, H]).
 *   q8_rows : [n_rows, H, D] codes of the listed rows
 *   k8      : [total_k, D] codes;  k_scale : [total_k]
 */
void dsa_oracle_indexer_fp8(int n_rows, const int64_t *rows, const uint8_t *q8_rows,
                            const double *qs_rows, int qs_per_head, const double *w_rows,
                            const uint8_t *k8, const double *k_scale, int H, int D,
                            int batch, const int32_t *cu_q, const int32_t *cu_k,
                            double *out, int64_t ld) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        int64_t kbase = 0, len_k = 0, pos = -1, seq = 0;
        double *orow = out + (int64_t)r * ld;
        for (int64_t s = 0; s < ld; ++s) orow[s] = -INFINITY;
        if (!row_info(rows[r], batch, cu_q, cu_k, &kbase, &len_k, &pos, &seq)) continue;
        const uint8_t *qr = q8_rows + (int64_t)r * H * D;
        const double *wr = w_rows + (int64_t)r * H;
        for (int64_t s = 0; s <= pos && s < len_k; ++s) {
            const uint8_t *ks = k8 + key_row(seq, kbase, s) * D;
            double kscale = k_scale[key_row(seq, kbase, s)];
            double score = 0.0;
            for (int j = 0; j < H; ++j) {
                double dot = 0.0;
                double qs = qs_per_head ? qs_rows[(int64_t)r * H + j] : qs_rows[r];
                for (int d = 0; d < D; ++d) {
                    double qv = dsa_oracle_e4m3_value(qr[(int64_t)j * D + d]) * qs;
                    double kv = dsa_oracle_e4m3_value(ks[d]) * kscale;
                    dot += qv * kv;
                }
                double relu = dot > 0.0 ? dot : 0.0;
                score += wr[j] * relu;
            }
            orow[s] = score;
        }
    }
}

/* --- ② top-k token selection ------------------------------------------------ */

typedef struct {
    double v;
    int64_t i;
} scored_t;

/* (score desc, index asc); -0.0 and +0.0 compare equal as values. */
static int cmp_scored(const void *pa, const void *pb) {
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    if (a->i < b->i) return -1;
    if (a->i > b->i) return 1;
    return 0;
}

/*
 * Per listed query row: sort the causal candidates 0..pos(t) of the score row by
 * (score desc, index asc) and keep the first k_eff = min(k, pos(t)+1) indices;
 * slots k_eff..k-1 are -1.  Output rows are in sorted (best-first) order.
 *   scores : [n_rows, ld] (only entries 0..pos(t) are read)
 *   idx    : [n_rows, k]
 * (section ② of [R]; "topk = min(index_topk, len)" of [M]).
 */
void dsa_oracle_topk(int n_rows, const int64_t *rows, const double *scores, int64_t ld,
                     int k, int batch, const int32_t *cu_q, const int32_t *cu_k,
                     int32_t *idx) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        int64_t kbase = 0, len_k = 0, pos = -1, seq = 0;
        int32_t *irow = idx + (int64_t)r * k;
        for (int j = 0; j < k; ++j) irow[j] = -1;
        if (!row_info(rows[r], batch, cu_q, cu_k, &kbase, &len_k, &pos, &seq)) continue;
        int64_t n = pos + 1;
        if (n > len_k) n = len_k;
        if (n <= 0) continue;
        scored_t *buf = (scored_t *)malloc(sizeof(scored_t) * (size_t)n);
        const double *srow = scores + (int64_t)r * ld;
        for (int64_t s = 0; s < n; ++s) {
            buf[s].v = srow[s];
            buf[s].i = s;
        }
        qsort(buf, (size_t)n, sizeof(scored_t), cmp_scored);
        int64_t keff = n < k ? n : k;
        for (int64_t j = 0; j < keff; ++j) irow[j] = (int32_t)buf[j].i;
        free(buf);
    }
}

/* --- sparse MLA in MQA mode ------------------------------------------------- */

/*
 * For each listed row t and head h, over the valid listed indices i
 * (0 <= idx[t,i] <= pos(t), idx < len_k):
 *     z_i   = scale * sum_{d<Dqk} q[t,h,d] * kv[kbase+idx_i, d]
 *     p_i   = exp(z_i - m) / sum_i exp(z_i - m),  m = max_i z_i
 *     o[t,h,e] = sum_i p_i * kv[kbase+idx_i, e]   for e < Dv
 *     lse[t,h] = m + log(sum_i exp(z_i - m))
 * The latent row is shared by all heads (MQA mode, "基于 MLA 的实现" of [R]);
 * the value is its first Dv dims.
 *   q_rows : [n_rows, H, Dqk];  idx_rows : [n_rows, k];  kv : [total_k, Dqk]
 *   o : [n_rows, H, Dv];  lse : [n_rows, H]
 */
void dsa_oracle_sparse_mla(int n_rows, const int64_t *rows, const double *q_rows,
                           const int32_t *idx_rows, int k, const double *kv, int H,
                           int Dqk, int Dv, double scale, int batch,
                           const int32_t *cu_q, const int32_t *cu_k, double *o,
                           double *lse) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        int64_t kbase = 0, len_k = 0, pos = -1, seq = 0;
        double *orow = o + (int64_t)r * H * Dv;
        double *lrow = lse + (int64_t)r * H;
        memset(orow, 0, sizeof(double) * (size_t)H * Dv);
        for (int h = 0; h < H; ++h) lrow[h] = -INFINITY;
        if (!row_info(rows[r], batch, cu_q, cu_k, &kbase, &len_k, &pos, &seq)) continue;
        const int32_t *irow = idx_rows + (int64_t)r * k;
        double *z = (double *)malloc(sizeof(double) * (size_t)k);
        for (int h = 0; h < H; ++h) {
            const double *qh = q_rows + ((int64_t)r * H + h) * Dqk;
            double m = -INFINITY;
            for (int i = 0; i < k; ++i) {
                int64_t s = irow[i];
                if (s < 0 || s > pos || s >= len_k) {
                    z[i] = -INFINITY;
                    continue;
                }
                const double *row = kv + key_row(seq, kbase, s) * Dqk;
                double dot = 0.0;
                for (int d = 0; d < Dqk; ++d) dot += qh[d] * row[d];
                z[i] = scale * dot;
                if (z[i] > m) m = z[i];
            }
            if (m == -INFINITY) continue; /* no valid key: o = 0, lse = -inf */
            double denom = 0.0;
            for (int i = 0; i < k; ++i)
                if (z[i] != -INFINITY) denom += exp(z[i] - m);
            double *oh = orow + (int64_t)h * Dv;
            for (int i = 0; i < k; ++i) {
                if (z[i] == -INFINITY) continue;
                double p = exp(z[i] - m) / denom;
                const double *row = kv + key_row(seq, kbase, irow[i]) * Dqk;
                for (int e = 0; e < Dv; ++e) oh[e] += p * row[e];
            }
            lrow[h] = m + log(denom);
        }
        free(z);
    }
}

/* --- upstream producer: the key-cache write --------------------------------- */

/*
 * The rows the path reads, made from the projections of new tokens ("DeepSeek-V3.2-Exp"
 * README, 2025-11-17 note: the indexer's RoPE takes its input in the non-interleaved
 * layout, MLA's RoPE in the interleaved one; "Model techniques map -- DeepSeek-V3.2": the
 * indexer's key passes through k_norm, the latent through kv_a_layernorm, RoPE acts on
 * the 64 RoPE dims only).  Readings: k_norm is a LayerNorm (mean and variance over the
 * 128 dims, affine weight and bias), kv_a_layernorm an RMSNorm over the 512 KV-LoRA dims
 * (weight), eps given; the indexer's RoPE dims are its first 64 (pairs (i, i + 32),
 * non-interleaved), the latent's are dims 512..575 (pairs (512 + 2i, 513 + 2i),
 * interleaved); both rotate pair i by the angle pos * inv_freq[i], i < 32.
 *   k_raw [n, 128], kv_raw [n, 576], pos [n], ln_w/ln_b [128], rms_w [512], inv_freq [32]
 *   out_k [n, 128], out_kv [n, 576]
 */
void dsa_oracle_cache_write(int n, const double *k_raw, const double *kv_raw, const int32_t *pos,
                            const double *ln_w, const double *ln_b, const double *rms_w,
                            const double *inv_freq, double eps, double *out_k, double *out_kv) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < n; ++t) {
        const double *x = k_raw + (int64_t)t * 128;
        double *y = out_k + (int64_t)t * 128;
        double mean = 0.0, var = 0.0;
        for (int d = 0; d < 128; ++d) mean += x[d];
        mean /= 128.0;
        for (int d = 0; d < 128; ++d) var += (x[d] - mean) * (x[d] - mean);
        var /= 128.0;
        const double inv = 1.0 / sqrt(var + eps);
        for (int d = 0; d < 128; ++d) y[d] = (x[d] - mean) * inv * ln_w[d] + ln_b[d];
        for (int i = 0; i < 32; ++i) {          /* non-interleaved: (i, i + 32) */
            const double a = (double)pos[t] * inv_freq[i];
            const double c = cos(a), s = sin(a);
            const double u = y[i], v = y[i + 32];
            y[i] = u * c - v * s;
            y[i + 32] = v * c + u * s;
        }
        const double *z = kv_raw + (int64_t)t * 576;
        double *o = out_kv + (int64_t)t * 576;
        double ms = 0.0;
        for (int d = 0; d < 512; ++d) ms += z[d] * z[d];
        const double rinv = 1.0 / sqrt(ms / 512.0 + eps);
        for (int d = 0; d < 512; ++d) o[d] = z[d] * rinv * rms_w[d];
        for (int i = 0; i < 32; ++i) {          /* interleaved: (512 + 2i, 513 + 2i) */
            const double a = (double)pos[t] * inv_freq[i];
            const double c = cos(a), s = sin(a);
            const double u = z[512 + 2 * i], v = z[513 + 2 * i];
            o[512 + 2 * i] = u * c - v * s;
            o[513 + 2 * i] = v * c + u * s;
        }
    }
}
