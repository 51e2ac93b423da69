/*
 * dsa.h -- C ABI of libdsa.so: the DeepSeek Sparse Attention (DSA) forward hot path
 * on one NVIDIA B200 (sm_100a).
 *
 * The path (definitions from "DeepSeek-V3.2 tech report summary", section 1
 * "DeepSeek Sparse Attention (DSA)"; shapes from "DeepSeek-V3.2" (miles docs) §1):
 *   1. lightning indexer   I[t,s] = sum_{j<H_I} w[t,j] * ReLU(q_I[t,j] . k_I[s]),  s <= pos(t)
 *   2. top-k selection     the k_eff = min(topk, pos(t)+1) largest I[t,.] per query
 *   3. sparse MLA (MQA)    softmax attention of 128 heads over only the selected latent
 *                          rows; each 576-d latent row (512 KV-LoRA + 64 RoPE) is shared
 *                          by all heads, the value is its first 512 dims, scale 1/sqrt(192)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Ownership: every data pointer is caller-owned DEVICE memory (except the
 *    dsa_problem_t itself, which is host memory read during the call).  The library
 *    never allocates, frees or synchronises; work is enqueued on `stream` and runs
 *    asynchronously in stream order.
 *  - Layout: dense row-major, last dimension innermost, every base pointer 16-byte
 *    aligned.  bf16 is IEEE bfloat16; e4m3 is OCP FP8 E4M3 ("fn": no infinities).
 *  - Ragged batches: sequence b owns query rows [cu_q[b], cu_q[b+1]) and key rows
 *    [cu_k[b], cu_k[b+1]).  Its queries are its LAST len_q(b) tokens, so the query in
 *    global row t of sequence b sits at position
 *        pos(t) = len_k(b) - len_q(b) + (t - cu_q[b])
 *    and sees keys 0..pos(t) of its own sequence ("preceding tokens", the token
 *    itself included).  Key indices are positions within the sequence.
 *  - Paged key caches ("DeepSeek-V3.2" (miles docs) §5.3: the sparse-attention KV cache
 *    is paged, 64 tokens per page): with a block table, key position s of sequence b is
 *    the row block_table[b * max_pages + s / 64] * 64 + s % 64 of k_idx, k_scale and kv,
 *    and cu_k only gives the sequence lengths (len_k(b) = cu_k[b+1] - cu_k[b]).
 *  - Errors: argument, shape and alignment checks run on the host before anything
 *    is launched and return DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED without side
 *    effects.  A failed launch returns DSA_ERR_CUDA.  Device-side bounded waits that
 *    give up set a sticky device flag, reported by dsa_check_device_errors().
 *    Nothing traps, nothing aborts, and no C++ exception crosses this ABI.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_ABI_VERSION 2

/* Same object as cudaStream_t; NULL = the legacy default stream. */
typedef struct CUstream_st *dsa_stream_t;

typedef enum dsa_status {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative or inconsistent size */
    DSA_ERR_UNSUPPORTED = 2,   /* a shape this build does not implement (see below) */
    DSA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than dsa_forward_workspace_size */
    DSA_ERR_CUDA = 4,          /* a CUDA launch or query failed */
    DSA_ERR_DEVICE_TIMEOUT = 5, /* a device-side bounded wait gave up (from dsa_check_device_errors) */
    DSA_ERR_DEVICE_BOUNDS = 6   /* a debug-mode device check failed (from dsa_check_device_errors) */
} dsa_status_t;

typedef enum dsa_dtype {
    DSA_BF16 = 0,
    DSA_E4M3 = 1,        /* e4m3 codes, fp32 scale per token (q_scale [T], k_scale [S]) */
    DSA_E4M3_UE8M0 = 2   /* e4m3 codes, power-of-two scales per 128-element block as ue8m0
                            bytes (value 2^(e - 127)): q_scale uint8 [T, H_I] (one block per
                            head of a token), k_scale uint8 [S] (one block per key token) */
} dsa_dtype_t;

/*
 * One DSA problem.  Sizes this build implements: n_idx_heads = 64, idx_dim = 128,
 * n_heads = 128, d_qk = 576, d_v = 512 (the DeepSeek-V3.2 shapes), 1 <= topk <= 2048.
 * Other values return DSA_ERR_UNSUPPORTED.
 */
typedef struct dsa_problem {
    int32_t batch;          /* B >= 1 */
    const int32_t *cu_q;    /* device [B+1] query-row offsets, cu_q[0] = 0; NULL only if B == 1 */
    const int32_t *cu_k;    /* device [B+1] key-row offsets, cu_k[0] = 0;   NULL only if B == 1 */
    int32_t total_q;        /* T  = cu_q[B] */
    int32_t total_k;        /* S  = cu_k[B] */
    int32_t max_len_q;      /* >= every len_q(b) */
    int32_t max_len_k;      /* >= every len_k(b); every len_q(b) <= len_k(b) */
    int32_t n_idx_heads;    /* H_I = 64 */
    int32_t idx_dim;        /* d_I = 128 */
    int32_t n_heads;        /* H = 128 */
    int32_t d_qk;           /* 576 = 512 latent + 64 RoPE */
    int32_t d_v;            /* 512 */
    int32_t topk;           /* index_topk, e.g. 2048 */
    dsa_dtype_t idx_dtype;  /* indexer inputs: DSA_BF16, DSA_E4M3 or DSA_E4M3_UE8M0 */
    float sm_scale;         /* attention softmax scale, 1/sqrt(192) for DeepSeek-V3.2 */
    /* Paged key caches (NULL: packed rows, cu_k gives the row offsets).  With a table,
     * cu_q / cu_k are required, page_size must be 64, total_k is the number of physical
     * rows (pages x 64) of k_idx / kv, and every len_k(b) <= max_pages * 64; entries past
     * a sequence's last page are not read. */
    const int32_t *block_table;  /* device [B, max_pages] int32 physical page numbers */
    int32_t page_size;           /* 64 */
    int32_t max_pages;           /* row stride of block_table */
} dsa_problem_t;

/*
 * Lightning indexer ("DeepSeek-V3.2 tech report summary", §1 DSA, ① Lightning
 * Indexer; heads/dims from "Model techniques map -- DeepSeek-V3.2", indexer wq_b/wk):
 *     scores[r, s] = sum_j w[t,j] * ReLU( sum_d q_idx[t,j,d] * k_idx[kbase(b)+s, d] )
 * for query rows t = row_begin + r, 0 <= r < row_count, and 0 <= s <= pos(t).
 * Entries with s > pos(t) are left unspecified (callers must not read them).
 *   q_idx   : [T, H_I, d_I]  bf16, or e4m3 codes (DSA_E4M3, DSA_E4M3_UE8M0)
 *   q_scale : DSA_E4M3: fp32 [T] per query token; DSA_E4M3_UE8M0: uint8 [T, H_I] ue8m0
 *             block scales (one per head of a token); NULL for bf16
 *   k_idx   : [S, d_I]       bf16 or e4m3 codes
 *   k_scale : DSA_E4M3: fp32 [S]; DSA_E4M3_UE8M0: uint8 [S] ue8m0; NULL for bf16
 *   w       : [T, H_I] fp32
 *   scores  : [row_count, ld_scores] fp32, ld_scores >= max_len_k, ld_scores % 4 == 0
 * Accumulation is fp32 (tensor cores); the e4m3 scales are applied in fp32.
 * The e4m3 scales must be finite and > 0: the kernel multiplies them into the finished
 * head sum (a per-head block scale into that head's weight), which equals the definition
 * only because ReLU(a*x) = a*ReLU(x) for a > 0 (a non-positive fp32 scale gives
 * unspecified scores; they live in device memory, so the host cannot check them; ue8m0
 * scales are positive by construction, 0xFF is NaN).
 */
dsa_status_t dsa_indexer_scores(const dsa_problem_t *p, const void *q_idx, const void *q_scale,
                                const void *k_idx, const void *k_scale, const float *w,
                                float *scores, int64_t ld_scores, int32_t row_begin,
                                int32_t row_count, dsa_stream_t stream);

/*
 * Top-k token selection ("DeepSeek-V3.2 tech report summary", §1 DSA, ② fine-grained
 * token selection; "Model techniques map -- DeepSeek-V3.2", Indexer-selected sparse
 * attention: topk = min(index_topk, len), int32 indices):
 * for each query row t = row_begin + r, idx[r, :] receives the k_eff = min(topk, pos(t)+1)
 * positions s <= pos(t) with the largest scores[r, s], ranked by (score desc, s asc)
 * with -0.0 == +0.0; slots k_eff..topk-1 are -1.  The order of the selected indices
 * within a row is unspecified.  Exact: no approximation, deterministic.
 *   scores : [row_count, ld_scores] fp32 (NaN-free in columns 0..pos(t))
 *   idx    : [row_count, topk] int32
 */
dsa_status_t dsa_topk(const dsa_problem_t *p, const float *scores, int64_t ld_scores,
                      int32_t row_begin, int32_t row_count, int32_t *idx, dsa_stream_t stream);

/*
 * Indexer and top-k fused without score rows ("DeepSeek-V3.2 tech report summary", §1 DSA,
 * ① and ②): idx[r, :] for the rows t = row_begin + r receives exactly what
 * dsa_indexer_scores followed by dsa_topk would write (the same indices in the same slots),
 * computed chunk_q rows at a time (0 = all rows at once) as follows.
 *  1. The indexer scores every 32nd tile of 128 keys of each row (a sample).
 *  2. A per-row threshold is taken from that sample, chosen so that about 1.4 * topk keys
 *     reach it.
 *  3. The indexer runs again over all keys and keeps only the scores that reach the
 *     threshold, as an unordered list of candidates.
 *  4. The selection runs over the candidates.
 * A row whose threshold let fewer than topk keys through, or more than the list holds, is
 * redone from its full score row.  So the result never depends on the threshold, only the
 * time does.
 * This path applies to one sequence without cu arrays and max_len_k <= 458752. Ragged
 * batches and longer rows run the two-pass kernels on the workspace, with the same result.
 *   idx       : [row_count, topk] int32
 *   workspace : device, >= dsa_indexer_topk_streaming_workspace_size(p, chunk_q) bytes,
 *               256-byte aligned (it includes one chunk of score rows for the rows that
 *               are redone)
 * Other tensors, scales and errors as dsa_indexer_scores.
 */
size_t dsa_indexer_topk_streaming_workspace_size(const dsa_problem_t *p, int32_t chunk_q);
dsa_status_t dsa_indexer_topk_streaming(const dsa_problem_t *p, const void *q_idx, const void *q_scale,
                                        const void *k_idx, const void *k_scale, const float *w,
                                        int32_t row_begin, int32_t row_count, int32_t chunk_q,
                                        int32_t *idx, void *workspace, size_t workspace_bytes,
                                        dsa_stream_t stream);

/*
 * Sparse MLA forward in MQA mode ("DeepSeek-V3.2 tech report summary", §1 DSA,
 * MLA-based implementation: each latent KV entry is shared by all query heads;
 * latent = 512 KV-LoRA + 64 RoPE per "Model techniques map -- DeepSeek-V3.2",
 * Multi-head latent attention):
 *   z[t,h,i] = sm_scale * q[t,h,:] . kv[kbase(b)+idx[t,i], :]        (576 dims)
 *   out[t,h,:] = sum_i softmax_i(z) * kv[kbase(b)+idx[t,i], 0:512]
 *   lse[t,h]   = log(sum_i exp(z[t,h,i]))                              (natural log)
 * over the slots i whose index satisfies 0 <= idx <= pos(t); every other slot (-1,
 * future or out-of-range positions) is masked, so causality holds for any input.
 * A row with no valid slot gets out = 0 and lse = -inf.  A repeated index counts once
 * per occurrence.
 *   q   : [T, 128, 576] bf16     kv  : [S, 576] bf16     idx : [T, topk] int32
 *   out : [T, 128, 512] bf16 (round-to-nearest-even from fp32)   lse : [T, 128] fp32
 */
dsa_status_t dsa_sparse_mla_fwd(const dsa_problem_t *p, const void *q, const void *kv,
                                const int32_t *idx, void *out, float *lse, dsa_stream_t stream);

/*
 * Dense ("masked MHA") form of the same attention, for short sequences ("DeepSeek-V3.2
 * tech report summary", §1 DSA, short-sequence optimisation: in short prefill, DSA is
 * simulated by masked MHA, which is more efficient there):
 *   z[t,h,s]   = sm_scale * q[t,h,:] . kv[kbase(b)+s, :]   for the keys 0 <= s <= pos(t)
 *   out, lse   as in dsa_sparse_mla_fwd, over those keys
 * restricted to the keys listed in idx[t, :] when idx is not NULL (each listed visible key
 * counts once; -1, future and out-of-range entries are ignored).  With idx = NULL every
 * causal key attends.  For an index row without repeated keys (every dsa_topk row) the
 * result equals dsa_sparse_mla_fwd on that row.  The keys are read as contiguous tiles, so
 * the work grows with pos(t) + 1 rather than with topk.
 *   idx : [T, topk] int32 or NULL; with idx, max_len_k <= 16384 (else DSA_ERR_UNSUPPORTED)
 * Packed caches only (a block table returns DSA_ERR_UNSUPPORTED).
 * dsa_forward uses this form (with idx = NULL, skipping the indexer and the top-k) whenever
 * max_len_k <= topk: every visible key is then selected, and the output is bit-identical
 * to the gathered form.  Above that, up to max_len_k <= 3584 (the short-sequence threshold
 * of this build), dsa_forward runs the indexer and the top-k and then this form restricted
 * to the selected keys; longer problems use dsa_sparse_mla_fwd.
 */
dsa_status_t dsa_dense_mla_fwd(const dsa_problem_t *p, const void *q, const void *kv,
                               const int32_t *idx, void *out, float *lse, dsa_stream_t stream);

/*
 * Bytes of workspace dsa_forward needs for this problem when it processes the
 * queries in chunks of `chunk_q` rows (0 = one chunk of max(T, 1) rows).
 */
size_t dsa_forward_workspace_size(const dsa_problem_t *p, int32_t chunk_q);

/*
 * The whole path: for each chunk of chunk_q query rows, indexer scores into the
 * workspace, top-k into idx_out (or the workspace when idx_out is NULL), then the
 * attention over the selected keys for all rows (gathered form, or the dense form for
 * short sequences: see dsa_dense_mla_fwd).  Same tensors and rules as the three calls above; the
 * full T x S score matrix is never materialised (at most chunk_q x max_len_k).
 *   idx_out   : [T, topk] int32 or NULL
 *   workspace : device, >= dsa_forward_workspace_size(p, chunk_q) bytes, 256-byte aligned
 */
dsa_status_t dsa_forward(const dsa_problem_t *p, const void *q_idx, const void *q_scale,
                         const void *k_idx, const void *k_scale, const float *w, const void *q,
                         const void *kv, int32_t chunk_q, int32_t *idx_out, void *out, float *lse,
                         void *workspace, size_t workspace_bytes, dsa_stream_t stream);

/*
 * dsa_forward without a workspace argument, for callers that cannot allocate device
 * memory where they run the path (host callbacks, runtimes that own all device memory,
 * serving loops that must not call cudaMalloc).  The pages have no counterpart: this is
 * a deployment convenience, not part of the method.
 * The per-chunk score scratch lives in a fixed device array of
 * dsa_forward_noalloc_scratch_bytes() bytes (32 MiB) inside the library, held by every GPU
 * that loads the library until the process exits.  Query rows are processed in chunks
 * of as many rows as fit; a problem whose longest score row alone (max_len_k rounded up
 * to 4 fp32) does not fit returns DSA_ERR_WORKSPACE before anything is launched.
 * idx_out is required here (it is the caller's output, not scratch).
 * Rows per chunk = 32 MiB / (4 * ceil4(max_len_k)) (8192 rows at 1K keys, 64 rows at
 * 128K keys): at long contexts the chunks get small and the indexer launches run with
 * few CTAs, so throughput falls far below dsa_forward with a large workspace.
 * The first call on a device looks up the array's device address (make it outside any
 * stream capture).  All calls share the array: calls that overlap on the GPU race on it.
 * Nothing is allocated or freed by this call.
 */
dsa_status_t dsa_forward_noalloc(const dsa_problem_t *p, const void *q_idx, const void *q_scale,
                                 const void *k_idx, const void *k_scale, const float *w, const void *q,
                                 const void *kv, int32_t *idx_out, void *out, float *lse, dsa_stream_t stream);

/* Size in bytes of the fixed scratch array used by dsa_forward_noalloc. */
size_t dsa_forward_noalloc_scratch_bytes(void);

/*
 * Synchronises `stream`, then reads and clears the device-side error flag of the
 * current device (set by a kernel whose bounded wait gave up, or by a debug-mode check).
 * Returns DSA_OK, DSA_ERR_DEVICE_TIMEOUT, DSA_ERR_DEVICE_BOUNDS, or DSA_ERR_CUDA if the
 * synchronisation itself failed.
 */
dsa_status_t dsa_check_device_errors(dsa_stream_t stream);

/*
 * Key-cache write: the rows the path reads, made from the projections of n new tokens
 * ("DeepSeek-V3.2-Exp" README, 2025-11-17 note: the indexer's RoPE input is
 * non-interleaved, MLA's RoPE input interleaved; "Model techniques map -- DeepSeek-V3.2":
 * the indexer key passes through k_norm, the latent through kv_a_layernorm, RoPE acts on
 * the 64 RoPE dims):
 *   k_idx_cache[rows[t]] = RoPE_ni(LayerNorm(k_idx_raw[t]) * k_norm_w + k_norm_b)
 *                          (LayerNorm over the 128 dims; RoPE on dims 0..63, pairs (i, i + 32))
 *   kv_cache[rows[t], 0:512]   = kv_raw[t, 0:512] / sqrt(mean(kv_raw[t, 0:512]^2) + eps) * kv_norm_w
 *   kv_cache[rows[t], 512:576] = RoPE_il(kv_raw[t, 512:576])   (pairs (512 + 2i, 513 + 2i))
 * where RoPE turns pair i (i < 32) by the angle positions[t] * inv_freq[i] (evaluated in
 * fp64).  Readings where the pages are silent: k_norm is a LayerNorm with weight and bias,
 * the indexer's RoPE dims are its first 64, the frequencies are the caller's (any scaled
 * schedule, e.g. YaRN, is computed once when the model is set up).  Arithmetic in fp32,
 * outputs rounded to bf16.
 *   k_idx_raw : [n, 128] bf16      kv_raw : [n, 576] bf16      positions, rows : [n] int32
 *   k_norm_w, k_norm_b : [128] fp32   kv_norm_w : [512] fp32   inv_freq : [32] fp32
 *   k_idx_cache : bf16 [.., 128]   kv_cache : bf16 [.., 576]   (rows[t]: the destination
 *   row, packed or through a block table; distinct rows, no two tokens write the same row)
 */
dsa_status_t dsa_cache_write(int32_t n_tokens, const void *k_idx_raw, const void *kv_raw,
                             const int32_t *positions, const int32_t *rows, const float *k_norm_w,
                             const float *k_norm_b, const float *kv_norm_w, const float *inv_freq,
                             float eps, void *k_idx_cache, void *kv_cache, dsa_stream_t stream);

/*
 * Self-test of the device-side failure path (no counterpart on the pages): launches one
 * CTA whose bounded wait on a barrier that nothing signals gives up after `limit_us`
 * microseconds (1 .. 10000), as a stalled pipeline wait would.  No copy or tensor-core
 * operation is in flight.  The next dsa_check_device_errors() then returns
 * DSA_ERR_DEVICE_TIMEOUT and clears the flag; the device stays usable.
 */
dsa_status_t dsa_selftest_bounded_wait(uint32_t limit_us, dsa_stream_t stream);

/*
 * Debug checks (process-wide, for the launches made after the call; off by default): every
 * kernel checks the sequence facts of each query row against the problem's sizes (cu_q /
 * cu_k inside total_k and max_len_k, block-table pages inside total_k) and, in the FP8
 * indexer with fp32 scales, that the scales are finite and > 0.  A failing row is counted
 * in the device flag (DSA_ERR_DEVICE_BOUNDS from dsa_check_device_errors) and treated as
 * having no keys, so no access leaves the arrays.  Costs a few loads per row.
 */
void dsa_set_debug_checks(int32_t enable);

/* Static English description of a status code (never NULL). */
const char *dsa_status_string(dsa_status_t s);

/* DSA_ABI_VERSION of the loaded library. */
int32_t dsa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
