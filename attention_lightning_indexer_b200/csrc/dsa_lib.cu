// dsa_lib.cu -- the C ABI of libdsa.so (declared in include/dsa.h): host-side argument
// checks, launch configuration and the chunked forward orchestration.  All arithmetic
// of the path runs in the kernels included below.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "../../include/dsa.h"
#include "cache_write.cuh"
#include "dsa_common.cuh"
#include "indexer_tc.cuh"
#include "select_stream.cuh"
#include "sparse_mla_pair.cuh"
#include "topk.cuh"

namespace {

using dsa::Problem;

int g_debug_checks = 0;   // dsa_set_debug_checks

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

dsa_status_t check_problem(const dsa_problem_t *p) {
    if (p == nullptr) return DSA_ERR_INVALID_ARG;
    if (p->batch < 1 || p->total_q < 0 || p->total_k < 0 || p->max_len_q < 0 || p->max_len_k < 0)
        return DSA_ERR_INVALID_ARG;
    if ((p->cu_q == nullptr) != (p->cu_k == nullptr)) return DSA_ERR_INVALID_ARG;
    if (p->cu_q == nullptr) {
        if (p->batch != 1 || p->total_q > p->total_k) return DSA_ERR_INVALID_ARG;
        if (p->max_len_k < p->total_k || p->max_len_q < p->total_q) return DSA_ERR_INVALID_ARG;
    }
    if (p->max_len_q > p->max_len_k && p->cu_q == nullptr) return DSA_ERR_INVALID_ARG;
    if (p->topk < 1) return DSA_ERR_INVALID_ARG;
    if (p->n_idx_heads != 64 || p->idx_dim != 128 || p->n_heads != 128 || p->d_qk != 576 || p->d_v != 512)
        return DSA_ERR_UNSUPPORTED;
    if (p->topk > 2048) return DSA_ERR_UNSUPPORTED;
    if (p->idx_dtype != DSA_BF16 && p->idx_dtype != DSA_E4M3 && p->idx_dtype != DSA_E4M3_UE8M0)
        return DSA_ERR_UNSUPPORTED;
    if (!(p->sm_scale > 0.0f)) return DSA_ERR_INVALID_ARG;
    if (p->block_table != nullptr) {
        if (p->cu_q == nullptr || p->max_pages < 1) return DSA_ERR_INVALID_ARG;
        if (p->page_size != 64) return DSA_ERR_UNSUPPORTED;
        if ((int64_t)p->max_len_k > (int64_t)p->max_pages * 64 || (p->total_k & 63) != 0) return DSA_ERR_INVALID_ARG;
    }
    return DSA_OK;
}

Problem to_dev(const dsa_problem_t *p) {
    Problem P;
    P.batch = p->batch;
    P.cu_q = p->cu_q;
    P.cu_k = p->cu_k;
    P.total_q = p->total_q;
    P.total_k = p->total_k;
    P.max_len_q = p->max_len_q;
    P.max_len_k = p->max_len_k;
    P.topk = p->topk;
    P.sm_scale = p->sm_scale;
    P.block_table = p->block_table;
    P.max_pages = p->block_table != nullptr ? p->max_pages : 0;
    P.ue8m0 = p->idx_dtype == DSA_E4M3_UE8M0 ? 1 : 0;
    P.debug = g_debug_checks;
    return P;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda needed).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D row-major tensor map (`cols` x `rows`, 1- or 2-byte elements) whose box is
// `box_rows` rows x 128 bytes, loaded with the 128-byte swizzle.
bool make_tmap_rows(CUtensorMap *m, const void *base, bool fp8, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    const uint32_t eb = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * eb};
    cuuint32_t box[2] = {128 / eb, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline dsa_status_t launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Opt-in to large dynamic shared memory for each kernel.  The attribute is a setting of
// the current device, so it is applied once per device (the first call made with that
// device current).
constexpr int MAX_DEVICES = 64;

// Longest key range the streaming selection takes (the sample of a row must fit the
// threshold kernel's shared memory); longer problems use the two-pass kernels.
constexpr int STREAM_MAX_KEYS = dsa::topk::STREAM_MAX_SAMPLES / 128 * (dsa::indexer::SAMPLE_STRIDE * 128);

size_t select_smem(int max_len_k) {
    return (size_t)dsa::topk::StreamCfg::SMEM + 8u * (size_t)((max_len_k + 31) / 32);
}

template <int QG, bool FP8, int MODE>
cudaError_t indexer_attr() {
    return cudaFuncSetAttribute(dsa::indexer::indexer_tc_kernel<QG, FP8, MODE>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, dsa::indexer::TcCfg<QG, FP8>::SMEM);
}

dsa_status_t set_smem_attrs() {
    static bool done[MAX_DEVICES] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return DSA_ERR_CUDA;
    if (done[dev]) return DSA_OK;
    cudaError_t e = cudaSuccess;
    e = cudaFuncSetAttribute(dsa::topk::topk_rows_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             dsa::topk::Cfg<256>::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(dsa::topk::topk_rows_kernel<1024>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dsa::topk::Cfg<1024>::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(dsa::mla::sparse_mla_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dsa::mla::PairCfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(dsa::mla::sparse_mla_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dsa::mla::PairCfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(dsa::mla::sparse_mla_pair_kernel<false, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, dsa::mla::PairCfg::SMEM);
    if (e == cudaSuccess) e = indexer_attr<8, false, dsa::indexer::SCORES>();
    if (e == cudaSuccess) e = indexer_attr<8, true, dsa::indexer::SCORES>();
    if (e == cudaSuccess) e = indexer_attr<8, false, dsa::indexer::SAMPLE>();
    if (e == cudaSuccess) e = indexer_attr<8, true, dsa::indexer::SAMPLE>();
    if (e == cudaSuccess) e = indexer_attr<8, false, dsa::indexer::FILTER>();
    if (e == cudaSuccess) e = indexer_attr<8, true, dsa::indexer::FILTER>();
    if (e == cudaSuccess) e = indexer_attr<1, false, dsa::indexer::SCORES>();
    if (e == cudaSuccess) e = indexer_attr<1, true, dsa::indexer::SCORES>();
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(dsa::topk::sample_threshold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dsa::topk::StreamCfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(dsa::topk::select_candidates_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)select_smem(STREAM_MAX_KEYS));
    if (e != cudaSuccess) return DSA_ERR_CUDA;
    done[dev] = true;
    return DSA_OK;
}

template <int QG, bool FP8, int MODE = dsa::indexer::SCORES>
dsa_status_t indexer_tc_launch(const dsa_problem_t *p, const void *q_idx, const void *q_scale, const void *k_idx,
                               const void *k_scale, const float *w, float *scores, int64_t ld, int row_begin,
                               int row_count, cudaStream_t stream,
                               dsa::indexer::StreamArgs sa = dsa::indexer::StreamArgs{}) {
    using C = dsa::indexer::TcCfg<QG, FP8>;
    CUtensorMap tq, tk;
    if (!make_tmap_rows(&tq, q_idx, FP8, 128, (uint64_t)p->total_q * 64, 64)) return DSA_ERR_CUDA;
    // key tiles: 128-row boxes, or 64-row boxes (one page) through the block table
    if (!make_tmap_rows(&tk, k_idx, FP8, 128, (uint64_t)p->total_k, p->block_table ? 64 : 128)) return DSA_ERR_CUDA;
    Problem P = to_dev(p);
    int nsplit = 1;
    unsigned grid;
    if (QG > 1) {
        grid = (unsigned)((row_count + QG - 1) / QG);
    } else {
        nsplit = (p->max_len_k + C::SPLIT_KEYS - 1) / C::SPLIT_KEYS;
        grid = (unsigned)row_count * (unsigned)nsplit;
    }
    dsa::indexer::indexer_tc_kernel<QG, FP8, MODE><<<grid, C::THREADS, C::SMEM, stream>>>(
        tq, tk, P, q_scale, k_scale, w, scores, ld, row_begin, row_count, nsplit, sa);
    return launch_status();
}

dsa_status_t indexer_launch(const dsa_problem_t *p, const void *q_idx, const void *q_scale, const void *k_idx,
                            const void *k_scale, const float *w, float *scores, int64_t ld, int row_begin,
                            int row_count, cudaStream_t stream) {
    if (row_count == 0 || p->max_len_k == 0 || p->total_k == 0) return DSA_OK;
    const bool fp8 = p->idx_dtype != DSA_BF16;
    // One sequence: groups of 8 consecutive queries share each key tile.  Ragged batches
    // (decode): one query per CTA, its key range split across CTAs.
    if (p->cu_q == nullptr)
        return fp8 ? indexer_tc_launch<8, true>(p, q_idx, q_scale, k_idx, k_scale, w, scores, ld, row_begin,
                                                row_count, stream)
                   : indexer_tc_launch<8, false>(p, q_idx, q_scale, k_idx, k_scale, w, scores, ld, row_begin,
                                                 row_count, stream);
    return fp8 ? indexer_tc_launch<1, true>(p, q_idx, q_scale, k_idx, k_scale, w, scores, ld, row_begin, row_count,
                                            stream)
               : indexer_tc_launch<1, false>(p, q_idx, q_scale, k_idx, k_scale, w, scores, ld, row_begin, row_count,
                                             stream);
}

dsa_status_t topk_launch(const dsa_problem_t *p, const float *scores, int64_t ld, int row_begin, int row_count,
                         int32_t *idx, cudaStream_t stream, const uint8_t *row_mask = nullptr) {
    if (row_count == 0) return DSA_OK;
    Problem P = to_dev(p);
    // Fewer rows than SMs (decode): 1024 threads per row; otherwise 256 threads, several
    // CTAs per SM.  Both produce the same indices in the same order.
    int dev = 0, n_sm = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DSA_ERR_CUDA;
    if (row_count < n_sm)
        dsa::topk::topk_rows_kernel<1024><<<row_count, 1024, dsa::topk::Cfg<1024>::SMEM, stream>>>(P, scores, ld,
                                                                                                    row_begin, idx, row_mask);
    else
        dsa::topk::topk_rows_kernel<256><<<row_count, 256, dsa::topk::Cfg<256>::SMEM, stream>>>(P, scores, ld,
                                                                                               row_begin, idx, row_mask);
    return launch_status();
}

// Sparse (gathered rows of idx) or dense (keys 0 .. pos(t), restricted to idx when idx is
// given) attention of every query row.
// CTA pairs the attention runs at once on one B200 (148 SMs, one CTA per SM), and the most
// pairs one token's index row is split over.
constexpr int MLA_PAIRS = 74;
constexpr int MLA_MAX_SPLITS = 8;

// Splits of each token's index row for the gathered attention: one unit per token when
// the tokens alone fill the SMs (prefill, large decode batches); otherwise several units
// (splits) per token, each over whole 256-slot blocks, each on its own CTA pair, merged by
// combine_splits_kernel.
void mla_split_plan(const dsa_problem_t *p, int *nsplit, int *bps) {
    const int T = p->total_q;
    const int nb = (p->topk + dsa::mla::PairCfg::BLK - 1) / dsa::mla::PairCfg::BLK;   // blocks of a row
    int sp = T > 0 ? MLA_PAIRS / T : 1;
    sp = sp < nb ? sp : nb;
    sp = sp < MLA_MAX_SPLITS ? sp : MLA_MAX_SPLITS;
    if (sp < 2) {
        *nsplit = 1;
        *bps = 1 << 24;
        return;
    }
    *bps = (nb + sp - 1) / sp;
    *nsplit = (nb + *bps - 1) / *bps;   // no split left without blocks
}

// Bytes of the split partials (0 without splits).
size_t mla_split_bytes(const dsa_problem_t *p) {
    int ns, bps;
    mla_split_plan(p, &ns, &bps);
    if (ns < 2) return 0;
    return align_up((size_t)p->total_q * (size_t)ns * 128 * 513 * sizeof(float), 256);
}

// CTA pairs of one attention instantiation that run at once on the current device (one
// CTA per SM; asked of the occupancy calculator once per device, after the shared-memory
// attribute is set).
template <bool DENSE, bool SPLIT>
int mla_resident_pairs() {
    static int pairs[MAX_DEVICES] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return 0;
    if (pairs[dev] > 0) return pairs[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(dsa::mla::PairCfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = dsa::mla::PairCfg::SMEM;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, dsa::mla::sparse_mla_pair_kernel<DENSE, SPLIT>, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    pairs[dev] = n;
    return n;
}

dsa_status_t mla_launch(const dsa_problem_t *p, const void *q, const void *kv, const int32_t *idx, void *out,
                        float *lse, cudaStream_t stream, bool dense = false, void *split_ws = nullptr) {
    if (p->total_q == 0) return DSA_OK;
    Problem P = to_dev(p);
    dsa::mla::SplitArgs sp{1, 1 << 24, nullptr, nullptr};
    if (!dense && split_ws != nullptr) {
        mla_split_plan(p, &sp.nsplit, &sp.bps);
        if (sp.nsplit > 1) {
            sp.o_part = static_cast<float *>(split_ws);
            sp.lse_part = sp.o_part + (size_t)p->total_q * (size_t)sp.nsplit * 128 * 512;
        }
    }
    CUtensorMap tq, tkv;
    // q: [T*128 rows, 576] read as 64-row boxes of 64 dims (each CTA of a pair loads its 64
    // heads; the latent rows are gathered by TMA, 4 rows per instruction)
    if (!make_tmap_rows(&tq, q, false, 576, (uint64_t)p->total_q * 128, 64)) return DSA_ERR_CUDA;
    // persistent pairs: no more than run at once, each taking units (token, split) in turn
    const long long units = (long long)p->total_q * sp.nsplit;
    const int resident = dense ? mla_resident_pairs<true, false>()
                               : (sp.nsplit > 1 ? mla_resident_pairs<false, true>() : mla_resident_pairs<false, false>());
    if (resident <= 0) return DSA_ERR_CUDA;
    const unsigned grid = 2u * (unsigned)(units < resident ? units : resident);
    auto *ob = reinterpret_cast<__nv_bfloat16 *>(out);
    if (dense) {
        // kv: [S rows, 576] read as 128-row boxes of 64 dims (contiguous keys)
        if (!make_tmap_rows(&tkv, kv, false, 576, (uint64_t)(p->total_k > 0 ? p->total_k : 1), 128)) return DSA_ERR_CUDA;
        dsa::mla::sparse_mla_pair_kernel<true><<<grid, dsa::mla::PairCfg::THREADS, dsa::mla::PairCfg::SMEM, stream>>>(
            tq, tkv, P, idx, ob, lse, sp);
    } else {
        // kv: [S rows, 576] gathered 4 rows x 64 dims at a time (one-row boxes)
        if (!make_tmap_rows(&tkv, kv, false, 576, (uint64_t)(p->total_k > 0 ? p->total_k : 1), 1)) return DSA_ERR_CUDA;
        if (sp.nsplit > 1)
            dsa::mla::sparse_mla_pair_kernel<false, true>
                <<<grid, dsa::mla::PairCfg::THREADS, dsa::mla::PairCfg::SMEM, stream>>>(tq, tkv, P, idx, ob, lse, sp);
        else
            dsa::mla::sparse_mla_pair_kernel<false, false>
                <<<grid, dsa::mla::PairCfg::THREADS, dsa::mla::PairCfg::SMEM, stream>>>(tq, tkv, P, idx, ob, lse, sp);
    }
    dsa_status_t st = launch_status();
    if (st != DSA_OK || sp.nsplit < 2) return st;
    dsa::mla::combine_splits_kernel<<<(unsigned)p->total_q * 128u, 128, 0, stream>>>(sp.nsplit, sp.o_part,
                                                                                   sp.lse_part, ob, lse);
    return launch_status();
}

// One CTA waits on an mbarrier that nothing arrives at, so its bounded wait runs out
// after `limit_ns`: exercises the give-up path (error flag, no hang) with no copy or MMA
// in flight.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
    using namespace dsa::sm100;
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
        mbar_wait_for(b, 0, limit_ns);
    }
}


// Key length up to which the fused forward runs the attention in the dense ("masked MHA")
// form over the selected keys: on B200 its contiguous TMA tile loads beat the row gathers
// up to here even though it multiplies every causal key.  Measured with index_topk 2048
// (dense vs gathered ms per prefill): 1.65 vs 2.01 at 2560 keys, 2.25 vs 2.50 at 3072,
// 2.93 vs 2.99 at 3584, 3.70 vs 3.49 at 4096.
constexpr int DENSE_KV_THRESHOLD = 3584;

bool dense_for(const dsa_problem_t *p) { return p->block_table == nullptr && p->max_len_k <= DENSE_KV_THRESHOLD; }

// The attention of the fused forward over its selected indices.  In one packed sequence the
// first rows see at most topk keys, so their selection is every visible key in order: the
// dense form over all causal keys computes them (the same MMAs on the same operands, so the
// same output) without gathering, and the gathered form takes the remaining rows.
dsa_status_t forward_attention(const dsa_problem_t *p, const void *q, const void *kv, const int32_t *idx, void *out,
                               float *lse, cudaStream_t s, void *split_ws) {
    if (dense_for(p)) return mla_launch(p, q, kv, idx, out, lse, s, true);
    const int T = p->total_q;
    int R = 0;   // rows with pos(t) + 1 <= topk
    if (p->cu_q == nullptr && p->block_table == nullptr) {
        const int64_t r = (int64_t)p->topk - ((int64_t)p->total_k - T);
        R = r < 0 ? 0 : (r > T ? T : (int)r);
    }
    if (R == 0 || R == T) return mla_launch(p, q, kv, idx, out, lse, s, false, split_ws);
    dsa_problem_t a = *p;   // rows 0 .. R-1 and the keys they see
    a.total_q = R;
    a.max_len_q = R;
    a.total_k = p->total_k - T + R;
    a.max_len_k = a.total_k;
    dsa_status_t st = mla_launch(&a, q, kv, nullptr, out, lse, s, true);
    if (st != DSA_OK) return st;
    dsa_problem_t b = *p;   // rows R .. T-1 (the same keys: pos = total_k - (T - R) + local row)
    b.total_q = T - R;
    b.max_len_q = T - R;
    const size_t qrow = 128u * 576u * 2u, orow = 128u * 512u * 2u;
    return mla_launch(&b, static_cast<const unsigned char *>(q) + (size_t)R * qrow, kv, idx + (int64_t)R * p->topk,
                      static_cast<unsigned char *>(out) + (size_t)R * orow, lse + (int64_t)R * 128, s, false,
                      split_ws);
}

int64_t scores_ld(const dsa_problem_t *p) { return (int64_t)align_up((size_t)(p->max_len_k > 0 ? p->max_len_k : 1), 4); }

int effective_chunk(const dsa_problem_t *p, int32_t chunk_q) {
    int T = p->total_q > 0 ? p->total_q : 1;
    if (chunk_q <= 0 || chunk_q > T) return T;
    return chunk_q;
}

// ---- streaming indexer -> top-k (no score rows; see select_stream.cuh)

struct StreamWs {
    float *scores;   // [chunk, ld]: rows the threshold misjudged are redone from full scores
    float *sample;   // [chunk, lds]
    float *f_lo;     // [chunk]
    int *cnt;        // [chunk]
    uint8_t *flag;   // [chunk]
    uint2 *cand;     // [chunk, cap]
    int64_t ld, lds;
    int cap;
};

bool streaming_applies(const dsa_problem_t *p) {
    return p->cu_q == nullptr && p->max_len_k > p->topk && p->max_len_k <= STREAM_MAX_KEYS;
}

// Bytes of the streaming workspace for chunks of `chunk` rows; fills *ws when base is given.
size_t stream_layout(const dsa_problem_t *p, int chunk, unsigned char *base, StreamWs *ws) {
    const int64_t ld = scores_ld(p);
    const int64_t span = (int64_t)dsa::indexer::SAMPLE_STRIDE * 128;
    const int64_t lds = ((p->max_len_k + span - 1) / span) * 128;
    const int cap = dsa::topk::STREAM_CAP;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, 256);
        return base ? base + at : nullptr;
    };
    unsigned char *sc = take((size_t)chunk * (size_t)ld * 4);
    unsigned char *sm = take((size_t)chunk * (size_t)lds * 4);
    unsigned char *fl = take((size_t)chunk * 4);
    unsigned char *cn = take((size_t)chunk * 4);
    unsigned char *fg = take((size_t)chunk);
    unsigned char *cd = take((size_t)chunk * (size_t)cap * 8);
    if (ws) {
        ws->scores = reinterpret_cast<float *>(sc);
        ws->sample = reinterpret_cast<float *>(sm);
        ws->f_lo = reinterpret_cast<float *>(fl);
        ws->cnt = reinterpret_cast<int *>(cn);
        ws->flag = fg;
        ws->cand = reinterpret_cast<uint2 *>(cd);
        ws->ld = ld;
        ws->lds = lds;
        ws->cap = cap;
    }
    return off;
}

template <bool FP8>
dsa_status_t stream_chunk(const dsa_problem_t *p, const void *q_idx, const void *q_scale, const void *k_idx,
                          const void *k_scale, const float *w, int r0, int rc, int32_t *idx, const StreamWs &ws,
                          cudaStream_t s) {
    using namespace dsa::indexer;
    dsa_status_t st;
    if (cudaMemsetAsync(ws.cnt, 0, (size_t)rc * 4, s) != cudaSuccess) return DSA_ERR_CUDA;
    if ((st = indexer_tc_launch<8, FP8, SAMPLE>(p, q_idx, q_scale, k_idx, k_scale, w, ws.sample, ws.lds, r0, rc,
                                                s)) != DSA_OK)
        return st;
    Problem P = to_dev(p);
    dsa::topk::sample_threshold_kernel<<<rc, dsa::topk::STREAM_NT, dsa::topk::StreamCfg::SMEM, s>>>(
        P, ws.sample, ws.lds, SAMPLE_STRIDE * 128, r0, ws.f_lo);
    if ((st = launch_status()) != DSA_OK) return st;
    StreamArgs fa{};
    fa.f_lo = ws.f_lo;
    fa.cnt = ws.cnt;
    fa.cand = ws.cand;
    fa.cap = ws.cap;
    if ((st = indexer_tc_launch<8, FP8, FILTER>(p, q_idx, q_scale, k_idx, k_scale, w, nullptr, 0, r0, rc, s, fa)) !=
        DSA_OK)
        return st;
    dsa::topk::select_candidates_kernel<<<rc, dsa::topk::STREAM_NT, select_smem(p->max_len_k), s>>>(
        P, ws.cnt, ws.cand, ws.cap, r0, idx, ws.flag);
    if ((st = launch_status()) != DSA_OK) return st;
    // rows whose candidates could not decide: full score rows and the two-pass selection
    StreamArgs ra{};
    ra.row_mask = ws.flag;
    if ((st = indexer_tc_launch<8, FP8, SCORES>(p, q_idx, q_scale, k_idx, k_scale, w, ws.scores, ws.ld, r0, rc, s,
                                                ra)) != DSA_OK)
        return st;
    return topk_launch(p, ws.scores, ws.ld, r0, rc, idx, s, ws.flag);
}

}  // namespace

extern "C" {

const char *dsa_status_string(dsa_status_t s) {
    switch (s) {
        case DSA_OK: return "success";
        case DSA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, or inconsistent size)";
        case DSA_ERR_UNSUPPORTED: return "unsupported problem shape for this build";
        case DSA_ERR_WORKSPACE: return "workspace missing or too small";
        case DSA_ERR_CUDA: return "CUDA launch or runtime error";
        case DSA_ERR_DEVICE_TIMEOUT: return "a device-side bounded wait gave up";
        case DSA_ERR_DEVICE_BOUNDS: return "a debug-mode device check found an inconsistent input (row skipped)";
    }
    return "unknown status";
}

int32_t dsa_abi_version(void) { return DSA_ABI_VERSION; }

dsa_status_t dsa_indexer_scores(const dsa_problem_t *p, const void *q_idx, const void *q_scale, const void *k_idx,
                                const void *k_scale, const float *w, float *scores, int64_t ld_scores,
                                int32_t row_begin, int32_t row_count, dsa_stream_t stream) {
    dsa_status_t st = check_problem(p);
    if (st != DSA_OK) return st;
    if (row_begin < 0 || row_count < 0 || (int64_t)row_begin + row_count > p->total_q) return DSA_ERR_INVALID_ARG;
    if (ld_scores < p->max_len_k || (ld_scores & 3) != 0) return DSA_ERR_INVALID_ARG;
    if (row_count > 0) {
        if (!q_idx || !k_idx || !w || !scores) return DSA_ERR_INVALID_ARG;
        if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
        if (p->idx_dtype != DSA_BF16 && (!q_scale || !k_scale)) return DSA_ERR_INVALID_ARG;
    }
    if ((st = set_smem_attrs()) != DSA_OK) return st;
    return indexer_launch(p, q_idx, q_scale, k_idx, k_scale, w, scores, ld_scores, row_begin, row_count,
                          (cudaStream_t)stream);
}

dsa_status_t dsa_topk(const dsa_problem_t *p, const float *scores, int64_t ld_scores, int32_t row_begin,
                      int32_t row_count, int32_t *idx, dsa_stream_t stream) {
    dsa_status_t st = check_problem(p);
    if (st != DSA_OK) return st;
    if (row_begin < 0 || row_count < 0 || (int64_t)row_begin + row_count > p->total_q) return DSA_ERR_INVALID_ARG;
    if (ld_scores < p->max_len_k || (ld_scores & 3) != 0) return DSA_ERR_INVALID_ARG;
    if (row_count > 0) {
        if (!scores || !idx || !aligned16(scores) || !aligned16(idx)) return DSA_ERR_INVALID_ARG;
    }
    if ((st = set_smem_attrs()) != DSA_OK) return st;
    return topk_launch(p, scores, ld_scores, row_begin, row_count, idx, (cudaStream_t)stream);
}

dsa_status_t dsa_sparse_mla_fwd(const dsa_problem_t *p, const void *q, const void *kv, const int32_t *idx, void *out,
                                float *lse, dsa_stream_t stream) {
    dsa_status_t st = check_problem(p);
    if (st != DSA_OK) return st;
    if (p->total_q > 0) {
        if (!q || !kv || !idx || !out || !lse) return DSA_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(kv) || !aligned16(idx) || !aligned16(out) || !aligned16(lse))
            return DSA_ERR_INVALID_ARG;
    }
    if ((st = set_smem_attrs()) != DSA_OK) return st;
    return mla_launch(p, q, kv, idx, out, lse, (cudaStream_t)stream);
}

dsa_status_t dsa_dense_mla_fwd(const dsa_problem_t *p, const void *q, const void *kv, const int32_t *idx, void *out,
                               float *lse, dsa_stream_t stream) {
    dsa_status_t st = check_problem(p);
    if (st != DSA_OK) return st;
    if (idx != nullptr && p->max_len_k > dsa::mla::PairCfg::DENSE_MAX_KEYS) return DSA_ERR_UNSUPPORTED;
    if (p->block_table != nullptr) return DSA_ERR_UNSUPPORTED;
    if (p->total_q > 0) {
        if (!q || !kv || !out || !lse) return DSA_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(kv) || !aligned16(out) || !aligned16(lse) || (idx && !aligned16(idx)))
            return DSA_ERR_INVALID_ARG;
    }
    if ((st = set_smem_attrs()) != DSA_OK) return st;
    return mla_launch(p, q, kv, idx, out, lse, (cudaStream_t)stream, true);
}

size_t dsa_forward_workspace_size(const dsa_problem_t *p, int32_t chunk_q) {
    if (check_problem(p) != DSA_OK) return 0;
    size_t chunk = (size_t)effective_chunk(p, chunk_q);
    size_t scores = align_up(chunk * (size_t)scores_ld(p) * sizeof(float), 256);
    size_t idx = align_up((size_t)(p->total_q > 0 ? p->total_q : 1) * (size_t)p->topk * sizeof(int32_t), 256);
    return scores + idx + mla_split_bytes(p);
}

dsa_status_t dsa_forward(const dsa_problem_t *p, const void *q_idx, const void *q_scale, const void *k_idx,
                         const void *k_scale, const float *w, const void *q, const void *kv, int32_t chunk_q,
                         int32_t *idx_out, void *out, float *lse, void *workspace, size_t workspace_bytes,
                         dsa_stream_t stream) {
    dsa_status_t st = check_problem(p);
    if (st != DSA_OK) return st;
    if (chunk_q < 0) return DSA_ERR_INVALID_ARG;
    if (p->total_q == 0) return DSA_OK;
    if (!q_idx || !k_idx || !w || !q || !kv || !out || !lse) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(q) || !aligned16(kv) ||
        !aligned16(out) || !aligned16(lse) || (idx_out && !aligned16(idx_out)))
        return DSA_ERR_INVALID_ARG;
    if (p->idx_dtype != DSA_BF16 && (!q_scale || !k_scale)) return DSA_ERR_INVALID_ARG;
    const size_t need = dsa_forward_workspace_size(p, chunk_q);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return DSA_ERR_WORKSPACE;
    if ((st = set_smem_attrs()) != DSA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const int chunk = effective_chunk(p, chunk_q);
    const int64_t ld = scores_ld(p);
    float *scores = reinterpret_cast<float *>(workspace);
    if (p->max_len_k <= p->topk && p->block_table == nullptr) {
        // Every row has at most topk visible keys, so the selection keeps all of them: no
        // scores are needed, and the attention runs over the contiguous keys (dense mode,
        // the same MMAs as the gathered form on the same operands).
        if (idx_out && (st = topk_launch(p, scores, ld, 0, p->total_q, idx_out, s)) != DSA_OK) return st;
        return mla_launch(p, q, kv, nullptr, out, lse, s, true);
    }
    int32_t *idx = idx_out;
    if (!idx) {
        size_t off = align_up((size_t)chunk * (size_t)ld * sizeof(float), 256);
        idx = reinterpret_cast<int32_t *>(reinterpret_cast<unsigned char *>(workspace) + off);
    }
    for (int r0 = 0; r0 < p->total_q; r0 += chunk) {
        const int rc = p->total_q - r0 < chunk ? p->total_q - r0 : chunk;
        st = indexer_launch(p, q_idx, q_scale, k_idx, k_scale, w, scores, ld, r0, rc, s);
        if (st != DSA_OK) return st;
        st = topk_launch(p, scores, ld, r0, rc, idx + (int64_t)r0 * p->topk, s);
        if (st != DSA_OK) return st;
    }
    // the partials of a split attention follow the score rows and the indices
    unsigned char *split_ws = static_cast<unsigned char *>(workspace) +
                              align_up((size_t)chunk * (size_t)ld * sizeof(float), 256) +
                              align_up((size_t)p->total_q * (size_t)p->topk * sizeof(int32_t), 256);
    return forward_attention(p, q, kv, idx, out, lse, s, split_ws);
}

size_t dsa_indexer_topk_streaming_workspace_size(const dsa_problem_t *p, int32_t chunk_q) {
    if (check_problem(p) != DSA_OK) return 0;
    const int chunk = effective_chunk(p, chunk_q);
    if (!streaming_applies(p)) return align_up((size_t)chunk * (size_t)scores_ld(p) * sizeof(float), 256);
    return stream_layout(p, chunk, nullptr, nullptr);
}

dsa_status_t dsa_indexer_topk_streaming(const dsa_problem_t *p, const void *q_idx, const void *q_scale,
                                        const void *k_idx, const void *k_scale, const float *w, int32_t row_begin,
                                        int32_t row_count, int32_t chunk_q, int32_t *idx, void *workspace,
                                        size_t workspace_bytes, dsa_stream_t stream) {
    dsa_status_t st = check_problem(p);
    if (st != DSA_OK) return st;
    if (row_begin < 0 || row_count < 0 || row_begin + row_count > p->total_q) return DSA_ERR_INVALID_ARG;
    if (row_count == 0) return DSA_OK;
    if (!q_idx || !k_idx || !w || !idx) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(idx)) return DSA_ERR_INVALID_ARG;
    if (p->idx_dtype != DSA_BF16 && (!q_scale || !k_scale)) return DSA_ERR_INVALID_ARG;
    const size_t need = dsa_indexer_topk_streaming_workspace_size(p, chunk_q);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return DSA_ERR_WORKSPACE;
    if ((st = set_smem_attrs()) != DSA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const int chunk = effective_chunk(p, chunk_q);
    const bool fp8 = p->idx_dtype != DSA_BF16;
    StreamWs ws{};
    const bool streaming = streaming_applies(p);
    if (streaming) stream_layout(p, chunk, static_cast<unsigned char *>(workspace), &ws);
    for (int r0 = row_begin; r0 < row_begin + row_count; r0 += chunk) {
        const int rc = row_begin + row_count - r0 < chunk ? row_begin + row_count - r0 : chunk;
        int32_t *out = idx + (int64_t)(r0 - row_begin) * p->topk;
        if (streaming) {
            st = fp8 ? stream_chunk<true>(p, q_idx, q_scale, k_idx, k_scale, w, r0, rc, out, ws, s)
                     : stream_chunk<false>(p, q_idx, q_scale, k_idx, k_scale, w, r0, rc, out, ws, s);
        } else {   // ragged batches and very long rows: the two-pass kernels (the same indices)
            float *scores = static_cast<float *>(workspace);
            const int64_t ld = scores_ld(p);
            st = indexer_launch(p, q_idx, q_scale, k_idx, k_scale, w, scores, ld, r0, rc, s);
            if (st == DSA_OK) st = topk_launch(p, scores, ld, r0, rc, out, s);
        }
        if (st != DSA_OK) return st;
    }
    return DSA_OK;
}

dsa_status_t dsa_cache_write(int32_t n_tokens, const void *k_idx_raw, const void *kv_raw, const int32_t *positions,
                             const int32_t *rows, const float *k_norm_w, const float *k_norm_b, const float *kv_norm_w,
                             const float *inv_freq, float eps, void *k_idx_cache, void *kv_cache, dsa_stream_t stream) {
    if (n_tokens < 0 || !(eps >= 0.0f)) return DSA_ERR_INVALID_ARG;
    if (n_tokens == 0) return DSA_OK;
    const void *ptrs[] = {k_idx_raw, kv_raw, positions, rows, k_norm_w, k_norm_b, kv_norm_w, inv_freq, k_idx_cache, kv_cache};
    for (const void *q : ptrs)
        if (q == nullptr || !aligned16(q)) return DSA_ERR_INVALID_ARG;
    const unsigned grid = (unsigned)((n_tokens + dsa::cache::WARPS - 1) / dsa::cache::WARPS);
    dsa::cache::cache_write_kernel<<<grid, 32 * dsa::cache::WARPS, 0, (cudaStream_t)stream>>>(
        n_tokens, reinterpret_cast<const __nv_bfloat16 *>(k_idx_raw), reinterpret_cast<const __nv_bfloat16 *>(kv_raw),
        positions, rows, k_norm_w, k_norm_b, kv_norm_w, inv_freq, eps, reinterpret_cast<__nv_bfloat16 *>(k_idx_cache),
        reinterpret_cast<__nv_bfloat16 *>(kv_cache));
    return launch_status();
}

dsa_status_t dsa_selftest_bounded_wait(uint32_t limit_us, dsa_stream_t stream) {
    if (limit_us < 1 || limit_us > 10000) return DSA_ERR_INVALID_ARG;
    bounded_wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_us * 1000ull);
    return launch_status();
}

dsa_status_t dsa_check_device_errors(dsa_stream_t stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return DSA_ERR_CUDA;
    unsigned int flag = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&flag, dsa::g_error_flag, sizeof(flag)) != cudaSuccess) return DSA_ERR_CUDA;
    if (flag != 0 && cudaMemcpyToSymbol(dsa::g_error_flag, &zero, sizeof(zero)) != cudaSuccess) return DSA_ERR_CUDA;
    if (flag & (dsa::sm100::ERR_WAIT_TIMEOUT | dsa::sm100::ERR_SMEM_ALIGN)) return DSA_ERR_DEVICE_TIMEOUT;
    return flag ? DSA_ERR_DEVICE_BOUNDS : DSA_OK;
}

void dsa_set_debug_checks(int32_t enable) { g_debug_checks = enable != 0; }

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Allocation-free variant of dsa_forward.
//
// Some callers cannot allocate device memory at the point where they run the path: code
// that runs inside a host callback or a custom allocator, runtimes that own all device
// memory up front and hand out nothing else, or deployments where a cudaMalloc in the
// serving loop would stall other streams.  dsa_forward_noalloc serves them: its only
// scratch (the fp32 index scores of one chunk of query rows) lives in the fixed array
// below, so the call itself never allocates or frees anything.
//
//   * The array holds NOALLOC_SCRATCH_BYTES (32 MiB).  Every GPU that loads this library
//     keeps it resident until the process exits.
//   * Its device address is looked up once per device, on the first call made with that
//     device current (cudaGetSymbolAddress); make that first call outside any stream
//     capture.
//   * All calls share the array and it keeps whatever the last call left: calls whose
//     work overlaps on the GPU (e.g. on two streams without ordering) race on it.  No
//     part of it needs to start at zero -- every score the top-k reads is written first by
//     the indexer of the same chunk.
// ---------------------------------------------------------------------------------------
namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(32) << 20;
constexpr int NOALLOC_MAX_DEVICES = MAX_DEVICES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Per-device address of g_noalloc_scratch (nullptr until looked up).
void *g_noalloc_addr[NOALLOC_MAX_DEVICES] = {};

dsa_status_t noalloc_scratch(float **scratch) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NOALLOC_MAX_DEVICES) return DSA_ERR_CUDA;
    if (g_noalloc_addr[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return DSA_ERR_CUDA;
        g_noalloc_addr[dev] = ptr;
    }
    *scratch = reinterpret_cast<float *>(g_noalloc_addr[dev]);
    return DSA_OK;
}

}  // namespace

extern "C" dsa_status_t dsa_forward_noalloc(const dsa_problem_t *p, const void *q_idx, const void *q_scale,
                                            const void *k_idx, const void *k_scale, const float *w, const void *q,
                                            const void *kv, int32_t *idx_out, void *out, float *lse,
                                            dsa_stream_t stream) {
    dsa_status_t st = check_problem(p);
    if (st != DSA_OK) return st;
    if (p->total_q == 0) return DSA_OK;
    if (!q_idx || !k_idx || !w || !q || !kv || !idx_out || !out || !lse) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(q) || !aligned16(kv) ||
        !aligned16(idx_out) || !aligned16(out) || !aligned16(lse))
        return DSA_ERR_INVALID_ARG;
    if (p->idx_dtype != DSA_BF16 && (!q_scale || !k_scale)) return DSA_ERR_INVALID_ARG;
    // rows of scores that fit in the fixed scratch; a single row must fit
    const int64_t ld = scores_ld(p);
    const int64_t rows_fit = (int64_t)(NOALLOC_SCRATCH_BYTES / ((size_t)ld * sizeof(float)));
    if (rows_fit < 1) return DSA_ERR_WORKSPACE;
    const int chunk = (int)(rows_fit < p->total_q ? rows_fit : p->total_q);
    float *scores = nullptr;
    if ((st = noalloc_scratch(&scores)) != DSA_OK) return st;
    if ((st = set_smem_attrs()) != DSA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (p->max_len_k <= p->topk && p->block_table == nullptr) {   // every visible key is selected
        if ((st = topk_launch(p, scores, ld, 0, p->total_q, idx_out, s)) != DSA_OK) return st;
        return mla_launch(p, q, kv, nullptr, out, lse, s, true);
    }
    for (int r0 = 0; r0 < p->total_q; r0 += chunk) {
        const int rc = p->total_q - r0 < chunk ? p->total_q - r0 : chunk;
        st = indexer_launch(p, q_idx, q_scale, k_idx, k_scale, w, scores, ld, r0, rc, s);
        if (st != DSA_OK) return st;
        st = topk_launch(p, scores, ld, r0, rc, idx_out + (int64_t)r0 * p->topk, s);
        if (st != DSA_OK) return st;
    }
    // the score rows are done: the scratch holds the partials of a split attention
    return forward_attention(p, q, kv, idx_out, out, lse, s,
                             mla_split_bytes(p) <= NOALLOC_SCRATCH_BYTES ? static_cast<void *>(scores) : nullptr);
}

extern "C" size_t dsa_forward_noalloc_scratch_bytes(void) { return NOALLOC_SCRATCH_BYTES; }
