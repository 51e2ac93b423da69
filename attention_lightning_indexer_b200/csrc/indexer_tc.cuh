// indexer_tc.cuh -- lightning indexer on the 5th-generation tensor cores (tcgen05).
//
// "DeepSeek-V3.2 tech report summary", §1 DSA, ① Lightning Indexer:
//     I[t,s] = sum_{j<64} w[t,j] * ReLU(q_I[t,j] . k_I[s]),  s <= pos(t),  d_I = 128,
// bf16 or FP8 (e4m3 with per-token scales).
//
// GEMM view: D[key, (query, head)] = k_I[key] . q_I[query, head], K = d_I = 128.
//  * keys sit on the MMA M axis (128 per tile, one TMEM lane each) and (query, head)
//    pairs on N (4 queries x 64 heads = 256 columns per MMA); a CTA keeps the q_I rows of
//    QG consecutive queries resident in shared memory and streams the key tiles of their
//    causal range through a TMA ring;
//  * accumulators live in TMEM, double-buffered: while the tensor core fills one buffer,
//    an epilogue warpgroup reads the other (tcgen05.ld), so each thread owns one key row
//    and sums w[t,j] * ReLU(.) over the 64 heads of a query in registers -- no shuffles;
//  * the fp32 score row is written coalesced (128 consecutive keys per query); keys past
//    pos(t) are never written, tiles past the group's last position are never loaded.
// FP8: kind::f8f6f4 MMA on e4m3 codes; since the scales are positive, ReLU(a*b*x) =
// a*b*ReLU(x): the query's scale (per token, or per head with ue8m0 block scales) joins
// w[t,j] when the weights are staged, and the key's scale multiplies the finished sum.
//
// Warp roles: 0 TMA producer, 1 MMA issuer, 2 TMEM allocator, 3 idle; then the epilogue
// warpgroups.  bf16 and decode: 4-7 for accumulator buffer 0, 8-11 for buffer 1 (12 warps).
// FP8 query groups: 4-7 and 12-15 for buffer 0 and 8-11 and 16-19 for buffer 1, each
// warpgroup summing two of the item's four queries (20 warps; setmaxnreg moves registers
// from the first warpgroup to the epilogue).
//
// Output modes (the streaming selection of the fused indexer -> top-k):
//   SCORES   the score rows (optionally only for the groups holding a row of row_mask);
//   SAMPLE   every SAMPLE_STRIDE-th key tile only, written compactly: sample column
//            j' * 128 + r holds key j' * SAMPLE_STRIDE * 128 + r;
//   FILTER   no score rows: each score >= the row's threshold f_lo is appended as (float
//            bits, key) to the row's candidate list (one atomic per warp and query for the
//            slots; the order of the list is not defined), the count in cnt.
#pragma once

#include "dsa_common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace indexer {

enum Mode { SCORES = 0, SAMPLE = 1, FILTER = 2 };
constexpr int SAMPLE_STRIDE = 32;

// Arguments of the streaming modes.
struct StreamArgs {
    const uint8_t *row_mask;   // SCORES: score only groups with a nonzero row_mask[t - row_begin] (nullptr: all)
    const float *f_lo;         // FILTER: per-row threshold
    int *cnt;                  // FILTER: per-row candidate count (zeroed by the caller)
    uint2 *cand;               // FILTER: [rows, cap] candidates (float bits, key)
    int cap;
};

template <int QG, bool FP8>
struct TcCfg {
    static constexpr int BM = 128;                          // keys per tile = MMA M
    static constexpr int EB = FP8 ? 1 : 2;                  // bytes per element
    static constexpr int ROWB = 128 * EB;                   // bytes per key / query-head row
    static constexpr int ATOMS = ROWB / 128;                // 128-byte swizzle atoms per row
    static constexpr int KSTEP = FP8 ? 32 : 16;             // K of one MMA instruction
    static constexpr int NKS = 128 / KSTEP;                 // MMAs per item
    static constexpr int KS_PER_ATOM = 128 / (KSTEP * EB);  // MMAs per swizzle atom
    static constexpr int QROWS = QG * 64;                   // B rows
    static constexpr int N = QROWS < 256 ? QROWS : 256;     // MMA N
    static constexpr int NSUB = QROWS / N;                  // items (MMA groups) per tile
    static constexpr int QPI = N / 64;                      // queries per item
    static constexpr int STAGES = (!FP8) ? 3 : 4;
    static constexpr int KTILE_BYTES = BM * ROWB;
    static constexpr int KATOM_BYTES = BM * 128;
    static constexpr int Q_BYTES = QROWS * ROWB;
    static constexpr int QATOM_BYTES = QROWS * 128;
    static constexpr int QBOX_BYTES = 64 * 128;             // one TMA box: 64 rows x 128 bytes
    static constexpr int TMEM_COLS = 2 * N < 32 ? 32 : 2 * N;
    static constexpr int OFF_K = Q_BYTES;
    static constexpr int OFF_W = OFF_K + STAGES * KTILE_BYTES;
    static constexpr int OFF_BAR = OFF_W + QROWS * 4;
    static constexpr int NBARS = 1 + 2 * STAGES + 4 + 1;   // ... + drain
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int SMEM = OFF_MISC + 16;
    // Epilogue warpgroups: two (one per accumulator buffer, each summing the buffer's QPI
    // queries), or for FP8 query groups four (two per buffer, QPI / 2 queries each): the
    // e4m3 MMA leaves the epilogue half the time, and more warps hide its latencies.
    static constexpr int EPI_WG = (FP8 && QG > 1) ? 4 : 2;
    static constexpr int EPI_SPLIT = EPI_WG / 2;            // warpgroups per accumulator buffer
    static constexpr int QPW = QPI / EPI_SPLIT;             // queries per warpgroup per item
    static constexpr int THREADS = 128 * (1 + EPI_WG);
    // register split when EPI_WG == 4 (setmaxnreg): 128 x REG_LOW + 512 x REG_HIGH must not
    // exceed 640 x the registers a thread is launched with (96)
    static constexpr int REG_LOW = 56, REG_HIGH = 104;
    static constexpr int SPLIT_KEYS = 4096;                 // key range of one CTA when QG == 1
    static_assert(EPI_WG == 2 || 128 * REG_LOW + 512 * REG_HIGH <= 640 * 96, "register split");
    static_assert(SMEM <= 232448, "shared memory budget");
};

template <int QG, bool FP8, int MODE>
__global__ void __launch_bounds__(TcCfg<QG, FP8>::THREADS, (QG == 1 && !FP8) ? 2 : 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, Problem P,
                  const void *__restrict__ q_scale, const void *__restrict__ k_scale, const float *__restrict__ w,
                  float *__restrict__ scores, int64_t ld, int row_begin, int row_count, int nsplit, StreamArgs sa) {
    using C = TcCfg<QG, FP8>;
    static_assert(MODE == SCORES || (QG > 1 && C::NSUB == 2), "streaming modes: one query group per CTA, "
                                                              "one item half per epilogue warpgroup");
    using namespace sm100;
    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- which query rows and which key range this CTA owns
    int t0, qcount, kbase, key0, nkeys_total;
    int pos0;   // position of query t0 (queries of a group are consecutive positions)
    RowInfo rk; // the group's sequence (key rows through key_row when the cache is paged)
    if (QG > 1) {
        const int ngroups = (row_count + QG - 1) / QG;
        const int g = ngroups - 1 - (int)blockIdx.x;          // heaviest (latest) groups first
        t0 = row_begin + g * QG;
        qcount = min(QG, row_begin + row_count - t0);
        const RowInfo ri = row_info(P, t0);                   // single sequence (cu arrays absent)
        rk = ri;
        kbase = ri.kbase;
        pos0 = ri.pos;
        key0 = 0;
        nkeys_total = row_ok(P, ri) ? min(ri.pos + qcount, ri.len_k) : 0;   // visible keys of the last query
    } else {
        const int r = (int)blockIdx.x / nsplit, split = (int)blockIdx.x % nsplit;
        t0 = row_begin + r;
        qcount = 1;
        const RowInfo ri = row_info_warp(P, t0);
        rk = ri;
        kbase = ri.kbase;
        pos0 = ri.pos;
        key0 = split * C::SPLIT_KEYS;
        nkeys_total = row_ok(P, ri) ? min(visible_keys(ri), key0 + C::SPLIT_KEYS) : 0;
    }
    if (nkeys_total <= key0) return;                          // uniform for the whole CTA
    if (MODE == SCORES && sa.row_mask != nullptr) {           // uniform: the same rows for every thread
        bool any = false;
        for (int q = 0; q < qcount; ++q) any = any || sa.row_mask[t0 + q - row_begin] != 0;
        if (!any) return;
    }
    const int tstride = MODE == SAMPLE ? SAMPLE_STRIDE : 1;  // key tiles advanced per tile processed
    const int ntiles = ((nkeys_total - key0 + C::BM - 1) / C::BM + tstride - 1) / tstride;
    const int nitems = ntiles * C::NSUB;

    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {                                      // SW128 operands need 1 KB alignment
        if (tid == 0) raise_error(ERR_SMEM_ALIGN);
        return;
    }
    const uint32_t q_s = sbase;
    const uint32_t k_s = sbase + C::OFF_K;
    float *w_s = reinterpret_cast<float *>(smem + C::OFF_W);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    const uint32_t q_full = bar0;
    auto k_full = [&](int s) { return bar0 + 8u * (1 + s); };
    auto k_empty = [&](int s) { return bar0 + 8u * (1 + C::STAGES + s); };
    auto acc_full = [&](int b) { return bar0 + 8u * (1 + 2 * C::STAGES + b); };
    auto acc_empty = [&](int b) { return bar0 + 8u * (1 + 2 * C::STAGES + 2 + b); };
    const uint32_t drain = bar0 + 8u * (1 + 2 * C::STAGES + 4);
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);  // [0] tmem base, [1] abort

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(k_full(s), 1);
            mbar_init(k_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), 4 * C::EPI_SPLIT);
        }
        mbar_init(drain, 1);
        misc[1] = 0;
        fence_barrier_init();
    }
    if (warp == 2) tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
    for (int i = tid; i < C::QROWS; i += C::THREADS) {
        const int q = i / 64;
        float wv = q < qcount ? __ldg(w + (int64_t)(t0 + q) * 64 + (i % 64)) : 0.f;
        if (FP8 && q < qcount) {   // the query's scale joins its head weights (scales are > 0)
            float qs;
            if (P.ue8m0) {
                qs = ue8m0_to_float(__ldg(reinterpret_cast<const uint8_t *>(q_scale) + (int64_t)(t0 + q) * 64 + (i % 64)));
            } else {
                qs = __ldg(reinterpret_cast<const float *>(q_scale) + t0 + q);
                if (P.debug && !(qs > 0.f && qs < INFINITY)) raise_error(ERR_BOUNDS);
            }
            wv *= qs;
        }
        w_s[i] = wv;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp < 4) {
    // with four epilogue warpgroups the first warpgroup gives registers to the epilogue
    if (C::EPI_WG == 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REG_LOW));
    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        mbar_expect_tx(q_full, (uint32_t)(qcount * 64 * C::ROWB));
        for (int a = 0; a < C::ATOMS; ++a)
            for (int q = 0; q < qcount; ++q)
                tma_load_2d(q_s + a * C::QATOM_BYTES + q * C::QBOX_BYTES, &tm_q, q_full, a * 128 / C::EB,
                            (t0 + q) * 64);
        int issued = 0;                                       // key tiles whose loads were issued
        for (int j = 0; j < ntiles; ++j) {
            const int s = j % C::STAGES;
            if (j >= C::STAGES && !mbar_wait(k_empty(s), ((j / C::STAGES) - 1) & 1)) { misc[1] = 1; break; }
            if (misc[1]) break;
            mbar_expect_tx(k_full(s), C::KTILE_BYTES);
            issued = j + 1;
            const int kk0 = key0 + j * tstride * C::BM;
            for (int a = 0; a < C::ATOMS; ++a) {
                const uint32_t dst = k_s + s * C::KTILE_BYTES + a * C::KATOM_BYTES;
                if (P.block_table == nullptr) {
                    tma_load_2d(dst, &tm_k, k_full(s), a * 128 / C::EB, kbase + kk0);
                } else {   // a 128-key tile is two pages of 64 rows (the map's box is 64 rows)
                    tma_load_2d(dst, &tm_k, k_full(s), a * 128 / C::EB, key_row(P, rk, kk0));
                    tma_load_2d(dst + 64 * 128, &tm_k, k_full(s), a * 128 / C::EB, key_row(P, rk, kk0 + 64));
                }
            }
        }
        // drain: the last commits on k_empty must land before the CTA may exit; after an
        // abort, at least every issued load must have landed (no copy into freed memory)
        for (int j = max(0, ntiles - C::STAGES); j < ntiles && !misc[1]; ++j)
            if (!mbar_wait(k_empty(j % C::STAGES), (j / C::STAGES) & 1)) misc[1] = 1;
        if (misc[1]) {
            mbar_wait(q_full, 0);
            for (int j = max(0, issued - C::STAGES); j < issued; ++j) mbar_wait(k_full(j % C::STAGES), (j / C::STAGES) & 1);
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idesc = FP8 ? idesc_e4m3(C::BM, C::N) : idesc_bf16(C::BM, C::N);
        bool ok = mbar_wait(q_full, 0);
        tc_fence_after();
        int it = 0;
        bool any = false;                                     // an MMA has been issued
        for (int j = 0; ok && j < ntiles && !misc[1]; ++j) {
            const int s = j % C::STAGES;
            if (!mbar_wait(k_full(s), (j / C::STAGES) & 1)) { ok = false; break; }
            tc_fence_after();
            for (int h = 0; h < C::NSUB; ++h, ++it) {
                const int b = it & 1;
                const int use = it >> 1;
                if (use > 0 && !mbar_wait(acc_empty(b), (use - 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(b * C::N);
#pragma unroll
                for (int kk = 0; kk < C::NKS; ++kk) {
                    const uint32_t a_addr = k_s + s * C::KTILE_BYTES + (kk / C::KS_PER_ATOM) * C::KATOM_BYTES +
                                            (kk % C::KS_PER_ATOM) * 32;
                    const uint32_t b_addr = q_s + (kk / C::KS_PER_ATOM) * C::QATOM_BYTES + h * C::N * 128 +
                                            (kk % C::KS_PER_ATOM) * 32;
                    if (FP8)
                        mma_f8(d, desc_sw128(a_addr), desc_sw128(b_addr), idesc, kk > 0 ? 1u : 0u);
                    else
                        mma_f16(d, desc_sw128(a_addr), desc_sw128(b_addr), idesc, kk > 0 ? 1u : 0u);
                }
                any = true;
                mma_commit(acc_full(b));
            }
            if (!ok) break;
            mma_commit(k_empty(s));
        }
        if (!ok) misc[1] = 1;
        if (misc[1] && any) {                                 // nothing in flight at dealloc
            mma_commit(drain);
            mbar_wait(drain, 0);
        }
    }
    } else {
        if (C::EPI_WG == 4) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REG_HIGH));
        // ------------------------------------------------ epilogue warpgroups
        const int e = (warp - 4) >> 2;            // epilogue warpgroup
        const int g = C::EPI_SPLIT > 1 ? e & 1 : e;   // accumulator buffer handled by this warpgroup
        const int qh = C::EPI_SPLIT > 1 ? e >> 1 : 0;   // which QPW queries of each item it sums
        const int quarter = warp & 3;             // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;      // key row inside the tile
        const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
        constexpr int QPW = C::QPW;
        const int qw0 = qh * QPW;                 // this warpgroup's first query within an item
        float th[QPW];      // FILTER: the thresholds of this warpgroup's queries (h == g)
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) {
            const int q = g * C::QPI + qw0 + qi;
            th[qi] = (MODE == FILTER && q < qcount) ? __ldg(sa.f_lo + (t0 + q - row_begin)) : 0.f;
        }
        for (int it = g; it < nitems; it += 2) {
            const int use = it >> 1;
            const int j = it / C::NSUB, h = it % C::NSUB;
            const int key = key0 + j * tstride * C::BM + row;
            float ks = 1.f;   // the key's scale, loaded before the accumulator wait
            if (FP8 && key < nkeys_total) {
                const int kr = key_row(P, rk, key);
                ks = P.ue8m0 ? ue8m0_to_float(__ldg(reinterpret_cast<const uint8_t *>(k_scale) + kr))
                             : __ldg(reinterpret_cast<const float *>(k_scale) + kr);
            }
            if (misc[1] || !mbar_wait(acc_full(g), use & 1)) { misc[1] = 1; break; }
            tc_fence_after();
            // This warpgroup's accumulator columns of the item are read in 2 * QPW chunks of 32
            // (query qi, head half): the load of chunk k + 1 is in flight while chunk k is
            // summed, and the buffer is released as soon as its last chunk has landed.
            // Sum over heads of w * ReLU(x) on packed fp32 FMAs: even heads in the low lane,
            // odd heads in the high lane (every lane rounds like a scalar fmaf).  FP8, whose
            // MMA leaves the epilogue less time, sums heads 0..31 and 32..63 in two
            // independent chains added at the end; bf16 keeps one chain in head order.
            float res[QPW];
            uint32_t va[32], vb[32];
            uint64_t acc = 0, acc_hi = 0;
            const uint32_t col0 = t_lane + (uint32_t)(g * C::N + qw0 * 64);
            tmem_ld32(col0, va);
            tmem_wait_ld();
            tmem_regs_ready(va);
#pragma unroll
            for (int k = 0; k < 2 * QPW; ++k) {
                const int qi = k >> 1, half = k & 1;
                uint32_t(&cur)[32] = half ? vb : va;
                uint32_t(&nxt)[32] = half ? va : vb;
                if (k + 1 < 2 * QPW) tmem_ld32(col0 + (uint32_t)((k + 1) * 32), nxt);
                if (half == 0) {
                    acc = 0;
                    acc_hi = 0;
                }
                const uint64_t *wq2 =
                    reinterpret_cast<const uint64_t *>(w_s + (h * C::QPI + qw0 + qi) * 64 + half * 32);
                uint64_t &dst = (FP8 && half) ? acc_hi : acc;
#pragma unroll
                for (int c = 0; c < 32; c += 2)
                    fma_f32x2(dst, pack_f32x2(fmaxf(__uint_as_float(cur[c]), 0.f), fmaxf(__uint_as_float(cur[c + 1]), 0.f)),
                              wq2[c / 2]);
                if (half == 1) {
                    float acc0, acc1, acc2, acc3;
                    unpack_f32x2(acc, acc0, acc1);
                    unpack_f32x2(acc_hi, acc2, acc3);
                    res[qi] = FP8 ? (acc0 + acc1) + (acc2 + acc3) : acc0 + acc1;
                }
                if (k + 1 < 2 * QPW) {
                    tmem_wait_ld();
                    tmem_regs_ready(nxt);
                    if (k + 2 == 2 * QPW) {   // this warpgroup's last chunk of the buffer has landed
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(acc_empty(g));
                    }
                }
            }
            if (FP8 && P.debug && key < nkeys_total && !P.ue8m0 && !(ks > 0.f && ks < INFINITY)) raise_error(ERR_BOUNDS);
            if (MODE == FILTER) {
                // each query is the same for the whole warp: the warp reserves its slots of
                // the QPI rows with independent atomics (issued together), then stores
                unsigned m[QPW];
                int base[QPW];
#pragma unroll
                for (int qi = 0; qi < QPW; ++qi) {
                    const int q = h * C::QPI + qw0 + qi;
                    const bool valid = q < qcount && key <= pos0 + q && key < nkeys_total;
                    res[qi] = FP8 ? res[qi] * ks : res[qi];
                    m[qi] = __ballot_sync(0xffffffffu, valid && res[qi] >= th[qi]);
                    base[qi] = 0;
                    if (lane == 0 && m[qi] != 0u) base[qi] = atomicAdd(sa.cnt + (t0 + q - row_begin), __popc(m[qi]));
                }
#pragma unroll
                for (int qi = 0; qi < QPW; ++qi) {
                    const int t = t0 + h * C::QPI + qw0 + qi;
                    const int b = __shfl_sync(0xffffffffu, base[qi], 0);
                    const int slot = b + __popc(m[qi] & ((1u << lane) - 1u));
                    if (((m[qi] >> lane) & 1u) && slot < sa.cap)
                        sa.cand[(int64_t)(t - row_begin) * sa.cap + slot] = make_uint2(__float_as_uint(res[qi]), (uint32_t)key);
                }
            } else {
#pragma unroll
                for (int qi = 0; qi < QPW; ++qi) {
                    const int q = h * C::QPI + qw0 + qi;
                    if (q < qcount && key <= pos0 + q && key < nkeys_total) {
                        const int t = t0 + q;
                        const float v = FP8 ? res[qi] * ks : res[qi];
                        const int col = MODE == SAMPLE ? j * C::BM + row : key;
                        scores[(int64_t)(t - row_begin) * ld + col] = v;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace indexer
}  // namespace dsa
