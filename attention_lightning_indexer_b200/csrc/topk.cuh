// topk.cuh -- exact causal top-k per query row by radix selection.
//
// "DeepSeek-V3.2 tech report summary", §1 DSA, ② fine-grained token selection: keep the
// top-k index scores of each query; "Model techniques map -- DeepSeek-V3.2",
// Indexer-selected sparse attention: k_eff = min(index_topk, #candidates), int32 out.
//
// Design (one CTA per query row, HBM-bound):
//   * scores are mapped to order-preserving 32-bit keys (-0.0 folded onto +0.0), so
//     comparing keys as unsigned integers compares the floats as values;
//   * an 11/11/10-bit MSB-first radix select finds the exact k-th largest key `thr`
//     and how many keys equal to `thr` are taken (the smallest indices win ties);
//   * after the first digit only the keys that share the selected digit are kept as
//     candidates (compacted in shared memory), so the later digits touch a few % of
//     the row;
//   * a final ordered pass writes keys > thr and the first `need_eq` keys == thr
//     using warp ballots, so the output is deterministic (ascending index within each
//     class) and independent of the launch shape.
// The row is staged once in shared memory when it fits; longer rows are re-read from
// global memory (L2) on each pass.
#pragma once

#include "dsa_common.cuh"

namespace dsa {
namespace topk {

constexpr int THREADS = 512;
constexpr int WARPS = THREADS / 32;
constexpr int BINS = 2048;        // 11-bit digits
constexpr int CAND_CAP = 8192;    // candidates kept after the first digit
constexpr unsigned FULL = 0xffffffffu;

// Shared-memory bytes besides the staged row.
constexpr int FIXED_SMEM = BINS * 4 + CAND_CAP * 4 + 64 * 4;

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Smem {
    uint32_t *hist;      // [BINS]
    int *cand;           // [CAND_CAP]
    int *scal;           // small scalars
    uint32_t *row;       // [row_cap] staged keys (may be unused)
};

// Finds the digit bin holding the `remaining`-th largest key of the histogram.
// Writes bin and the count of keys in strictly higher bins to scal[0], scal[1].
__device__ __forceinline__ void select_bin(const uint32_t *hist, int nbins, int remaining, int *scal) {
    const int lane = threadIdx.x & 31;
    const int per = nbins / 32;                // bins per lane (64 or 32)
    // lane 0 owns the highest bins
    const int top = nbins - 1 - lane * per;
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) mine += hist[top - i];
    uint32_t incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        uint32_t v = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += v;
    }
    uint32_t above = incl - mine;              // keys in bins of lanes before mine
    bool here = (above < (uint32_t)remaining) && ((uint32_t)remaining <= incl);
    if (here) {
        uint32_t acc = above;
        for (int i = 0; i < per; ++i) {
            uint32_t h = hist[top - i];
            if (acc + h >= (uint32_t)remaining) {
                scal[0] = top - i;
                scal[1] = (int)acc;
                break;
            }
            acc += h;
        }
    }
}

template <bool STAGED>
__device__ __forceinline__ uint32_t key_at(const Smem &sm, const float *src, int i) {
    if (STAGED) return sm.row[i];
    return order_key(__ldg(src + i));
}

template <bool STAGED>
__device__ void select_row(const Smem &sm, const float *src, int n, int K, int32_t *out) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int *scal = sm.scal;
    // scal: [0] bin, [1] above, [2] ncand, [3..3+WARPS) gt counts, [3+WARPS..3+2W) eq counts

    // ---- digit 0: bits 31..21 over the whole row
    for (int i = tid; i < BINS; i += THREADS) sm.hist[i] = 0;
    if (tid == 0) scal[2] = 0;
    __syncthreads();
    const int n_pad = (n + 31) & ~31;
    for (int i = tid; i < n_pad; i += THREADS) {
        uint32_t d = i < n ? (key_at<STAGED>(sm, src, i) >> 21) : (uint32_t)BINS;
        unsigned peers = __match_any_sync(FULL, d);
        if (d < (uint32_t)BINS && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[d], (uint32_t)__popc(peers));
    }
    __syncthreads();
    if (warp == 0) select_bin(sm.hist, BINS, K, scal);
    __syncthreads();
    int remaining = K - scal[1];
    uint32_t prefix = (uint32_t)scal[0] << 21;
    uint32_t mask = 0xFFE00000u;
    __syncthreads();

    // ---- compact candidates that share digit 0
    for (int i = tid; i < n; i += THREADS) {
        if ((key_at<STAGED>(sm, src, i) & mask) == prefix) {
            int slot = atomicAdd(&scal[2], 1);
            if (slot < CAND_CAP) sm.cand[slot] = i;
        }
    }
    __syncthreads();
    const int ncand = scal[2];
    const bool use_cand = ncand <= CAND_CAP;

    // ---- digits 1 (bits 20..10) and 2 (bits 9..0)
    for (int pass = 1; pass <= 2; ++pass) {
        const int shift = pass == 1 ? 10 : 0;
        const int nb = pass == 1 ? 2048 : 1024;
        for (int i = tid; i < nb; i += THREADS) sm.hist[i] = 0;
        __syncthreads();
        const int m = use_cand ? ncand : n;
        const int m_pad = (m + 31) & ~31;
        for (int j = tid; j < m_pad; j += THREADS) {
            uint32_t d = (uint32_t)BINS;
            if (j < m) {
                int i = use_cand ? sm.cand[j] : j;
                uint32_t key = key_at<STAGED>(sm, src, i);
                if ((key & mask) == prefix) d = (key >> shift) & (uint32_t)(nb - 1);
            }
            unsigned peers = __match_any_sync(FULL, d);
            if (d < (uint32_t)BINS && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[d], (uint32_t)__popc(peers));
        }
        __syncthreads();
        if (warp == 0) select_bin(sm.hist, nb, remaining, scal);
        __syncthreads();
        remaining -= scal[1];
        prefix |= (uint32_t)scal[0] << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        __syncthreads();
    }
    const uint32_t thr = prefix;
    const int need_eq = remaining;       // >= 1
    const int count_gt = K - need_eq;

    // ---- ordered output: warp w owns the index range [w*R, min(n, (w+1)*R))
    const int R = ((n + WARPS * 32 - 1) / (WARPS * 32)) * 32;
    const int wb = warp * R;
    const int we = min(n, wb + R);
    int gt = 0, eq = 0;
    for (int base = wb; base < we; base += 32) {
        int i = base + lane;
        uint32_t key = i < we ? key_at<STAGED>(sm, src, i) : 0u;
        gt += __popc(__ballot_sync(FULL, i < we && key > thr));
        eq += __popc(__ballot_sync(FULL, i < we && key == thr));
    }
    if (lane == 0) {
        scal[3 + warp] = gt;
        scal[3 + WARPS + warp] = eq;
    }
    __syncthreads();
    int gt_off = 0, eq_off = 0;
    for (int w2 = 0; w2 < warp; ++w2) {
        gt_off += scal[3 + w2];
        eq_off += scal[3 + WARPS + w2];
    }
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = wb; base < we; base += 32) {
        int i = base + lane;
        uint32_t key = i < we ? key_at<STAGED>(sm, src, i) : 0u;
        unsigned bg = __ballot_sync(FULL, i < we && key > thr);
        unsigned be = __ballot_sync(FULL, i < we && key == thr);
        if (i < we && key > thr) {
            int slot = gt_off + __popc(bg & lt_mask);
            if (slot < count_gt) out[slot] = i;      // always true when the counts agree
        }
        if (i < we && key == thr) {
            int rank = eq_off + __popc(be & lt_mask);
            if (rank < need_eq && count_gt + rank < K) out[count_gt + rank] = i;
        }
        gt_off += __popc(bg);
        eq_off += __popc(be);
    }
}

// grid = row_count CTAs of THREADS threads; dynamic smem = FIXED_SMEM + row_cap*4.
__global__ void __launch_bounds__(THREADS) topk_rows_kernel(Problem P, const float *__restrict__ scores,
                                                            int64_t ld, int row_begin, int32_t *__restrict__ idx,
                                                            int row_cap) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem sm;
    sm.hist = reinterpret_cast<uint32_t *>(smem_raw);
    sm.cand = reinterpret_cast<int *>(smem_raw + BINS * 4);
    sm.scal = reinterpret_cast<int *>(smem_raw + BINS * 4 + CAND_CAP * 4);
    sm.row = reinterpret_cast<uint32_t *>(smem_raw + FIXED_SMEM);

    const int r = blockIdx.x;
    const int t = row_begin + r;
    const int K = P.topk;
    int32_t *out = idx + (int64_t)r * K;
    const RowInfo ri = row_info(P, t);
    const int n = visible_keys(ri);
    if (n <= K) {   // select all visible keys
        for (int j = threadIdx.x; j < K; j += THREADS) out[j] = j < n ? j : -1;
        return;
    }
    const float *src = scores + (int64_t)r * ld;
    if (n <= row_cap) {
        const int n4 = n >> 2;
        const float4 *s4 = reinterpret_cast<const float4 *>(src);
        for (int i = threadIdx.x; i < n4; i += THREADS) {
            float4 v = __ldg(s4 + i);
            uint4 k;
            k.x = order_key(v.x);
            k.y = order_key(v.y);
            k.z = order_key(v.z);
            k.w = order_key(v.w);
            reinterpret_cast<uint4 *>(sm.row)[i] = k;
        }
        for (int i = (n4 << 2) + threadIdx.x; i < n; i += THREADS) sm.row[i] = order_key(__ldg(src + i));
        __syncthreads();
        select_row<true>(sm, src, n, K, out);
    } else {
        select_row<false>(sm, src, n, K, out);
    }
}

}  // namespace topk
}  // namespace dsa
