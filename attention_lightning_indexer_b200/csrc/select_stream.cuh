// select_stream.cuh -- the selection half of the streaming indexer -> top-k (no score rows).
//
// "DeepSeek-V3.2 tech report summary", §1 DSA, ② fine-grained token selection: the top-k
// index scores of each query, exact, with the same tie rule and the same output layout as
// topk_rows_kernel (keys above the k-th key in ascending index order, then the keys equal
// to it that are taken, smallest indices first, in ascending index order).
//
// The indexer runs twice on the tensor cores: once over every SAMPLE_STRIDE-th key tile
// (a sample row per query), once over all tiles writing only the scores that reach a
// per-row threshold f_lo (an unordered candidate list).  In between,
// sample_threshold_kernel takes f_lo from the sample (the two-digit radix estimate of the
// top-k's fast path, with a wider margin: about 1.4 k keys of the row are expected to
// reach it).
// select_candidates_kernel then selects over the candidates.  This is exact whenever at
// least k keys reached f_lo and none was dropped: the k-th largest score is then >= f_lo,
// so every key that can be selected, ties included, is a candidate.  Otherwise the row is
// flagged, and the two-pass kernels (full score row, topk_rows_kernel) redo it.
#pragma once

#include "topk.cuh"

namespace dsa {
namespace topk {

constexpr int STREAM_NT = 256;
using StreamCfg = Cfg<STREAM_NT, 7168>;   // room for ~1.4 k candidates and long rows' samples
constexpr int STREAM_CAP = StreamCfg::WARPS * StreamCfg::SEG;          // candidates a row may hold
constexpr int STREAM_MAX_SAMPLES = 2 * StreamCfg::WARPS * StreamCfg::SEG;

// Exclusive block-wide prefix sum of v (all threads); wtot: WARPS ints of shared memory.
__device__ __forceinline__ int block_excl_scan(int v, int *wtot, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int wt;
    const int ex = warp_excl_scan(v, lane, wt);
    if (lane == 0) wtot[warp] = wt;
    __syncthreads();
    const int base = warp_sum(lane < warp ? wtot[lane] : 0);
    total = warp_sum(lane < StreamCfg::WARPS ? wtot[lane] : 0);
    __syncthreads();
    return base + ex;
}

// Writes the positions of the set bits of bits[0, nw) in ascending order to out[0, ..).
__device__ __forceinline__ void ordered_bits(const uint32_t *bits, int nw, int32_t *out, int *wtot) {
    const int per = (nw + STREAM_NT - 1) / STREAM_NT;
    const int w0 = min(nw, (int)threadIdx.x * per), w1 = min(nw, w0 + per);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(bits[w]);
    int total;
    int off = block_excl_scan(c, wtot, total);
    for (int w = w0; w < w1; ++w) {
        uint32_t b = bits[w];
        while (b != 0u) {
            const int bit = __ffs(b) - 1;
            out[off++] = w * 32 + bit;
            b &= b - 1u;
        }
    }
}

// grid = row_count CTAs of STREAM_NT threads, dynamic shared memory StreamCfg::SMEM.
// sample [rows, lds]: column j * 128 + c holds the score of key j * span + c, span =
// SAMPLE_STRIDE * 128; keys at or past the row's visible count are not valid.
__global__ void __launch_bounds__(STREAM_NT, 2)
sample_threshold_kernel(Problem P, const float *__restrict__ sample, int64_t lds, int span, int row_begin,
                        float *__restrict__ f_lo) {
    using C = StreamCfg;
    extern __shared__ __align__(16) unsigned char smem[];
    const int r = blockIdx.x, tid = threadIdx.x;
    const int K = P.topk;
    const RowInfo ri = row_info(P, row_begin + r);
    const int n = row_ok(P, ri) ? visible_keys(ri) : 0;
    if (n <= K) {   // every visible key is selected: no candidate is needed
        if (tid == 0) f_lo[r] = INFINITY;
        return;
    }
    const int ntile = (n + span - 1) / span;                 // sampled tiles holding a visible key
    const int ns = (ntile - 1) * 128 + min(128, n - (ntile - 1) * span);
    if (ns > STREAM_MAX_SAMPLES) {   // cannot happen within the host's size limit: take every key
        if (tid == 0) f_lo[r] = -INFINITY;
        return;
    }
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem + C::OFF_SEGK);   // spans both segment arrays
    const float *src = sample + (int64_t)r * lds;
    for (int i = tid; i < ns; i += STREAM_NT) keys[i] = order_key(__ldg(src + i));
    clear_hist<C>(smem, 0);
    __syncthreads();
    // about 1.4 k keys of the row are expected to reach the threshold: a row that falls
    // short of k is redone from full scores, which costs more than the extra candidates
    const int target = min(ns, (int)((1.4 * K * (double)ns) / (double)n) + 8);
    const int ns_pad = (ns + STREAM_NT - 1) / STREAM_NT * STREAM_NT;
    int dummy;
    const uint32_t t_lo = radix_select<C>(
        target,
        [&](auto fn) {
            for (int j = tid; j < ns_pad; j += STREAM_NT) fn(j < ns ? keys[j] : 0u, j < ns);
        },
        smem, &dummy, 2);
    if (tid == 0) f_lo[r] = key_float(t_lo);
}

// grid = row_count CTAs of STREAM_NT threads, dynamic shared memory StreamCfg::SMEM +
// 8 * nw_max bytes (two bitmaps of nw_max = ceil(max_len_k / 32) words).
// cand [rows, cap] holds cnt[r] candidates of row r (float bits of the score, key).
// Writes idx[r, :] and flag[r] = 0, or only flag[r] = 1 when the row must be redone.
__global__ void __launch_bounds__(STREAM_NT, 2)
select_candidates_kernel(Problem P, const int *__restrict__ cnt, const uint2 *__restrict__ cand, int cap,
                         int row_begin, int32_t *__restrict__ idx, uint8_t *__restrict__ flag) {
    using C = StreamCfg;
    extern __shared__ __align__(16) unsigned char smem[];
    const int r = blockIdx.x, tid = threadIdx.x;
    const int K = P.topk;
    int32_t *out = idx + (int64_t)r * K;
    const RowInfo ri = row_info(P, row_begin + r);
    const int n = row_ok(P, ri) ? visible_keys(ri) : 0;
    if (n <= K) {   // select every visible key
        for (int j = tid; j < K; j += STREAM_NT) out[j] = j < n ? j : -1;
        if (tid == 0) flag[r] = 0;
        return;
    }
    const int m = cnt[r];
    if (m < K || m > cap || m > STREAM_CAP) {   // the threshold misjudged this row
        if (tid == 0) flag[r] = 1;
        return;
    }
    if (tid == 0) flag[r] = 0;
    uint32_t *ck = reinterpret_cast<uint32_t *>(smem + C::OFF_SEGK);
    int *ci = reinterpret_cast<int *>(smem + C::OFF_SEGI);
    int *scal = reinterpret_cast<int *>(smem + C::OFF_SCAL);
    int *wtot = scal + 8;
    const int nw = (n + 31) / 32;
    uint32_t *gt = reinterpret_cast<uint32_t *>(smem + C::SMEM);
    uint32_t *eq = gt + nw;
    const uint2 *src = cand + (int64_t)r * cap;
    for (int j = tid; j < m; j += STREAM_NT) {
        const uint2 e = src[j];
        ck[j] = cand_key(e.x);
        ci[j] = (int)e.y;
    }
    for (int i = tid; i < 2 * nw; i += STREAM_NT) gt[i] = 0u;
    clear_hist<C>(smem, 0);
    __syncthreads();

    // ---- the k-th largest key among the candidates
    const int m_pad = (m + STREAM_NT - 1) / STREAM_NT * STREAM_NT;
    int above;
    const uint32_t thr = radix_select<C>(
        K,
        [&](auto fn) {
            for (int j = tid; j < m_pad; j += STREAM_NT) fn(j < m ? ck[j] : 0u, j < m);
        },
        smem, &above);
    const int need_eq = K - above;   // >= 1

    // ---- keys equal to it: all of them, or the need_eq smallest indices
    int e = 0;
    for (int j = tid; j < m; j += STREAM_NT) e += ck[j] == thr;
    int e_total;
    block_excl_scan(e, wtot, e_total);
    int idx_thr = 0x7fffffff;
    if (need_eq < e_total) {   // uniform
        clear_hist<C>(smem, 0);
        __syncthreads();
        int dummy;
        // the need_eq-th largest of ~index over the ties is the need_eq-th smallest index
        const uint32_t kmax = radix_select<C>(
            need_eq,
            [&](auto fn) {
                for (int j = tid; j < m_pad; j += STREAM_NT) {
                    const bool tie = j < m && ck[j] == thr;
                    fn(tie ? ~(uint32_t)ci[j] : 0u, tie);
                }
            },
            smem, &dummy);
        idx_thr = (int)~kmax;
    }

    // ---- bitmaps of the taken keys, then ordered writes
    for (int j = tid; j < m; j += STREAM_NT) {
        const uint32_t k = ck[j];
        const int i = ci[j];
        if (k > thr) atomicOr(gt + (i >> 5), 1u << (i & 31));
        else if (k == thr && i <= idx_thr) atomicOr(eq + (i >> 5), 1u << (i & 31));
    }
    __syncthreads();
    ordered_bits(gt, nw, out, wtot);
    ordered_bits(eq, nw, out + above, wtot);
}

}  // namespace topk
}  // namespace dsa
