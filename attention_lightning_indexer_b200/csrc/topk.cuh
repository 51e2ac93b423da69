// topk.cuh -- exact causal top-k per query row by radix selection.
//
// "DeepSeek-V3.2 tech report summary", §1 DSA, ② fine-grained token selection: keep the
// top-k index scores of each query; "Model techniques map -- DeepSeek-V3.2",
// Indexer-selected sparse attention: k_eff = min(index_topk, #candidates), int32 out.
//
// Design (one 256-thread CTA per query row; HBM-bound, several CTAs per SM):
//   * scores map to order-preserving 32-bit keys (-0.0 folded onto +0.0), so comparing
//     keys as unsigned integers compares the floats as values;
//   * pass 1 (the only HBM read of the row): histogram of the top 11 key bits, 4 float4
//     loads in flight per thread, warp-aggregated shared atomics (match.any);
//   * the bin holding the k-th largest key is found; pass 2 (an L2 re-read) counts, per
//     warp range, the keys in higher bins (certainly selected) and compacts the indices
//     of the keys in that bin (the candidates) into shared memory;
//   * digits 2 (bits 20..10) and 3 (bits 9..0) are resolved on the candidates only,
//     giving the exact k-th largest key `thr` and the number `need_eq` of keys equal to
//     it that are taken (smallest indices first);
//   * pass 3 (an L2 re-read) writes, in ascending index order, every key > thr followed
//     by the first need_eq keys == thr, from per-warp offsets and in-warp prefix sums:
//     the output is deterministic and independent of the launch shape.
// When the candidates overflow the shared buffer (e.g. a row of identical scores) the
// later digits and the per-warp counts are taken from the row itself instead (slower,
// same result).
#pragma once

#include "dsa_common.cuh"

namespace dsa {
namespace topk {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int BINS = 2048;        // 11-bit digits
constexpr int CAND_CAP = 6144;    // candidates kept after the first digit
constexpr unsigned FULL = 0xffffffffu;

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Smem {
    uint32_t hist[BINS];
    int cand[CAND_CAP];
    int warp_gt0[WARPS];   // keys whose first digit is above the threshold bin, per warp range
    int warp_gt[WARPS];    // candidates above thr, per warp range
    int warp_eq[WARPS];    // candidates equal to thr, per warp range
    int scal[8];           // [0] bin  [1] above  [2] ncand
};

// Warp-aggregated histogram increment; d == BINS means "no key" (lane still participates).
__device__ __forceinline__ void hist_add(uint32_t *hist, uint32_t d, int lane) {
    const unsigned peers = __match_any_sync(FULL, d);
    if (d < (uint32_t)BINS && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (uint32_t)__popc(peers));
}

// Warp 0: the bin holding the `remaining`-th largest key; writes bin and the count of
// keys in strictly higher bins to scal[0], scal[1].
__device__ __forceinline__ void select_bin(const uint32_t *hist, int nbins, int remaining, int *scal) {
    const int lane = threadIdx.x & 31;
    const int per = nbins / 32;
    const int top = nbins - 1 - lane * per;   // lane 0 owns the highest bins
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) mine += hist[top - i];
    uint32_t incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += v;
    }
    const uint32_t above = incl - mine;
    if (above < (uint32_t)remaining && (uint32_t)remaining <= incl) {
        uint32_t acc = above;
        for (int i = 0; i < per; ++i) {
            const uint32_t h = hist[top - i];
            if (acc + h >= (uint32_t)remaining) {
                scal[0] = top - i;
                scal[1] = (int)acc;
                break;
            }
            acc += h;
        }
    }
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(FULL, v, off);
    return v;
}

__device__ __forceinline__ int warp_excl_scan(int v, int lane, int &total) {
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int x = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += x;
    }
    total = __shfl_sync(FULL, incl, 31);
    return incl - v;
}

// The lane's 4 consecutive keys i0..i0+3 of the warp range [.., we); invalid ones get 0.
__device__ __forceinline__ int load4(const float *src, int i0, int we, uint32_t (&k)[4]) {
    if (i0 + 3 < we) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(src + i0));
        k[0] = order_key(v.x);
        k[1] = order_key(v.y);
        k[2] = order_key(v.z);
        k[3] = order_key(v.w);
        return 4;
    }
    int nv = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        k[c] = 0u;
        if (i0 + c < we) {
            k[c] = order_key(__ldg(src + i0 + c));
            ++nv;
        }
    }
    return nv;
}

// Pass 3: warp w writes, in ascending index order, the keys of its range [wb, we) that
// are > thr (from slot gt_off on) and those == thr whose rank among equal keys is below
// need_eq (from slot count_gt + eq_off on).
__device__ __forceinline__ void ordered_output(const float *src, int wb, int we, int lane, uint32_t thr, int need_eq,
                                               int count_gt, int K, int gt_off, int eq_off, int32_t *out) {
    for (int base = wb; base < we; base += 128) {
        const int i0 = base + lane * 4;
        uint32_t k[4];
        load4(src, i0, we, k);
        int cg = 0, ce = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const bool v = i0 + c < we;
            cg += v && k[c] > thr;
            ce += v && k[c] == thr;
        }
        int tg, te;
        int og = warp_excl_scan(cg, lane, tg) + gt_off;
        int oe = warp_excl_scan(ce, lane, te) + eq_off;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (i0 + c >= we) continue;
            if (k[c] > thr) {
                if (og < count_gt) out[og] = i0 + c;
                ++og;
            } else if (k[c] == thr) {
                if (oe < need_eq && count_gt + oe < K) out[count_gt + oe] = i0 + c;
                ++oe;
            }
        }
        gt_off += tg;
        eq_off += te;
    }
}

__global__ void __launch_bounds__(THREADS) topk_rows_kernel(Problem P, const float *__restrict__ scores, int64_t ld,
                                                            int row_begin, int32_t *__restrict__ idx) {
    __shared__ Smem sm;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = blockIdx.x;
    const int K = P.topk;
    int32_t *out = idx + (int64_t)r * K;
    const RowInfo ri = row_info(P, row_begin + r);
    const int n = visible_keys(ri);
    if (n <= K) {   // select every visible key
        for (int j = tid; j < K; j += THREADS) out[j] = j < n ? j : -1;
        return;
    }
    const float *src = scores + (int64_t)r * ld;
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    const int n4 = n >> 2;
    const int R = ((n + WARPS * 128 - 1) / (WARPS * 128)) * 128;   // warp range, multiple of 128
    const int wb = warp * R;
    const int we = min(n, wb + R);

    // ---- fast path: a sample fixes a lower digit bound; only keys at or above it are counted
    for (int i = tid; i < BINS; i += THREADS) sm.hist[i] = 0;
    if (tid < WARPS) {
        sm.warp_gt[tid] = 0;
        sm.warp_eq[tid] = 0;
    }
    if (tid < 8) sm.scal[tid] = 0;
    __syncthreads();
    int ns = 0;                                            // sampled keys (every 16th float4)
    for (int m = tid; 16 * m < n4; m += THREADS) {
        const float4 v = __ldg(s4 + 16 * m);
        atomicAdd(&sm.hist[order_key(v.x) >> 21], 1u);
        atomicAdd(&sm.hist[order_key(v.y) >> 21], 1u);
        atomicAdd(&sm.hist[order_key(v.z) >> 21], 1u);
        atomicAdd(&sm.hist[order_key(v.w) >> 21], 1u);
    }
    ns = 4 * ((n4 + 15) / 16);
    __syncthreads();
    if (warp == 0) {
        // lowest bin b_lo whose sampled tail covers ~1.5 K keys of the full row (+ margin)
        const uint32_t target = (uint32_t)((1.5 * K * (double)ns) / (double)n) + 16u;
        select_bin(sm.hist, BINS, (int)min(target, (uint32_t)ns), sm.scal);   // scal[0] = b_lo
    }
    __syncthreads();
    const uint32_t b_lo = (uint32_t)sm.scal[0];
    __syncthreads();
    for (int i = tid; i < BINS; i += THREADS) sm.hist[i] = 0;
    if (tid == 0) sm.scal[2] = 0;
    __syncthreads();
    {
        for (int base = 0; base < n4; base += THREADS * 4) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = base + u * THREADS + tid;
                v[u] = i < n4 ? __ldg(s4 + i) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i4 = base + u * THREADS + tid;
                const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t key = order_key(e[c]);
                    const bool is = i4 < n4 && (key >> 21) >= b_lo;
                    const unsigned bal = __ballot_sync(FULL, is);
                    if (bal) {
                        int slot0 = 0;
                        if (lane == __ffs(bal) - 1) slot0 = atomicAdd(&sm.scal[2], __popc(bal));
                        slot0 = __shfl_sync(FULL, slot0, __ffs(bal) - 1);
                        if (is) {
                            const int slot = slot0 + __popc(bal & ((1u << lane) - 1u));
                            if (slot < CAND_CAP) sm.cand[slot] = 4 * i4 + c;
                            atomicAdd(&sm.hist[key >> 21], 1u);
                        }
                    }
                }
            }
        }
        const int tail = n - (n4 << 2);
        if (tid < tail) {
            const int i = (n4 << 2) + tid;
            const uint32_t key = order_key(__ldg(src + i));
            if ((key >> 21) >= b_lo) {
                const int slot = atomicAdd(&sm.scal[2], 1);
                if (slot < CAND_CAP) sm.cand[slot] = i;
                atomicAdd(&sm.hist[key >> 21], 1u);
            }
        }
    }
    __syncthreads();
    const int ncand_fast = sm.scal[2];
    const bool fast = ncand_fast >= K && ncand_fast <= CAND_CAP;
    if (fast) {
        // exact digits 1..3 on the candidates (bins below b_lo hold no count)
        if (warp == 0) select_bin(sm.hist, BINS, K, sm.scal);
        __syncthreads();
        int remaining = K - sm.scal[1];
        uint32_t prefix = (uint32_t)sm.scal[0] << 21, mask = 0xFFE00000u;
        __syncthreads();
        for (int pass = 1; pass <= 2; ++pass) {
            const int shift = pass == 1 ? 10 : 0;
            const int nb = pass == 1 ? 2048 : 1024;
            for (int i = tid; i < nb; i += THREADS) sm.hist[i] = 0;
            __syncthreads();
            const int m_pad = (ncand_fast + 31) & ~31;
            for (int j = tid; j < m_pad; j += THREADS) {
                uint32_t d = (uint32_t)BINS;
                if (j < ncand_fast) {
                    const uint32_t key = order_key(__ldg(src + sm.cand[j]));
                    if ((key & mask) == prefix) d = (key >> shift) & (uint32_t)(nb - 1);
                }
                hist_add(sm.hist, d, lane);
            }
            __syncthreads();
            if (warp == 0) select_bin(sm.hist, nb, remaining, sm.scal);
            __syncthreads();
            remaining -= sm.scal[1];
            prefix |= (uint32_t)sm.scal[0] << shift;
            mask |= (uint32_t)(nb - 1) << shift;
            __syncthreads();
        }
        const uint32_t thr = prefix;
        const int need_eq = remaining;
        const int count_gt = K - need_eq;
        // every key > thr is a candidate: per-warp-range counts from the candidate list
        for (int j = tid; j < ncand_fast; j += THREADS) {
            const int i = sm.cand[j];
            const uint32_t key = order_key(__ldg(src + i));
            if (key > thr) atomicAdd(&sm.warp_gt[i / R], 1);
            else if (key == thr) atomicAdd(&sm.warp_eq[i / R], 1);
        }
        __syncthreads();
        int gt_off = 0, eq_off = 0;
        for (int w2 = 0; w2 < warp; ++w2) {
            gt_off += sm.warp_gt[w2];
            eq_off += sm.warp_eq[w2];
        }
        ordered_output(src, wb, we, lane, thr, need_eq, count_gt, K, gt_off, eq_off, out);
        return;
    }
    // ---- general path (the sample was not representative): full radix selection
    for (int i = tid; i < BINS; i += THREADS) sm.hist[i] = 0;
    if (tid < WARPS) {
        sm.warp_gt[tid] = 0;
        sm.warp_eq[tid] = 0;
    }
    if (tid == 0) sm.scal[2] = 0;
    __syncthreads();

    // ---- pass 1: histogram of bits 31..21
    {
        for (int base = 0; base < n4; base += THREADS * 4) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = base + u * THREADS + tid;
                v[u] = i < n4 ? __ldg(s4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const bool ok = base + u * THREADS + tid < n4;
                hist_add(sm.hist, ok ? order_key(v[u].x) >> 21 : (uint32_t)BINS, lane);
                hist_add(sm.hist, ok ? order_key(v[u].y) >> 21 : (uint32_t)BINS, lane);
                hist_add(sm.hist, ok ? order_key(v[u].z) >> 21 : (uint32_t)BINS, lane);
                hist_add(sm.hist, ok ? order_key(v[u].w) >> 21 : (uint32_t)BINS, lane);
            }
        }
        const int tail = n - (n4 << 2);
        if (tid < tail) atomicAdd(&sm.hist[order_key(__ldg(src + (n4 << 2) + tid)) >> 21], 1u);
    }
    __syncthreads();
    if (warp == 0) select_bin(sm.hist, BINS, K, sm.scal);
    __syncthreads();
    const uint32_t b0 = (uint32_t)sm.scal[0];
    int remaining = K - sm.scal[1];

    // ---- pass 2: per-warp count of keys above bin b0, compaction of the keys in b0
    {
        int g0 = 0;
        for (int base = wb; base < we; base += 128) {
            const int i0 = base + lane * 4;
            uint32_t k[4];
            load4(src, i0, we, k);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (i0 + c >= we) continue;
                const uint32_t d = k[c] >> 21;
                if (d > b0) {
                    ++g0;
                } else if (d == b0) {
                    const int slot = atomicAdd(&sm.scal[2], 1);
                    if (slot < CAND_CAP) sm.cand[slot] = i0 + c;
                }
            }
        }
        g0 = warp_sum(g0);
        if (lane == 0) sm.warp_gt0[warp] = g0;
    }
    __syncthreads();
    const int ncand = sm.scal[2];
    const bool use_cand = ncand <= CAND_CAP;

    // ---- digits 2 and 3 on the candidates (or on the whole row after an overflow)
    uint32_t prefix = b0 << 21, mask = 0xFFE00000u;
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
                const uint32_t key = order_key(__ldg(src + (use_cand ? sm.cand[j] : j)));
                if ((key & mask) == prefix) d = (key >> shift) & (uint32_t)(nb - 1);
            }
            hist_add(sm.hist, d, lane);
        }
        __syncthreads();
        if (warp == 0) select_bin(sm.hist, nb, remaining, sm.scal);
        __syncthreads();
        remaining -= sm.scal[1];
        prefix |= (uint32_t)sm.scal[0] << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        __syncthreads();
    }
    const uint32_t thr = prefix;
    const int need_eq = remaining;       // >= 1
    const int count_gt = K - need_eq;

    // ---- per-warp counts of the keys > thr and == thr inside bin b0
    if (use_cand) {
        for (int j = tid; j < ncand; j += THREADS) {
            const int i = sm.cand[j];
            const uint32_t key = order_key(__ldg(src + i));
            if (key > thr) atomicAdd(&sm.warp_gt[i / R], 1);
            else if (key == thr) atomicAdd(&sm.warp_eq[i / R], 1);
        }
    } else {
        int cg = 0, ce = 0;
        for (int base = wb; base < we; base += 128) {
            const int i0 = base + lane * 4;
            uint32_t k[4];
            load4(src, i0, we, k);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (i0 + c >= we || (k[c] >> 21) != b0) continue;
                cg += k[c] > thr;
                ce += k[c] == thr;
            }
        }
        cg = warp_sum(cg);
        ce = warp_sum(ce);
        if (lane == 0) {
            sm.warp_gt[warp] = cg;
            sm.warp_eq[warp] = ce;
        }
    }
    __syncthreads();
    int gt_off0 = 0, eq_off0 = 0;
    for (int w2 = 0; w2 < warp; ++w2) {
        gt_off0 += sm.warp_gt0[w2] + sm.warp_gt[w2];
        eq_off0 += sm.warp_eq[w2];
    }
    ordered_output(src, wb, we, lane, thr, need_eq, count_gt, K, gt_off0, eq_off0, out);
}

}  // namespace topk
}  // namespace dsa
