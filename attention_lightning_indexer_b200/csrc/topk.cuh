// topk.cuh -- exact causal top-k per query row by radix selection.
//
// "DeepSeek-V3.2 tech report summary", §1 DSA, ② fine-grained token selection: keep the
// top-k index scores of each query; "Model techniques map -- DeepSeek-V3.2",
// Indexer-selected sparse attention: k_eff = min(index_topk, #candidates), int32 out.
//
// Scores map to order-preserving 32-bit keys (-0.0 folded onto +0.0), so comparing keys
// as unsigned integers compares the floats as values.  One CTA per row: 256 threads when
// there are many rows (several CTAs share an SM), 512 when a launch has fewer rows than
// SMs (decode), so a long row is not left to 8 warps.
//
// Fast path (one HBM read of the row):
//   * every 16th float4 of the row is sampled; a radix select on the sample (two 11-bit
//     digits) gives a key t_lo that about 1.2 k keys of the full row are expected to reach;
//   * one pass over the row keeps the keys >= t_lo with their indices, each warp in its
//     own shared-memory segment and in ascending index order (ballot prefix sums, no
//     atomics);
//   * an exact radix select (11/11/10-bit digits) over these candidates gives the k-th
//     largest key `thr` and how many keys equal to it are taken (smallest indices first);
//   * the candidates > thr and the first `need_eq` == thr are written in ascending index
//     order from per-warp offsets: deterministic, independent of the launch shape.
// If the sample misjudged (fewer than k candidates, or a warp's segment overflows) the
// general path runs instead: a full-row radix select with candidate compaction and an
// ordered final pass over the row (same result, more passes).
#pragma once

#include "dsa_common.cuh"

namespace dsa {
namespace topk {

constexpr int BINS = 2048;        // 11-bit digits
constexpr unsigned FULL = 0xffffffffu;

template <int NT>
struct Cfg {
    static constexpr int THREADS = NT;
    static constexpr int WARPS = NT / 32;
    static constexpr int SEG = 8192 / WARPS;                  // candidate slots per warp (fast path)
    static constexpr int CAND_CAP = WARPS * SEG * 2;          // general-path candidate indices (same bytes)
    // Dynamic shared memory layout.
    static constexpr int OFF_HIST = 0;                        // [BINS] u32
    static constexpr int OFF_SEGK = OFF_HIST + BINS * 4;      // [WARPS][SEG] u32 keys (also: samples)
    static constexpr int OFF_SEGI = OFF_SEGK + WARPS * SEG * 4;   // [WARPS][SEG] int indices
    static constexpr int OFF_SCAL = OFF_SEGI + WARPS * SEG * 4;   // scalars, see below
    // scal: [0..1] select_bin result, [2] candidate count, [3] overflow flag, then three
    // per-warp arrays A = scal + 8, B = A + WARPS, C = B + WARPS
    static constexpr int NSCAL = 8 + 3 * WARPS;
    static constexpr int SMEM = OFF_SCAL + NSCAL * 4;
    static_assert(CAND_CAP * 4 == 2 * WARPS * SEG * 4, "general-path candidates reuse both segment arrays");
    static_assert(NT % 32 == 0 && 2048 % (NT / 32) == 0, "whole warps; select_bin splits 2048 bins over 32 lanes");
};

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp-aggregated histogram increment; d == BINS means "no key" (lane still participates).
__device__ __forceinline__ void hist_add(uint32_t *hist, uint32_t d, int lane) {
    const unsigned peers = __match_any_sync(FULL, d);
    if (d < (uint32_t)BINS && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (uint32_t)__popc(peers));
}

// Warp 0: the bin holding the `remaining`-th largest key; writes bin and the count of
// keys in strictly higher bins to scal[0], scal[1].  Lane L first sums its block of
// nbins/32 consecutive bins (lane 0 owns the highest; the loop is skewed by the lane so the
// 32 lanes hit 32 different banks), a warp scan finds the lane whose block holds the
// target, and the warp then scans that block (per/32 bins per lane) to find the bin.
__device__ __forceinline__ void select_bin(const uint32_t *hist, int nbins, int remaining, int *scal) {
    const int lane = threadIdx.x & 31;
    const int per = nbins / 32;               // 64 or 32 bins per lane
    const int top = nbins - 1 - lane * per;   // lane 0 owns the highest bins
    uint32_t mine = 0;
    for (int i = 0; i < per; ++i) mine += hist[top - ((i + lane) & (per - 1))];
    uint32_t incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(FULL, incl, off);
        if (lane >= off) incl += v;
    }
    // the lane whose block holds the target (exactly one: remaining <= total keys)
    const unsigned hit = __ballot_sync(FULL, (incl - mine) < (uint32_t)remaining && (uint32_t)remaining <= incl);
    const int src = hit ? __ffs(hit) - 1 : 0;  // hit == 0 cannot happen (remaining <= count); stay in range
    const uint32_t above_blk = __shfl_sync(FULL, incl - mine, src);
    const int btop = nbins - 1 - src * per;
    // that block, highest bin first: lane l holds bins btop - l*q .. btop - l*q - (q-1), q = per/32
    const int q = per / 32;
    uint32_t h[2] = {0, 0};
    for (int j = 0; j < q; ++j) h[j] = hist[btop - lane * q - j];
    const uint32_t lsum = h[0] + (q > 1 ? h[1] : 0u);
    uint32_t lincl = lsum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(FULL, lincl, off);
        if (lane >= off) lincl += v;
    }
    const uint32_t lbefore = above_blk + lincl - lsum;
    const bool mine_hit = lbefore < (uint32_t)remaining && (uint32_t)remaining <= lbefore + lsum;
    if (hit != 0 && mine_hit) {
        if (lbefore + h[0] >= (uint32_t)remaining) {
            scal[0] = btop - lane * q;
            scal[1] = (int)lbefore;
        } else {
            scal[0] = btop - lane * q - 1;
            scal[1] = (int)(lbefore + h[0]);
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
__device__ __forceinline__ void load4(const float *src, int i0, int we, uint32_t (&k)[4]) {
    if (i0 + 3 < we) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(src + i0));
        k[0] = order_key(v.x);
        k[1] = order_key(v.y);
        k[2] = order_key(v.z);
        k[3] = order_key(v.w);
        return;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) k[c] = i0 + c < we ? order_key(__ldg(src + i0 + c)) : 0u;
}

// Exact radix selection (11/11/10-bit digits, MSB first) of the `rank`-th largest key among
// the keys get(j), j < m, for which valid(j) holds.  Returns the key; *above receives the
// number of keys strictly greater.  All threads call it; uses hist and scal[0..1].
// With passes == 2 the result is only a lower bound of that key: the smallest key of the
// 22-bit bin that holds it (enough for a candidate threshold).
template <class C, class Get>
__device__ uint32_t radix_select(int m, int rank, Get get, uint32_t *hist, int *scal, int *above, int passes = 3) {
    constexpr int THREADS = C::THREADS;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t prefix = 0, mask = 0;
    int remaining = rank, above_total = 0;
    const int m_pad = (m + 31) & ~31;
    for (int pass = 0; pass < passes; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int i = tid; i < nb; i += THREADS) hist[i] = 0;
        __syncthreads();
        for (int j = tid; j < m_pad; j += THREADS) {
            uint32_t d = (uint32_t)BINS, key = 0;
            if (j < m && get(j, key) && (key & mask) == prefix) d = (key >> shift) & (uint32_t)(nb - 1);
            hist_add(hist, d, lane);
        }
        __syncthreads();
        if (warp == 0) select_bin(hist, nb, remaining, scal);
        __syncthreads();
        remaining -= scal[1];
        above_total += scal[1];
        prefix |= (uint32_t)scal[0] << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        __syncthreads();
    }
    *above = above_total;
    return prefix;
}

// The same selection when each warp holds its own items: warp w's items are get(j),
// j < m_w (m_w differs per warp); every warp walks only its own items.
template <class C, class Get>
__device__ uint32_t radix_select_per_warp(int m_w, int rank, Get get, uint32_t *hist, int *scal, int *above) {
    constexpr int THREADS = C::THREADS;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t prefix = 0, mask = 0;
    int remaining = rank, above_total = 0;
    const int m_pad = (m_w + 31) & ~31;
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int i = tid; i < nb; i += THREADS) hist[i] = 0;
        __syncthreads();
        for (int j = lane; j < m_pad; j += 32) {
            uint32_t d = (uint32_t)BINS;
            if (j < m_w) {
                const uint32_t key = get(j);
                if ((key & mask) == prefix) d = (key >> shift) & (uint32_t)(nb - 1);
            }
            hist_add(hist, d, lane);
        }
        __syncthreads();
        if (warp == 0) select_bin(hist, nb, remaining, scal);
        __syncthreads();
        remaining -= scal[1];
        above_total += scal[1];
        prefix |= (uint32_t)scal[0] << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        __syncthreads();
    }
    *above = above_total;
    return prefix;
}

// Warp w writes, in ascending index order, the keys of its range [wb, we) of the row that
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

// Fast path.  Returns false (nothing written) when the sample misjudged the row.
template <class C>
__device__ bool select_row_sampled(const float *src, int n, int K, unsigned char *smem, int32_t *out) {
    constexpr int THREADS = C::THREADS, WARPS = C::WARPS, SEG = C::SEG;
    constexpr int OFF_HIST = C::OFF_HIST, OFF_SEGK = C::OFF_SEGK, OFF_SEGI = C::OFF_SEGI, OFF_SCAL = C::OFF_SCAL;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem + OFF_HIST);
    uint32_t *segk = reinterpret_cast<uint32_t *>(smem + OFF_SEGK);
    int *segi = reinterpret_cast<int *>(smem + OFF_SEGI);
    int *scal = reinterpret_cast<int *>(smem + OFF_SCAL);
    int *seg_cnt = scal + 8, *wgt = scal + 8 + WARPS, *weq = scal + 8 + 2 * WARPS;
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    const int n4 = n >> 2;
    const int nsamp4 = (n4 + 15) / 16;                       // sampled float4 (every 16th)
    const int ns = 4 * nsamp4;
    if (ns < 64 || ns > WARPS * SEG) return false;

    // ---- sample keys into the segment key array (free at this point)
    for (int m = tid; m < nsamp4; m += THREADS) {
        const float4 v = __ldg(s4 + 16 * m);
        segk[4 * m + 0] = order_key(v.x);
        segk[4 * m + 1] = order_key(v.y);
        segk[4 * m + 2] = order_key(v.z);
        segk[4 * m + 3] = order_key(v.w);
    }
    if (tid < WARPS) seg_cnt[tid] = 0;
    if (tid == 0) scal[3] = 0;
    __syncthreads();
    const int target = min(ns, (int)((1.2 * K * (double)ns) / (double)n) + 16);
    int dummy;
    // a lower bound of the sample's target-th key is all the candidate pass needs: two
    // digit passes (22 bits)
    const uint32_t t_lo = radix_select<C>(
        ns, target, [&](int j, uint32_t &key) { key = segk[j]; return true; }, hist, scal, &dummy, 2);
    __syncthreads();   // samples no longer needed

    // ---- candidates: keys >= t_lo, per warp in ascending index order
    const int R = ((n + WARPS * 128 - 1) / (WARPS * 128)) * 128;
    const int wb = warp * R, we = min(n, wb + R);
    uint32_t *mk = segk + warp * SEG;
    int *mi = segi + warp * SEG;
    int cnt = 0;
    bool overflow = false;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = wb; base < we; base += 512) {
        // 16 coalesced loads per lane, keys base + 32 j + lane: the order (j, lane) is the
        // index order, so ballot prefix counts keep the segment sorted by index
        uint32_t kk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int i = base + 32 * j + lane;
            kk[j] = i < we ? order_key(__ldg(src + i)) : 0u;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int i = base + 32 * j + lane;
            const bool take = i < we && kk[j] >= t_lo;
            const unsigned m = __ballot_sync(FULL, take);
            if (take) {
                const int off = cnt + __popc(m & lt);
                if (off < SEG) {
                    mk[off] = kk[j];
                    mi[off] = i;
                }
            }
            cnt += __popc(m);
        }
    }
    overflow = cnt > SEG;
    if (lane == 0) {
        seg_cnt[warp] = overflow ? 0 : cnt;
        if (overflow) scal[3] = 1;
    }
    __syncthreads();
    int total = 0;
    for (int w = 0; w < WARPS; ++w) total += seg_cnt[w];
    if (scal[3] != 0 || total < K) return false;   // uniform decision

    // ---- exact k-th largest among the candidates
    int above;
    const uint32_t thr = radix_select_per_warp<C>(cnt, K, [&](int j) { return mk[j]; }, hist, scal, &above);
    const int need_eq = K - above;                   // >= 1
    const int count_gt = above;

    // ---- per-warp counts of > thr and == thr, then ordered writes
    int cg = 0, ce = 0;
    for (int j = lane; j < cnt; j += 32) {
        cg += mk[j] > thr;
        ce += mk[j] == thr;
    }
    cg = warp_sum(cg);
    ce = warp_sum(ce);
    __syncthreads();
    if (lane == 0) {
        wgt[warp] = cg;
        weq[warp] = ce;
    }
    __syncthreads();
    int gt_off = 0, eq_off = 0;
    for (int w2 = 0; w2 < warp; ++w2) {
        gt_off += wgt[w2];
        eq_off += weq[w2];
    }
    for (int base = 0; base < cnt; base += 32) {
        const int j = base + lane;
        const uint32_t key = j < cnt ? mk[j] : 0u;
        const bool g = j < cnt && key > thr, e = j < cnt && key == thr;
        const unsigned bg = __ballot_sync(FULL, g), be = __ballot_sync(FULL, e);
        if (g) {
            const int slot = gt_off + __popc(bg & lt);
            if (slot < count_gt) out[slot] = mi[j];
        }
        if (e) {
            const int rank = eq_off + __popc(be & lt);
            if (rank < need_eq && count_gt + rank < K) out[count_gt + rank] = mi[j];
        }
        gt_off += __popc(bg);
        eq_off += __popc(be);
    }
    return true;
}

// General path: full radix selection over the row.
template <class C>
__device__ void select_row_general(const float *src, int n, int K, unsigned char *smem, int32_t *out) {
    constexpr int THREADS = C::THREADS, WARPS = C::WARPS, CAND_CAP = C::CAND_CAP;
    constexpr int OFF_HIST = C::OFF_HIST, OFF_SEGK = C::OFF_SEGK, OFF_SCAL = C::OFF_SCAL;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem + OFF_HIST);
    int *cand = reinterpret_cast<int *>(smem + OFF_SEGK);   // CAND_CAP entries over both segment arrays
    int *scal = reinterpret_cast<int *>(smem + OFF_SCAL);
    // per warp: keys above bin b0, keys in b0 above thr, keys == thr
    int *w_above = scal + 8, *w_gt = scal + 8 + WARPS, *w_eq = scal + 8 + 2 * WARPS;
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    const int n4 = n >> 2;
    const int R = ((n + WARPS * 128 - 1) / (WARPS * 128)) * 128;
    const int wb = warp * R, we = min(n, wb + R);

    __syncthreads();
    for (int i = tid; i < BINS; i += THREADS) hist[i] = 0;
    for (int i = tid; i < 3 * WARPS; i += THREADS) scal[8 + i] = 0;
    if (tid == 0) scal[2] = 0;
    __syncthreads();

    // ---- pass 1: histogram of bits 31..21 over the whole row
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
            hist_add(hist, ok ? order_key(v[u].x) >> 21 : (uint32_t)BINS, lane);
            hist_add(hist, ok ? order_key(v[u].y) >> 21 : (uint32_t)BINS, lane);
            hist_add(hist, ok ? order_key(v[u].z) >> 21 : (uint32_t)BINS, lane);
            hist_add(hist, ok ? order_key(v[u].w) >> 21 : (uint32_t)BINS, lane);
        }
    }
    {
        const int tail = n - (n4 << 2);
        if (tid < tail) atomicAdd(&hist[order_key(__ldg(src + (n4 << 2) + tid)) >> 21], 1u);
    }
    __syncthreads();
    if (warp == 0) select_bin(hist, BINS, K, scal);
    __syncthreads();
    const uint32_t b0 = (uint32_t)scal[0];
    int remaining = K - scal[1];
    __syncthreads();

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
                    const int slot = atomicAdd(&scal[2], 1);
                    if (slot < CAND_CAP) cand[slot] = i0 + c;
                }
            }
        }
        g0 = warp_sum(g0);
        if (lane == 0) w_above[warp] = g0;
    }
    __syncthreads();
    const int ncand = scal[2];
    const bool use_cand = ncand <= CAND_CAP;

    // ---- digits 2 and 3 on the candidates (or on the whole row after an overflow)
    uint32_t prefix = b0 << 21, mask = 0xFFE00000u;
    for (int pass = 1; pass <= 2; ++pass) {
        const int shift = pass == 1 ? 10 : 0;
        const int nb = pass == 1 ? 2048 : 1024;
        for (int i = tid; i < nb; i += THREADS) hist[i] = 0;
        __syncthreads();
        const int m = use_cand ? ncand : n;
        const int m_pad = (m + 31) & ~31;
        for (int j = tid; j < m_pad; j += THREADS) {
            uint32_t d = (uint32_t)BINS;
            if (j < m) {
                const uint32_t key = order_key(__ldg(src + (use_cand ? cand[j] : j)));
                if ((key & mask) == prefix) d = (key >> shift) & (uint32_t)(nb - 1);
            }
            hist_add(hist, d, lane);
        }
        __syncthreads();
        if (warp == 0) select_bin(hist, nb, remaining, scal);
        __syncthreads();
        remaining -= scal[1];
        prefix |= (uint32_t)scal[0] << shift;
        mask |= (uint32_t)(nb - 1) << shift;
        __syncthreads();
    }
    const uint32_t thr = prefix;
    const int need_eq = remaining;       // >= 1
    const int count_gt = K - need_eq;

    // ---- per-warp counts of the keys > thr and == thr inside bin b0
    if (use_cand) {
        for (int j = tid; j < ncand; j += THREADS) {
            const int i = cand[j];
            const uint32_t key = order_key(__ldg(src + i));
            if (key > thr) atomicAdd(&w_gt[i / R], 1);
            else if (key == thr) atomicAdd(&w_eq[i / R], 1);
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
            w_gt[warp] = cg;
            w_eq[warp] = ce;
        }
    }
    __syncthreads();
    int gt_off = 0, eq_off = 0;
    for (int w2 = 0; w2 < warp; ++w2) {
        gt_off += w_above[w2] + w_gt[w2];
        eq_off += w_eq[w2];
    }
    ordered_output(src, wb, we, lane, thr, need_eq, count_gt, K, gt_off, eq_off, out);
}

// grid = row_count CTAs of NT threads, dynamic shared memory Cfg<NT>::SMEM bytes.
template <int NT>
__global__ void __launch_bounds__(NT, NT >= 512 ? 1 : 3) topk_rows_kernel(Problem P, const float *__restrict__ scores, int64_t ld,
                                                       int row_begin, int32_t *__restrict__ idx) {
    using C = Cfg<NT>;
    extern __shared__ __align__(16) unsigned char smem[];
    const int r = blockIdx.x;
    const int K = P.topk;
    int32_t *out = idx + (int64_t)r * K;
    const RowInfo ri = row_info(P, row_begin + r);
    const int n = row_ok(P, ri) ? visible_keys(ri) : 0;
    if (n <= K) {   // select every visible key
        for (int j = threadIdx.x; j < K; j += NT) out[j] = j < n ? j : -1;
        return;
    }
    const float *src = scores + (int64_t)r * ld;
    if (!select_row_sampled<C>(src, n, K, smem, out)) select_row_general<C>(src, n, K, smem, out);
}

}  // namespace topk
}  // namespace dsa
