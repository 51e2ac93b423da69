// topk.cuh -- exact causal top-k per query row by radix selection.
//
// "DeepSeek-V3.2 tech report summary", §1 DSA, ② fine-grained token selection: keep the
// top-k index scores of each query; "Model techniques map -- DeepSeek-V3.2",
// Indexer-selected sparse attention: k_eff = min(index_topk, #candidates), int32 out.
//
// Scores map to order-preserving 32-bit keys (-0.0 folded onto +0.0), so comparing keys
// as unsigned integers compares the floats as values.  One CTA per row: 256 threads when
// there are many rows (four CTAs share an SM), 1024 when a launch has fewer rows than
// SMs (decode), so a long row is not left to 8 warps.
//
// Fast path (one HBM read of the row):
//   * every 16th float4 of the row is sampled; a radix select on the sample (two 11-bit
//     digits) gives a key t_lo that about 1.2 k keys of the full row are expected to reach;
//   * one pass over the row (float4 loads, the next chunk in flight while the current one
//     is filtered) keeps the scores >= t_lo (as raw float bits) with their indices, each
//     warp in its own shared-memory segment and in ascending index order (ballot prefix
//     sums, predicated stores, no atomics);
//   * an exact radix select (11/11/10-bit digits) over these candidates gives the k-th
//     largest key `thr` and how many keys equal to it are taken (smallest indices first);
//   * the candidates > thr and the first `need_eq` == thr are written in ascending index
//     order from per-warp offsets: deterministic, independent of the launch shape.
// If the sample misjudged (fewer than k candidates, or a warp's segment overflows) the
// general path runs instead: a full-row radix select with candidate compaction and an
// ordered final pass over the row (same result, more passes).
//
// Every digit pass takes two block barriers: the histograms are double-buffered (a pass
// clears the other buffer for the next pass while it counts), and the bin holding the
// target rank is found from 32 group sums kept beside each histogram (two dependent
// shared-memory loads per lane instead of a walk over 64 bins).
#pragma once

#include "dsa_common.cuh"

namespace dsa {
namespace topk {

constexpr int BINS = 2048;        // 11-bit digits
constexpr int GROUPS = 32;        // group sums per histogram (one per lane of the bin search)
constexpr unsigned FULL = 0xffffffffu;

// NT threads; CAP candidate slots in all (about 1.2 k = 2.5 K are expected per row).  The
// 256-thread shape keeps 4096, so that four CTAs share an SM (49.5 KB of shared memory each).
template <int NT, int CAP = (NT >= 512 ? 7168 : 4096)>
struct Cfg {
    static constexpr int THREADS = NT;
    static constexpr int WARPS = NT / 32;
    static constexpr int SEG = CAP / WARPS;                   // candidate slots per warp (fast path)
    static constexpr int CAND_CAP = WARPS * SEG * 2;          // general-path candidate indices (same bytes)
    // Dynamic shared memory layout.
    static constexpr int OFF_HIST = 0;                             // [2][BINS] u32
    static constexpr int OFF_GRP = OFF_HIST + 2 * BINS * 4;        // [2][GROUPS] u32
    static constexpr int OFF_SEGK = OFF_GRP + 2 * GROUPS * 4;      // [WARPS][SEG] u32 keys
    static constexpr int OFF_SEGI = OFF_SEGK + WARPS * SEG * 4;    // [WARPS][SEG] int indices
    // (the samples of the fast path, up to 2 * WARPS * SEG keys, span both arrays)
    static constexpr int OFF_SCAL = OFF_SEGI + WARPS * SEG * 4;    // scalars, see below
    // scal: [0..1] and [4..5] digit-pass results (by pass parity), [2] candidate count,
    // [3] overflow flag, then three per-warp arrays A = scal + 8, B = A + WARPS, C = B + WARPS
    static constexpr int NSCAL = 8 + 3 * WARPS;
    static constexpr int SMEM = OFF_SCAL + NSCAL * 4;
    static_assert(CAP % WARPS == 0 && NT % 32 == 0, "whole warps, equal segments");
    static_assert(CAND_CAP * 4 == 2 * WARPS * SEG * 4, "general-path candidates reuse both segment arrays");
};

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float whose key is k (inverse of order_key; key 0x80000000 gives +0.0).  For finite
// v: order_key(v) >= k  <=>  v >= key_float(k), signed zeros included.
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Histogram buffers of parity p.
template <class C>
__device__ __forceinline__ uint32_t *hist_of(unsigned char *smem, int p) {
    return reinterpret_cast<uint32_t *>(smem + C::OFF_HIST) + p * BINS;
}
template <class C>
__device__ __forceinline__ uint32_t *grp_of(unsigned char *smem, int p) {
    return reinterpret_cast<uint32_t *>(smem + C::OFF_GRP) + p * GROUPS;
}

// Clears the histogram and group sums of parity p (all threads).
template <class C>
__device__ __forceinline__ void clear_hist(unsigned char *smem, int p) {
    uint4 *h = reinterpret_cast<uint4 *>(hist_of<C>(smem, p));
    for (int i = threadIdx.x; i < BINS / 4; i += C::THREADS) h[i] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x < GROUPS) grp_of<C>(smem, p)[threadIdx.x] = 0u;
}

// Count of digit d (d >= NB: no key; the lane still takes part) into the bin and its group
// (NB / GROUPS consecutive bins).  A warp whose lanes all hold one digit (a run of equal
// keys) adds 32 with one atomic; otherwise each lane adds its own.
template <int NB>
__device__ __forceinline__ void hist_add(uint32_t *hist, uint32_t *grp, uint32_t d, int lane) {
    constexpr uint32_t PER = NB / GROUPS;
    const uint32_t d0 = __shfl_sync(FULL, d, 0);
    if (__all_sync(FULL, d == d0)) {
        if (lane == 0 && d0 < (uint32_t)NB) {
            atomicAdd(&hist[d0], 32u);
            atomicAdd(&grp[d0 / PER], 32u);
        }
        return;
    }
    if (d < (uint32_t)NB) {
        atomicAdd(&hist[d], 1u);
        atomicAdd(&grp[d / PER], 1u);
    }
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t x = __shfl_up_sync(FULL, v, off);
        if (lane >= off) v += x;
    }
    return v;
}

// Warp 0: the bin of an NB-bin histogram holding the `remaining`-th largest key; writes the
// bin and the count of keys in strictly higher bins to res[0], res[1].  Lane l first takes
// group 31 - l (highest first), a warp scan finds the group holding the target, then each
// lane takes Q = NB / 1024 bins of that group (highest first) and a second scan finds the
// bin.  remaining <= the histogram's total.
template <int NB>
__device__ __forceinline__ void select_bin(const uint32_t *hist, const uint32_t *grp, int remaining, int *res) {
    constexpr int PER = NB / GROUPS;   // bins per group: 64 or 32
    constexpr int Q = PER / 32;        // bins per lane within the group: 2 or 1
    const int lane = threadIdx.x & 31;
    const uint32_t rem = (uint32_t)remaining;
    const uint32_t mine = grp[GROUPS - 1 - lane];
    const uint32_t incl = warp_incl_scan(mine, lane);
    const unsigned hit = __ballot_sync(FULL, (incl - mine) < rem && rem <= incl);
    const int src = hit ? __ffs(hit) - 1 : 0;  // hit == 0 cannot happen; stay in range
    const uint32_t above_grp = __shfl_sync(FULL, incl - mine, src);
    const int btop = (GROUPS - src) * PER - 1;  // highest bin of that group
    uint32_t h[Q];
#pragma unroll
    for (int j = 0; j < Q; ++j) h[j] = hist[btop - lane * Q - j];
    uint32_t lsum = 0;
#pragma unroll
    for (int j = 0; j < Q; ++j) lsum += h[j];
    const uint32_t lbefore = above_grp + warp_incl_scan(lsum, lane) - lsum;
    if (hit != 0 && lbefore < rem && rem <= lbefore + lsum) {
        uint32_t acc = lbefore;
#pragma unroll
        for (int j = 0; j < Q; ++j) {
            if (acc + h[j] >= rem) {
                res[0] = btop - lane * Q - j;
                res[1] = (int)acc;
                break;
            }
            acc += h[j];
        }
    }
}

// One digit pass.  On entry the buffers of parity `cur` are zero and visible to all
// threads; this pass clears parity cur ^ 1 for the next one, counts with add(hist, grp),
// and returns {bin, keys in higher bins} of the `remaining`-th largest.  Two barriers.
template <class C, int NB, class Add>
__device__ __forceinline__ int2 digit_pass(unsigned char *smem, int cur, int remaining, Add add) {
    int *res = reinterpret_cast<int *>(smem + C::OFF_SCAL) + 4 * cur;
    uint32_t *hist = hist_of<C>(smem, cur), *grp = grp_of<C>(smem, cur);
    clear_hist<C>(smem, cur ^ 1);
    add(hist, grp);
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) select_bin<NB>(hist, grp, remaining, res);
    __syncthreads();
    return make_int2(res[0], res[1]);
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(FULL, v, off);
    return v;
}

__device__ __forceinline__ int warp_excl_scan(int v, int lane, int &total) {
    const int incl = (int)warp_incl_scan((uint32_t)v, lane);
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

// The lane's 4 consecutive scores i0..i0+3, reading only below we (the rest are 0 and
// must be masked by the caller).
__device__ __forceinline__ float4 load4f(const float *src, int i0, int we) {
    if (i0 + 3 < we) return __ldg(reinterpret_cast<const float4 *>(src + i0));
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i0 < we) v.x = __ldg(src + i0);
    if (i0 + 1 < we) v.y = __ldg(src + i0 + 1);
    if (i0 + 2 < we) v.z = __ldg(src + i0 + 2);
    return v;
}

// Exact radix selection (11/11/10-bit digits, MSB first) of the `rank`-th largest key.
// for_items(fn) calls fn(key, valid) once per item of the calling thread; the lanes of a
// warp must make the same number of calls.  Starts on zeroed buffers of parity 0 and
// leaves parity 0 zeroed after an even number of passes.  Returns the key; *above
// receives the number of keys strictly greater.  With passes == 2 the result is only a
// lower bound of that key: the smallest key of the 22-bit bin that holds it.
template <class C, class ForItems>
__device__ uint32_t radix_select(int rank, ForItems for_items, unsigned char *smem, int *above, int passes = 3) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, mask = 0;
    int remaining = rank, above_total = 0;
    for (int pass = 0; pass < passes; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        int2 r;
        if (pass < 2) {
            r = digit_pass<C, 2048>(smem, pass & 1, remaining, [&](uint32_t *hist, uint32_t *grp) {
                for_items([&](uint32_t key, bool valid) {
                    const bool in = valid && (key & mask) == prefix;
                    hist_add<2048>(hist, grp, in ? (key >> shift) & 2047u : 2048u, lane);
                });
            });
        } else {
            r = digit_pass<C, 1024>(smem, pass & 1, remaining, [&](uint32_t *hist, uint32_t *grp) {
                for_items([&](uint32_t key, bool valid) {
                    const bool in = valid && (key & mask) == prefix;
                    hist_add<1024>(hist, grp, in ? key & 1023u : 1024u, lane);
                });
            });
        }
        remaining -= r.y;
        above_total += r.y;
        prefix |= (uint32_t)r.x << shift;
        mask |= (pass == 2 ? 1023u : 2047u) << shift;
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

// Appends the scores of one float4 group (indices i0..i0+3 of the lane's slot, nv of them
// valid) that reach f_lo, as float bits, to the warp's segment in index order: lanes in
// order, then the four components.  CHECKED = false: all four valid and the segment has
// room for 128 more (the caller's warp-uniform test), so the stores need no guard.
template <bool CHECKED>
__device__ __forceinline__ void keep_group(const float4 v, int i0, int nv, float f_lo, unsigned lt, int seg, int &cnt,
                                          uint32_t *mk, int *mi) {
    const bool t0 = (!CHECKED || nv > 0) && v.x >= f_lo, t1 = (!CHECKED || nv > 1) && v.y >= f_lo;
    const bool t2 = (!CHECKED || nv > 2) && v.z >= f_lo, t3 = (!CHECKED || nv > 3) && v.w >= f_lo;
    const unsigned b0 = __ballot_sync(FULL, t0), b1 = __ballot_sync(FULL, t1);
    const unsigned b2 = __ballot_sync(FULL, t2), b3 = __ballot_sync(FULL, t3);
    int off = cnt + __popc(b0 & lt) + __popc(b1 & lt) + __popc(b2 & lt) + __popc(b3 & lt);
    if (t0 && (!CHECKED || off < seg)) { mk[off] = __float_as_uint(v.x); mi[off] = i0; }
    off += t0;
    if (t1 && (!CHECKED || off < seg)) { mk[off] = __float_as_uint(v.y); mi[off] = i0 + 1; }
    off += t1;
    if (t2 && (!CHECKED || off < seg)) { mk[off] = __float_as_uint(v.z); mi[off] = i0 + 2; }
    off += t2;
    if (t3 && (!CHECKED || off < seg)) { mk[off] = __float_as_uint(v.w); mi[off] = i0 + 3; }
    cnt += __popc(b0) + __popc(b1) + __popc(b2) + __popc(b3);
}

// Key of a candidate stored as float bits.
__device__ __forceinline__ uint32_t cand_key(uint32_t bits) { return order_key(__uint_as_float(bits)); }

// Fast path.  Returns false (nothing written) when the sample misjudged the row.
template <class C>
__device__ bool select_row_sampled(const float *src, int n, int K, unsigned char *smem, int32_t *out) {
    constexpr int THREADS = C::THREADS, WARPS = C::WARPS, SEG = C::SEG;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t *segk = reinterpret_cast<uint32_t *>(smem + C::OFF_SEGK);
    int *segi = reinterpret_cast<int *>(smem + C::OFF_SEGI);
    int *scal = reinterpret_cast<int *>(smem + C::OFF_SCAL);
    int *seg_cnt = scal + 8, *wgt = scal + 8 + WARPS, *weq = scal + 8 + 2 * WARPS;
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    const int n4 = n >> 2;
    const int nsamp4 = (n4 + 15) / 16;                       // sampled float4 (every 16th)
    const int ns = 4 * nsamp4;
    if (ns < 64 || ns > 2 * WARPS * SEG) return false;

    // ---- sample keys into the segment arrays (keys, then indices: contiguous, free now)
    for (int m = tid; m < nsamp4; m += THREADS) {
        const float4 v = __ldg(s4 + 16 * m);
        segk[4 * m + 0] = order_key(v.x);
        segk[4 * m + 1] = order_key(v.y);
        segk[4 * m + 2] = order_key(v.z);
        segk[4 * m + 3] = order_key(v.w);
    }
    clear_hist<C>(smem, 0);
    if (tid == 0) scal[3] = 0;
    __syncthreads();
    const int target = min(ns, (int)((1.2 * K * (double)ns) / (double)n) + 16);
    int dummy;
    // a lower bound of the sample's target-th key is all the candidate pass needs: two
    // digit passes (22 bits); the samples are last read before the first barrier of the
    // second pass, so the candidate pass below may overwrite them
    const int ns_pad = (ns + THREADS - 1) / THREADS * THREADS;
    const uint32_t t_lo = radix_select<C>(
        target,
        [&](auto fn) {
            for (int j = tid; j < ns_pad; j += THREADS) fn(j < ns ? segk[j] : 0u, j < ns);
        },
        smem, &dummy, 2);
    const float f_lo = key_float(t_lo);

    // ---- candidates: scores >= f_lo, per warp in ascending index order.  Chunks of 512
    // scores per warp (4 float4 per lane); the next chunk is loaded before the current one
    // is filtered.
    const int R = ((n + WARPS * 128 - 1) / (WARPS * 128)) * 128;
    const int wb = min(n, warp * R), we = min(n, wb + R);
    uint32_t *mk = segk + warp * SEG;
    int *mi = segi + warp * SEG;
    int cnt = 0;
    const unsigned lt = (1u << lane) - 1u;
    float4 v[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) v[g] = load4f(src, wb + 128 * g + 4 * lane, we);
    for (int base = wb; base < we; base += 512) {
        float4 nx[4];
        const int nbase = base + 512;
        if (nbase < we) {
#pragma unroll
            for (int g = 0; g < 4; ++g) nx[g] = load4f(src, nbase + 128 * g + 4 * lane, we);
        }
        const bool whole = base + 512 <= we;   // warp-uniform
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int i0 = base + 128 * g + 4 * lane;
            if (whole && cnt + 128 <= SEG)
                keep_group<false>(v[g], i0, 4, f_lo, lt, SEG, cnt, mk, mi);
            else
                keep_group<true>(v[g], i0, min(max(we - i0, 0), 4), f_lo, lt, SEG, cnt, mk, mi);
        }
        if (nbase < we) {
#pragma unroll
            for (int g = 0; g < 4; ++g) v[g] = nx[g];
        }
    }
    if (lane == 0) {
        seg_cnt[warp] = cnt > SEG ? 0 : cnt;
        if (cnt > SEG) scal[3] = 1;
    }
    __syncthreads();
    const int total = warp_sum(lane < WARPS ? seg_cnt[lane] : 0);
    if (scal[3] != 0 || total < K) return false;   // uniform decision

    // ---- exact k-th largest among the candidates (each warp walks its own segment)
    int above;
    const int cnt_pad = (cnt + 31) & ~31;
    const uint32_t thr = radix_select<C>(
        K,
        [&](auto fn) {
            for (int j = lane; j < cnt_pad; j += 32) fn(j < cnt ? cand_key(mk[j]) : 0u, j < cnt);
        },
        smem, &above);
    const int need_eq = K - above;                   // >= 1
    const int count_gt = above;

    // ---- per-warp counts of > thr and == thr, then ordered writes
    int cg = 0, ce = 0;
    for (int j = lane; j < cnt; j += 32) {
        const uint32_t key = cand_key(mk[j]);
        cg += key > thr;
        ce += key == thr;
    }
    cg = warp_sum(cg);
    ce = warp_sum(ce);
    if (lane == 0) {
        wgt[warp] = cg;
        weq[warp] = ce;
    }
    __syncthreads();
    int gt_off = warp_sum(lane < warp ? wgt[lane] : 0);
    int eq_off = warp_sum(lane < warp ? weq[lane] : 0);
    for (int base = 0; base < cnt; base += 32) {
        const int j = base + lane;
        const uint32_t key = j < cnt ? cand_key(mk[j]) : 0u;
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
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int *cand = reinterpret_cast<int *>(smem + C::OFF_SEGK);   // CAND_CAP entries over both segment arrays
    int *scal = reinterpret_cast<int *>(smem + C::OFF_SCAL);
    // per warp: keys above bin b0, keys in b0 above thr, keys == thr
    int *w_above = scal + 8, *w_gt = scal + 8 + WARPS, *w_eq = scal + 8 + 2 * WARPS;
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    const int n4 = n >> 2;
    const int R = ((n + WARPS * 128 - 1) / (WARPS * 128)) * 128;
    const int wb = min(n, warp * R), we = min(n, wb + R);

    __syncthreads();   // the fast path's last reads of shared memory are done
    clear_hist<C>(smem, 0);
    for (int i = tid; i < 3 * WARPS; i += THREADS) scal[8 + i] = 0;
    if (tid == 0) scal[2] = 0;
    __syncthreads();

    // ---- pass 1: histogram of bits 31..21 over the whole row (float4 body, scalar tail)
    const int n4_pad = (n4 + THREADS - 1) / THREADS * THREADS;
    const int tail = n - (n4 << 2);
    const int2 r0 = digit_pass<C, 2048>(smem, 0, K, [&](uint32_t *hist, uint32_t *grp) {
        for (int i = tid; i < n4_pad; i += THREADS) {
            const bool ok = i < n4;
            const float4 v = ok ? __ldg(s4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            hist_add<2048>(hist, grp, ok ? order_key(v.x) >> 21 : 2048u, lane);
            hist_add<2048>(hist, grp, ok ? order_key(v.y) >> 21 : 2048u, lane);
            hist_add<2048>(hist, grp, ok ? order_key(v.z) >> 21 : 2048u, lane);
            hist_add<2048>(hist, grp, ok ? order_key(v.w) >> 21 : 2048u, lane);
        }
        if (warp == 0) {   // the tail (< 4 keys): the whole warp takes part
            const bool ok = lane < tail;
            hist_add<2048>(hist, grp, ok ? order_key(__ldg(src + (n4 << 2) + lane)) >> 21 : 2048u, lane);
        }
    });
    const uint32_t b0 = (uint32_t)r0.x;
    int remaining = K - r0.y;

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

    // ---- digits 2 and 3 on the candidates (or on the whole row after an overflow); the
    // first pass left parity 1 cleared
    uint32_t prefix = b0 << 21, mask = 0xFFE00000u;
    const int m = use_cand ? ncand : n;
    const int m_pad = (m + THREADS - 1) / THREADS * THREADS;
    auto key_at = [&](int j) { return order_key(__ldg(src + (use_cand ? cand[j] : j))); };
    const int2 r1 = digit_pass<C, 2048>(smem, 1, remaining, [&](uint32_t *hist, uint32_t *grp) {
        for (int j = tid; j < m_pad; j += THREADS) {
            uint32_t d = 2048u;
            if (j < m) {
                const uint32_t key = key_at(j);
                if ((key & mask) == prefix) d = (key >> 10) & 2047u;
            }
            hist_add<2048>(hist, grp, d, lane);
        }
    });
    remaining -= r1.y;
    prefix |= (uint32_t)r1.x << 10;
    mask |= 2047u << 10;
    const int2 r2 = digit_pass<C, 1024>(smem, 0, remaining, [&](uint32_t *hist, uint32_t *grp) {
        for (int j = tid; j < m_pad; j += THREADS) {
            uint32_t d = 1024u;
            if (j < m) {
                const uint32_t key = key_at(j);
                if ((key & mask) == prefix) d = key & 1023u;
            }
            hist_add<1024>(hist, grp, d, lane);
        }
    });
    remaining -= r2.y;
    prefix |= (uint32_t)r2.x;
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
    int gt_off = warp_sum(lane < warp ? w_above[lane] + w_gt[lane] : 0);
    int eq_off = warp_sum(lane < warp ? w_eq[lane] : 0);
    ordered_output(src, wb, we, lane, thr, need_eq, count_gt, K, gt_off, eq_off, out);
}

// grid = row_count CTAs of NT threads, dynamic shared memory Cfg<NT>::SMEM bytes.  With a
// row_mask only the rows r with row_mask[r] != 0 are selected (the others are untouched).
template <int NT>
__global__ void __launch_bounds__(NT, NT >= 512 ? 1 : 4) topk_rows_kernel(Problem P, const float *__restrict__ scores, int64_t ld,
                                                       int row_begin, int32_t *__restrict__ idx,
                                                       const uint8_t *__restrict__ row_mask) {
    using C = Cfg<NT>;
    extern __shared__ __align__(16) unsigned char smem[];
    const int r = blockIdx.x;
    if (row_mask != nullptr && row_mask[r] == 0) return;
    const int K = P.topk;
    int32_t *out = idx + (int64_t)r * K;
    const RowInfo ri = row_info_warp(P, row_begin + r);
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
