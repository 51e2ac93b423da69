// sparse_mla_pair.cuh -- attention over the selected latent rows (MLA in MQA mode) on
// pairs of SMs: persistent 2-CTA clusters that take query tokens in turn, 2-SM tensor-core
// MMAs (cta_group::2).
//
// "DeepSeek-V3.2 tech report summary", §1 DSA: full attention only over the k selected
// tokens; MLA-based implementation in MQA mode (every 576-d latent row is shared by all
// 128 query heads); value = first 512 dims; softmax scale 1/sqrt(192).
//
// The index row is cut into blocks of 256 slots.  CTA c of the pair owns slots
// [256 b + 128 c, 256 b + 128 c + 128) of block b ("its keys") and heads 64 c .. 64 c + 63.
//   QK_b   S^T[key, h] = kv[key, :576] . q[h, :576]          M = 256 keys (128 per CTA,
//          A = the gathered rows in each CTA), N = 128 heads (B = q, 64 heads per CTA),
//          K = 576: each CTA receives S^T of its own 128 keys for all heads in TMEM.
//   softmax  each CTA turns its S^T into P^T = exp2(S^T * scale * log2 e - m[h]) for its
//          keys; m[h] is the pair's running per-head reference maximum (exact block maxima
//          are exchanged every block, the reference moves lazily, only when a block
//          maximum exceeds it by more than TAU).
//   PV_b   O^T[d, h] += V^T[d, key] . P^T[key, h] over the 256 keys of the block:
//          M = 256 value dims per instruction (two instructions cover 512), A = value
//          atoms in each CTA (CTA c holds dims 256 i + 128 c .. + 127 for every key of the
//          block), N = 128 heads (B = P^T, CTA c holds heads 64 c .. + 63 for all 256
//          keys): each CTA stores the P^T of its keys for the other CTA's heads straight
//          into the other CTA's shared memory (16 KB per block).
// So every flop of the definition is executed once, each selected row is gathered once
// whole (QK) plus the value dims each CTA needs for PV, and q is split between the CTAs.
//
// Tensor memory per CTA (512 columns): S^T double buffer [0,128) [128,256) (lanes = the
// CTA's keys, columns = heads); O^T [256,384) for value dims 128 c + [0,128) and
// [384,512) for 256 + 128 c + [0,128) (lanes = value dims, columns = heads).
// Shared memory per CTA: q half (9 swizzled 64-dim atoms of 64 heads, 72 KB), P^T buffer
// (256 keys x 64 heads, MN-major, 32 KB), a 7-slot ring of gathered 16 KB atoms (128 keys x
// 64 dims, 128-byte swizzle applied in the address) fed in MMA order QK_0, QK_1, PV_0,
// QK_2, PV_1, ..., PV_{n-1}:
//   QK_b  9 atoms of the CTA's own keys;
//   PV_b  8 atoms: for i = 0, 1 and key half h = 0, 1 (the keys of CTA h), the CTA's two
//         64-dim value atoms 4 i + 2 c + {0, 1}.
// Both CTAs lay the ring out identically (same positions, same slots); the even CTA
// issues every MMA once both CTAs' operands have landed and commits to the barriers of
// both.  Rows are gathered by TMA (tile::gather4: 4 rows x 128 bytes per instruction, the
// 128-byte swizzle applied by the copy engine), each lane of a loader warp issuing one
// instruction of an atom; the 2-SM form completes the bytes of both CTAs on the even
// CTA's barrier of the slot (one expect-tx by the even CTA), so neither CTA relays the
// other's ring state.  Seven loader warps take the ring positions in turn, one slot each.
// The softmax warps of both CTAs signal the even CTA's P^T barrier with cluster-scope
// arrivals after their stores.
// Dense mode (DENSE = true, the short-sequence "masked MHA" form of the same attention):
// slot s of block b is key 256 b + s itself, keys 0 .. pos(t) in order, restricted to the
// keys listed in idx when idx is given (a bitmask built in shared memory; each listed key
// counts once).  The keys of an atom are contiguous rows, so one thread per CTA loads each
// atom with a 2-SM TMA tile load that completes on the even CTA's barrier.  With all
// visible keys listed in order the two modes run the same MMAs on the same operands.
//
// Warp roles (16 warps per CTA): 0-6 gather and each scan a unit's index row for its block
// count (0 also publishes the count, issues the q TMA and allocates tensor memory; in dense
// mode only warp 0 loads, one tile per atom), 7 issues the MMAs (even CTA), 8-15 run the
// softmax and the epilogue: warp w owns TMEM lane quarter w % 4 and head half (w - 8) / 4.
// The first two warpgroups give registers to the last two (setmaxnreg).
#pragma once

#include "dsa_common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace mla {

struct PairCfg {
    static constexpr int BLK = 256;                 // index slots per block (128 per CTA)
    static constexpr int NATOM = 9;                 // 64-dim atoms per 576-d row
    static constexpr int ATOM = 128 * 128;          // one gathered atom: 128 keys x 128 bytes
    static constexpr int QATOM = 64 * 128;          // one q atom: 64 heads x 128 bytes
    static constexpr int NSLOT = 7;
    static constexpr int NLOAD = 7;                 // loader warps, one ring slot each
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_P = OFF_Q + NATOM * QATOM;        // 73728
    static constexpr int OFF_RING = OFF_P + 256 * 128;         // 106496
    static constexpr int OFF_RED = OFF_RING + NSLOT * ATOM;    // [4][128] f32
    static constexpr int OFF_XM = OFF_RED + 4 * 128 * 4;       // [2][128] f32, peer block maxima
    static constexpr int OFF_XL = OFF_XM + 2 * 128 * 4;        // [128] f32, peer row sums
    static constexpr int OFF_MR = OFF_XL + 128 * 4;            // [128] f32, running reference max
    static constexpr int OFF_FS = OFF_MR + 128 * 4;            // [128] f32, rescale factor / 1/l
    static constexpr int OFF_MASK = OFF_FS + 128 * 4;          // dense mode: listed-key bitmask
    static constexpr int DENSE_MAX_KEYS = 16384;               // keys a masked dense row may have
    static constexpr int OFF_BAR = OFF_MASK + DENSE_MAX_KEYS / 8;
    // empty[7] pfull[7] q_full q_free s_full[2] s_free[2] p_full pv_done o_ready xbar[2]
    // lbar drain unit_full[2] unit_free[2]
    static constexpr int NBARS = 2 * NSLOT + 2 + 2 + 2 + 3 + 2 + 2 + 2 + 2;
    // [0] TMEM base, [1] abort, [2..3] unit blocks, [4] the peer CTA's abort flag at teardown
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    // even CTA: [2][NSLOT] int, the last ring position each CTA issued into each slot
    static constexpr int OFF_LASTPOS = OFF_MISC + 32;
    static constexpr int SMEM = OFF_LASTPOS + 2 * NSLOT * 4;
    static constexpr int THREADS = 512;
    static constexpr int SOFT0 = 8;                 // first softmax warp
    static constexpr int REG_LOW = 88, REG_HIGH = 168;   // 256 x 88 + 256 x 168 = 512 x 128
    static constexpr int TMEM_S = 0, TMEM_O = 256;
    static constexpr float TAU = 8.0f;              // lazy-rescale threshold (log2 units)
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(NLOAD <= NSLOT, "ring waits need NLOAD <= NSLOT");
    static_assert(256 * REG_LOW + 256 * REG_HIGH <= 65536 / THREADS * THREADS, "register split");
};

__device__ __forceinline__ bool pair_visible(int e, const RowInfo &ri) { return e >= 0 && e <= ri.pos && e < ri.len_k; }

// Group g (0 .. 2n-1) of the ring order QK_0, QK_1, PV_0, QK_2, PV_1, ..., PV_{n-1}.
__device__ __forceinline__ void pair_group(int g, int n, bool &qk, int &blk) {
    if (g == 0) { qk = true; blk = 0; }
    else if (g == 2 * n - 1) { qk = false; blk = n - 1; }
    else if (g & 1) { qk = true; blk = (g + 1) >> 1; }
    else { qk = false; blk = (g >> 1) - 1; }
}

// PV position m (0..7) of a group starting at ring position p: instruction i, key half h,
// and the 64-dim value atom it holds.  The two atoms of one (i, h) pair form one MN-major
// operand whose lower-addressed slot must hold the lower dims.
__device__ __forceinline__ int pv_value_atom(int c, int p, int m) {
    const int i = m >> 2, h = (m >> 1) & 1, e = m & 1;
    const int s0 = (p + 4 * i + 2 * h) % PairCfg::NSLOT;
    const int s1 = (s0 + 1) % PairCfg::NSLOT;
    const bool lo_first = s0 < s1;
    return 4 * i + 2 * c + (lo_first ? e : 1 - e);
}

// Lane l ends with the reduction (max or sum) over the 32 lanes of element l of v.
template <bool MAX>
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
    for (int m = 16, n = 32; m >= 1; m >>= 1, n >>= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? v[i] : v[i + n / 2];
            const float keep = upper ? v[i + n / 2] : v[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, m);
            v[i] = MAX ? fmaxf(keep, recv) : keep + recv;
        }
    }
    return v[0];
}

// Split of each token's index row over several CTA pairs (sparse form only): split c of a
// token takes blocks [c * bps, (c + 1) * bps) of its 256-slot blocks and writes, instead of
// out / lse, its normalised partial output in fp32 and the lse of its slots to
// o_part [T * nsplit, 128, 512] / lse_part [T * nsplit, 128] (row t * nsplit + c);
// combine_splits_kernel merges them.  The SPLIT = false instantiation (one unit per token)
// writes out / lse directly.
struct SplitArgs {
    int nsplit;
    int bps;
    float *o_part;
    float *lse_part;
};

// Blocks of one unit (token row ri, split `split` of `bps` blocks): the 256-slot blocks up
// to the last visible slot of the index row (every lane of the warp returns the same
// count).  Dense form: keys 0 .. pos(t) are the slots.
template <bool DENSE>
__device__ __forceinline__ int pair_unit_blocks(const Problem &P, const RowInfo &ri, const int32_t *irow, int K,
                                                int split, int bps, int lane) {
    if (!row_ok(P, ri)) return 0;
    int last = -1;
    if (DENSE) {
        last = min(ri.pos, ri.len_k - 1);
    } else {
        if ((K & 3) == 0) {
            const int n4 = K >> 2;
#pragma unroll 4
            for (int i4 = lane; i4 < n4; i4 += 32) {
                const int4 x = __ldg(reinterpret_cast<const int4 *>(irow) + i4);
                if (pair_visible(x.x, ri)) last = 4 * i4;
                if (pair_visible(x.y, ri)) last = 4 * i4 + 1;
                if (pair_visible(x.z, ri)) last = 4 * i4 + 2;
                if (pair_visible(x.w, ri)) last = 4 * i4 + 3;
            }
        } else {
            for (int i = lane; i < K; i += 32)
                if (pair_visible(__ldg(irow + i), ri)) last = i;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
    }
    const int nb_row = (last + PairCfg::BLK) / PairCfg::BLK;   // 0 when no slot is visible
    const int b_begin = split * bps;
    return max(0, min(nb_row, b_begin + bps) - b_begin);
}

// Persistent schedule.  The grid holds at most as many pairs as run at once; pair g takes
// the units g, g + npairs, g + 2 npairs, ... (unit u = token T - 1 - u / nsplit, split
// u % nsplit: later, heavier tokens first).  Ring positions, the S^T double buffer and
// every per-block barrier keep counting across units, so the gathers and the first QKs of
// the next unit run while the current one finishes its last PV and its epilogue.  Per
// unit, loader warp 0 publishes the unit's block count (a two-entry table guarded by
// unit_full / unit_free) and loads its q as soon as the previous unit's last QK has read
// q_s (q_free).  PV_0 of a unit overwrites O^T only once the P^T of its block 0 is in
// place, and the softmax warps write that P^T after their epilogue of the previous unit
// has read O^T out of tensor memory (loads waited for, then a tcgen05 fence before the
// arrivals), so O^T needs no barrier of its own.
template <bool DENSE, bool SPLIT = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(512, 1)
sparse_mla_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                       Problem P, const int32_t *__restrict__ idx, __nv_bfloat16 *__restrict__ out,
                       float *__restrict__ lse, SplitArgs sp) {
    using C = PairCfg;
    using namespace sm100;
    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cr = (int)cluster_ctarank();                   // 0: issues the MMAs
    const int peer = cr ^ 1;
    const int T = P.total_q;
    static_assert(!(DENSE && SPLIT), "the dense form is not split");
    const int nsplit = SPLIT ? sp.nsplit : 1;
    const int bps = SPLIT ? sp.bps : (1 << 24);
    const int units = T * nsplit;
    const int npairs = (int)(gridDim.x >> 1);
    const int pair0 = (int)(blockIdx.x >> 1);
    constexpr bool partial = SPLIT;
    const int K = P.topk;
    const bool masked = DENSE && idx != nullptr;

    const uint32_t sbase = smem_u32(smem);
    const bool misaligned = (sbase & 1023u) != 0;           // uniform; no unit runs then
    const uint32_t q_s = sbase + C::OFF_Q;
    const uint32_t p_s = sbase + C::OFF_P;
    const uint32_t ring_s = sbase + C::OFF_RING;
    float *red = reinterpret_cast<float *>(smem + C::OFF_RED);
    float *xm = reinterpret_cast<float *>(smem + C::OFF_XM);
    float *xl = reinterpret_cast<float *>(smem + C::OFF_XL);
    float *mr = reinterpret_cast<float *>(smem + C::OFF_MR);
    float *fs = reinterpret_cast<float *>(smem + C::OFF_FS);
    uint32_t *maskw = reinterpret_cast<uint32_t *>(smem + C::OFF_MASK);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto empty = [&](int s) { return bar0 + 8u * s; };
    auto pfull = [&](int s) { return bar0 + 8u * (C::NSLOT + s); };
    const uint32_t q_full = bar0 + 8u * (2 * C::NSLOT);      // even CTA: q of both CTAs landed
    const uint32_t q_free = q_full + 8;                      // the unit's last QK has read q_s
    auto s_full = [&](int b) { return q_full + 16 + 8u * b; };
    auto s_free = [&](int b) { return q_full + 32 + 8u * b; };
    const uint32_t p_full = q_full + 48;                    // P^T of both CTAs written (even CTA)
    const uint32_t pv_done = q_full + 56;
    const uint32_t o_ready = q_full + 64;
    auto xbar = [&](int b) { return q_full + 72 + 8u * b; };
    const uint32_t lbar = q_full + 88;
    const uint32_t drain = q_full + 96;
    auto unit_full = [&](int i) { return q_full + 104 + 8u * i; };
    auto unit_free = [&](int i) { return q_full + 120 + 8u * i; };
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    volatile int *unit_nb = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);

    // ---- setup (every thread of both CTAs reaches the cluster barriers below)
    if (tid == 0 && !misaligned) {
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(empty(s), 1);
            mbar_init(pfull(s), 1);       // the even CTA's expect-tx for both CTAs' bytes
        }
        mbar_init(q_full, 1);             // likewise
        mbar_init(q_free, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(s_full(b), 1);
            mbar_init(s_free(b), 16);     // 8 softmax warps of each CTA
            mbar_init(xbar(b), 1);
            mbar_init(unit_full(b), 1);   // loader warp 0
            mbar_init(unit_free(b), cr == 0 ? 2 : 1);   // the MMA thread (even CTA), the softmax warps
        }
        mbar_init(p_full, 16);            // 8 softmax warps of each CTA
        mbar_init(pv_done, 1);
        mbar_init(o_ready, 1);
        mbar_init(lbar, 1);
        mbar_init(drain, 1);
        misc[1] = 0;
        misc[4] = 0;
        for (int i = 0; i < 2 * C::NSLOT; ++i) reinterpret_cast<int *>(smem + C::OFF_LASTPOS)[i] = -1;
        fence_barrier_init();
    }
    if (tid == 0 && misaligned) {
        raise_error(ERR_SMEM_ALIGN);
        misc[1] = 1;
    }
    cluster_sync();   // both CTAs running, their barriers initialised
    if (warp == 0) tmem_alloc_pair(sbase + C::OFF_MISC, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const bool run = !misaligned;
    const uint32_t peer_misc1 = mapa_shared(sbase + C::OFF_MISC + 4, (uint32_t)peer);
    auto abort_pair = [&]() {                                // stop both CTAs of the pair
        misc[1] = 1;
        st_cluster_u32(peer_misc1, 1u);
    };
    const int lw = warp;                                     // loader warps 0 .. NLOAD-1
    const bool loader = warp < C::NLOAD && (!DENSE || warp == 0);

    if (warp < C::SOFT0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REG_LOW));
    if (loader) {
        // ------------------------------------------------ loads: q per unit, ring atoms
        const uint32_t lead_pfull = mapa_shared(pfull(0), 0);
        const uint32_t lead_q_full = mapa_shared(q_full, 0);
        if (lw == 0 && lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_kv);
        }
        bool ok = run;
        int p = 0;                                           // ring position, counted across units
        int nq = 0;                                          // units with blocks so far
        int last_issued = -1;                                // the last ring position this warp issued
        for (int j = 0, u = pair0; ok && u < units; ++j, u += npairs) {
            const int t = T - 1 - u / nsplit;
            const int split = u % nsplit;
            const RowInfo ri = row_info_warp(P, t);
            const int32_t *irow = idx != nullptr ? idx + (int64_t)t * K : nullptr;
            const int nblocks = pair_unit_blocks<DENSE>(P, ri, irow, K, split, bps, lane);
            if (lw == 0) {
                bool okw = true;
                if (lane == 0) {
                    if (j >= 2) okw = mbar_wait(unit_free(j & 1), ((j >> 1) - 1) & 1);
                    if (okw) {
                        unit_nb[j & 1] = nblocks;
                        mbar_arrive(unit_full(j & 1));
                    }
                    if (okw && nblocks > 0 && nq > 0) okw = mbar_wait(q_free, (nq - 1) & 1);
                    if (okw && nblocks > 0) {
                        if (cr == 0) mbar_expect_tx(q_full, 2 * C::NATOM * C::QATOM);   // both CTAs' q
                        for (int a = 0; a < C::NATOM; ++a)
                            tma_load_2d_pair(q_s + a * C::QATOM, &tm_q, lead_q_full, 64 * a, t * 128 + 64 * cr);
                    }
                }
                if (!__shfl_sync(0xffffffffu, okw, 0)) {
                    ok = false;
                    break;
                }
            }
            if (nblocks == 0) continue;
            ++nq;
            if (DENSE) {
                // ---- TMA tile loads of contiguous keys (lane 0 of warp 0)
                bool okd = true;
                if (lane == 0) {
                    for (int g = 0; okd && g < 2 * nblocks; ++g) {
                        bool qk;
                        int b;
                        pair_group(g, nblocks, qk, b);
                        const int natoms = qk ? C::NATOM : 8;
                        for (int m = 0; m < natoms; ++m) {
                            const int pp = p + m, slot = pp % C::NSLOT;
                            if (pp >= C::NSLOT && !mbar_wait(empty(slot), ((pp / C::NSLOT) - 1) & 1)) {
                                okd = false;
                                break;
                            }
                            if (misc[1]) {
                                okd = false;
                                break;
                            }
                            const int h = qk ? cr : ((m >> 1) & 1);
                            const int a = qk ? m : pv_value_atom(cr, p, m);
                            if (cr == 0) mbar_expect_tx(pfull(slot), 2 * C::ATOM);   // both CTAs' tiles
                            tma_load_2d_pair(ring_s + slot * C::ATOM, &tm_kv, lead_pfull + 8u * slot, 64 * a,
                                             ri.kbase + C::BLK * b + 128 * h);
                            last_issued = pp;
                        }
                        p += natoms;
                    }
                }
                ok = __shfl_sync(0xffffffffu, okd, 0);
                p = __shfl_sync(0xffffffffu, p, 0);
            } else {
                // ---- row gathers (TMA gather4: 4 rows per lane, one atom per warp and ring
                // position; the loader warps take the positions in turn).  All atoms of a group
                // gather the same rows, so each lane loads the index entries of the next group
                // while the current one is issued.
                const int b_begin = split * bps;
                const int32_t *irow_s = irow + b_begin * C::BLK;
                const int ks_left = K - b_begin * C::BLK;
                auto entries = [&](int b, int h) {               // raw entries of this lane's 4 slots
                    const int s0 = C::BLK * b + 128 * h + 4 * lane;
                    int4 x;
                    if ((K & 3) == 0 && s0 + 3 < ks_left) {
                        x = __ldg(reinterpret_cast<const int4 *>(irow_s + s0));
                    } else {
                        x.x = s0 < ks_left ? __ldg(irow_s + s0) : -1;
                        x.y = s0 + 1 < ks_left ? __ldg(irow_s + s0 + 1) : -1;
                        x.z = s0 + 2 < ks_left ? __ldg(irow_s + s0 + 2) : -1;
                        x.w = s0 + 3 < ks_left ? __ldg(irow_s + s0 + 3) : -1;
                    }
                    return x;
                };
                // group g needs key half cr of block b (QK_b, kept in e0) or both halves (PV_b)
                int4 e0 = entries(0, cr), e1 = make_int4(-1, -1, -1, -1);
                for (int g = 0; ok && g < 2 * nblocks; ++g) {
                    bool qk;
                    int b;
                    pair_group(g, nblocks, qk, b);
                    int4 n0 = e0, n1 = e1;
                    if (g + 1 < 2 * nblocks) {
                        bool qk1;
                        int b1;
                        pair_group(g + 1, nblocks, qk1, b1);
                        n0 = entries(b1, qk1 ? cr : 0);
                        if (!qk1) n1 = entries(b1, 1);
                    }
                    const int natoms = qk ? C::NATOM : 8;
                    for (int m = 0; m < natoms; ++m) {
                        const int pp = p + m;
                        if (pp % C::NLOAD != lw) continue;
                        const int4 x = (!qk && ((m >> 1) & 1)) ? e1 : e0;
                        const int r[4] = {x.x, x.y, x.z, x.w};
                        int e[4];
#pragma unroll
                        for (int v = 0; v < 4; ++v) e[v] = key_row(P, ri, pair_visible(r[v], ri) ? r[v] : 0);
                        const int a = qk ? m : pv_value_atom(cr, p, m);
                        const int slot = pp % C::NSLOT;
                        bool okw = true;
                        if (lane == 0) {
                            if (pp >= C::NSLOT) okw = mbar_wait(empty(slot), ((pp / C::NSLOT) - 1) & 1);
                            if (okw && cr == 0) mbar_expect_tx(pfull(slot), 2 * C::ATOM);   // both CTAs' rows
                        }
                        if (!__shfl_sync(0xffffffffu, okw, 0) || misc[1]) {
                            ok = false;
                            break;
                        }
                        tma_gather4_pair(ring_s + slot * C::ATOM + 512 * lane, &tm_kv, lead_pfull + 8u * slot, 64 * a,
                                         e[0], e[1], e[2], e[3]);
                        last_issued = pp;
                    }
                    e0 = n0;
                    e1 = n1;
                    p += natoms;
                }
            }
        }
        if (!ok && lane == 0) abort_pair();
        // the last position this warp issued into each of its slots, recorded in the even CTA
        // for the drain after an abort (gathered form: warp lw owns slot lw; dense form: warp 0
        // issued every position up to last_issued in order)
        static_assert(C::NLOAD == C::NSLOT, "one ring slot per gathering warp");
        if (lane == 0) {
            const uint32_t rec = mapa_shared(sbase + C::OFF_LASTPOS + 4u * (uint32_t)(cr * C::NSLOT), 0);
            if (DENSE) {
                for (int sl = 0; sl < C::NSLOT; ++sl) {
                    const int v = last_issued >= sl ? last_issued - (last_issued - sl) % C::NSLOT : -1;
                    st_cluster_u32(rec + 4u * sl, (uint32_t)v);
                }
            } else {
                st_cluster_u32(rec + 4u * lw, (uint32_t)last_issued);
            }
        }
        // the last q load has landed before the pair may exit (both CTAs' bytes complete on
        // the even CTA's barrier; the cluster barrier at teardown holds the odd CTA)
        if (lw == 0 && lane == 0 && cr == 0 && nq > 0) mbar_wait_cluster(q_full, (nq - 1) & 1);
    } else if (warp == 7 && lane == 0 && cr == 0) {
        // ------------------------------------------------ MMA issuer (even CTA)
        const uint32_t idesc_qk = idesc_bf16(256, 128);
        const uint32_t idesc_pv = idesc_bf16_mn_mn(256, 128);
        bool ok = run;
        bool issued = false;
        int pos = 0;                                         // ring position, counted across units
        int gb0 = 0;                                         // blocks of the earlier units
        int nq = 0;                                          // units with blocks so far
        for (int j = 0, u = pair0; ok && u < units; ++j, u += npairs) {
            if (!mbar_wait(unit_full(j & 1), (j >> 1) & 1)) {
                ok = false;
                break;
            }
            const int nblocks = unit_nb[j & 1];
            mbar_arrive(unit_free(j & 1));
            if (nblocks == 0) continue;
            if (!mbar_wait_cluster(q_full, nq & 1) || misc[1]) {
                ok = false;
                break;
            }
            for (int g = 0; ok && g < 2 * nblocks; ++g) {
                bool qk;
                int b;
                pair_group(g, nblocks, qk, b);
                const int gb = gb0 + b;
                if (qk) {                                    // QK_b -> S^T buffer gb & 1
                    if (gb >= 2 && !mbar_wait_cluster(s_free(gb & 1), ((gb >> 1) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = tmem + C::TMEM_S + 128 * (gb & 1);
                    for (int a = 0; a < C::NATOM; ++a, ++pos) {
                        const int slot = pos % C::NSLOT;
                        const uint32_t par = (pos / C::NSLOT) & 1;
                        if (!mbar_wait_cluster(pfull(slot), par) || misc[1]) {
                            ok = false;
                            break;
                        }
                        const uint32_t sa = ring_s + slot * C::ATOM;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_f16_pair(d, desc_sw128(sa + kk * 32), desc_sw128(q_s + a * C::QATOM + kk * 32),
                                         idesc_qk, (a > 0 || kk > 0) ? 1u : 0u);
                        issued = true;
                        mma_commit_pair_both(empty(slot));
                    }
                    if (!ok) break;
                    if (b == nblocks - 1) mma_commit_pair_both(q_free);   // the unit's last read of q_s
                    mma_commit_pair_both(s_full(gb & 1));
                } else {                                     // PV_b
                    if (!mbar_wait_cluster(p_full, gb & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int i = 0; ok && i < 2; ++i) {
                        const uint32_t d = tmem + C::TMEM_O + 128 * i;
                        for (int h = 0; h < 2; ++h, pos += 2) {
                            const int s0 = pos % C::NSLOT, s1 = (pos + 1) % C::NSLOT;
                            const uint32_t par0 = (pos / C::NSLOT) & 1, par1 = ((pos + 1) / C::NSLOT) & 1;
                            if (!mbar_wait_cluster(pfull(s0), par0) || !mbar_wait_cluster(pfull(s1), par1) ||
                                misc[1]) {
                                ok = false;
                                break;
                            }
                            const int slo = s0 < s1 ? s0 : s1, shi = s0 < s1 ? s1 : s0;
                            const uint32_t vb = ring_s + slo * C::ATOM;
                            const uint32_t lbo = (uint32_t)(shi - slo) * C::ATOM;
#pragma unroll
                            for (int k8 = 0; k8 < 8; ++k8)
                                mma_f16_pair(d, desc_sw128_mn(vb + k8 * 2048, lbo),
                                             desc_sw128_mn(p_s + (8 * h + k8) * 2048, 16384), idesc_pv,
                                             (b > 0 || h > 0 || k8 > 0) ? 1u : 0u);
                            issued = true;
                            mma_commit_pair_both(empty(s0));
                            mma_commit_pair_both(empty(s1));
                        }
                    }
                    if (!ok) break;
                    mma_commit_pair_both(pv_done);
                    if (b == nblocks - 1) mma_commit_pair_both(o_ready);
                }
            }
            gb0 += nblocks;
            ++nq;
        }
        if (!ok) {
            abort_pair();
            if (issued) {                                    // nothing may be in flight at dealloc
                mma_commit_pair_both(drain);
                mbar_wait(drain, 0);
            }
        }
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REG_HIGH));
        // ------------------------------------------------ softmax + epilogue
        const int st = tid - 32 * C::SOFT0;                  // 0 .. 255
        const int quarter = warp & 3;
        const int h2 = (warp - C::SOFT0) >> 2;               // head half handled by this warp
        const int key = quarter * 32 + lane;                 // this thread's key among the CTA's 128
        const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
        const float sl2 = P.sm_scale * 1.4426950408889634f;
        const uint32_t xm_peer = mapa_shared(sbase + C::OFF_XM, (uint32_t)peer);
        const uint32_t xbar_peer = mapa_shared(xbar(0), (uint32_t)peer);
        const uint32_t s_free_lead = mapa_shared(s_free(0), 0);
        const uint32_t p_full_lead = mapa_shared(p_full, 0);
        const uint32_t p_peer_s = mapa_shared(p_s, (uint32_t)peer);
        const int sown = 128 * cr + key;                     // slot of this thread's key within a block
        bool ok = run;
        int gb0 = 0;                                         // blocks of the earlier units
        int nq = 0;                                          // units with blocks so far
        for (int j = 0, u = pair0; ok && u < units; ++j, u += npairs) {
            const int t = T - 1 - u / nsplit;
            const int split = u % nsplit;
            const RowInfo ri = row_info_warp(P, t);
            const bool got = mbar_wait(unit_full(j & 1), (j >> 1) & 1);
            const int nblocks = got ? unit_nb[j & 1] : 0;
            if (named_bar_or(1, 256, !got || misc[1] != 0)) {
                ok = false;
                break;
            }
            if (st == 0) mbar_arrive(unit_free(j & 1));
            const int32_t *irow_s = idx != nullptr ? idx + (int64_t)t * K + split * bps * C::BLK : nullptr;
            const int ks_left = K - split * bps * C::BLK;
            if (masked && nblocks > 0) {
                // bitmask of the listed keys (keys 0 .. last)
                const int last = min(ri.pos, ri.len_k - 1);
                for (int i = st; i <= (last >> 5); i += 256) maskw[i] = 0u;
                named_bar(1, 256);
                for (int i = st; i < K; i += 256) {
                    const int e = __ldg(irow_s + i);
                    if (pair_visible(e, ri)) atomicOr(maskw + (e >> 5), 1u << (e & 31));
                }
                named_bar(1, 256);
            }
            if (st < 128) mr[st] = -INFINITY;                // reference maxima of the 128 heads
            float l[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) l[i] = 0.f;
            int ent = !DENSE && nblocks > 0 && sown < ks_left ? __ldg(irow_s + sown) : -1;
            for (int b = 0; b < nblocks; ++b) {
                const int gb = gb0 + b;
                bool vis;
                if (DENSE) {
                    const int sk = C::BLK * b + sown;        // the key itself
                    vis = sk <= ri.pos && sk < ri.len_k && (!masked || ((maskw[sk >> 5] >> (sk & 31)) & 1u));
                } else {
                    vis = pair_visible(ent, ri);
                    const int s = C::BLK * (b + 1) + sown;
                    ent = (b + 1 < nblocks && s < ks_left) ? __ldg(irow_s + s) : -1;
                }
                const bool fail = misc[1] != 0 || !mbar_wait_cluster(s_full(gb & 1), (gb >> 1) & 1);
                if (named_bar_or(1, 256, fail)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sb = t_lane + C::TMEM_S + 128 * (gb & 1) + 64 * h2;
                // ---- exact block maxima of this CTA's keys (per head), then of the pair
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    uint32_t sr[32];
                    float v[32];
                    tmem_ld32(sb + 32 * jj, sr);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = vis ? __uint_as_float(sr[i]) : -INFINITY;
                    red[quarter * 128 + 64 * h2 + 32 * jj + lane] = transpose_reduce32<true>(v, lane);
                }
                named_bar(1, 256);
                bool need = false;
                if (st < 128) {
                    const int h = st;
                    const float m_cta = fmaxf(fmaxf(red[h], red[128 + h]), fmaxf(red[256 + h], red[384 + h]));
                    st_async_f32(xm_peer + 4u * (128 * (gb & 1) + h), m_cta, xbar_peer + 8u * (gb & 1));
                    if (st == 0) mbar_expect_tx(xbar(gb & 1), 128 * 4);
                    const bool okx = mbar_wait_cluster(xbar(gb & 1), (gb >> 1) & 1);
                    const float m_blk = fmaxf(m_cta, okx ? xm[128 * (gb & 1) + h] : m_cta) * sl2;
                    const float m_old = mr[h];
                    need = m_blk > m_old + C::TAU;
                    const float m_new = need ? m_blk : m_old;
                    fs[h] = (need && m_old != -INFINITY) ? exp2f(m_old - m_new) : 1.0f;
                    mr[h] = m_new;
                    if (!okx) misc[1] = 1;
                }
                // every exit decision below is taken through a barrier, so the 8 warps stay together
                const bool any = named_bar_or(1, 256, need);
                bool pv_waited = false;
                if (any) {
#pragma unroll
                    for (int i = 0; i < 64; ++i) l[i] *= fs[64 * h2 + i];
                    if (b > 0) {
                        // O^T must hold PV_{b-1} before it is rescaled; PV_b cannot start before
                        // this CTA's P^T arrives below
                        const bool okp = mbar_wait_cluster(pv_done, (gb - 1) & 1);
                        pv_waited = true;
                        tc_fence_after();
                        if (__all_sync(0xffffffffu, okp)) {
#pragma unroll 1
                            for (int ch = 0; ch < 4; ++ch) {
                                uint32_t o[32];
                                const uint32_t oa = t_lane + C::TMEM_O + 128 * h2 + 32 * ch;
                                tmem_ld32(oa, o);
                                tmem_wait_ld();
#pragma unroll
                                for (int i = 0; i < 32; ++i)
                                    o[i] = __float_as_uint(__uint_as_float(o[i]) * fs[32 * ch + i]);
                                tmem_st32(oa, o);
                            }
                            tmem_wait_st();
                        }
                    }
                }
                // ---- P^T of this thread's key for its 64 heads (bf16 pairs)
                uint32_t pk[32];
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    uint32_t sr[32];
                    tmem_ld32(sb + 32 * jj, sr);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 m2 = reinterpret_cast<const float2 *>(mr)[32 * h2 + 16 * jj + i];
                        const float p0 = vis ? ex2_approx(fmaf(__uint_as_float(sr[2 * i]), sl2, -m2.x)) : 0.f;
                        const float p1 = vis ? ex2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), sl2, -m2.y)) : 0.f;
                        l[32 * jj + 2 * i] += p0;
                        l[32 * jj + 2 * i + 1] += p1;
                        pk[16 * jj + i] = pack_bf16x2(p0, p1);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(s_free_lead + 8u * (gb & 1));   // S^T consumed
                if (b > 0 && !pv_waited) {
                    // PV_{b-1} still reads the P^T buffer (block 0's predecessor, the previous
                    // unit's last PV, completed before that unit's epilogue)
                    const bool okp = mbar_wait_cluster(pv_done, (gb - 1) & 1);
                    if (!okp) misc[1] = 1;
                }
                {
                    // row 128 cr + key of the P^T buffer of the CTA holding heads 64 h2 .. + 63
                    const uint32_t row = (uint32_t)(128 * cr + key);
                    if (h2 == cr) {
                        const uint32_t base = p_s + row * 128;
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            st_shared_v4(base + ((v ^ (row & 7)) << 4), pk[4 * v], pk[4 * v + 1], pk[4 * v + 2],
                                         pk[4 * v + 3]);
                        fence_proxy_async_smem();
                    } else {
                        const uint32_t base = p_peer_s + row * 128;
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            st_cluster_v4(base + ((v ^ (row & 7)) << 4), pk[4 * v], pk[4 * v + 1], pk[4 * v + 2],
                                          pk[4 * v + 3]);
                        fence_proxy_async_cluster();
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(p_full_lead);   // this warp's 32 rows are in place
                if (named_bar_or(1, 256, misc[1] != 0)) {
                    ok = false;
                    break;
                }
            }
            if (!ok && st == 0) abort_pair();

            // ---- epilogue: row sums of the pair, lse, O^T / l transposed into out
            const int64_t obase = (int64_t)t * 128;
            const int64_t pbase = ((int64_t)t * nsplit + split) * 128;   // partial rows (split mode)
            if (nblocks > 0 && ok) {
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = l[32 * jj + i];
                    red[quarter * 128 + 64 * h2 + 32 * jj + lane] = transpose_reduce32<false>(v, lane);
                }
                named_bar(1, 256);
                if (st < 128) {
                    const int h = st;
                    const float l_cta = (red[h] + red[128 + h]) + (red[256 + h] + red[384 + h]);
                    st_async_f32(mapa_shared(sbase + C::OFF_XL + 4u * h, (uint32_t)peer), l_cta,
                                 mapa_shared(lbar, (uint32_t)peer));
                    if (st == 0) mbar_expect_tx(lbar, 128 * 4);
                    const bool okl = mbar_wait_cluster(lbar, nq & 1);
                    // the two CTAs add the same two numbers in the same order
                    const float l_tot = cr == 0 ? l_cta + xl[h] : xl[h] + l_cta;
                    const bool fine = okl && l_tot > 0.f;
                    fs[h] = fine ? 1.0f / l_tot : 0.f;
                    if ((h >> 6) == cr) {
                        const float lv =
                            okl ? (l_tot > 0.f ? (mr[h] + log2f(l_tot)) * 0.6931471805599453f : -INFINITY) : NAN;
                        if (partial) sp.lse_part[pbase + h] = lv;
                        else lse[obase + h] = lv;
                    }
                }
                const bool oko = mbar_wait_cluster(o_ready, nq & 1);
                named_bar(1, 256);
                tc_fence_after();
                // O^T block i = h2: lanes = value dims 256 h2 + 128 cr + quarter*32 + lane, columns = heads
                if (partial) {   // fp32 partial rows, written from registers (32 lanes: 128 bytes per head)
                    float *op = sp.o_part + pbase * 512 + 256 * h2 + 128 * cr + key;
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t o[32];
                        tmem_ld32(t_lane + C::TMEM_O + 128 * h2 + 32 * ch, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int h = 32 * ch + i;
                            op[(int64_t)h * 512] = oko ? __uint_as_float(o[i]) * fs[h] : 0.f;
                        }
                    }
                } else {
                    // bf16 rows from registers: lanes 2m and 2m + 1 swap one value per head pair, so
                    // each stores two adjacent dims of one head (64 contiguous bytes per head per warp)
                    const bool odd = (lane & 1) != 0;
                    __nv_bfloat16 *orow = out + obase * 512 + 256 * h2 + 128 * cr + 32 * quarter + (lane & ~1);
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t o[32];
                        tmem_ld32(t_lane + C::TMEM_O + 128 * h2 + 32 * ch, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            const int h = 32 * ch + i;
                            const float v0 = oko ? __uint_as_float(o[i]) * fs[h] : 0.f;
                            const float v1 = oko ? __uint_as_float(o[i + 1]) * fs[h + 1] : 0.f;
                            const float recv = __shfl_xor_sync(0xffffffffu, odd ? v0 : v1, 1);
                            const uint32_t w = odd ? pack_bf16x2(recv, v1) : pack_bf16x2(v0, recv);
                            *reinterpret_cast<uint32_t *>(orow + (int64_t)(h + (odd ? 1 : 0)) * 512) = w;
                        }
                    }
                }
                // O^T read out: ordered before this warp's next arrivals (s_free, p_full) by the
                // tcgen05 fence that precedes them
            } else {
                // no visible slot (or an aborted pipeline): out = 0, lse = -inf (NaN if aborted)
                for (int e = st; e < 128 * 32; e += 256) {
                    const int h = e >> 5, part = e & 31;      // 32 x 16 bytes per head: the CTA's 2 x 128 dims
                    const int d0 = 256 * (part >> 4) + 128 * cr + 8 * (part & 15);
                    if (partial) {
                        float4 *op = reinterpret_cast<float4 *>(sp.o_part + (pbase + h) * 512 + d0);
                        op[0] = make_float4(0.f, 0.f, 0.f, 0.f);
                        op[1] = make_float4(0.f, 0.f, 0.f, 0.f);
                    } else {
                        *reinterpret_cast<uint4 *>(out + (obase + h) * 512 + d0) = make_uint4(0, 0, 0, 0);
                    }
                }
                if (st < 128 && (st >> 6) == cr) {
                    const float lv = nblocks == 0 ? -INFINITY : NAN;
                    if (partial) sp.lse_part[pbase + st] = lv;
                    else lse[obase + st] = lv;
                }
            }
            gb0 += nblocks;
            if (nblocks > 0) ++nq;
        }
    }
    // ---- teardown: nothing of either CTA is in flight past this point.  After an abort
    // (either CTA's flag, so both take the same branch) the even CTA first waits, bounded,
    // until the last position either CTA issued into each slot has landed.  Each CTA hands
    // its final flag to the peer before the cluster barrier: past that barrier the peer may
    // already have exited, so nothing reads the peer's shared memory there.
    tc_fence_before();
    __syncthreads();                                         // this CTA's roles are done
    if (tid == 0) st_cluster_u32(mapa_shared(sbase + C::OFF_MISC + 16, (uint32_t)peer), misc[1]);
    cluster_sync();
    const bool aborted = misc[1] != 0u || misc[4] != 0u;     // the same in both CTAs
    if (aborted) {
        if (cr == 0 && run && tid < C::NSLOT) {
            const int *lp = reinterpret_cast<const int *>(smem + C::OFF_LASTPOS);
            const int pmax = max(lp[tid], lp[C::NSLOT + tid]);
            if (pmax >= 0) mbar_wait_cluster(pfull(tid), (uint32_t)(pmax / C::NSLOT) & 1u);
        }
        cluster_sync();
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

// Merges the nsplit partial results of each (token, head): lse = log sum_c exp(lse_c),
// out = sum_c exp(lse_c - lse) o_c, rounded once to bf16.  Splits without a visible slot
// (lse_c = -inf) weigh 0; a row without any gives out = 0, lse = -inf.  grid = T * 128
// blocks of 128 threads (4 value dims each).
__global__ void __launch_bounds__(128) combine_splits_kernel(int nsplit, const float *__restrict__ o_part,
                                                            const float *__restrict__ lse_part,
                                                            __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    const int row = blockIdx.x;                              // t * 128 + h
    const int t = row >> 7, h = row & 127;
    float m = -INFINITY;
    for (int c = 0; c < nsplit; ++c) m = fmaxf(m, lse_part[((int64_t)t * nsplit + c) * 128 + h]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (m != -INFINITY) {
        for (int c = 0; c < nsplit; ++c) {
            const int64_t pr = ((int64_t)t * nsplit + c) * 128 + h;
            const float lc = lse_part[pr];
            const float wgt = lc == -INFINITY ? 0.f : expf(lc - m);
            wsum += wgt;
            const float4 v = reinterpret_cast<const float4 *>(o_part + pr * 512)[threadIdx.x];
            acc.x = fmaf(wgt, v.x, acc.x);
            acc.y = fmaf(wgt, v.y, acc.y);
            acc.z = fmaf(wgt, v.z, acc.z);
            acc.w = fmaf(wgt, v.w, acc.w);
        }
    }
    const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
    __nv_bfloat16 *o = out + (int64_t)row * 512 + 4 * threadIdx.x;
    o[0] = __float2bfloat16_rn(acc.x * inv);
    o[1] = __float2bfloat16_rn(acc.y * inv);
    o[2] = __float2bfloat16_rn(acc.z * inv);
    o[3] = __float2bfloat16_rn(acc.w * inv);
    if (threadIdx.x == 0) lse[row] = m == -INFINITY ? -INFINITY : m + logf(wsum);
}

}  // namespace mla
}  // namespace dsa
