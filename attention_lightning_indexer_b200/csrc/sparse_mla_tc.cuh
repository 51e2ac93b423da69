// sparse_mla_tc.cuh -- attention over the selected latent rows (MLA in MQA mode) on the
// 5th-generation tensor cores.
//
// "DeepSeek-V3.2 tech report summary", §1 DSA: full attention only over the k selected
// tokens; MLA-based implementation in MQA mode (every 576-d latent row is shared by all
// 128 query heads); value = first 512 dims; softmax scale 1/sqrt(192).
//
// One CTA per (query token, value half v).  The selected-index row is cut into blocks
// of 128 slots; for block b:
//   S_b[h, key] = q[h, :] . kv[key, :]                 (M = 128 heads, N = 128 keys, K = 576)
//   P_b         = exp2(S_b * scale * log2 e - m[h])     (online softmax, lazy rescale)
//   O_v[h, :]  += P_b[h, key] kv[key, 256 v : 256 v + 256]
// A slot whose index is not a visible key (-1, a future position, out of range) is
// gathered as key 0 of the sequence and masked out of the softmax.  Blocks past the last
// visible slot are skipped, so the top-k output (visible slots first, -1 after) costs
// ceil(k_eff / 128) blocks.
// Tensor memory (512 columns): O_v [0,256) fp32 and two S/P buffers [256,384), [384,512):
// S_b lands in buffer b & 1 and is overwritten in place by P_b (bf16 pairs), the A operand
// of the PV product.  With two buffers the tensor core computes S_{b+1} while the softmax
// warps turn S_b into P_b.
// Shared memory: all of q (9 swizzled 64-dim atoms of 128 heads, 144 KB), so every QK MMA
// reads both operands from shared memory (mixing tensor-memory and shared-memory A
// operands into one accumulator runs at about half rate), and a 5-slot ring of 64-dim
// atoms of gathered latent rows (16 KB each) fed in MMA issue order:
//   QK_0, QK_1, PV_0, QK_2, PV_1, ..., QK_{n-1}, PV_{n-2}, PV_{n-1}
// (QK: the 9 atoms of the block; PV: the 4 value atoms of the block, gathered again and
// consumed as two N = 128 pairs; the lower atom of a pair sits in the lower ring slot).
// Atoms are gathered with 16-byte cp.async (one warp instruction moves 128 bytes of 4
// rows; the 128-byte swizzle is applied in the shared-memory address) from row numbers
// held in registers, so the copies issue back to back; each lane signals the slot
// asynchronously when its copies land (cp.async mbarrier arrive).  One warp issues about
// 20 bytes per clock and three reach the SM's gather rate of about 57, so three loader
// warps take the ring positions in turn.
//
// Warp roles (12 warps): 0, 2, 3 gather (2 also allocates tensor memory), 1 issues the
// MMAs (one thread), 4-11 scan the index row for its last visible slot, then run the
// softmax and the epilogue: warp w owns TMEM lane quarter w % 4 (32 heads) and key/column
// half c = (w - 4) / 4.  Thread 0 issues the q TMA right after initialising the barriers,
// and the loaders gather the first five atoms of block 0 while the row is scanned.
#pragma once

#include "dsa_common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace mla {

struct TcCfg {
    static constexpr int BK = 128;                  // index slots (keys) per block
    static constexpr int NATOM = 9;                 // 64-dim atoms per 576-d row
    static constexpr int ATOM_BYTES = BK * 128;     // one atom of a 128-row tile
    static constexpr int NSLOT = 5;                 // gather ring slots
    static constexpr int NLOAD = 3;                 // loader warps, taking ring positions in turn
    // A loader waiting for position p - NSLOT to be consumed has itself seen position
    // p - NLOAD's slot freed, i.e. p - NLOAD - NSLOT consumed; with NLOAD <= NSLOT that
    // covers p - 2 NSLOT, so the parity wait cannot alias an older phase.
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_RING = NATOM * ATOM_BYTES;                  // 147456
    static constexpr int OFF_RED = OFF_RING + NSLOT * ATOM_BYTES;         // [2][128] floats
    static constexpr int OFF_BAR = OFF_RED + 2 * 128 * 4;
    // ring_full[5], ring_empty[5], q_full, s_full[2], p_full[2], pv_done, o_ready
    static constexpr int NBARS = 2 * NSLOT + 1 + 2 + 2 + 1 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int SMEM = OFF_MISC + 16;
    static constexpr int THREADS = 384;
    static constexpr int TMEM_O = 0, TMEM_S = 256;
    static constexpr float TAU = 8.0f;              // lazy-rescale threshold (log2 units)
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(NLOAD <= NSLOT, "ring waits need NLOAD <= NSLOT");
};

// Value atom at offset m (0..3) of a PV group starting at ring position pv_start: pair
// (m >> 1) holds atoms 4v + 2*pair + {0,1}; the lower atom goes to the lower-addressed
// ring slot so that the pair is one MN-major operand with a positive atom stride.
__device__ __forceinline__ int pv_atom(int v, int pv_start, int m) {
    const int pp = pv_start + (m & ~1);
    const bool lo_first = (pp % TcCfg::NSLOT) < ((pp + 1) % TcCfg::NSLOT);
    const int e = m & 1;
    return 4 * v + 2 * (m >> 1) + (lo_first ? e : 1 - e);
}

// Group g (0 .. 2n-1) of the ring order QK_0, QK_1, PV_0, QK_2, PV_1, ..., PV_{n-1}:
// whether it is a QK group, and its block.
__device__ __forceinline__ void ring_group(int g, int n, bool &qk, int &blk) {
    if (g == 0) { qk = true; blk = 0; }
    else if (g == 2 * n - 1) { qk = false; blk = n - 1; }
    else if (g & 1) { qk = true; blk = (g + 1) >> 1; }
    else { qk = false; blk = (g >> 1) - 1; }
}

__device__ __forceinline__ bool visible(int e, const RowInfo &ri) { return e >= 0 && e <= ri.pos && e < ri.len_k; }

// One loader warp's part of the ring: the positions p with p % NLOAD == lw, each a whole
// atom (32 copy instructions; instruction i moves 128 bytes of rows i, 32+i, 64+i, 96+i:
// lane l copies 16-byte chunk l % 8 of row 32 (l / 8) + i).  Returns false if a wait gave
// up or another role aborted.
// Index entries of block j for lane `lane`'s rows (32 (lane / 8) + i, i < 32); slots past
// the end of the row read as -1.
__device__ __forceinline__ void fetch_rows(const int32_t *irow, int K, int j, int lane, int (&e)[32]) {
    const int s0 = j * TcCfg::BK + (lane >> 3) * 32;
    if ((K & 3) == 0 && s0 + 31 < K) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int4 x = __ldg(reinterpret_cast<const int4 *>(irow + s0) + i);
            e[4 * i] = x.x; e[4 * i + 1] = x.y; e[4 * i + 2] = x.z; e[4 * i + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) e[i] = s0 + i < K ? __ldg(irow + s0 + i) : -1;
    }
}

// One atom's 32 copy instructions into a ring slot, then the lane's asynchronous arrival on
// the slot's ring_full barrier.
__device__ __forceinline__ void gather_atom(const char *kv_bytes, const int (&rows)[32], int a, uint32_t slot,
                                            uint32_t full_bar, int lane) {
    using namespace sm100;
    const int ch = lane & 7;
    const int r0 = (lane >> 3) * 32;
    const char *src = kv_bytes + a * 128 + ch * 16;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int r = r0 + i;
        cp_async16(slot + r * 128 + ((ch ^ (r & 7)) << 4), src + (int64_t)rows[i] * 1152);
    }
    cp_async_arrive_noinc(full_bar);                         // fires when this lane's copies land
}

// Before the visible extent of the row is known: the first NSLOT atoms of QK_0 (ring
// positions 0 .. NSLOT-1 need no slot wait), this warp's share of them.  `rows` keeps
// block 0's row numbers for gather_turns.
__device__ __forceinline__ void gather_first(int lw, const int32_t *irow, int K, const RowInfo &ri,
                                             const char *kv_bytes, uint32_t ring_s, uint32_t bar0, int lane,
                                             int (&rows)[32]) {
    using C = TcCfg;
    fetch_rows(irow, K, 0, lane, rows);
#pragma unroll
    for (int i = 0; i < 32; ++i) rows[i] = ri.kbase + (visible(rows[i], ri) ? rows[i] : 0);
    for (int pp = lw; pp < C::NSLOT; pp += C::NLOAD)
        gather_atom(kv_bytes, rows, pp, ring_s + pp * C::ATOM_BYTES, bar0 + 8u * pp, lane);
}

__device__ __forceinline__ bool gather_turns(int lw, const int32_t *irow, int K, const RowInfo &ri,
                                             const char *kv_bytes, uint32_t ring_s, uint32_t bar0, int v, int nblocks,
                                             volatile uint32_t *misc, int lane, int (&rows)[32]) {
    using C = TcCfg;
    using namespace sm100;
    static_assert(C::NSLOT <= C::NATOM, "the early positions all belong to QK_0");
    // index entries of block j for this lane's rows
    auto fetch = [&](int j, int (&e)[32]) {
        fetch_rows(irow, K, j, lane, e);
    };
    // raw: entries of the next QK block (prefetched); rows: row numbers of the current
    // group's block (block 0's on entry; a PV group re-reads its block's entries, by then in L1)
    int raw[32];
    if (nblocks > 1) fetch(1, raw);
    int p = 0;                                               // ring position of the group's first atom
    for (int g = 0; g < 2 * nblocks; ++g) {
        bool qk;
        int blk;
        ring_group(g, nblocks, qk, blk);
        if (qk && blk > 0) {                                 // rows of block blk; prefetch blk + 1
#pragma unroll
            for (int i = 0; i < 32; ++i) rows[i] = ri.kbase + (visible(raw[i], ri) ? raw[i] : 0);
            if (blk + 1 < nblocks) fetch(blk + 1, raw);
        } else if (!qk) {
            fetch(blk, rows);
#pragma unroll
            for (int i = 0; i < 32; ++i) rows[i] = ri.kbase + (visible(rows[i], ri) ? rows[i] : 0);
        }
        const int natoms = qk ? C::NATOM : 4;
        for (int m = 0; m < natoms; ++m) {
            const int pp = p + m;
            if (pp % C::NLOAD != lw || pp < C::NSLOT) continue;   // positions < NSLOT: gather_first
            const int a = qk ? m : pv_atom(v, p, m);
            const int slot_i = pp % C::NSLOT;
            bool okw = true;
            if (lane == 0) okw = mbar_wait(bar0 + 8u * (C::NSLOT + slot_i), ((pp / C::NSLOT) - 1) & 1);
            if (!__shfl_sync(0xffffffffu, okw, 0) || misc[1]) return false;
            gather_atom(kv_bytes, rows, a, ring_s + slot_i * C::ATOM_BYTES, bar0 + 8u * slot_i, lane);
        }
        p += natoms;
    }
    return true;
}

__global__ void __launch_bounds__(384, 1)
sparse_mla_tc_kernel(const __grid_constant__ CUtensorMap tm_q, Problem P, const __nv_bfloat16 *__restrict__ q,
                     const __nv_bfloat16 *__restrict__ kv, const int32_t *__restrict__ idx,
                     __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    using C = TcCfg;
    using namespace sm100;
    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = P.total_q;
    const int t = T - 1 - (int)(blockIdx.x >> 1);           // heavier (later) tokens first
    const int v = (int)(blockIdx.x & 1);                     // value half
    const int K = P.topk;
    const RowInfo ri = row_info(P, t);
    const int32_t *irow = idx + (int64_t)t * K;
    const bool vec4 = (K & 3) == 0;                          // rows of idx are 16-byte aligned

    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {
        if (tid == 0) raise_error(ERR_SMEM_ALIGN);
        return;
    }
    const uint32_t q_s = sbase + C::OFF_Q;
    const uint32_t ring_s = sbase + C::OFF_RING;
    float *red = reinterpret_cast<float *>(smem + C::OFF_RED);       // [2 halves][128]
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto ring_full = [&](int s) { return bar0 + 8u * s; };
    auto ring_empty = [&](int s) { return bar0 + 8u * (C::NSLOT + s); };
    const uint32_t q_full = bar0 + 8u * (2 * C::NSLOT);
    auto s_full = [&](int b) { return q_full + 8u * (1 + b); };
    auto p_full = [&](int b) { return q_full + 8u * (3 + b); };
    const uint32_t pv_done = q_full + 40;
    // o_ready completes once, after the last PV: pv_done may still have two phases in
    // flight when the epilogue starts, so its parity alone cannot tell them apart
    const uint32_t o_ready = q_full + 48;
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);  // tmem, abort

    // ---- setup
    if (tid == 0) {
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(ring_full(s), 32);   // every lane of the loading warp arrives
            mbar_init(ring_empty(s), 1);
        }
        mbar_init(q_full, 1);
        mbar_init(s_full(0), 1);
        mbar_init(s_full(1), 1);
        mbar_init(p_full(0), 8);
        mbar_init(p_full(1), 8);
        mbar_init(pv_done, 1);
        mbar_init(o_ready, 1);
        misc[1] = 0;
        fence_barrier_init();
        // q lands while the index row is scanned (waited for before exit even when the row
        // has no visible slot)
        prefetch_tmap(&tm_q);
        mbar_expect_tx(q_full, C::NATOM * C::ATOM_BYTES);
        for (int a = 0; a < C::NATOM; ++a) tma_load_2d(q_s + a * C::ATOM_BYTES, &tm_q, q_full, 64 * a, t * 128);
    }
    if (warp == 2) tmem_alloc(sbase + C::OFF_MISC, 512);
    const char *kv_bytes = reinterpret_cast<const char *>(kv);
    const int lw = warp == 0 ? 0 : warp - 1;                 // loader warps 0, 2, 3: ring positions p % 3 == lw
    int rows0[32];                                           // a loader's row numbers of block 0
    if (warp == 0 || warp == 2 || warp == 3) {
        // the first ring positions are gathered while the row is scanned: they hold atoms of
        // block 0, which exists whenever any slot is visible (otherwise nothing consumes them)
        __syncwarp();
        named_bar(3, 96);                                    // the barriers are initialised
        gather_first(lw, irow, K, ri, kv_bytes, ring_s, bar0, lane, rows0);
    }
    if (warp >= 4) {   // last visible slot of this row (8 warps, interleaved int4 groups)
        int last = -1;
        const int part = warp - 4;
        if (vec4) {
            const int n4 = K >> 2;
#pragma unroll 2
            for (int i4 = part * 32 + lane; i4 < n4; i4 += 256) {
                const int4 x = __ldg(reinterpret_cast<const int4 *>(irow) + i4);
                if (visible(x.x, ri)) last = 4 * i4;
                if (visible(x.y, ri)) last = 4 * i4 + 1;
                if (visible(x.z, ri)) last = 4 * i4 + 2;
                if (visible(x.w, ri)) last = 4 * i4 + 3;
            }
        } else {
            for (int i = part * 32 + lane; i < K; i += 256)
                if (visible(__ldg(irow + i), ri)) last = i;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
        if (lane == 0) reinterpret_cast<int *>(red)[part] = last;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    int last_slot = -1;
#pragma unroll
    for (int i = 0; i < 8; ++i) last_slot = max(last_slot, reinterpret_cast<int *>(red)[i]);
    const int nblocks = (last_slot + C::BK) / C::BK;         // 0 when no slot is visible
    __syncthreads();   // red is reused by the softmax warps

    if (warp == 0 || warp == 2 || warp == 3) {
        // ------------------------------------------------ gather loaders (+ q TMA)
        const bool ok_run = gather_turns(lw, irow, K, ri, kv_bytes, ring_s, bar0, v, nblocks, misc, lane, rows0);
        if (!ok_run) misc[1] = 1;
        cp_async_wait<0>();
        // a row without a visible slot: the q tile was still loaded; let it land before exit
        if (nblocks == 0 && warp == 0 && lane == 0) mbar_wait(q_full, 0);
    } else if (warp == 1 && lane == 0 && nblocks > 0) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idesc_qk = idesc_bf16(128, C::BK);
        const uint32_t idesc_pv = idesc_bf16_bmn(128, 128);
        bool ok = mbar_wait(q_full, 0);
        int pos = 0;
        for (int g = 0; ok && g < 2 * nblocks; ++g) {
            bool qk;
            int b;
            ring_group(g, nblocks, qk, b);
            if (qk) {                                        // QK_b -> S buffer b & 1
                const uint32_t d = tmem + C::TMEM_S + 128 * (b & 1);
                for (int a = 0; a < C::NATOM; ++a, ++pos) {
                    if (!mbar_wait(ring_full(pos % C::NSLOT), (pos / C::NSLOT) & 1)) { ok = false; break; }
                    fence_proxy_async_smem();
                    const uint32_t slot = ring_s + (pos % C::NSLOT) * C::ATOM_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(d, desc_sw128(q_s + a * C::ATOM_BYTES + kk * 32), desc_sw128(slot + kk * 32), idesc_qk,
                                (a > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(ring_empty(pos % C::NSLOT));
                }
                if (!ok) break;
                mma_commit(s_full(b & 1));
            } else {                                         // PV_b
                if (!mbar_wait(p_full(b & 1), (b >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t pa = tmem + C::TMEM_S + 128 * (b & 1);   // P_b as bf16 pairs
                for (int pair = 0; pair < 2; ++pair, pos += 2) {
                    if (!mbar_wait(ring_full(pos % C::NSLOT), (pos / C::NSLOT) & 1) ||
                        !mbar_wait(ring_full((pos + 1) % C::NSLOT), ((pos + 1) / C::NSLOT) & 1)) { ok = false; break; }
                    fence_proxy_async_smem();
                    const int s0 = pos % C::NSLOT, s1 = (pos + 1) % C::NSLOT;
                    const int slo = s0 < s1 ? s0 : s1, shi = s0 < s1 ? s1 : s0;
                    const uint32_t vb = ring_s + slo * C::ATOM_BYTES;
                    const uint32_t lbo = (uint32_t)(shi - slo) * C::ATOM_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::BK / 16; ++kk)
                        mma_f16_ts(tmem + C::TMEM_O + 128 * pair, pa + kk * 8, desc_sw128_mn(vb + kk * 2048, lbo),
                                   idesc_pv, (b > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(ring_empty(s0));
                    mma_commit(ring_empty(s1));
                }
                if (!ok) break;
                mma_commit(pv_done);
                if (b == nblocks - 1) mma_commit(o_ready);
            }
        }
        if (!ok) misc[1] = 1;
    } else if (warp >= 4) {
        // ------------------------------------------------ softmax + epilogue
        const int quarter = warp & 3;
        const int c = (warp - 4) >> 2;                  // key half of S, column half of O
        const int h = quarter * 32 + lane;              // head (TMEM lane)
        const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
        const float sl2 = P.sm_scale * 1.4426950408889634f;   // scale * log2(e)
        float m_run = -INFINITY, l_part = 0.f;
        bool ok = true;
        // index entries of this thread's key half of block b: slots 64c + lane (e[0]) and
        // 64c + 32 + lane (e[1]), fetched a block ahead
        auto fetch_mask = [&](int b, int (&e)[2]) {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int s = b * C::BK + 64 * c + 32 * u + lane;
                e[u] = s < K ? __ldg(irow + s) : -1;
            }
        };
        int ent[2] = {-1, -1};
        if (nblocks > 0) fetch_mask(0, ent);
        for (int b = 0; b < nblocks; ++b) {
            // bit i of w0 / w1: key 64c + i / 64c + 32 + i of the block is visible
            const unsigned w0 = __ballot_sync(0xffffffffu, visible(ent[0], ri));
            const unsigned w1 = __ballot_sync(0xffffffffu, visible(ent[1], ri));
            if (b + 1 < nblocks) fetch_mask(b + 1, ent);
            const bool fail = misc[1] != 0 || !mbar_wait(s_full(b & 1), (b >> 1) & 1);
            if (named_bar_or(1, 256, fail)) { ok = false; misc[1] = 1; break; }   // all 8 warps leave together
            tc_fence_after();
            const uint32_t sb = t_lane + C::TMEM_S + 128 * (b & 1);
            uint32_t s0[32], s1[32];
            tmem_ld32(sb + 64 * c, s0);
            tmem_ld32(sb + 64 * c + 32, s1);
            tmem_wait_ld();
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if ((w0 >> i) & 1u) mx = fmaxf(mx, __uint_as_float(s0[i]));
                if ((w1 >> i) & 1u) mx = fmaxf(mx, __uint_as_float(s1[i]));
            }
            // red is single-buffered: every thread passed this block's opening barrier
            // only after reading the previous block's values
            red[c * 128 + h] = mx;
            named_bar(1, 256);
            const float m_blk = fmaxf(red[h], red[128 + h]) * sl2;
            // Lazy rescale: a row moves its reference max only when the block max exceeds it
            // by more than TAU.  The TMEM load/store is warp-collective, so the whole warp
            // takes that path when any of its rows needs it (factor 1 for the others).
            // A block without a visible slot has m_blk = -inf and never moves it.
            const bool need = m_blk > m_run + C::TAU;
            const float f = (need && m_run != -INFINITY) ? exp2f(m_run - m_blk) : 1.0f;
            if (need) m_run = m_blk;
            uint32_t pk[32];
            float ls = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float p0 = (w0 >> (2 * i)) & 1u ? ex2_approx(fmaf(__uint_as_float(s0[2 * i]), sl2, -m_run)) : 0.f;
                const float p1 = (w0 >> (2 * i + 1)) & 1u ? ex2_approx(fmaf(__uint_as_float(s0[2 * i + 1]), sl2, -m_run)) : 0.f;
                ls += p0 + p1;
                pk[i] = pack_bf16x2(p0, p1);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float p0 = (w1 >> (2 * i)) & 1u ? ex2_approx(fmaf(__uint_as_float(s1[2 * i]), sl2, -m_run)) : 0.f;
                const float p1 = (w1 >> (2 * i + 1)) & 1u ? ex2_approx(fmaf(__uint_as_float(s1[2 * i + 1]), sl2, -m_run)) : 0.f;
                ls += p0 + p1;
                pk[16 + i] = pack_bf16x2(p0, p1);
            }
            tmem_st32(sb + 32 * c, pk);
            if (b > 0 && __any_sync(0xffffffffu, need)) {
                // Rescale O (done after storing P_b, when S_b is no longer live).  O must
                // include PV_{b-1} first; QK_b was issued after PV_{b-2}, so pv_done has
                // completed b-1 or b phases here and the parity of phase b-1 is unambiguous.
                // PV_b cannot start before this warp's p_full arrival below.
                const bool okp = mbar_wait(pv_done, (b - 1) & 1);
                tc_fence_after();
                l_part *= f;
                if (__all_sync(0xffffffffu, okp)) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t o[32];
                        const uint32_t oa = t_lane + C::TMEM_O + 128 * c + 32 * ch;
                        tmem_ld32(oa, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                        tmem_st32(oa, o);
                    }
                }
            }
            l_part += ls;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full(b & 1));
        }
        // ---- epilogue
        const int64_t orow = ((int64_t)t * 128 + h) * 512 + 256 * v + 128 * c;
        if (nblocks == 0 || !ok) {
            uint4 z = make_uint4(0, 0, 0, 0);
            for (int i = 0; i < 16; ++i) reinterpret_cast<uint4 *>(out + orow)[i] = z;
            if (v == 0 && c == 0) lse[(int64_t)t * 128 + h] = nblocks == 0 ? -INFINITY : NAN;
        } else {
            bool okw = mbar_wait(o_ready, 0);
            tc_fence_after();
            // the last block's max was read before its p_full arrival, which the last PV
            // (hence o_ready) waited for: red may be reused
            red[c * 128 + h] = l_part;
            named_bar(1, 256);
            const float l = red[h] + red[128 + h];
            const float inv = (l > 0.f && okw) ? 1.0f / l : 0.f;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t o[32];
                tmem_ld32(t_lane + C::TMEM_O + 128 * c + 32 * ch, o);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
                uint4 *dst = reinterpret_cast<uint4 *>(out + orow + 32 * ch);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
            if (v == 0 && c == 0) lse[(int64_t)t * 128 + h] = (m_run + log2f(l)) * 0.6931471805599453f;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace mla
}  // namespace dsa
