// sparse_mla_tc.cuh -- attention over the selected latent rows (MLA in MQA mode) on the
// 5th-generation tensor cores.
//
// "DeepSeek-V3.2 tech report summary", §1 DSA: full attention only over the k selected
// tokens; MLA-based implementation in MQA mode (every 576-d latent row is shared by all
// 128 query heads); value = first 512 dims; softmax scale 1/sqrt(192).
//
// One CTA per (query token, value half v).  Per block of 128 selected keys:
//   S[h, key]  = q[h, :] . kv[key, :]        (M = 128 heads, N = 128 keys, K = 576)
//   P          = exp2(S * scale * log2 e - m[h])   (online softmax, lazy rescale)
//   O_v[h, :] += P[h, key] kv[key, 256 v : 256 v + 256]   (M = 128, N = 256, K = 128 keys)
// Tensor memory (512 columns): O_v [0,256) fp32; q dims 0..255 as the A operand of
// the first 16 QK k-steps [256,384) (bf16 pairs); S [384,512) fp32, overwritten in
// place by P as bf16 pairs [384,448) -- the A operand of the PV product.
// Shared memory: q dims 256..575 (5 swizzled 128-byte atoms, 80 KB) and a 9-slot ring,
// one slot per 64-dim atom of the current block's 128 gathered latent rows (144 KB);
// slot a always holds atom a, so the 4 atoms of this CTA's value half are 4
// consecutive slots and serve directly as the MN-major B operand of the PV product.
// Rows are gathered by three producer warps with 16-byte cp.async (each warp
// instruction moves 4 rows x 128 bytes of one atom; the 128-byte swizzle is applied in
// the shared-memory address).  Small TMA gathers were issue-bound here; the LSU path
// keeps the gather off the critical path.  The selected indices are compacted on the
// fly (invalid slots -- -1, future or out-of-range positions -- are skipped); the tail
// of the last block is padded with a duplicate row and masked in the softmax.
//
// Warp roles (12 warps): 0 index compaction + gathers + q TMA, 1 MMA issuer, 2 TMEM
// allocator then gathers, 3 gathers, 4-11 softmax/epilogue: warp w owns TMEM lane
// quarter w % 4 (32 heads) and key/column half c = (w - 4) / 4.
#pragma once

#include "dsa_common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace mla {

struct TcCfg {
    static constexpr int BK = 128;                  // keys per block
    static constexpr int NATOM = 9;                 // 64-dim atoms per 576-d row
    static constexpr int ATOM_BYTES = BK * 128;     // one atom of a 128-row tile
    static constexpr int QHI_ATOMS = 5;             // q dims 256..575 in shared memory
    static constexpr int OFF_QHI = 0;
    static constexpr int OFF_KV = QHI_ATOMS * ATOM_BYTES;            // 81920
    static constexpr int OFF_RED = OFF_KV + NATOM * ATOM_BYTES;      // 229376
    static constexpr int OFF_STAGE = OFF_RED + 2 * 128 * 4;          // row-max / sum exchange
    static constexpr int STAGE_CAP = 256;                            // compacted indices
    static constexpr int OFF_BAR = OFF_STAGE + STAGE_CAP * 4;
    static constexpr int NBARS = 2 * NATOM + 5;
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int SMEM = OFF_MISC + 16;
    static constexpr int THREADS = 384;
    static constexpr int TMEM_O = 0, TMEM_QLO = 256, TMEM_S = 384;
    static constexpr float TAU = 8.0f;              // lazy-rescale threshold (log2 units)
    static_assert(SMEM <= 232448, "shared memory budget");
};

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

    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {
        if (tid == 0) raise_error(ERR_SMEM_ALIGN);
        return;
    }
    const uint32_t qhi_s = sbase + C::OFF_QHI;
    const uint32_t kv_s = sbase + C::OFF_KV;
    float *red = reinterpret_cast<float *>(smem + C::OFF_RED);      // [2 halves][128]
    int *stage = reinterpret_cast<int *>(smem + C::OFF_STAGE);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto kv_full = [&](int a) { return bar0 + 8u * a; };
    auto kv_empty = [&](int a) { return bar0 + 8u * (C::NATOM + a); };
    const uint32_t q_full = bar0 + 8u * (2 * C::NATOM);
    const uint32_t qlo_ready = q_full + 8;
    const uint32_t s_full = q_full + 16;
    const uint32_t p_full = q_full + 24;
    const uint32_t pv_done = q_full + 32;
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);  // tmem, nvalid, abort

    // ---- setup
    if (tid == 0) {
        for (int a = 0; a < C::NATOM; ++a) {
            mbar_init(kv_full(a), 32);   // one arrival per lane of the producing warp
            mbar_init(kv_empty(a), 1);
        }
        mbar_init(q_full, 1);
        mbar_init(qlo_ready, 8);
        mbar_init(s_full, 1);
        mbar_init(p_full, 8);
        mbar_init(pv_done, 1);
        misc[2] = 0;
        fence_barrier_init();
    }
    if (warp == 2) tmem_alloc(sbase + C::OFF_MISC, 512);
    if (warp == 0 || warp == 3) {   // number of valid selected indices of this row (2 warps)
        int cnt = 0;
        const int32_t *irow = idx + (int64_t)t * K;
        const int half = (warp == 0) ? 0 : 1;
        if ((K & 3) == 0) {
            // 16-byte loads, all issued before use
            const int n4 = K >> 2;
#pragma unroll 4
            for (int i4 = half * 32 + lane; i4 < n4; i4 += 64) {
                const int4 x = __ldg(reinterpret_cast<const int4 *>(irow) + i4);
                cnt += (x.x >= 0 && x.x <= ri.pos && x.x < ri.len_k) + (x.y >= 0 && x.y <= ri.pos && x.y < ri.len_k) +
                       (x.z >= 0 && x.z <= ri.pos && x.z < ri.len_k) + (x.w >= 0 && x.w <= ri.pos && x.w < ri.len_k);
            }
        } else {
            for (int i = half * 32 + lane; i < K; i += 64) {
                const int s = __ldg(irow + i);
                cnt += s >= 0 && s <= ri.pos && s < ri.len_k;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        if (lane == 0) red[half] = (float)cnt;   // exact for counts <= 2^24
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int nvalid = (int)red[0] + (int)red[1];
    __syncthreads();   // red is reused by the softmax warps
    const int nblocks = (nvalid + C::BK - 1) / C::BK;
    // QK atom order: the 5 atoms outside this CTA's value half first, then its 4 value atoms
    auto atom_of = [&](int ai) { return ai < 5 ? (ai + 4 * (1 - v) + (ai >= 4 ? 4 * v : 0)) % 9 : ai - 5 + 4 * v; };

    if (warp == 0 || warp == 2 || warp == 3) {
        // ------------------------------------------------ index compaction, gathers, q TMA
        const int pw = warp == 0 ? 0 : warp - 1;            // producer 0, 1, 2
        if (warp == 0 && lane == 0 && nblocks > 0) {
            prefetch_tmap(&tm_q);
            mbar_expect_tx(q_full, C::QHI_ATOMS * C::ATOM_BYTES);
            for (int a = 0; a < C::QHI_ATOMS; ++a)
                tma_load_2d(qhi_s + a * C::ATOM_BYTES, &tm_q, q_full, 256 + 64 * a, t * 128);
        }
        const int32_t *irow = idx + (int64_t)t * K;
        const bool vec4 = (K & 3) == 0;                      // rows of idx are 16-byte aligned
        auto load_chunk = [&](int rd, int (&e)[4]) {         // entries rd + 4*lane .. +3
            const int i = rd + 4 * lane;
            if (vec4 && i + 3 < K) {
                const int4 x = __ldg(reinterpret_cast<const int4 *>(irow + i));
                e[0] = x.x; e[1] = x.y; e[2] = x.z; e[3] = x.w;
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u) e[u] = i + u < K ? __ldg(irow + i + u) : -1;
            }
        };
        int rd = 0, cnt = 0;
        int nxt[4] = {-1, -1, -1, -1};
        if (warp == 0 && nblocks > 0) load_chunk(0, nxt);
        const char *kv_bytes = reinterpret_cast<const char *>(kv);
        bool ok_run = true;
        for (int j = 0; j < nblocks; ++j) {
            // the three producer warps leave together when any of them gave up
            if (named_bar_or(2, 96, !ok_run || misc[2] != 0)) { ok_run = false; break; }
            if (warp == 0) {
                while (cnt < C::BK && rd < K) {
                    int cur[4] = {nxt[0], nxt[1], nxt[2], nxt[3]};
                    rd += 128;
                    if (rd < K) load_chunk(rd, nxt);            // prefetch the next chunk
                    int vc = 0;
                    bool okv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        okv[u] = cur[u] >= 0 && cur[u] <= ri.pos && cur[u] < ri.len_k;
                        vc += okv[u];
                    }
                    int incl = vc;                            // in-warp prefix of valid entries
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int x = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += x;
                    }
                    const int tot = __shfl_sync(0xffffffffu, incl, 31);
                    int off = cnt + incl - vc;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (okv[u]) stage[off++] = ri.kbase + cur[u];
                    cnt += tot;
                }
                if (lane == 0) misc[3] = (uint32_t)min(cnt, C::BK);
            }
            named_bar(2, 96);                                 // stage holds this block's rows
            const int nb = (int)misc[3];
            const int base_row = stage[0];
            int rows[32];
#pragma unroll
            for (int g = 0; g < 32; ++g) {
                const int k = 4 * g + (lane >> 3);
                rows[g] = k < nb ? stage[k] : base_row;
            }
            named_bar(2, 96);                                 // all rows read: stage may be rewritten
            if (warp == 0) {                                  // keep the entries beyond this block
                const int left = cnt - nb;                    // < 128
                int keep[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) keep[u] = lane + 32 * u < left ? stage[C::BK + lane + 32 * u] : 0;
                __syncwarp();
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (lane + 32 * u < left) stage[lane + 32 * u] = keep[u];
                __syncwarp();
                cnt = left;
            }
            // phase 1: atoms outside this CTA's value half (free once QK of the previous
            // block consumed them); phase 2: the value atoms (free after the previous PV)
            for (int phase = 0; phase < 2 && ok_run; ++phase) {
                // this warp's atoms in QK order: ai = first + pw, first + pw + 3 (when in range)
                const int first = phase == 0 ? 0 : 5, last = phase == 0 ? 5 : 9;
                const int nmine = (first + pw < last) + (first + pw + 3 < last);
                for (int q = 0; q < nmine; ++q) {
                    const int a = atom_of(first + pw + 3 * q);
                    if (j > 0) {
                        bool okw = true;
                        if (lane == 0) okw = mbar_wait(kv_empty(a), (j - 1) & 1);
                        okw = __shfl_sync(0xffffffffu, okw, 0);
                        if (!okw || misc[2]) { misc[2] = 1; ok_run = false; break; }
                    }
                    const uint32_t slot = kv_s + a * C::ATOM_BYTES;
                    const int ch = lane & 7;
#pragma unroll
                    for (int g = 0; g < 32; ++g) {
                        const int r = 4 * g + (lane >> 3);
                        cp_async16(slot + r * 128 + ((ch ^ (r & 7)) << 4),
                                   kv_bytes + (int64_t)rows[g] * 1152 + a * 128 + ch * 16);
                    }
                    cp_async_commit();
                }
                if (!ok_run) break;
                // signal each atom once its copies have landed
                if (nmine == 2) {
                    cp_async_wait<1>();
                    fence_proxy_async_smem();
                    mbar_arrive(kv_full(atom_of(first + pw)));
                }
                if (nmine >= 1) {
                    cp_async_wait<0>();
                    fence_proxy_async_smem();
                    mbar_arrive(kv_full(atom_of(first + pw + 3 * (nmine - 1))));
                }
            }
        }
        // drain: the MMA commits on the value atoms of the last block must land before exit
        if (warp == 0 && lane == 0 && ok_run && nblocks > 0)
            for (int ai = 5; ai < C::NATOM; ++ai)
                if (!mbar_wait(kv_empty(atom_of(ai)), (nblocks - 1) & 1)) { misc[2] = 1; break; }
    } else if (warp == 1 && lane == 0 && nblocks > 0) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idesc_qk = idesc_bf16(128, C::BK);
        const uint32_t idesc_pv = idesc_bf16_bmn(128, 256);
        bool ok = mbar_wait(q_full, 0) && mbar_wait(qlo_ready, 0);
        tc_fence_after();
        for (int j = 0; ok && j < nblocks; ++j) {
            for (int ai = 0; ai < C::NATOM; ++ai) {
                const int a = atom_of(ai);
                // shared-memory operands only: the mbarrier (after the producers' proxy fence)
                // orders them; no tcgen05 fence is needed here
                if (!mbar_wait(kv_full(a), j & 1)) { ok = false; break; }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bdesc = desc_sw128(kv_s + a * C::ATOM_BYTES + kk * 32);
                    const uint32_t acc = (ai > 0 || kk > 0) ? 1u : 0u;
                    if (a < 4)
                        mma_f16_ts(tmem + C::TMEM_S, tmem + C::TMEM_QLO + a * 32 + kk * 8, bdesc, idesc_qk, acc);
                    else
                        mma_f16(tmem + C::TMEM_S, desc_sw128(qhi_s + (a - 4) * C::ATOM_BYTES + kk * 32), bdesc,
                                idesc_qk, acc);
                }
                if (ai < 5) mma_commit(kv_empty(a));
            }
            if (!ok) break;
            mma_commit(s_full);
            if (!mbar_wait(p_full, j & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t vbase = kv_s + 4 * v * C::ATOM_BYTES;
#pragma unroll
            for (int kk = 0; kk < C::BK / 16; ++kk)
                mma_f16_ts(tmem + C::TMEM_O, tmem + C::TMEM_S + kk * 8, desc_sw128_mn(vbase + kk * 2048, C::ATOM_BYTES),
                           idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
            for (int ai = 5; ai < C::NATOM; ++ai) mma_commit(kv_empty(atom_of(ai)));
            mma_commit(pv_done);
        }
        if (!ok) misc[2] = 1;
    } else if (warp >= 4) {
        // ------------------------------------------------ softmax + epilogue
        const int quarter = warp & 3;
        const int c = (warp - 4) >> 2;                  // key half of S, column half of O
        const int h = quarter * 32 + lane;              // head (TMEM lane)
        const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
        const float sl2 = P.sm_scale * 1.4426950408889634f;   // scale * log2(e)
        if (nblocks > 0) {
            // q dims [128c, 128c+128) of head h -> TMEM A operand columns
            const uint4 *qsrc = reinterpret_cast<const uint4 *>(q + ((int64_t)t * 128 + h) * 576 + 128 * c);
            uint32_t regs[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 x = __ldg(qsrc + half * 8 + i);
                    regs[4 * i + 0] = x.x;
                    regs[4 * i + 1] = x.y;
                    regs[4 * i + 2] = x.z;
                    regs[4 * i + 3] = x.w;
                }
                tmem_st32(t_lane + C::TMEM_QLO + 64 * c + 32 * half, regs);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(qlo_ready);
        }
        float m_run = -INFINITY, l_part = 0.f;
        bool ok = true;
        for (int j = 0; j < nblocks; ++j) {
            const bool fail = misc[2] != 0 || !mbar_wait(s_full, j & 1);
            if (named_bar_or(1, 256, fail)) { ok = false; misc[2] = 1; break; }   // all 8 warps leave together
            tc_fence_after();
            uint32_t s0[32], s1[32];
            tmem_ld32(t_lane + C::TMEM_S + 64 * c, s0);
            tmem_ld32(t_lane + C::TMEM_S + 64 * c + 32, s1);
            tmem_wait_ld();
            const int nb = min(C::BK, nvalid - j * C::BK);
            const int kbase_c = 64 * c;                  // first key of this thread's half
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (kbase_c + i < nb) mx = fmaxf(mx, __uint_as_float(s0[i]));
                if (kbase_c + 32 + i < nb) mx = fmaxf(mx, __uint_as_float(s1[i]));
            }
            // red is single-buffered: every thread passed this block's opening barrier
            // only after reading the previous block's values
            red[c * 128 + h] = mx;
            named_bar(1, 256);
            const float m_blk = fmaxf(red[h], red[128 + h]) * sl2;
            // Lazy rescale: a row moves its reference max only when the block max exceeds it
            // by more than TAU.  The TMEM load/store is warp-collective, so the whole warp
            // takes that path when any of its rows needs it (factor 1 for the others).
            const bool need = m_blk > m_run + C::TAU;
            const float f = (need && j > 0) ? exp2f(m_run - m_blk) : 1.0f;
            if (need) m_run = m_blk;
            if (j > 0 && __any_sync(0xffffffffu, need)) {   // previous PV is complete (s_full)
                l_part *= f;
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
            uint32_t pk[32];
            float ls = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int k0 = kbase_c + 2 * i;
                const float p0 = k0 < nb ? ex2_approx(fmaf(__uint_as_float(s0[2 * i]), sl2, -m_run)) : 0.f;
                const float p1 = k0 + 1 < nb ? ex2_approx(fmaf(__uint_as_float(s0[2 * i + 1]), sl2, -m_run)) : 0.f;
                ls += p0 + p1;
                pk[i] = pack_bf16x2(p0, p1);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int k0 = kbase_c + 32 + 2 * i;
                const float p0 = k0 < nb ? ex2_approx(fmaf(__uint_as_float(s1[2 * i]), sl2, -m_run)) : 0.f;
                const float p1 = k0 + 1 < nb ? ex2_approx(fmaf(__uint_as_float(s1[2 * i + 1]), sl2, -m_run)) : 0.f;
                ls += p0 + p1;
                pk[16 + i] = pack_bf16x2(p0, p1);
            }
            l_part += ls;
            tmem_st32(t_lane + C::TMEM_S + 32 * c, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // ---- epilogue
        const int64_t orow = ((int64_t)t * 128 + h) * 512 + 256 * v + 128 * c;
        if (nblocks == 0 || !ok) {
            uint4 z = make_uint4(0, 0, 0, 0);
            for (int i = 0; i < 16; ++i) reinterpret_cast<uint4 *>(out + orow)[i] = z;
            if (v == 0 && c == 0) lse[(int64_t)t * 128 + h] = nblocks == 0 ? -INFINITY : NAN;
        } else {
            bool okw = mbar_wait(pv_done, (nblocks - 1) & 1);
            tc_fence_after();
            // the last block's max was read before its p_full arrival, which the last PV
            // (hence pv_done) waited for: red may be reused
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
