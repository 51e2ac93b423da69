// indexer.cuh -- lightning indexer scores.
//
// "DeepSeek-V3.2 tech report summary", §1 DSA, ① Lightning Indexer:
//     I[t,s] = sum_{j<H_I} w[t,j] * ReLU(q_I[t,j] . k_I[s])   over preceding tokens s <= t,
// 64 heads of dim 128 ("DeepSeek-V3.2" miles docs §1); FP8-capable.
#pragma once

#include "dsa_common.cuh"

namespace dsa {
namespace indexer {

constexpr int HI = 64;     // indexer heads
constexpr int DI = 128;    // indexer head dim

template <bool FP8>
__device__ __forceinline__ float load_val(const void *base, int64_t i) {
    if (FP8) {
        __nv_fp8_e4m3 v;
        v.__x = reinterpret_cast<const __nv_fp8_storage_t *>(base)[i];
        return float(v);
    }
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[i]);
}

// CUDA-core reference-shaped kernel: one CTA per (64-key tile, query row).
// 256 threads: thread = (key kk = tid/4, head quarter hq = tid%4).
// Dynamic shared memory: CUDA_CORE_SMEM bytes.
constexpr int CUDA_CORE_SMEM = (2 * 64 * (DI + 1) + HI) * 4;
template <bool FP8>
__global__ void __launch_bounds__(256) indexer_cuda_core_kernel(Problem P, const void *__restrict__ q_idx,
                                                                const float *__restrict__ q_scale,
                                                                const void *__restrict__ k_idx,
                                                                const float *__restrict__ k_scale,
                                                                const float *__restrict__ w, float *__restrict__ scores,
                                                                int64_t ld, int row_begin) {
    extern __shared__ float smem_f[];
    float (*qs)[DI + 1] = reinterpret_cast<float (*)[DI + 1]>(smem_f);
    float (*ks)[DI + 1] = reinterpret_cast<float (*)[DI + 1]>(smem_f + HI * (DI + 1));
    float *ws = smem_f + 2 * 64 * (DI + 1);
    const int r = blockIdx.y;
    const int t = row_begin + r;
    const RowInfo ri = row_info(P, t);
    const int n = visible_keys(ri);
    const int s0 = blockIdx.x * 64;
    if (s0 >= n) return;
    const float qsc = FP8 ? __ldg(q_scale + t) : 1.0f;
    for (int i = threadIdx.x; i < HI * DI; i += 256)
        qs[i / DI][i % DI] = load_val<FP8>(q_idx, (int64_t)t * HI * DI + i) * qsc;
    if (threadIdx.x < HI) ws[threadIdx.x] = __ldg(w + (int64_t)t * HI + threadIdx.x);
    for (int i = threadIdx.x; i < 64 * DI; i += 256) {
        int kk = i / DI, d = i % DI;
        int s = s0 + kk;
        float v = 0.f;
        if (s < n) {
            int64_t row = (int64_t)ri.kbase + s;
            v = load_val<FP8>(k_idx, row * DI + d);
            if (FP8) v *= __ldg(k_scale + row);
        }
        ks[kk][d] = v;
    }
    __syncthreads();
    const int kk = threadIdx.x >> 2, hq = threadIdx.x & 3;
    float acc = 0.f;
    for (int h = hq * 16; h < hq * 16 + 16; ++h) {
        float dot = 0.f;
#pragma unroll 8
        for (int d = 0; d < DI; ++d) dot = fmaf(qs[h][d], ks[kk][d], dot);
        acc = fmaf(ws[h], fmaxf(dot, 0.f), acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (hq == 0 && s0 + kk < n) scores[(int64_t)r * ld + s0 + kk] = acc;
}

}  // namespace indexer
}  // namespace dsa
