// sparse_mla.cuh -- attention over the selected latent rows, MLA in MQA mode.
//
// "DeepSeek-V3.2 tech report summary", §1 DSA: full attention only over the k selected
// tokens; MLA-based implementation in MQA mode (each latent KV entry shared by all query
// heads).  Latent = 512 KV-LoRA + 64 RoPE dims, value = the first 512 dims, softmax
// scale 1/sqrt(192) (128 NoPE + 64 RoPE query/key head dims, "DeepSeek-V3.2" §1).
#pragma once

#include "dsa_common.cuh"

namespace dsa {
namespace mla {

constexpr int H = 128;
constexpr int DQK = 576;
constexpr int DV = 512;

// CUDA-core kernel: one CTA per (query row, group of 16 heads), 256 threads.
// Thread (head hl = tid/16, value slice vs = tid%16 of 32 dims) keeps its output slice
// in registers; keys are processed in blocks of 32 with an online softmax.
constexpr int CC_HG = 16, CC_KB = 32;
constexpr int CUDA_CORE_SMEM = CC_KB * DQK * 2 + CC_HG * DQK * 4 + CC_HG * (CC_KB + 1) * 4 + CC_KB * 4;
__global__ void __launch_bounds__(256) sparse_mla_cuda_core_kernel(Problem P, const __nv_bfloat16 *__restrict__ q,
                                                                   const __nv_bfloat16 *__restrict__ kv,
                                                                   const int32_t *__restrict__ idx,
                                                                   __nv_bfloat16 *__restrict__ out,
                                                                   float *__restrict__ lse) {
    constexpr int HG = CC_HG, KB = CC_KB;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __nv_bfloat16 (*kvs)[DQK] = reinterpret_cast<__nv_bfloat16 (*)[DQK]>(smem_raw);
    float (*qs)[DQK] = reinterpret_cast<float (*)[DQK]>(smem_raw + KB * DQK * 2);
    float (*S)[KB + 1] = reinterpret_cast<float (*)[KB + 1]>(smem_raw + KB * DQK * 2 + HG * DQK * 4);
    int *rows = reinterpret_cast<int *>(smem_raw + KB * DQK * 2 + HG * DQK * 4 + HG * (KB + 1) * 4);
    const int t = blockIdx.x;
    const int h0 = blockIdx.y * HG;
    const RowInfo ri = row_info(P, t);
    const int K = P.topk;
    for (int i = threadIdx.x; i < HG * DQK; i += 256)
        qs[i / DQK][i % DQK] = __bfloat162float(q[((int64_t)t * H + h0) * DQK + i]);
    const int hl = threadIdx.x >> 4, vs = threadIdx.x & 15;
    float o[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f;
    for (int b0 = 0; b0 < K; b0 += KB) {
        __syncthreads();
        if (threadIdx.x < KB) {
            int j = b0 + threadIdx.x;
            int s = j < K ? __ldg(idx + (int64_t)t * K + j) : -1;
            rows[threadIdx.x] = (s >= 0 && s <= ri.pos && s < ri.len_k) ? ri.kbase + s : -1;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < KB * (DQK / 8); i += 256) {
            int j = i / (DQK / 8), c = i % (DQK / 8);
            int row = rows[j];
            uint4 v = make_uint4(0, 0, 0, 0);
            if (row >= 0) v = __ldg(reinterpret_cast<const uint4 *>(kv + (int64_t)row * DQK) + c);
            reinterpret_cast<uint4 *>(&kvs[j][0])[c] = v;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < HG * KB; e += 256) {
            int h = e / KB, j = e % KB;
            float dot = 0.f;
            for (int d = 0; d < DQK; ++d) dot = fmaf(qs[h][d], __bfloat162float(kvs[j][d]), dot);
            S[h][j] = rows[j] >= 0 ? dot * P.sm_scale : -INFINITY;
        }
        __syncthreads();
        float mb = -INFINITY;
        for (int j = 0; j < KB; ++j) mb = fmaxf(mb, S[hl][j]);
        float mn = fmaxf(m, mb);
        if (mn == -INFINITY) continue;
        float corr = expf(m - mn);
        l *= corr;
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= corr;
        for (int j = 0; j < KB; ++j) {
            float s = S[hl][j];
            if (s == -INFINITY) continue;
            float p = expf(s - mn);
            l += p;
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = fmaf(p, __bfloat162float(kvs[j][vs * 32 + i]), o[i]);
        }
        m = mn;
    }
    const int h = h0 + hl;
    __nv_bfloat16 *op = out + ((int64_t)t * H + h) * DV + vs * 32;
    const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) op[i] = __float2bfloat16_rn(o[i] * inv);
    if (vs == 0) lse[(int64_t)t * H + h] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace mla
}  // namespace dsa
