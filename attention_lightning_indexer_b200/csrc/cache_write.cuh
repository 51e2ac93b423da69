// cache_write.cuh -- the rows the DSA path reads, written from the projections of new
// tokens: the indexer key k_I through k_norm and RoPE in the non-interleaved layout, the
// MLA latent through its RMSNorm and RoPE in the interleaved layout ("DeepSeek-V3.2-Exp"
// README, 2025-11-17 note: the indexer's RoPE input is non-interleaved, MLA's interleaved;
// "Model techniques map -- DeepSeek-V3.2": k_norm on the indexer key, kv_a_layernorm on
// the latent, RoPE on the 64 RoPE dims only).
//
//   k_I[row]      = RoPE_half(LayerNorm(k_raw) * ln_w + ln_b)   pairs (i, i + 32), i < 32
//   kv[row, :512] = k_raw_latent[:512] / rms * rms_w
//   kv[row, 512:] = RoPE_interleaved(latent[512:])             pairs (512 + 2i, 513 + 2i)
// with the angle pos * inv_freq[i] of pair i, evaluated in fp64 (positions reach 163,840)
// once per token and pair (lane i) and shared by both RoPEs through warp shuffles.
// One warp per token: 1.4 KB read and 1.4 KB written per token.
#pragma once

#include "dsa_common.cuh"

namespace dsa {
namespace cache {

constexpr int WARPS = 8;

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void rot_cs(int pos, float inv_freq, float &c, float &s) {
    double sd, cd;
    sincos((double)pos * (double)inv_freq, &sd, &cd);
    c = (float)cd;
    s = (float)sd;
}

__global__ void __launch_bounds__(32 * WARPS)
cache_write_kernel(int n, const __nv_bfloat16 *__restrict__ k_raw, const __nv_bfloat16 *__restrict__ kv_raw,
                   const int32_t *__restrict__ pos, const int32_t *__restrict__ rows,
                   const float *__restrict__ ln_w, const float *__restrict__ ln_b, const float *__restrict__ rms_w,
                   const float *__restrict__ inv_freq, float eps, __nv_bfloat16 *__restrict__ k_cache,
                   __nv_bfloat16 *__restrict__ kv_cache) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * WARPS + (threadIdx.x >> 5);
    if (t >= n) return;                                       // whole warp
    const int p = __ldg(pos + t);
    const int64_t row = __ldg(rows + t);
    // the 32 rotation angles of this position, pair i by lane i (both RoPEs use the same
    // frequencies); lanes read the ones they need by shuffles
    float c_lane, s_lane;
    rot_cs(p, __ldg(inv_freq + lane), c_lane, s_lane);

    // ---- indexer key: lane l holds dims 4l .. 4l+3
    float x[4];
    {
        const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(k_raw + (int64_t)t * 128) + lane);
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
        x[0] = __low2float(a); x[1] = __high2float(a); x[2] = __low2float(b); x[3] = __high2float(b);
    }
    const float mean = warp_sum_f((x[0] + x[1]) + (x[2] + x[3])) * (1.0f / 128.0f);
    float dv = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) dv += (x[j] - mean) * (x[j] - mean);
    const float inv = rsqrtf(warp_sum_f(dv) * (1.0f / 128.0f) + eps);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int d = 4 * lane + j;
        x[j] = (x[j] - mean) * inv * __ldg(ln_w + d) + __ldg(ln_b + d);
    }
    // RoPE, non-interleaved: dims i (lanes 0-7) pair with i + 32 (lanes 8-15)
    float partner[4], ck[4], sk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        partner[j] = __shfl_xor_sync(0xffffffffu, x[j], 8);
        ck[j] = __shfl_sync(0xffffffffu, c_lane, 4 * (lane & 7) + j);   // pair i = 4 (lane & 7) + j
        sk[j] = __shfl_sync(0xffffffffu, s_lane, 4 * (lane & 7) + j);
    }
    if (lane < 16) {
        const bool lower = lane < 8;
#pragma unroll
        for (int j = 0; j < 4; ++j) x[j] = lower ? x[j] * ck[j] - partner[j] * sk[j] : x[j] * ck[j] + partner[j] * sk[j];
    }
    {
        uint2 o;
        __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
        o.x = *reinterpret_cast<uint32_t *>(&a);
        o.y = *reinterpret_cast<uint32_t *>(&b);
        reinterpret_cast<uint2 *>(k_cache + row * 128)[lane] = o;
    }

    // ---- latent: 16-byte chunks; lane l holds chunks l and l + 32 of the 512 KV-LoRA dims,
    // lanes 0-7 also chunk 64 + l of the 64 RoPE dims
    const uint4 *src = reinterpret_cast<const uint4 *>(kv_raw + (int64_t)t * 576);
    float z[16];
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
        const uint4 v = __ldg(src + lane + 32 * c2);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w4[j]);
            z[8 * c2 + 2 * j] = __low2float(h);
            z[8 * c2 + 2 * j + 1] = __high2float(h);
        }
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) ss += z[j] * z[j];
    const float rinv = rsqrtf(warp_sum_f(ss) * (1.0f / 512.0f) + eps);
    uint4 *dst = reinterpret_cast<uint4 *>(kv_cache + row * 576);
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t o4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int d = 8 * (lane + 32 * c2) + 2 * j;
            __nv_bfloat162 h = __floats2bfloat162_rn(z[8 * c2 + 2 * j] * rinv * __ldg(rms_w + d),
                                                     z[8 * c2 + 2 * j + 1] * rinv * __ldg(rms_w + d + 1));
            o4[j] = *reinterpret_cast<uint32_t *>(&h);
        }
        dst[lane + 32 * c2] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
    float cl[4], sl[4];   // lanes 0-7: pairs i = 4 lane .. 4 lane + 3 of the latent's RoPE dims
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        cl[j] = __shfl_sync(0xffffffffu, c_lane, (4 * lane + j) & 31);
        sl[j] = __shfl_sync(0xffffffffu, s_lane, (4 * lane + j) & 31);
    }
    if (lane < 8) {   // RoPE, interleaved: pairs (512 + 2i, 513 + 2i), i = 4 lane .. 4 lane + 3
        const uint4 v = __ldg(src + 64 + lane);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        uint32_t o4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w4[j]);
            const float u = __low2float(h), w = __high2float(h);
            __nv_bfloat162 r = __floats2bfloat162_rn(u * cl[j] - w * sl[j], w * cl[j] + u * sl[j]);
            o4[j] = *reinterpret_cast<uint32_t *>(&r);
        }
        dst[64 + lane] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
}

}  // namespace cache
}  // namespace dsa
