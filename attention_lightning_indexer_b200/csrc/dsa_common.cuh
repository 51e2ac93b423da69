// dsa_common.cuh -- device-side problem description and small helpers shared by the
// DSA kernels (indexer, top-k, sparse MLA).  Included once, by dsa_lib.cu.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsa {

// Plain-value copy of dsa_problem_t passed to kernels by value.
struct Problem {
    int batch;
    const int32_t *cu_q;   // nullptr when batch == 1
    const int32_t *cu_k;
    int total_q, total_k, max_len_q, max_len_k;
    int topk;
    float sm_scale;
};

// Sequence facts for one global query row t (the boundary's ragged reading: the
// queries of a sequence are its last len_q tokens).
struct RowInfo {
    int seq;
    int kbase;   // first key row of the sequence in k_idx / kv
    int len_k;
    int pos;     // position of the query inside its sequence; keys 0..pos are visible
};

__device__ __forceinline__ RowInfo row_info(const Problem &P, int t) {
    RowInfo r;
    if (P.cu_q == nullptr) {
        r.seq = 0;
        r.kbase = 0;
        r.len_k = P.total_k;
        r.pos = P.total_k - P.total_q + t;
        return r;
    }
    // upper_bound over cu_q[1..batch]: first b with cu_q[b+1] > t
    int lo = 0, hi = P.batch - 1;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (__ldg(P.cu_q + mid + 1) > t) hi = mid; else lo = mid + 1;
    }
    int q0 = __ldg(P.cu_q + lo), q1 = __ldg(P.cu_q + lo + 1);
    int k0 = __ldg(P.cu_k + lo), k1 = __ldg(P.cu_k + lo + 1);
    r.seq = lo;
    r.kbase = k0;
    r.len_k = k1 - k0;
    r.pos = (k1 - k0) - (q1 - q0) + (t - q0);
    return r;
}

// Number of visible keys of a row: keys 0..pos that exist in the sequence.
__device__ __forceinline__ int visible_keys(const RowInfo &r) {
    int n = r.pos + 1;
    if (n > r.len_k) n = r.len_k;
    return n < 0 ? 0 : n;
}

// Sticky error flag of this device (bounded waits that give up set it).
__device__ unsigned int g_error_flag;

__device__ __forceinline__ void raise_error(unsigned int code) { atomicOr(&g_error_flag, code); }

}  // namespace dsa
