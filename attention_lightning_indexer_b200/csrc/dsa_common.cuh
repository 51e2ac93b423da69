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
    const int32_t *block_table;   // nullptr: packed rows; else [batch, max_pages] pages of 64 keys
    int max_pages;
    int ue8m0;                    // FP8 indexer scales: 0 fp32 per token, 1 ue8m0 per 128-element block
    int debug;                    // check each row's sequence facts against the sizes (see row_ok)
};

// Value 2^(e - 127) of a ue8m0 scale byte, built exactly from its bits (e = 0 is the
// subnormal 2^-127, e = 255 is NaN).
__device__ __forceinline__ float ue8m0_to_float(uint32_t e) {
    if (e == 0u) return __uint_as_float(0x00400000u);
    if (e == 255u) return __uint_as_float(0x7fc00000u);
    return __uint_as_float(e << 23);
}

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

// row_info for a whole warp (all 32 lanes converged, the same t): a 32-way search over
// cu_q.  The sequence of t is the last b with cu_q[b] <= t (cu_q[0] = 0 <= t keeps lane 0's
// candidate true), found in ceil(log32(batch)) rounds of parallel loads instead of a binary
// search's log2(batch) dependent ones; the same answer as row_info.
__device__ __forceinline__ RowInfo row_info_warp(const Problem &P, int t) {
    if (P.cu_q == nullptr) return row_info(P, t);
    const int lane = threadIdx.x & 31;
    int lo = 0, hi = P.batch;                                // the answer lies in [lo, hi)
    while (hi - lo > 1) {
        const int stride = (hi - lo + 31) >> 5;
        const int b = lo + lane * stride;
        const bool le = b < hi && __ldg(P.cu_q + b) <= t;
        const unsigned m = __ballot_sync(0xffffffffu, le);
        const int j = m != 0u ? 31 - __clz(m) : 0;
        lo += j * stride;
        hi = min(hi, lo + stride);
    }
    const int q0 = __ldg(P.cu_q + lo), q1 = __ldg(P.cu_q + lo + 1);
    const int k0 = __ldg(P.cu_k + lo), k1 = __ldg(P.cu_k + lo + 1);
    RowInfo r;
    r.seq = lo;
    r.kbase = k0;
    r.len_k = k1 - k0;
    r.pos = (k1 - k0) - (q1 - q0) + (t - q0);
    return r;
}

// Row of the key arrays (k_idx, k_scale, kv) that holds key position s of the row's
// sequence: packed (kbase + s) or through the block table (pages of 64 keys).  A position
// past the sequence's last page maps to the sequence's first page (only loaded, never used).
__device__ __forceinline__ int key_row(const Problem &P, const RowInfo &r, int s) {
    if (P.block_table == nullptr) return r.kbase + s;
    const int pg = s >> 6;
    const int npg = (r.len_k + 63) >> 6;
    const int32_t *tab = P.block_table + (int64_t)r.seq * P.max_pages;
    return __ldg(tab + (pg < npg ? pg : 0)) * 64 + (s & 63);
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

constexpr unsigned ERR_BOUNDS = 4u;   // a debug-mode check found an inconsistent input

// Debug mode: the row's sequence must lie inside the key arrays (cu_q / cu_k consistent with
// total_k and max_len_k, block-table pages inside total_k).  A row that fails is counted
// in the error flag and treated by every kernel as having no keys, so no access leaves
// the arrays.  Always true outside debug mode.
__device__ __forceinline__ bool row_ok(const Problem &P, const RowInfo &r) {
    if (!P.debug) return true;
    bool ok = r.len_k >= 1 && r.pos >= 0 && r.pos < r.len_k && r.len_k <= P.max_len_k;
    if (P.block_table == nullptr) {
        ok = ok && r.kbase >= 0 && (int64_t)r.kbase + r.len_k <= P.total_k;
    } else if (ok) {
        const int32_t *tab = P.block_table + (int64_t)r.seq * P.max_pages;
        for (int pg = 0; pg < ((r.len_k + 63) >> 6) && ok; ++pg) {
            const int e = __ldg(tab + pg);
            ok = e >= 0 && ((int64_t)e + 1) * 64 <= P.total_k;
        }
    }
    if (!ok) raise_error(ERR_BOUNDS);
    return ok;
}

}  // namespace dsa
