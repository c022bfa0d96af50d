// common.cuh -- small device helpers shared by the dynamic short convolution kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace dynconv {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// First token of the sequence / packed document holding token n.
//  cu == nullptr: dense batch of sequences of length seqlen.
//  otherwise:     largest s with cu[s] <= n, by binary search over cu[0..n_docs].
// The result is clamped to [0, n] so that a malformed cu_seqlens can never send
// a tap outside the tensor (the pre-check kernel reports it instead).
__device__ __forceinline__ int64_t seg_start(int64_t n, const int32_t* __restrict__ cu, int64_t n_docs,
                                             int64_t seqlen) {
    int64_t s;
    if (cu == nullptr) {
        s = (n / seqlen) * seqlen;
    } else {
        int64_t lo = 0, hi = n_docs;
        while (hi - lo > 1) {
            const int64_t mid = (lo + hi) >> 1;
            if ((int64_t)__ldg(cu + mid) <= n) lo = mid; else hi = mid;
        }
        s = (int64_t)__ldg(cu + lo);
    }
    s = s < 0 ? 0 : s;
    return s > n ? n : s;
}

// seg_start for token indices below 2^31 (32-bit arithmetic: the tensor-core
// kernels require N < 2^31).
__device__ __forceinline__ int32_t seg_start32(int32_t n, const int32_t* __restrict__ cu, int32_t n_docs,
                                               int32_t seqlen) {
    int32_t s;
    if (cu == nullptr) {
        s = n - (int32_t)((uint32_t)n % (uint32_t)seqlen);
    } else {
        int32_t lo = 0, hi = n_docs;
        while (hi - lo > 1) {
            const int32_t mid = (lo + hi) >> 1;
            if (__ldg(cu + mid) <= n) lo = mid; else hi = mid;
        }
        s = __ldg(cu + lo);
    }
    s = s < 0 ? 0 : s;
    return s > n ? n : s;
}

// seg_bounds for token indices below 2^31 (32-bit arithmetic).
__device__ __forceinline__ void seg_bounds32(int32_t n, const int32_t* __restrict__ cu, int32_t n_docs,
                                             int32_t seqlen, int32_t N, int32_t& s, int32_t& e) {
    if (cu == nullptr) {
        s = n - (int32_t)((uint32_t)n % (uint32_t)seqlen);
        e = s + seqlen;
    } else {
        int32_t lo = 0, hi = n_docs;
        while (hi - lo > 1) {
            const int32_t mid = (lo + hi) >> 1;
            if (__ldg(cu + mid) <= n) lo = mid; else hi = mid;
        }
        s = __ldg(cu + lo);
        e = __ldg(cu + lo + 1);
    }
    s = s < 0 ? 0 : (s > n ? n : s);
    e = e <= n ? n + 1 : (e > N ? N : e);
}

// Start s (first token) and end e (one past the last token) of the sequence /
// packed document holding token n < N, clamped so that s <= n < e <= N whatever
// cu_seqlens holds.
__device__ __forceinline__ void seg_bounds(int64_t n, const int32_t* __restrict__ cu, int64_t n_docs,
                                           int64_t seqlen, int64_t N, int64_t& s, int64_t& e) {
    if (cu == nullptr) {
        s = (n / seqlen) * seqlen;
        e = s + seqlen;
    } else {
        int64_t lo = 0, hi = n_docs;
        while (hi - lo > 1) {
            const int64_t mid = (lo + hi) >> 1;
            if ((int64_t)__ldg(cu + mid) <= n) lo = mid; else hi = mid;
        }
        s = (int64_t)__ldg(cu + lo);
        e = (int64_t)__ldg(cu + lo + 1);
    }
    s = s < 0 ? 0 : (s > n ? n : s);
    e = e <= n ? n + 1 : (e > N ? N : e);
}

}  // namespace dynconv
