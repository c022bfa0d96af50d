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

// Rotary position embedding of 8 consecutive channels (4 interleaved pairs) of one token, with
// cs the fp32 table row of its position at the pairs' head-local offset (cos and sin of each pair):
//   inverse = false: (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos)
//   inverse = true:  (x0, x1) -> (x0 cos + x1 sin, x1 cos - x0 sin)   (the transpose)
__device__ __forceinline__ void rope_pairs8(float (&x)[8], const float* __restrict__ cs, bool inverse) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(cs));
    const float4 b = __ldg(reinterpret_cast<const float4*>(cs) + 1);
    const float co[4] = {a.x, a.z, b.x, b.z};
    const float si[4] = {inverse ? -a.y : a.y, inverse ? -a.w : a.w, inverse ? -b.y : b.y, inverse ? -b.w : b.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float x0 = x[2 * q], x1 = x[2 * q + 1];
        x[2 * q] = fmaf(x0, co[q], -x1 * si[q]);
        x[2 * q + 1] = fmaf(x0, si[q], x1 * co[q]);
    }
}

// The same with the table slice already in registers: a = (cos, sin) of pairs 0, 1; b = of pairs 2, 3.
__device__ __forceinline__ void rope_pairs8v(float (&x)[8], const float4& a, const float4& b, bool inverse) {
    const float co[4] = {a.x, a.z, b.x, b.z};
    const float si[4] = {inverse ? -a.y : a.y, inverse ? -a.w : a.w, inverse ? -b.y : b.y, inverse ? -b.w : b.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float x0 = x[2 * q], x1 = x[2 * q + 1];
        x[2 * q] = fmaf(x0, co[q], -x1 * si[q]);
        x[2 * q + 1] = fmaf(x0, si[q], x1 * co[q]);
    }
}

// The same on 8 bf16 values packed in a uint4 (rotated in fp32, rounded once back to bf16).
// The same with the table slice already in registers (a = entries 0..3, b = entries 4..7).
__device__ __forceinline__ uint4 rope_bf16x8v(const uint4& v, const float4& a, const float4& b, bool inverse) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float x[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        x[2 * q] = __uint_as_float(w[q] << 16);
        x[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
    }
    rope_pairs8v(x, a, b, inverse);
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        __nv_bfloat162 t = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
        o[q] = *reinterpret_cast<uint32_t*>(&t);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ uint4 rope_bf16x8(const uint4& v, const float* __restrict__ cs, bool inverse) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float x[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        x[2 * q] = __uint_as_float(w[q] << 16);
        x[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
    }
    rope_pairs8(x, cs, inverse);
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        __nv_bfloat162 t = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
        o[q] = *reinterpret_cast<uint32_t*>(&t);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// out[n, c] = (R^T or R) x[n, c] for the rotated channels c < rope_n and x[n, c] for rope_n <= c <
// out_w (bf16, token-major; out has row stride out_w >= rope_n, a multiple of 8).  Warp `wid` of `nwarps` takes tokens wid, wid + nwarps, ...: its position (and table
// row) once per token, its lanes the token's 8-channel groups (two per round, loads first).  Positions
// are clamped below rope_max.
__device__ __forceinline__ void rope_rows_bf16(const __nv_bfloat16* __restrict__ x, int64_t x_stride,
                                               __nv_bfloat16* __restrict__ out, int out_w, int64_t N, int64_t wid,
                                               int64_t nwarps, int rope_n, int rope_hd, int rope_max,
                                               const float* __restrict__ cs, const int32_t* __restrict__ cu,
                                               int64_t n_docs, int64_t seqlen, bool inverse) {
    const int lane = threadIdx.x & 31;
    const int Gr = rope_n / 8, G = out_w / 8;
    for (int64_t n = wid; n < N; n += nwarps) {
        int64_t pos;
        if (cu == nullptr && N < (int64_t(1) << 31) && seqlen < (int64_t(1) << 31))
            pos = (int64_t)((uint32_t)n % (uint32_t)seqlen);
        else
            pos = n - seg_start(n, cu, n_docs, seqlen);
        pos = pos < rope_max ? pos : rope_max - 1;
        const __nv_bfloat16* xr = x + n * x_stride;
        __nv_bfloat16* orow = out + n * out_w;
        const float* crow = cs + pos * rope_hd;
        for (int g = lane; g < G; g += 64) {
            const bool two = g + 32 < G;
            const int c0 = 8 * g, c1 = 8 * (g + 32);
            const uint4 v0 = *reinterpret_cast<const uint4*>(xr + c0);
            float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), b0 = a0, a1 = a0, b1 = a0;
            if (g < Gr) {
                const float4* t0 = reinterpret_cast<const float4*>(crow + c0 % rope_hd);
                a0 = __ldg(t0);
                b0 = __ldg(t0 + 1);
            }
            uint4 v1 = make_uint4(0, 0, 0, 0);
            if (two) {
                v1 = *reinterpret_cast<const uint4*>(xr + c1);
                if (g + 32 < Gr) {
                    const float4* t1 = reinterpret_cast<const float4*>(crow + c1 % rope_hd);
                    a1 = __ldg(t1);
                    b1 = __ldg(t1 + 1);
                }
            }
            *reinterpret_cast<uint4*>(orow + c0) = g < Gr ? rope_bf16x8v(v0, a0, b0, inverse) : v0;
            if (two) *reinterpret_cast<uint4*>(orow + c1) = g + 32 < Gr ? rope_bf16x8v(v1, a1, b1, inverse) : v1;
        }
    }
}

}  // namespace dynconv
