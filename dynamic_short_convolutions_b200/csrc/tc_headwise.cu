// tc_headwise.cu -- the head-wise dynamic short convolution, bf16 storage, fp32 accumulation.
//
// Parameterization 2 of "Dynamic Short Convolutions Improve Transformers"
// (gist.science technical summary, "Dynamic Short Convolutions"): one K-tap filter
// per head, shared by the head's head_dim consecutive channels,
//   wh[n, q*K + j] = sum_i h[n, i] W[i, q*K + j]                      (tensor cores)
//   y[n, c]  = u[n, c] + sum_{j <= n - s(n)} wh[n, (c/hd)*K + j] u[n-j, c]
// and the adjoint
//   du[m, c] = g[m, c] + sum_{j < e(m) - m} wh[m+j, (c/hd)*K + j] g[m+j, c]
//   dwh[n, q*K + j] = sum_{c in head q} [j <= n - s(n)] g[n, c] u[n-j, c]   (warp shuffles)
//   dW = h^T dwh,  dh = dwh W^T                                        (tensor cores)
// The conv kernels are memory-bound CUDA-core kernels: token-major (16-byte loads and stores
// along C, packed fp32 FMAs, a reduce-scatter over each head's lanes for dwh) and channel-first
// (loads along the token rows of [batch * C, seqlen], a lane's filter taps held across the
// head's channels, dwh summed per warp and then over the block's warps in order).
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "prof.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace dynconv {

cudaError_t tc_gen_backward(const void* X, int R, const void* h, int64_t hs, const void* P, int64_t N, int64_t d,
                            void* dh, float* dP, float* dP_part, uint32_t* err, cudaStream_t st);
int gen_bwd_splits(int64_t N, int64_t d, int R);
int gen_bwd_dblk(int64_t d, int R);

namespace {

using namespace tc;

// A block covers kTokPerBlock tokens x 256 channels: 8 warps, each lane 8 channels (16-byte
// loads and stores along C) of two consecutive tokens per step; the rows beyond the pair were
// just read by the block's other warps and come from L1 / L2.
constexpr int kTokPerBlock = 64;

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16_lo(w[i]);
        f[2 * i + 1] = bf16_hi(w[i]);
    }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
}

// acc[0..8) += w * x (8 bf16 in a uint4) on the packed fp32 FMA.
__device__ __forceinline__ void axpy8(float (&acc)[8], float w, const uint4& x) {
    const uint32_t* v = reinterpret_cast<const uint32_t*>(&x);
#pragma unroll
    for (int p = 0; p < 4; ++p) ffma2(acc[2 * p], acc[2 * p + 1], w, w, bf16_lo(v[p]), bf16_hi(v[p]));
}

// sum_i a[i] b[i] over 8 values given as bf16 (two fp32 lanes, then their sum).
__device__ __forceinline__ float dot8(const uint4& a, const uint4& b) {
    const uint32_t* x = reinterpret_cast<const uint32_t*>(&a);
    const uint32_t* y = reinterpret_cast<const uint32_t*>(&b);
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int p = 0; p < 4; ++p) ffma2(s0, s1, bf16_lo(x[p]), bf16_hi(x[p]), bf16_lo(y[p]), bf16_hi(y[p]));
    return s0 + s1;
}

// The K taps of one head's filter for one token, as floats (8- or 4-byte loads when aligned,
// which holds for K = 4 and K = 2 since R = H K).
template <int K>
__device__ __forceinline__ void load_taps(const __nv_bfloat16* __restrict__ p, float (&w)[K]) {
    if constexpr (K == 4) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        w[0] = bf16_lo(v.x);
        w[1] = bf16_hi(v.x);
        w[2] = bf16_lo(v.y);
        w[3] = bf16_hi(v.y);
    } else if constexpr (K == 2) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
        w[0] = bf16_lo(v);
        w[1] = bf16_hi(v);
    } else {
#pragma unroll
        for (int j = 0; j < K; ++j) w[j] = __bfloat162float(p[j]);
    }
}

// A thread takes two consecutive tokens n, n + 1, which share K of their K + 1 rows of u.
template <int K>
__global__ void __launch_bounds__(256) hw_conv_fwd_kernel(const __nv_bfloat16* __restrict__ u, int64_t us,
                                                          const __nv_bfloat16* __restrict__ wh, int R, int hd,
                                                          int64_t N, int64_t C, int64_t seqlen,
                                                          const int32_t* __restrict__ cu, int64_t n_docs,
                                                          __nv_bfloat16* __restrict__ y,
                                                          const float* __restrict__ rope_cs, int rope_n, int rope_hd,
                                                          int rope_max) {
    pdl_trigger();
    pdl_wait();
    const int gl = threadIdx.x & 31, tl = threadIdx.x >> 5;
    const int64_t c = (int64_t)blockIdx.x * 256 + gl * 8;
    const int q = (int)(c / hd);
    const int64_t n0 = (int64_t)blockIdx.y * kTokPerBlock;
    const int64_t n1 = min(N, n0 + kTokPerBlock);
    for (int64_t n = n0 + 2 * tl; n < n1; n += 16) {
        const bool two = n + 1 < n1;                     // uniform over the warp
        // rows n - K + 1 .. n + 1 of u (zero outside [0, N)); the filters of n and n + 1
        uint4 ur[K + 1];
        float w[2][K];
#pragma unroll
        for (int i = 0; i <= K; ++i) {
            const int64_t m = n - K + 1 + i;
            ur[i] = (m >= 0 && m < N) ? *reinterpret_cast<const uint4*>(u + m * us + c) : make_uint4(0, 0, 0, 0);
        }
        load_taps<K>(wh + n * R + q * K, w[0]);
        if (two) load_taps<K>(wh + (n + 1) * R + q * K, w[1]);
        int32_t pos[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int32_t m = (int32_t)n + (two ? t : 0);
            pos[t] = m - seg_start32(m, cu, (int32_t)n_docs, (int32_t)seqlen);
        }
        // RoPE: the two tokens' table slices, loaded with the rows above
        const bool rot = rope_cs && c < rope_n;
        float4 rc[2][2];
        if (rot) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const float4* t4 = reinterpret_cast<const float4*>(
                    rope_cs + (int64_t)min(pos[t], rope_max - 1) * rope_hd + c % rope_hd);
                rc[t][0] = __ldg(t4);
                rc[t][1] = __ldg(t4 + 1);
            }
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            if (t == 1 && !two) break;
            const int32_t m = (int32_t)n + t;
            float acc[8];
            unpack8(ur[K - 1 + t], acc);
#pragma unroll
            for (int j = 0; j < K; ++j) axpy8(acc, j <= pos[t] ? w[t][j] : 0.f, ur[K - 1 + t - j]);
            if (rot) rope_pairs8v(acc, rc[t][0], rc[t][1], false);
            *reinterpret_cast<uint4*>(y + (int64_t)m * C + c) = pack8(acc);
        }
    }
}

// Sums p[0..K) over the L lanes (a power of two) that hold one head and stores dst[j] for
// j < K, masked to 0 for j > pos.  For K >= 3 and L >= 4 a reduce-scatter: two exchange
// steps leave each lane one tap, then a butterfly finishes it (log2(L) + 1 shuffles instead
// of K log2(L)); otherwise a plain butterfly over all K values.
template <int K>
__device__ __forceinline__ void head_sum_store(float (&p)[K], int L, int gl, int32_t pos,
                                               __nv_bfloat16* __restrict__ dst) {
    if constexpr (K >= 3) {
        if (L >= 4) {
            const float q3 = K > 3 ? p[K - 1] : 0.f;
            const int h1 = L >> 1, h2 = L >> 2;
            const bool b1 = (gl & h1) != 0, b2 = (gl & h2) != 0;
            const float s0 = b1 ? p[0] : p[2], s1 = b1 ? p[1] : q3;
            float k0 = b1 ? p[2] : p[0], k1 = b1 ? q3 : p[1];
            k0 += __shfl_xor_sync(0xffffffffu, s0, h1);
            k1 += __shfl_xor_sync(0xffffffffu, s1, h1);
            const float s = b2 ? k0 : k1;
            float k = b2 ? k1 : k0;
            k += __shfl_xor_sync(0xffffffffu, s, h2);
            for (int off = h2 >> 1; off > 0; off >>= 1) k += __shfl_xor_sync(0xffffffffu, k, off);
            const int tap = (b1 ? 2 : 0) + (b2 ? 1 : 0);
            if ((gl & (h2 - 1)) == 0 && tap < K) dst[tap] = __float2bfloat16_rn(tap <= pos ? k : 0.f);
            return;
        }
    }
#pragma unroll
    for (int j = 0; j < K; ++j)
        for (int off = L >> 1; off > 0; off >>= 1) p[j] += __shfl_xor_sync(0xffffffffu, p[j], off);
    const int l = gl & (L - 1);
#pragma unroll
    for (int j = 0; j < K; ++j)
        if (j % L == l) dst[j] = __float2bfloat16_rn(j <= pos ? p[j] : 0.f);
}

// L = head_dim / 8 lanes hold one head's channels (a power of two <= 32, aligned in the warp).
// A thread takes two consecutive tokens n, n + 1, which share K of their K + 1 rows of g, of u
// and of the filter: each row is loaded once for both.
template <int K>
__global__ void __launch_bounds__(256) hw_conv_bwd_kernel(const __nv_bfloat16* __restrict__ g,
                                                          const __nv_bfloat16* __restrict__ u, int64_t us,
                                                          const __nv_bfloat16* __restrict__ wh, int R, int hd,
                                                          int64_t N, int64_t C, int64_t seqlen,
                                                          const int32_t* __restrict__ cu, int64_t n_docs,
                                                          __nv_bfloat16* __restrict__ du,
                                                          __nv_bfloat16* __restrict__ dwh,
                                                          const __nv_bfloat16* __restrict__ gr, int rope_n) {
    pdl_trigger();
    pdl_wait();
    const int gl = threadIdx.x & 31, tl = threadIdx.x >> 5;
    const int64_t c = (int64_t)blockIdx.x * 256 + gl * 8;
    const int q = (int)(c / hd);
    const int L = hd >> 3;
    const int64_t n0 = (int64_t)blockIdx.y * kTokPerBlock;
    const int64_t n1 = min(N, n0 + kTokPerBlock);
    // RoPE: the rotated channels' rows of g come from R^T g (gr [N, rope_n]), written beforehand
    const bool rot = gr != nullptr && c < rope_n;
    const __nv_bfloat16* gsrc = rot ? gr : g;
    const int64_t gstride = rot ? rope_n : C;
    for (int64_t n = n0 + 2 * tl; n < n1; n += 16) {
        const bool two = n + 1 < n1;                     // uniform over the warp
        int32_t sb[2], eb[2];
        seg_bounds32((int32_t)n, cu, (int32_t)n_docs, (int32_t)seqlen, (int32_t)N, sb[0], eb[0]);
        if (two) seg_bounds32((int32_t)n + 1, cu, (int32_t)n_docs, (int32_t)seqlen, (int32_t)N, sb[1], eb[1]);
        else { sb[1] = sb[0]; eb[1] = eb[0]; }
        // rows n .. n + K of g and of the filter, rows n - K + 1 .. n + 1 of u (zero outside [0, N))
        uint4 gr[K + 1], ur[K + 1];
        float wr[K + 1][K];
#pragma unroll
        for (int i = 0; i <= K; ++i) {                   // every load of the pair first
            const int64_t mg = n + i, mu = n - K + 1 + i;
            gr[i] = mg < N ? *reinterpret_cast<const uint4*>(gsrc + mg * gstride + c) : make_uint4(0, 0, 0, 0);
            ur[i] = (mu >= 0 && mu < N) ? *reinterpret_cast<const uint4*>(u + mu * us + c) : make_uint4(0, 0, 0, 0);
            if (mg < N) load_taps<K>(wh + mg * R + q * K, wr[i]);
            else
#pragma unroll
                for (int j = 0; j < K; ++j) wr[i][j] = 0.f;
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            if (t == 1 && !two) break;
            const int32_t m = (int32_t)n + t;
            const int32_t pos = m - sb[t], epos = eb[t] - 1 - m;
            float acc[8];
            unpack8(gr[t], acc);
            float part[K];
#pragma unroll
            for (int j = 0; j < K; ++j) {
                axpy8(acc, j <= epos ? wr[t + j][j] : 0.f, gr[t + j]);   // filter of token m+j, tap j
                part[j] = dot8(gr[t], ur[K - 1 + t - j]);                 // g[m] . u[m-j] over 8 channels
            }
            *reinterpret_cast<uint4*>(du + (int64_t)m * C + c) = pack8(acc);
            head_sum_store<K>(part, L, gl, pos, dwh + (int64_t)m * R + q * K);
        }
    }
}

// ---- channel-first layout: u, y, g, du are [batch * C, seqlen] rows (tokens contiguous) ----
// A block is 8 warps on one sequence b, tokens t0 .. t0 + 32 V - 1 (V consecutive tokens per
// lane, one 8- or 16-byte load per row), and one head q; warp w takes channels w, w + 8, ... of
// the head, so a lane's filter taps stay in registers across the head's channels.  The K - 1
// tokens before a lane's first come from the previous lane by shuffle (lane 0 loads them), the
// K - 1 after its last from the next lane (lane 31 loads them).  seqlen is a multiple of 8, so a
// lane's V tokens are all inside the sequence or all past its end.

// V bf16 values of one row, as V / 2 packed pairs.
template <int V>
__device__ __forceinline__ void ldrow(const __nv_bfloat16* __restrict__ p, uint32_t (&w)[V / 2]) {
    if constexpr (V == 8) {
        const uint4 t = *reinterpret_cast<const uint4*>(p);
        w[0] = t.x; w[1] = t.y; w[2] = t.z; w[3] = t.w;
    } else {
        const uint2 t = *reinterpret_cast<const uint2*>(p);
        w[0] = t.x; w[1] = t.y;
    }
}
template <int V>
__device__ __forceinline__ void strow(__nv_bfloat16* __restrict__ p, const float (&f)[V]) {
    if constexpr (V == 8) {
        *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                                                  pack_bf16(f[6], f[7]));
    } else {
        *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]));
    }
}
// Element i (0 <= i < 2 P) of P packed bf16 pairs.
template <int P>
__device__ __forceinline__ float elem(const uint32_t (&w)[P], int i) {
    return (i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]);
}

// Row values of tokens t - 4 .. t + V - 1 (prev = the 4 before the lane's first) and, for the
// backward, t + V .. t + V + 3 (next), for a lane whose V tokens start at t.
template <int V>
__device__ __forceinline__ void row_halo_prev(const __nv_bfloat16* __restrict__ row, const uint32_t (&cur)[V / 2],
                                              int lane, int64_t t, bool live, uint32_t (&prev)[2]) {
    prev[0] = __shfl_up_sync(0xffffffffu, cur[V / 2 - 2], 1);
    prev[1] = __shfl_up_sync(0xffffffffu, cur[V / 2 - 1], 1);
    if (lane == 0) {
        if (live && t >= 4) {
            const uint2 v = *reinterpret_cast<const uint2*>(row + t - 4);
            prev[0] = v.x;
            prev[1] = v.y;
        } else {
            prev[0] = prev[1] = 0u;
        }
    }
}
template <int V>
__device__ __forceinline__ void row_halo_next(const __nv_bfloat16* __restrict__ row, const uint32_t (&cur)[V / 2],
                                              int lane, int64_t t, int64_t T, uint32_t (&next)[2]) {
    next[0] = __shfl_down_sync(0xffffffffu, cur[0], 1);
    next[1] = __shfl_down_sync(0xffffffffu, cur[1], 1);
    if (lane == 31) {
        if (t + V < T) {
            const uint2 v = *reinterpret_cast<const uint2*>(row + t + V);
            next[0] = v.x;
            next[1] = v.y;
        } else {
            next[0] = next[1] = 0u;
        }
    }
}

// y[c, t] = u[c, t] + sum_{j <= t - s(t)} wh[t, q K + j] u[c, t - j]  (the same FMA order as the
// token-major kernel, so both layouts give the same bits).
template <int K, int V>
__global__ void __launch_bounds__(256) hw_conv_fwd_cf_kernel(const __nv_bfloat16* __restrict__ u, int64_t us,
                                                             const __nv_bfloat16* __restrict__ wh, int R, int hd,
                                                             int64_t N, int64_t C, int64_t T, int64_t tps,
                                                             const int32_t* __restrict__ cu, int64_t n_docs,
                                                             __nv_bfloat16* __restrict__ y) {
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.x / tps;
    const int64_t t = (blockIdx.x - b * tps) * (32 * V) + lane * V;
    const int q = blockIdx.y;
    const bool live = t < T;
    const int64_t n0 = b * T + t;
    float w[V][K];
    int32_t pos[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
        if (live) {
            load_taps<K>(wh + (n0 + i) * R + q * K, w[i]);
            pos[i] = (int32_t)(n0 + i - seg_start(n0 + i, cu, n_docs, T));
        } else {
#pragma unroll
            for (int j = 0; j < K; ++j) w[i][j] = 0.f;
            pos[i] = 0;
        }
    }
    for (int c = q * hd + warp; c < (q + 1) * hd; c += 8) {
        const __nv_bfloat16* urow = u + (b * C + c) * us;
        uint32_t cur[V / 2], prev[2];
        if (live) ldrow<V>(urow + t, cur);
        else
#pragma unroll
            for (int k = 0; k < V / 2; ++k) cur[k] = 0u;
        row_halo_prev<V>(urow, cur, lane, t, live, prev);
        float acc[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            acc[i] = elem(cur, i);
#pragma unroll
            for (int j = 0; j < K; ++j) {
                const float x = i - j >= 0 ? elem(cur, i - j) : elem(prev, 4 + i - j);
                acc[i] = fmaf(j <= pos[i] ? w[i][j] : 0.f, x, acc[i]);
            }
        }
        if (live) strow<V>(y + (b * C + c) * T + t, acc);
    }
}

// du[c, t] = g[c, t] + sum_{j < e(t) - t} wh[t + j, q K + j] g[c, t + j]; dwh[t, q K + j] =
// sum_{c in q} [j <= t - s(t)] g[c, t] u[c, t - j]: each warp sums its channels in order, then
// the block sums the 8 warps' partials in order (no atomics).
template <int K, int V>
__global__ void __launch_bounds__(256) hw_conv_bwd_cf_kernel(const __nv_bfloat16* __restrict__ g,
                                                             const __nv_bfloat16* __restrict__ u, int64_t us,
                                                             const __nv_bfloat16* __restrict__ wh, int R, int hd,
                                                             int64_t N, int64_t C, int64_t T, int64_t tps,
                                                             const int32_t* __restrict__ cu, int64_t n_docs,
                                                             __nv_bfloat16* __restrict__ du,
                                                             __nv_bfloat16* __restrict__ dwh) {
    __shared__ float red[8][32 * V][K];
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t b = blockIdx.x / tps;
    const int64_t tb = (blockIdx.x - b * tps) * (32 * V);
    const int64_t t = tb + lane * V;
    const int q = blockIdx.y;
    const bool live = t < T;
    const int64_t n0 = b * T + t;
    // wf[i][j]: tap j of the filter of token t + i (i < V + K - 1), zero past the sequence end
    float wf[V + K - 1][K];
    int32_t pos[V], epos[V];
#pragma unroll
    for (int i = 0; i < V + K - 1; ++i) {
        if (live && t + i < T) load_taps<K>(wh + (n0 + i) * R + q * K, wf[i]);
        else
#pragma unroll
            for (int j = 0; j < K; ++j) wf[i][j] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < V; ++i) {
        if (live) {
            int64_t sb, eb;
            seg_bounds(n0 + i, cu, n_docs, T, N, sb, eb);
            pos[i] = (int32_t)(n0 + i - sb);
            epos[i] = (int32_t)(eb - 1 - (n0 + i));
        } else {
            pos[i] = epos[i] = -1;
        }
    }
    float dacc[V][K];
#pragma unroll
    for (int i = 0; i < V; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j) dacc[i][j] = 0.f;
    for (int c = q * hd + warp; c < (q + 1) * hd; c += 8) {
        const __nv_bfloat16* grow = g + (b * C + c) * T;
        const __nv_bfloat16* urow = u + (b * C + c) * us;
        uint32_t gc[V / 2], uc[V / 2], gn[2], up[2];
        if (live) {
            ldrow<V>(grow + t, gc);
            ldrow<V>(urow + t, uc);
        } else {
#pragma unroll
            for (int k = 0; k < V / 2; ++k) gc[k] = uc[k] = 0u;
        }
        row_halo_next<V>(grow, gc, lane, t, T, gn);
        row_halo_prev<V>(urow, uc, lane, t, live, up);
        float acc[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const float gi = elem(gc, i);
            acc[i] = gi;
#pragma unroll
            for (int j = 0; j < K; ++j) {
                const float gx = i + j < V ? elem(gc, i + j) : elem(gn, i + j - V);
                acc[i] = fmaf(j <= epos[i] ? wf[i + j][j] : 0.f, gx, acc[i]);
                const float ux = i - j >= 0 ? elem(uc, i - j) : elem(up, 4 + i - j);
                dacc[i][j] = fmaf(gi, ux, dacc[i][j]);
            }
        }
        if (live) strow<V>(du + (b * C + c) * T + t, acc);
    }
#pragma unroll
    for (int i = 0; i < V; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j) red[warp][lane * V + i][j] = dacc[i][j];
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * V * K; e += 256) {
        const int k = e / K, j = e - k * K;
        const int64_t tt = tb + k;
        if (tt >= T) continue;
        float sum = 0.f;
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) sum += red[w8][k][j];
        const int64_t n = b * T + tt;
        const int32_t ps = (int32_t)(n - seg_start(n, cu, n_docs, T));
        dwh[n * R + q * K + j] = __float2bfloat16_rn(j <= ps ? sum : 0.f);
    }
}

// gr[n, c] = (R^T g)[n, c] for the rotated channels c < rope_n (bf16, token-major), blocks striding over tokens.
__global__ void __launch_bounds__(128) rope_rows_kernel(const __nv_bfloat16* __restrict__ g, int64_t C,
                                                        __nv_bfloat16* __restrict__ gr, int64_t N, int rope_n,
                                                        int rope_hd, int rope_max, const float* __restrict__ cs,
                                                        const int32_t* __restrict__ cu, int64_t n_docs,
                                                        int64_t seqlen) {
    pdl_trigger();
    pdl_wait();
    rope_rows_bf16(g, C, gr, N, (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5),
                   (int64_t)gridDim.x * (blockDim.x / 32), rope_n, rope_hd, rope_max, cs, cu, n_docs, seqlen, true);
}

inline size_t al256(size_t x) { return (x + 255) / 256 * 256; }

// Rows of the RoPE table as an int (at least 1; positions are clamped below it).
inline int rope_rows(const Prob& p) { return (int)std::max<int64_t>(1, std::min<int64_t>(p.rope_max, INT32_MAX)); }

}  // namespace


TcHwLayout tc_hw_layout(const Prob& p) {
    TcHwLayout L{};
    size_t off = 0;
    L.wh = off;     off = al256(off + (size_t)p.N * p.R * 2);
    L.dwh = off;    off = al256(off + (size_t)p.N * p.R * 2);
    L.dpart = off;  off = al256(off + (size_t)gen_bwd_splits(p.N, p.d, (int)p.R) * p.d * p.R * 4);
    L.gr = off;     off = al256(off + (size_t)p.N * p.rope_n * 2);                  // RoPE: R^T g, rotated channels
    L.total = off;
    return L;
}

bool tc_headwise_supported(const Prob& p) {
    if (p.dtype != 1 || p.kind != 1) return false;
    if (p.R > 128 || p.R % 8 != 0 || p.d % 8 != 0) return false;
    if (p.K < 1 || p.K > 4) return false;
    if (p.layout == 1) return cf_tiles_ok(p) && p.H < 65536;
    if (p.hd < 8 || p.hd > 256 || (p.hd & (p.hd - 1)) != 0) return false;
    // one grid row per kTokPerBlock tokens (grid y up to 65535), 32-bit token indices
    return p.C % 256 == 0 && p.N < int64_t(kTokPerBlock) * 65535;
}

// Channel-first: 8 tokens per lane in the forward, 4 in the backward (fewer registers for
// the look-ahead filters and the dwh partials).
constexpr int kCfFwdV = 8, kCfBwdV = 4;

template <int K>
static cudaError_t launch_hw_fwd(const Prob& p, const void* u, const void* wh, void* y, cudaStream_t st) {
    cudaError_t e;
    if (p.layout == 1) {
        const int64_t tps = (p.seqlen + 32 * kCfFwdV - 1) / (32 * kCfFwdV);
        const dim3 grid((unsigned)(p.batch * tps), (unsigned)p.H);
        DC_LAUNCH(kTcHeadwiseFwd, st, e = launch_pdl(hw_conv_fwd_cf_kernel<K, kCfFwdV>, grid, dim3(256), 0, st,
            static_cast<const __nv_bfloat16*>(u), p.us, static_cast<const __nv_bfloat16*>(wh), (int)p.R, (int)p.hd,
            p.N, p.C, p.seqlen, tps, p.cu, p.n_docs, static_cast<__nv_bfloat16*>(y)));
        return e;
    }
    const dim3 grid((unsigned)(p.C / 256), (unsigned)((p.N + kTokPerBlock - 1) / kTokPerBlock));
    DC_LAUNCH(kTcHeadwiseFwd, st, e = launch_pdl(hw_conv_fwd_kernel<K>, grid, dim3(256), 0, st,
        static_cast<const __nv_bfloat16*>(u), p.us, static_cast<const __nv_bfloat16*>(wh), (int)p.R, (int)p.hd,
        p.N, p.C, p.seqlen, p.cu, p.n_docs, static_cast<__nv_bfloat16*>(y), p.rope_n > 0 ? p.rope_cs : nullptr,
        (int)p.rope_n, p.rope_n > 0 ? (int)p.rope_hd : 1, rope_rows(p)));
    return e;
}

template <int K>
static cudaError_t launch_hw_bwd(const Prob& p, const void* g, const void* u, const void* wh, void* du, void* dwh,
                                 const void* gr, cudaStream_t st) {
    cudaError_t e;
    if (p.layout == 1) {
        const int64_t tps = (p.seqlen + 32 * kCfBwdV - 1) / (32 * kCfBwdV);
        const dim3 grid((unsigned)(p.batch * tps), (unsigned)p.H);
        DC_LAUNCH(kTcHeadwiseBwd, st, e = launch_pdl(hw_conv_bwd_cf_kernel<K, kCfBwdV>, grid, dim3(256), 0, st,
            static_cast<const __nv_bfloat16*>(g), static_cast<const __nv_bfloat16*>(u), p.us,
            static_cast<const __nv_bfloat16*>(wh), (int)p.R, (int)p.hd, p.N, p.C, p.seqlen, tps, p.cu, p.n_docs,
            static_cast<__nv_bfloat16*>(du), static_cast<__nv_bfloat16*>(dwh)));
        return e;
    }
    const dim3 grid((unsigned)(p.C / 256), (unsigned)((p.N + kTokPerBlock - 1) / kTokPerBlock));
    DC_LAUNCH(kTcHeadwiseBwd, st, e = launch_pdl(hw_conv_bwd_kernel<K>, grid, dim3(256), 0, st,
        static_cast<const __nv_bfloat16*>(g), static_cast<const __nv_bfloat16*>(u), p.us,
        static_cast<const __nv_bfloat16*>(wh), (int)p.R, (int)p.hd, p.N, p.C, p.seqlen, p.cu, p.n_docs,
        static_cast<__nv_bfloat16*>(du), static_cast<__nv_bfloat16*>(dwh), static_cast<const __nv_bfloat16*>(gr),
        (int)p.rope_n));
    return e;
}

cudaError_t tc_headwise_forward(const Prob& p, const void* u, const void* h, const void* W, void* y, void* z_save,
                                char* tcws, uint32_t* err, cudaStream_t st) {
    const TcHwLayout L = tc_hw_layout(p);
    void* wh = z_save ? z_save : static_cast<void*>(tcws + L.wh);
    cudaError_t e = tc_gen_launch(h, p.hs, W, p.N, p.d, (int)p.R, wh, p.R, err, st);
    if (e != cudaSuccess) return e;
    switch (p.K) {
        case 1: return launch_hw_fwd<1>(p, u, wh, y, st);
        case 2: return launch_hw_fwd<2>(p, u, wh, y, st);
        case 3: return launch_hw_fwd<3>(p, u, wh, y, st);
        default: return launch_hw_fwd<4>(p, u, wh, y, st);
    }
}

cudaError_t tc_headwise_backward(const Prob& p, const void* g, const void* u, const void* h, const void* W,
                                 const void* z_saved, void* du, void* dh, float* dW, char* tcws, uint32_t* err,
                                 cudaStream_t st) {
    const TcHwLayout L = tc_hw_layout(p);
    const void* wh = z_saved;
    if (!wh) {
        void* whs = tcws + L.wh;
        cudaError_t e = tc_gen_launch(h, p.hs, W, p.N, p.d, (int)p.R, whs, p.R, err, st);
        if (e != cudaSuccess) return e;
        wh = whs;
    }
    void* dwh = tcws + L.dwh;
    cudaError_t e;
    void* gr = nullptr;
    if (p.rope_n > 0) {                    // R^T g of the rotated channels, read by the conv backward
        gr = tcws + L.gr;
        DC_LAUNCH(kTcPrep, st, e = launch_pdl(rope_rows_kernel, dim3((unsigned)std::min<int64_t>(p.N, 148 * 8)),
                                              dim3(128), 0, st, static_cast<const __nv_bfloat16*>(g), p.C,
                                              static_cast<__nv_bfloat16*>(gr), p.N, (int)p.rope_n, (int)p.rope_hd,
                                              rope_rows(p), p.rope_cs, p.cu, p.n_docs, p.seqlen));
        if (e != cudaSuccess) return e;
    }
    switch (p.K) {
        case 1: e = launch_hw_bwd<1>(p, g, u, wh, du, dwh, gr, st); break;
        case 2: e = launch_hw_bwd<2>(p, g, u, wh, du, dwh, gr, st); break;
        case 3: e = launch_hw_bwd<3>(p, g, u, wh, du, dwh, gr, st); break;
        default: e = launch_hw_bwd<4>(p, g, u, wh, du, dwh, gr, st); break;
    }
    if (e != cudaSuccess) return e;
    return tc_gen_backward(dwh, (int)p.R, h, p.hs, W, p.N, p.d, dh, dW, reinterpret_cast<float*>(tcws + L.dpart),
                           err, st);
}

}  // namespace dynconv
