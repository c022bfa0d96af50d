// simt.cu -- generic CUDA-core kernels for dynamic short convolutions.
//
// These cover every shape the C ABI accepts, in fp32 or bf16 storage with fp32
// accumulation.  They are the fp32 path (fp32 inputs must not be rounded to a
// tensor-core operand type) and the path for bf16 shapes outside the
// tensor-core kernels' coverage.  One thread block per token for the per-token
// steps; one thread per output entry for the token reductions, each summed in
// token order (deterministic).  u, y, g and du are addressed through their
// strides, so the same kernels serve the token-major [N, C] and the
// channel-first [batch, C, seqlen] layouts, any seqlen and channel stride.
//
// Operation ("Dynamic Short Convolutions Improve Transformers", gist.science
// technical summary, "Dynamic Short Convolutions": Mechanism, Parameterization,
// Placement):
//   y[n,c] = u[n,c] + sum_{j<K, n-j >= s(n)} w[n,c,j] u[n-j,c]
//   w[n,c,j] = sum_k z[n,k] B[k,c*K+j], z = h A        (low-rank)
//   w[n,c,j] = (h W)[n, (c/head_dim)*K + j]            (head-wise)
// and its adjoint (du, then dz or dwh, dA/dB or dW, dh).
#include "common.cuh"
#include "internal.h"
#include "prof.h"

namespace dynconv {
namespace {

constexpr int kThreads = 256;

// Element (token n, channel c) of a conv-side tensor (u, y, g, du) in either layout:
//   token-major   n * ts + c
//   channel-first (n / T) * bs + (n % T) + c * cs    (T = seqlen; sequences bs apart, channels cs apart)
struct Ax {
    int64_t T, bs, ts, cs;
    int cf;
    __device__ __forceinline__ int64_t operator()(int64_t n, int64_t c) const {
        return cf ? (n / T) * bs + (n % T) + c * cs : n * ts + c;
    }
};

// u (strided) and the dense conv-side tensors of a problem.
inline Ax ax_u(const Prob& p) {
    const int64_t T = p.seqlen > 0 ? p.seqlen : 1;
    return p.layout ? Ax{T, p.C * p.us, 1, p.us, 1} : Ax{T, 0, p.us, 1, 0};
}
inline Ax ax_dense(const Prob& p) {
    const int64_t T = p.seqlen > 0 ? p.seqlen : 1;
    return p.layout ? Ax{T, p.C * T, 1, T, 1} : Ax{T, 0, p.C, 1, 0};
}

// X[n, k] = sum_i h[n, i] P[i, k]   (z = h A or head-wise filters h W), fp32 out;
// optionally also stored to zsave in the storage type.
template <typename T>
__global__ void __launch_bounds__(kThreads) gen_kernel(const T* __restrict__ h, int64_t hs,
                                                        const T* __restrict__ P, int64_t d, int64_t R,
                                                        float* __restrict__ X, T* __restrict__ zsave) {
    const int64_t n = blockIdx.x;
    for (int64_t k = threadIdx.x; k < R; k += blockDim.x) {
        float acc = 0.f;
        for (int64_t i = 0; i < d; ++i) acc = fmaf(to_f32(h[n * hs + i]), to_f32(P[i * R + k]), acc);
        X[n * R + k] = acc;
        if (zsave) zsave[n * R + k] = from_f32<T>(acc);
    }
}

// z_saved (storage type) -> fp32 generator buffer.
template <typename T>
__global__ void widen_kernel(const T* __restrict__ src, float* __restrict__ dst, int64_t count) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = to_f32(src[i]);
}

// Filter tap j of channel c at a token whose generator row (z or head-wise filters) is xs.
template <typename T, int KIND>
__device__ __forceinline__ float filter_tap(const float* xs, const T* __restrict__ B, int64_t R, int64_t C,
                                            int64_t K, int64_t hd, int64_t c, int64_t j) {
    if (KIND == 0) {
        float w = 0.f;
        for (int64_t k = 0; k < R; ++k) w = fmaf(xs[k], to_f32(B[k * C * K + c * K + j]), w);
        return w;
    } else {
        return xs[(c / hd) * K + j];
    }
}

template <typename T, int KIND>
__global__ void __launch_bounds__(kThreads) conv_fwd_kernel(
    const T* __restrict__ u, Ax au, const float* __restrict__ X, int64_t R, const T* __restrict__ B,
    int64_t C, int64_t K, int64_t hd, const int32_t* __restrict__ cu, int64_t n_docs, int64_t seqlen,
    T* __restrict__ y, Ax ay) {
    extern __shared__ float xs[];
    const int64_t n = blockIdx.x;
    for (int64_t k = threadIdx.x; k < R; k += blockDim.x) xs[k] = X[n * R + k];
    __syncthreads();
    const int64_t s = seg_start(n, cu, n_docs, seqlen);
    for (int64_t c = threadIdx.x; c < C; c += blockDim.x) {
        float acc = to_f32(u[au(n, c)]);
        for (int64_t j = 0; j < K; ++j)
            if (n - j >= s) acc = fmaf(filter_tap<T, KIND>(xs, B, R, C, K, hd, c, j), to_f32(u[au(n - j, c)]), acc);
        y[ay(n, c)] = from_f32<T>(acc);
    }
}

// Per token m: du[m,c] = g[m,c] + sum_j w[m+j,c,j] g[m+j,c] over taps whose source
// token m lies in the segment of m+j; and the generator-space gradient of token m:
// dz[m,k] = sum_{c,j} dw[m,c,j] B[k,c*K+j] (low-rank) or dwh[m,q,j] = sum_{c in q} dw[m,c,j],
// with dw[m,c,j] = g[m,c] u[m-j,c] for m-j >= s(m).
template <typename T, int KIND>
__global__ void __launch_bounds__(kThreads) conv_bwd_kernel(
    const T* __restrict__ g, const T* __restrict__ u, Ax au, Ax ad, const float* __restrict__ X, int64_t R,
    const T* __restrict__ B, int64_t N, int64_t C, int64_t K, int64_t hd, const int32_t* __restrict__ cu,
    int64_t n_docs, int64_t seqlen, T* __restrict__ du, float* __restrict__ dgen) {
    extern __shared__ float sm[];
    float* xs = sm;                       // [K][R] generator rows of tokens m .. m+K-1
    float* red = sm + K * R;              // [kThreads/32] warp partials
    __shared__ int valid[4];
    const int64_t m = blockIdx.x;
    const int64_t sm_ = seg_start(m, cu, n_docs, seqlen);
    for (int64_t e = threadIdx.x; e < K * R; e += blockDim.x) {
        const int64_t j = e / R, n = m + j;
        xs[e] = n < N ? X[n * R + (e % R)] : 0.f;
    }
    if (threadIdx.x < K) {
        const int64_t n = m + threadIdx.x;
        valid[threadIdx.x] = (n < N) && (m >= seg_start(n, cu, n_docs, seqlen));
    }
    __syncthreads();
    for (int64_t c = threadIdx.x; c < C; c += blockDim.x) {
        float acc = to_f32(g[ad(m, c)]);
        for (int64_t j = 0; j < K; ++j)
            if (valid[j]) acc = fmaf(filter_tap<T, KIND>(xs + j * R, B, R, C, K, hd, c, j), to_f32(g[ad(m + j, c)]), acc);
        du[ad(m, c)] = from_f32<T>(acc);
    }
    if (KIND == 0) {
        // dz[m, k] for every k: block reduction over channels in a fixed order.
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        for (int64_t k = 0; k < R; ++k) {
            float part = 0.f;
            for (int64_t c = threadIdx.x; c < C; c += blockDim.x) {
                const float gm = to_f32(g[ad(m, c)]);
                for (int64_t j = 0; j < K; ++j)
                    if (m - j >= sm_) part = fmaf(gm * to_f32(u[au(m - j, c)]), to_f32(B[k * C * K + c * K + j]), part);
            }
            for (int off = 16; off > 0; off >>= 1) part += __shfl_down_sync(0xffffffffu, part, off);
            if (lane == 0) red[warp] = part;
            __syncthreads();
            if (threadIdx.x == 0) {
                float t = 0.f;
                for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
                dgen[m * R + k] = t;
            }
            __syncthreads();
        }
    } else {
        // dwh[m, q, j]: one thread per (q, j), summing the head's channels in order.
        for (int64_t e = threadIdx.x; e < R; e += blockDim.x) {
            const int64_t q = e / K, j = e % K;
            float t = 0.f;
            if (m - j >= sm_)
                for (int64_t c = q * hd; c < (q + 1) * hd; ++c) t = fmaf(to_f32(g[ad(m, c)]), to_f32(u[au(m - j, c)]), t);
            dgen[m * R + e] = t;
        }
    }
}

// dB[k, c*K+j] = sum_n z[n,k] g[n,c] u[n-j,c]  (n-j >= s(n)), one thread per entry.
template <typename T>
__global__ void __launch_bounds__(kThreads) dB_kernel(
    const float* __restrict__ Z, int64_t r, const T* __restrict__ g, const T* __restrict__ u, Ax au, Ax ad,
    int64_t N, int64_t C, int64_t K, const int32_t* __restrict__ cu, int64_t n_docs, int64_t seqlen,
    float* __restrict__ dB) {
    const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (e >= r * C * K) return;
    const int64_t k = e / (C * K), col = e % (C * K), c = col / K, j = col % K;
    float acc = 0.f;
    for (int64_t n = j; n < N; ++n)
        if (n - j >= seg_start(n, cu, n_docs, seqlen))
            acc = fmaf(Z[n * r + k], to_f32(g[ad(n, c)]) * to_f32(u[au(n - j, c)]), acc);
    dB[e] = acc;
}

// dP[i, k] = sum_n h[n, i] X[n, k]  (dA = h^T dz, dW = h^T dwh), one thread per entry.
template <typename T>
__global__ void __launch_bounds__(kThreads) hTX_kernel(const T* __restrict__ h, int64_t hs,
                                                        const float* __restrict__ X, int64_t N, int64_t d,
                                                        int64_t R, float* __restrict__ dP) {
    const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (e >= d * R) return;
    const int64_t i = e / R, k = e % R;
    float acc = 0.f;
    for (int64_t n = 0; n < N; ++n) acc = fmaf(to_f32(h[n * hs + i]), X[n * R + k], acc);
    dP[e] = acc;
}

// dh[n, i] = sum_k X[n, k] P[i, k]  (dz A^T or dwh W^T), one thread per entry.
template <typename T>
__global__ void __launch_bounds__(kThreads) dh_kernel(const float* __restrict__ X, const T* __restrict__ P,
                                                       int64_t N, int64_t d, int64_t R, T* __restrict__ dh) {
    const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (e >= N * d) return;
    const int64_t n = e / d, i = e % d;
    float acc = 0.f;
    for (int64_t k = 0; k < R; ++k) acc = fmaf(X[n * R + k], to_f32(P[i * R + k]), acc);
    dh[e] = from_f32<T>(acc);
}

__global__ void check_seqlens_kernel(const int32_t* __restrict__ cu, int64_t n_docs, int64_t N,
                                     uint32_t* __restrict__ err, int64_t max_doc_len) {
    bool bad = false, longdoc = false;
    for (int64_t i = threadIdx.x; i < n_docs; i += blockDim.x) {
        bad |= cu[i + 1] < cu[i];
        longdoc |= max_doc_len > 0 && (int64_t)cu[i + 1] - (int64_t)cu[i] > max_doc_len;
    }
    if (threadIdx.x == 0) bad |= (cu[0] != 0) || ((int64_t)cu[n_docs] != N);
    if (bad) atomicOr(err, kErrBadSeqlens);
    if (longdoc) atomicOr(err, kErrRopePos);
}

// x -> R x (forward) or R^T x (inverse) on the rotated channels of every token, one block per token:
// pairs (2i, 2i+1) of each rope_hd-channel head below rope_n turn by the table's angle at the token's
// position in its sequence / document; the other channels are copied (nothing to do in place).
template <typename T>
__global__ void __launch_bounds__(kThreads) rope_kernel(const T* __restrict__ x, Ax ax, T* __restrict__ out, Ax ao,
                                                         int64_t C, int64_t rope_n, int64_t rope_hd, int64_t rope_max,
                                                         const float* __restrict__ cs, const int32_t* __restrict__ cu,
                                                         int64_t n_docs, int64_t seqlen, int inverse, int copy_rest) {
    const int64_t n = blockIdx.x;
    int64_t pos = n - seg_start(n, cu, n_docs, seqlen);
    pos = pos < rope_max ? pos : rope_max - 1;            // in bounds even when the device check fails
    for (int64_t c = 2 * (int64_t)threadIdx.x; c < C; c += 2 * blockDim.x) {
        if (c < rope_n) {
            const float x0 = to_f32(x[ax(n, c)]), x1 = to_f32(x[ax(n, c + 1)]);
            const float co = cs[pos * rope_hd + (c % rope_hd)];
            const float si = inverse ? -cs[pos * rope_hd + (c % rope_hd) + 1] : cs[pos * rope_hd + (c % rope_hd) + 1];
            out[ao(n, c)] = from_f32<T>(fmaf(x0, co, -x1 * si));
            out[ao(n, c + 1)] = from_f32<T>(fmaf(x0, si, x1 * co));
        } else if (copy_rest) {
            out[ao(n, c)] = x[ax(n, c)];
            if (c + 1 < C) out[ao(n, c + 1)] = x[ax(n, c + 1)];
        }
    }
}

inline unsigned blocks_for(int64_t n) { return (unsigned)((n + kThreads - 1) / kThreads); }

template <typename T>
cudaError_t forward_t(const Prob& p, const void* u, const void* h, const void* A, const void* BW, void* y,
                      void* z_save, void* ws, cudaStream_t st) {
    const WsLayout L = ws_layout(p);
    float* X = reinterpret_cast<float*>(static_cast<char*>(ws) + L.gen);
    const T* P = static_cast<const T*>(p.kind == 0 ? A : BW);
    DC_LAUNCH(kSimtGen, st, gen_kernel<T><<<(unsigned)p.N, kThreads, 0, st>>>(
        static_cast<const T*>(h), p.hs, P, p.d, p.R, X, static_cast<T*>(z_save)));
    const size_t smem = sizeof(float) * (size_t)p.R;
    if (p.kind == 0)
        DC_LAUNCH(kSimtConvFwd, st, conv_fwd_kernel<T, 0><<<(unsigned)p.N, kThreads, smem, st>>>(
            static_cast<const T*>(u), ax_u(p), X, p.R, static_cast<const T*>(BW), p.C, p.K, 1, p.cu, p.n_docs,
            p.seqlen, static_cast<T*>(y), ax_dense(p)));
    else
        DC_LAUNCH(kSimtConvFwd, st, conv_fwd_kernel<T, 1><<<(unsigned)p.N, kThreads, smem, st>>>(
            static_cast<const T*>(u), ax_u(p), X, p.R, nullptr, p.C, p.K, p.hd, p.cu, p.n_docs, p.seqlen,
            static_cast<T*>(y), ax_dense(p)));
    return cudaGetLastError();
}

template <typename T>
cudaError_t backward_t(const Prob& p, const void* g, const void* u, const void* h, const void* A,
                       const void* BW, const void* z_saved, void* du, void* dh, float* dA, float* dBW,
                       void* ws, cudaStream_t st) {
    const WsLayout L = ws_layout(p);
    float* X = reinterpret_cast<float*>(static_cast<char*>(ws) + L.gen);
    float* DG = reinterpret_cast<float*>(static_cast<char*>(ws) + L.dgen);
    const T* P = static_cast<const T*>(p.kind == 0 ? A : BW);
    if (z_saved) {
        const int64_t cnt = p.N * p.R;
        const unsigned nb = (unsigned)(cnt < 148 * 64 * kThreads ? blocks_for(cnt) : 148 * 64);
        DC_LAUNCH(kSimtWiden, st, widen_kernel<T><<<nb, kThreads, 0, st>>>(static_cast<const T*>(z_saved), X, cnt));
    } else {
        DC_LAUNCH(kSimtGen, st, gen_kernel<T><<<(unsigned)p.N, kThreads, 0, st>>>(
            static_cast<const T*>(h), p.hs, P, p.d, p.R, X, nullptr));
    }
    const size_t smem = sizeof(float) * (size_t)(p.K * p.R + kThreads / 32);
    if (p.kind == 0)
        DC_LAUNCH(kSimtConvBwd, st, conv_bwd_kernel<T, 0><<<(unsigned)p.N, kThreads, smem, st>>>(
            static_cast<const T*>(g), static_cast<const T*>(u), ax_u(p), ax_dense(p), X, p.R,
            static_cast<const T*>(BW), p.N, p.C, p.K, 1, p.cu, p.n_docs, p.seqlen, static_cast<T*>(du), DG));
    else
        DC_LAUNCH(kSimtConvBwd, st, conv_bwd_kernel<T, 1><<<(unsigned)p.N, kThreads, smem, st>>>(
            static_cast<const T*>(g), static_cast<const T*>(u), ax_u(p), ax_dense(p), X, p.R, nullptr, p.N, p.C,
            p.K, p.hd, p.cu, p.n_docs, p.seqlen, static_cast<T*>(du), DG));
    if (p.kind == 0) {
        DC_LAUNCH(kSimtDB, st, dB_kernel<T><<<blocks_for(p.r * p.C * p.K), kThreads, 0, st>>>(
            X, p.r, static_cast<const T*>(g), static_cast<const T*>(u), ax_u(p), ax_dense(p), p.N, p.C, p.K, p.cu,
            p.n_docs, p.seqlen, dBW));
        DC_LAUNCH(kSimtHTX, st, hTX_kernel<T><<<blocks_for(p.d * p.R), kThreads, 0, st>>>(
            static_cast<const T*>(h), p.hs, DG, p.N, p.d, p.R, dA));
    } else {
        DC_LAUNCH(kSimtHTX, st, hTX_kernel<T><<<blocks_for(p.d * p.R), kThreads, 0, st>>>(
            static_cast<const T*>(h), p.hs, DG, p.N, p.d, p.R, dBW));
    }
    if (dh)
        DC_LAUNCH(kSimtDh, st, dh_kernel<T><<<blocks_for(p.N * p.d), kThreads, 0, st>>>(
            DG, P, p.N, p.d, p.R, static_cast<T*>(dh)));
    return cudaGetLastError();
}

}  // namespace

cudaError_t simt_forward(const Prob& p, const void* u, const void* h, const void* A, const void* BW, void* y,
                         void* z_save, void* ws, cudaStream_t st) {
    cudaError_t e = p.dtype == 0 ? forward_t<float>(p, u, h, A, BW, y, z_save, ws, st)
                                 : forward_t<__nv_bfloat16>(p, u, h, A, BW, y, z_save, ws, st);
    if (e != cudaSuccess || p.rope_n == 0) return e;
    return simt_rope(p, y, y, false, st);             // y <- R y, in place
}

cudaError_t simt_backward(const Prob& p, const void* g, const void* u, const void* h, const void* A,
                          const void* BW, const void* z_saved, void* du, void* dh, float* dA, float* dBW,
                          void* ws, cudaStream_t st) {
    if (p.rope_n > 0) {                                // the conv backward is fed with R^T g
        void* gt = static_cast<char*>(ws) + ws_layout(p).rope;
        cudaError_t e = simt_rope(p, g, gt, true, st);
        if (e != cudaSuccess) return e;
        g = gt;
    }
    return p.dtype == 0 ? backward_t<float>(p, g, u, h, A, BW, z_saved, du, dh, dA, dBW, ws, st)
                        : backward_t<__nv_bfloat16>(p, g, u, h, A, BW, z_saved, du, dh, dA, dBW, ws, st);
}

cudaError_t launch_check_seqlens(const int32_t* cu, int64_t n_docs, int64_t N, uint32_t* err, cudaStream_t st,
                                 int64_t max_doc_len) {
    DC_LAUNCH(kCheckSeqlens, st, check_seqlens_kernel<<<1, kThreads, 0, st>>>(cu, n_docs, N, err, max_doc_len));
    return cudaGetLastError();
}

cudaError_t simt_rope(const Prob& p, const void* x, void* out, bool inverse, cudaStream_t st) {
    if (p.N == 0) return cudaSuccess;
    const bool in_place = x == out;
    if (p.dtype == 0)
        DC_LAUNCH(kSimtRope, st, rope_kernel<float><<<(unsigned)p.N, kThreads, 0, st>>>(
            static_cast<const float*>(x), ax_dense(p), static_cast<float*>(out), ax_dense(p), p.C, p.rope_n,
            p.rope_hd, p.rope_max, p.rope_cs, p.cu, p.n_docs, p.seqlen, inverse ? 1 : 0, in_place ? 0 : 1));
    else
        DC_LAUNCH(kSimtRope, st, rope_kernel<__nv_bfloat16><<<(unsigned)p.N, kThreads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), ax_dense(p), static_cast<__nv_bfloat16*>(out), ax_dense(p), p.C,
            p.rope_n, p.rope_hd, p.rope_max, p.rope_cs, p.cu, p.n_docs, p.seqlen, inverse ? 1 : 0, in_place ? 0 : 1));
    return cudaGetLastError();
}

}  // namespace dynconv
