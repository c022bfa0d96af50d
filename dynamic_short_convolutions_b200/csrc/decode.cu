// decode.cu -- one decode step of the dynamic short convolution: the newest token of each of
// `batch` sequences, with the K - 1 previous conv inputs of each sequence kept in a rolling
// state.  The operation is the Mechanism formula of "Dynamic Short Convolutions Improve
// Transformers" (gist.science technical summary, "Dynamic Short Convolutions") applied at the
// last position, with the Parameterization's generated filter and the residual Placement:
//   y[b,c] = u[b,c] + sum_{j<K} w[b,c,j] x_j[b,c],   x_0 = u[b,c],  x_j = state[b, j-1, c]
//   w[b,c,j] = sum_k z[b,k] B[k, c K + j], z = h A      (low-rank)
//   w[b,c,j] = (h W)[b, (c / head_dim) K + j]           (head-wise)
// then state[b, j, c] <- x_j[b,c] for j = 0 .. K-2 (the state rolls by one token).  The pages
// leave inference unoptimised (atlas.scime.ai summary, "Limitations"); this is the step a
// generation loop needs.  A zero state is the start of a sequence: taps before the start read
// zero, as in the training forward.
//
// Kernels (CUDA cores, fp32 accumulation; the work per step is a few MB, latency-bound):
//   decode_gen_kernel   partial generator rows h[b, slice] P[slice, :] (P = A or W) per d-slice,
//                       32 outputs per block and every sequence of the batch.
//   decode_conv_kernel  per (128 channels, kDecRows sequences): the generator rows (the slices
//                       summed in order), the filter taps from them and B (each B element read
//                       once per block and applied to all of its sequences), the conv, the
//                       output row and the rolled state.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "prof.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace dynconv {
namespace {

using tc::pdl_trigger;
using tc::pdl_wait;

constexpr int kGenThreads = 256;
constexpr int kGenWarps = kGenThreads / 32;
constexpr int kConvThreads = 128;
constexpr int kDecRows = 4;           // sequences per block of decode_conv_kernel

// Split-d partial generator rows: part[s][b][k] = sum_{i in slice s} h[b, i] P[i, k] for the d-slice s
// of this block (blockIdx.y), 32 outputs k per block (one per lane), the sequences spread over the
// warps.  The slices are summed in order by decode_conv_kernel (deterministic).
template <typename T>
__global__ void __launch_bounds__(kGenThreads) decode_gen_kernel(const T* __restrict__ h, int64_t hs,
                                                                 const T* __restrict__ P, int64_t d, int64_t R,
                                                                 int64_t batch, int n_split,
                                                                 float* __restrict__ part) {
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t k = (int64_t)blockIdx.x * 32 + lane;
    const int split = blockIdx.y;
    const int64_t i0 = d * split / n_split, i1 = d * (split + 1) / n_split;
    // blockIdx.z: a chunk of 4 * kGenWarps sequences (four per warp)
    for (int64_t b0 = (int64_t)blockIdx.z * 4 * kGenWarps; b0 < batch; b0 += (int64_t)gridDim.z * 4 * kGenWarps) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        int64_t rows[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) rows[q] = b0 + warp + q * kGenWarps;
        if (k < R) {
#pragma unroll 4
            for (int64_t i = i0; i < i1; ++i) {
                const float pk = to_f32(P[i * R + k]);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (rows[q] < batch) acc[q] = fmaf(to_f32(h[rows[q] * hs + i]), pk, acc[q]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (rows[q] < batch) part[((int64_t)split * batch + rows[q]) * R + k] = acc[q];
        }
    }
}

template <typename T, int KIND, int K>
__global__ void __launch_bounds__(kConvThreads) decode_conv_kernel(const T* __restrict__ u, int64_t us,
                                                                   const float* __restrict__ part, int n_split,
                                                                   int64_t R, const T* __restrict__ B, int64_t C,
                                                                   int64_t hd, int64_t batch, T* __restrict__ state,
                                                                   T* __restrict__ y) {
    extern __shared__ float xs[];   // [kDecRows][R]: the generator rows of this block's sequences
    pdl_trigger();
    pdl_wait();
    const int64_t b0 = (int64_t)blockIdx.y * kDecRows;
    const int nb = batch - b0 < kDecRows ? (int)(batch - b0) : kDecRows;
    for (int64_t i = threadIdx.x; i < nb * R; i += blockDim.x) {
        float acc = 0.f;
        for (int sp = 0; sp < n_split; ++sp) acc += part[((int64_t)sp * batch + b0) * R + i];
        xs[i] = acc;
    }
    __syncthreads();
    const int64_t c = (int64_t)blockIdx.x * kConvThreads + threadIdx.x;
    if (c >= C) return;
    float w[kDecRows][K];
    if (KIND == 0) {
#pragma unroll
        for (int r = 0; r < kDecRows; ++r)
#pragma unroll
            for (int j = 0; j < K; ++j) w[r][j] = 0.f;
        const T* bc = B + c * K;
#pragma unroll 4
        for (int64_t k = 0; k < R; ++k) {
            float bk[K];
#pragma unroll
            for (int j = 0; j < K; ++j) bk[j] = to_f32(bc[k * C * K + j]);
#pragma unroll
            for (int r = 0; r < kDecRows; ++r)
#pragma unroll
                for (int j = 0; j < K; ++j) w[r][j] = fmaf(xs[r * R + k], bk[j], w[r][j]);
        }
    } else {
        const int64_t q = c / hd;
#pragma unroll
        for (int r = 0; r < kDecRows; ++r)
#pragma unroll
            for (int j = 0; j < K; ++j) w[r][j] = r < nb ? xs[r * R + q * K + j] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < kDecRows; ++r) {
        if (r >= nb) break;
        const int64_t b = b0 + r;
        float x[K];
        x[0] = to_f32(u[b * us + c]);
#pragma unroll
        for (int j = 1; j < K; ++j) x[j] = to_f32(state[(b * (K - 1) + (j - 1)) * C + c]);
        float acc = x[0];
#pragma unroll
        for (int j = 0; j < K; ++j) acc = fmaf(w[r][j], x[j], acc);
        y[b * C + c] = from_f32<T>(acc);
#pragma unroll
        for (int j = 0; j + 1 < K; ++j) state[(b * (K - 1) + j) * C + c] = from_f32<T>(x[j]);
    }
}

// Sequence chunks (grid z) and d-slices (grid y) of the generator: enough blocks to cover the
// SMs about twice, slices of at least 32.
inline int gen_chunks(const Prob& p) { return (int)std::max<int64_t>(1, (p.N + 4 * kGenWarps - 1) / (4 * kGenWarps)); }
inline int gen_splits(const Prob& p) {
    const int64_t blocks = ((p.R + 31) / 32) * gen_chunks(p);
    const int64_t want = (2 * 148 + blocks - 1) / blocks;
    return (int)std::max<int64_t>(1, std::min<int64_t>(want, (p.d + 31) / 32));
}

template <typename T, int KIND, int K>
cudaError_t launch_conv(const Prob& p, const void* u, const float* part, int n_split, const void* BW, void* state,
                        void* y, cudaStream_t st) {
    const dim3 grid((unsigned)((p.C + kConvThreads - 1) / kConvThreads), (unsigned)((p.batch + kDecRows - 1) / kDecRows));
    const size_t smem = sizeof(float) * (size_t)kDecRows * (size_t)p.R;
    cudaError_t e;
    DC_LAUNCH(kDecodeConv, st, e = launch_pdl(decode_conv_kernel<T, KIND, K>, grid, dim3(kConvThreads), smem, st,
                                              static_cast<const T*>(u), p.us, (const float*)part, n_split, p.R,
                                              KIND == 0 ? static_cast<const T*>(BW) : nullptr, p.C,
                                              p.hd > 0 ? p.hd : 1, p.batch, static_cast<T*>(state),
                                              static_cast<T*>(y)));
    return e;
}

template <typename T, int KIND>
cudaError_t conv_k(const Prob& p, const void* u, const float* part, int n_split, const void* BW, void* state,
                   void* y, cudaStream_t st) {
    switch (p.K) {
        case 1: return launch_conv<T, KIND, 1>(p, u, part, n_split, BW, state, y, st);
        case 2: return launch_conv<T, KIND, 2>(p, u, part, n_split, BW, state, y, st);
        case 3: return launch_conv<T, KIND, 3>(p, u, part, n_split, BW, state, y, st);
        default: return launch_conv<T, KIND, 4>(p, u, part, n_split, BW, state, y, st);
    }
}

template <typename T>
cudaError_t decode_t(const Prob& p, const void* u, const void* h, const void* A, const void* BW, void* state,
                     void* y, void* ws, cudaStream_t st) {
    const WsLayout L = ws_layout(p);
    float* part = reinterpret_cast<float*>(static_cast<char*>(ws) + L.dec);
    const T* P = static_cast<const T*>(p.kind == 0 ? A : BW);
    const int n_split = gen_splits(p);
    const dim3 grid((unsigned)((p.R + 31) / 32), (unsigned)n_split, (unsigned)gen_chunks(p));
    cudaError_t e;
    DC_LAUNCH(kDecodeGen, st, e = launch_pdl(decode_gen_kernel<T>, grid, dim3(kGenThreads), 0, st,
                                             static_cast<const T*>(h), p.hs, P, p.d, p.R, p.batch, n_split, part));
    if (e != cudaSuccess) return e;
    return p.kind == 0 ? conv_k<T, 0>(p, u, part, n_split, BW, state, y, st)
                       : conv_k<T, 1>(p, u, part, n_split, BW, state, y, st);
}

}  // namespace

size_t decode_partial_bytes(const Prob& p) { return sizeof(float) * (size_t)gen_splits(p) * p.N * p.R; }

cudaError_t decode_step(const Prob& p, const void* u, const void* h, const void* A, const void* BW, void* state,
                        void* y, void* ws, cudaStream_t st) {
    return p.dtype == 1 ? decode_t<__nv_bfloat16>(p, u, h, A, BW, state, y, ws, st)
                        : decode_t<float>(p, u, h, A, BW, state, y, ws, st);
}

}  // namespace dynconv
