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
// The conv kernels are memory-bound CUDA-core kernels: token-major (a warp streams consecutive
// tokens through per-lane cp.async rings in shared memory, 16-byte loads and stores along C,
// packed fp32 FMAs, a reduce-scatter over each head's lanes for dwh) and channel-first (a warp
// streams a head's token rows of [batch * C, seqlen] through a TMA ring, a lane's filter taps held
// across the head's channels, dwh summed per warp and then over the block's warps in order).
#include <algorithm>
#include <type_traits>

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

// Token-major kernels: a warp streams a run of consecutive tokens over 256 channels, each lane 8
// channels (16-byte stores along C, packed fp32 FMAs).  The rows of each token -- u; g; the
// filter taps of the block's heads; with RoPE the table row of the token's position -- come into
// a shared-memory ring by TMA, a few tokens at a time, so ~8 tokens of every warp are in flight
// without registers held for them, and rows outside [0, N) read zero through the tensor maps'
// bounds.  The rows of u (and the backward's pending du rows) sit in rolling register windows,
// so a row is read and unpacked once; only the K - 1 rows of u before a run (and of g after it)
// are read twice.
constexpr int kHwRunFwd = 16, kHwRunBwd = 32;      // tokens per run (one warp, one block)
constexpr int kHwMaxRopeHd = 256;                  // RoPE table rows of up to 256 floats (1 KB)

// Segment bounds [s, e) of the tokens a warp walks through in increasing order: looked up again
// (seg_bounds32) only when the walk leaves the current segment.
struct SegWalk {
    int32_t s = 0, e = 0;
    __device__ __forceinline__ int32_t pos(int32_t n, const int32_t* __restrict__ cu, int32_t n_docs, int32_t seqlen,
                                           int32_t N) {
        if (n >= e) seg_bounds32(n, cu, n_docs, seqlen, N, s, e);
        return n - s;
    }
};

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

// acc[0..8) += w * x[0..8) on the packed fp32 FMA.
__device__ __forceinline__ void axpy8f(float (&acc)[8], float w, const float (&x)[8]) {
#pragma unroll
    for (int p = 0; p < 4; ++p) ffma2(acc[2 * p], acc[2 * p + 1], w, w, x[2 * p], x[2 * p + 1]);
}

// sum_i a[i] b[i] over 8 values (two fp32 lanes, then their sum).
__device__ __forceinline__ float dot8f(const float (&a)[8], const float (&b)[8]) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int p = 0; p < 4; ++p) ffma2(s0, s1, a[2 * p], a[2 * p + 1], b[2 * p], b[2 * p + 1]);
    return s0 + s1;
}

// The K taps of one head's filter for one token, as floats: 8- or 4-byte loads for K = 4 and
// K = 2 (aligned since R = H K and the taps boxes start at multiples of 8 columns), else
// element by element.  p is global (channel-first kernels) or shared memory (token-major).
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

// Sums p[0..K) over the L lanes (a power of two <= 32) that hold one head and stores dst[j]
// for j < K, masked to 0 for j > pos, when `store`.  For K >= 3 and L >= 4 a reduce-scatter:
// two exchange steps leave each lane one tap, then a butterfly finishes it (log2(L) + 1
// shuffles instead of K log2(L)); otherwise a plain butterfly over all K values.  Every lane
// of the warp takes part in the shuffles.
template <int K>
__device__ __forceinline__ void head_sum_store(float (&p)[K], int L, int gl, int32_t pos, bool store,
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
#pragma unroll
            for (int it = 1; it <= 3; ++it) {            // offsets h2 / 2, h2 / 4, h2 / 8 (h2 <= 8)
                const int off = h2 >> it;
                if (off > 0) k += __shfl_xor_sync(0xffffffffu, k, off);
            }
            const int tap = (b1 ? 2 : 0) + (b2 ? 1 : 0);
            if (store && (gl & (h2 - 1)) == 0 && tap < K) dst[tap] = __float2bfloat16_rn(tap <= pos ? k : 0.f);
            return;
        }
    }
#pragma unroll
    for (int j = 0; j < K; ++j)
#pragma unroll
        for (int it = 1; it <= 5; ++it) {
            const int off = L >> it;
            if (off > 0) p[j] += __shfl_xor_sync(0xffffffffu, p[j], off);
        }
    const int l = gl & (L - 1);
#pragma unroll
    for (int j = 0; j < K; ++j)
        if (store && j % L == l) dst[j] = __float2bfloat16_rn(j <= pos ? p[j] : 0.f);
}

// Rows come in chunks of T stream rows (T a multiple of K, so a row's place in the rolling windows
// is fixed by its place in the chunk): one TMA box per tensor and chunk, one mbarrier per ring
// slot, kept Q - 1 chunks ahead of the chunk being computed.  A block is one warp and one run:
// block b takes channel block b % n_cblk and tokens (b / n_cblk) * run onwards, so everything
// that depends on the token position is uniform over the block and only the channel offset
// varies by lane.  Chunks whose rows are all interior (no look-back, look-ahead or end of the
// tensor among them) run a body without the per-row range tests, and without the taps' segment
// mask when none of their rows is within K - 1 tokens of a segment start.
template <int K>
struct HwTile {
    static constexpr int T = K >= 3 ? K : 4;     // stream rows per chunk
    static constexpr int Q = (12 + T - 1) / T;   // ring slots (chunks)
};

__host__ __device__ constexpr uint32_t al128(uint32_t x) { return (x + 127u) & ~127u; }

// Forward.  A run covers tokens n0 .. n0 + run - 1; its stream starts K - 1 rows earlier (the
// taps' reach back).  Chunk: u rows [T][512 B], taps rows [T][taps_box], RoPE table rows
// [T][rope_hd floats].
template <int K>
__global__ void __launch_bounds__(32, 24) hw_conv_fwd_kernel(const __grid_constant__ CUtensorMap tm_u,
                                                         const __grid_constant__ CUtensorMap tm_w, int hd, int32_t N,
                                                         int64_t C, int32_t seqlen, const int32_t* __restrict__ cu,
                                                         int32_t n_docs, int n_cblk, __nv_bfloat16* __restrict__ y,
                                                         const float* __restrict__ rope_cs, int rope_n, int rope_hd,
                                                         int rope_max, int run, int taps_box, uint32_t* err) {
    constexpr int T = HwTile<K>::T, Q = HwTile<K>::Q;
    extern __shared__ __align__(128) uint8_t hw_smem[];
    __shared__ uint64_t bars[Q];
    __shared__ int abort_flag;
    const int lane = threadIdx.x;
    if (lane == 0) {
        for (int s = 0; s < Q; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        abort_flag = 0;
        tma_prefetch(&tm_u);
        tma_prefetch(&tm_w);
    }
    __syncwarp();
    pdl_trigger();
    pdl_wait();
    const int32_t cb = (int32_t)(blockIdx.x % (uint32_t)n_cblk);
    const int32_t n0 = (int32_t)(blockIdx.x / (uint32_t)n_cblk) * run;
    const int32_t c0 = cb * 256, c = c0 + lane * 8;
    const int q = c / hd, x0 = ((c0 / hd) * K) & ~7;
    const int len = min(run, N - n0) + K - 1, nch = (len + T - 1) / T;
    const bool rope_blk = rope_cs != nullptr && c0 < rope_n;      // the block holds rotated channels
    const bool rot = rope_blk && c < rope_n;
    const uint32_t tpitch = (uint32_t)taps_box * 2u, toff = al128(T * 512u);
    const uint32_t rrow = (uint32_t)rope_hd * 4u, roff = toff + al128(T * tpitch);
    const uint32_t chunk = al128(roff + (rope_cs ? T * rrow : 0u));
    const int tl = q * K - x0, rl = rot ? (c % rope_hd) : 0;
    SegWalk walk_in, walk;
    auto issue = [&](int k) {                        // lane 0
        if (k >= nch) return;
        const int32_t row0 = n0 - (K - 1) + k * T;
        uint8_t* sl = hw_smem + (uint32_t)(k % Q) * chunk;
        uint64_t* bar = &bars[k % Q];
        mbar_arrive_expect_tx(bar, T * 512u + T * tpitch + (rope_blk ? T * rrow : 0u));
        tma_load_2d(sl, &tm_u, bar, c0, row0);
        tma_load_2d(sl + toff, &tm_w, bar, x0, row0);
        if (rope_blk) {
#pragma unroll
            for (int t = 0; t < T; ++t) {            // the table row of each token's position
                const int32_t n = row0 + t;
                const int32_t p = (n >= n0 && n < N) ? min(walk_in.pos(n, cu, n_docs, seqlen, N), rope_max - 1) : 0;
                bulk_load(sl + roff + t * rrow, rope_cs + (int64_t)p * rope_hd, rrow, bar);
            }
        }
    };
    if (lane == 0)
        for (int k = 0; k < Q - 1; ++k) issue(k);
    __nv_bfloat16* yp = y + (int64_t)n0 * C + c;
    float win[K][8];                                 // u row of stream index r at win[r mod K]
    auto body = [&](const uint8_t* sl, int r0, auto full, auto masked) {
        constexpr bool FULL = decltype(full)::value, MASK = decltype(masked)::value;
#pragma unroll
        for (int s = 0; s < T; ++s) {
            const int r = r0 + s;
            if (!FULL && r >= len) break;
            unpack8(*reinterpret_cast<const uint4*>(sl + s * 512 + lane * 16), win[s % K]);
            const int32_t n = n0 - (K - 1) + r;
            if (!FULL && n < n0) continue;
            const int32_t pos = MASK ? walk.pos(n, cu, n_docs, seqlen, N) : K;
            float w[K];
            load_taps<K>(reinterpret_cast<const __nv_bfloat16*>(sl + toff + s * tpitch) + tl, w);
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = win[s % K][e];
#pragma unroll
            for (int j = 0; j < K; ++j) axpy8f(acc, (!MASK || j <= pos) ? w[j] : 0.f, win[(s - j + K) % K]);
            if (rot) {
                const float4* t = reinterpret_cast<const float4*>(sl + roff + s * rrow + rl * 4);
                rope_pairs8v(acc, t[0], t[1], false);
            }
            *reinterpret_cast<uint4*>(yp) = pack8(acc);
            yp += C;
        }
    };
    int k_fail = -1;
    for (int k = 0; k < nch; ++k) {
        __syncwarp();                                // slot k - 1, which chunk k + Q - 1 refills, is read
        if (lane == 0) {
            fence_async_smem();
            issue(k + Q - 1);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bars[k % Q], (uint32_t)(k / Q) & 1u, &abort_flag, err))) {
            k_fail = k;
            break;
        }
        const uint8_t* sl = hw_smem + (uint32_t)(k % Q) * chunk;
        const int r0 = k * T;
        if (r0 >= K - 1 && r0 + T <= len) {
            // no row of the chunk within K - 1 of a segment start: the taps need no mask
            const int32_t nf = n0 - (K - 1) + r0;
            if (walk.pos(nf, cu, n_docs, seqlen, N) >= K - 1 && nf + T <= walk.e)
                body(sl, r0, std::true_type{}, std::false_type{});
            else
                body(sl, r0, std::true_type{}, std::true_type{});
        } else {
            body(sl, r0, std::false_type{}, std::true_type{});
        }
    }
    if (k_fail >= 0 && lane == 0)                    // let the copies already issued land
        for (int k = k_fail; k < min(nch, k_fail + Q); ++k) mbar_wait_drain(&bars[k % Q], (uint32_t)(k / Q) & 1u);
}

// Backward.  A run covers tokens n0 .. n_end - 1 (du and dwh rows); its stream runs from
// n0 - K + 1 (the rows of u that dwh reaches back to) to n_end + K - 2 (the rows of g whose
// filters reach back into the run).  du is accumulated forward: token n adds wh[n, j] g[n] to
// the pending du row n - j, which takes the terms of du[m] in the order j = 0 .. K - 1; row
// n - K + 1 is then complete and stored.  Chunk: g rows, u rows ([T][512 B] each), taps rows.
// With RoPE the blocks of rotated channels read g from R^T g (tm_gr, written beforehand).
template <int K>
__global__ void __launch_bounds__(32, 16) hw_conv_bwd_kernel(const __grid_constant__ CUtensorMap tm_g,
                                                         const __grid_constant__ CUtensorMap tm_gr,
                                                         const __grid_constant__ CUtensorMap tm_u,
                                                         const __grid_constant__ CUtensorMap tm_w, int R, int hd,
                                                         int32_t N, int64_t C, int32_t seqlen,
                                                         const int32_t* __restrict__ cu, int32_t n_docs, int n_cblk,
                                                         __nv_bfloat16* __restrict__ du,
                                                         __nv_bfloat16* __restrict__ dwh, int rope_n, int run,
                                                         int taps_box, uint32_t* err) {
    constexpr int T = HwTile<K>::T, Q = HwTile<K>::Q;
    extern __shared__ __align__(128) uint8_t hw_smem[];
    __shared__ uint64_t bars[Q];
    __shared__ int abort_flag;
    const int lane = threadIdx.x;
    if (lane == 0) {
        for (int s = 0; s < Q; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        abort_flag = 0;
        tma_prefetch(&tm_g);
        tma_prefetch(&tm_gr);
        tma_prefetch(&tm_u);
        tma_prefetch(&tm_w);
    }
    __syncwarp();
    pdl_trigger();
    pdl_wait();
    const int32_t cb = (int32_t)(blockIdx.x % (uint32_t)n_cblk);
    const int32_t n0 = (int32_t)(blockIdx.x / (uint32_t)n_cblk) * run;
    const int32_t c0 = cb * 256, c = c0 + lane * 8;
    const int q = c / hd, x0 = ((c0 / hd) * K) & ~7;
    const int L = hd >> 3, tl = q * K - x0;
    const int32_t n_end = min(n0 + run, N);
    const int nb = n_end - n0, len = nb + 2 * (K - 1), nch = (len + T - 1) / T;
    const CUtensorMap* tg = c0 < rope_n ? &tm_gr : &tm_g;
    const uint32_t tpitch = (uint32_t)taps_box * 2u, toff = T * 1024u;
    const uint32_t chunk = al128(toff + T * tpitch);
    auto issue = [&](int k) {                        // lane 0
        if (k >= nch) return;
        const int32_t row0 = n0 - (K - 1) + k * T;
        uint8_t* sl = hw_smem + (uint32_t)(k % Q) * chunk;
        uint64_t* bar = &bars[k % Q];
        mbar_arrive_expect_tx(bar, T * 1024u + T * tpitch);
        tma_load_2d(sl, tg, bar, c0, row0);
        tma_load_2d(sl + T * 512, &tm_u, bar, c0, row0);
        tma_load_2d(sl + toff, &tm_w, bar, x0, row0);
    };
    if (lane == 0)
        for (int k = 0; k < Q - 1; ++k) issue(k);
    SegWalk walk;
    __nv_bfloat16* dup = du + (int64_t)n0 * C + c;
    __nv_bfloat16* dwp = dwh + (int64_t)n0 * R + q * K;
    float uw[K][8];                                  // u row of stream index r at uw[r mod K]
    float acc[K][8];                                 // pending du row of stream index r at acc[r mod K]
    auto body = [&](const uint8_t* sl, int r0, auto full, auto masked) {
        constexpr bool FULL = decltype(full)::value, MASK = decltype(masked)::value;
#pragma unroll
        for (int s = 0; s < T; ++s) {
            const int r = r0 + s;
            if (!FULL && r >= len) break;
            const int32_t n = n0 - (K - 1) + r;
            if (FULL || n < n_end) unpack8(*reinterpret_cast<const uint4*>(sl + (T + s) * 512 + lane * 16), uw[s % K]);
            if (!FULL && n < n0) continue;
            const int32_t pos = !MASK ? K : (FULL || n < N) ? walk.pos(n, cu, n_docs, seqlen, N) : 0;
            float gf[8], w[K];
            unpack8(*reinterpret_cast<const uint4*>(sl + s * 512 + lane * 16), gf);
            load_taps<K>(reinterpret_cast<const __nv_bfloat16*>(sl + toff + s * tpitch) + tl, w);
            // du: a new row for token n, then token n's term of the pending rows n - 1 .. n - K + 1
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[s % K][e] = gf[e];
            axpy8f(acc[s % K], w[0], gf);
#pragma unroll
            for (int j = 1; j < K; ++j)
                if (FULL || n - j >= n0) axpy8f(acc[(s - j + K) % K], (!MASK || j <= pos) ? w[j] : 0.f, gf);
            if (FULL || n < n_end) {                 // dwh[n, q K + j] = sum over the head of g[n] . u[n - j]
                float part[K];
#pragma unroll
                for (int j = 0; j < K; ++j) part[j] = dot8f(gf, uw[(s - j + K) % K]);
                head_sum_store<K>(part, L, lane, pos, true, dwp);
                dwp += R;
            }
            if (FULL || n - (K - 1) >= n0) {         // row n - K + 1 is complete
                *reinterpret_cast<uint4*>(dup) = pack8(acc[(s + 1) % K]);
                dup += C;
            }
        }
    };
    int k_fail = -1;
    for (int k = 0; k < nch; ++k) {
        __syncwarp();                                // slot k - 1, which chunk k + Q - 1 refills, is read
        if (lane == 0) {
            fence_async_smem();
            issue(k + Q - 1);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bars[k % Q], (uint32_t)(k / Q) & 1u, &abort_flag, err))) {
            k_fail = k;
            break;
        }
        const uint8_t* sl = hw_smem + (uint32_t)(k % Q) * chunk;
        const int r0 = k * T;
        if (r0 >= 2 * (K - 1) && r0 + T <= K - 1 + nb) {
            // no row of the chunk within K - 1 of a segment start: the taps need no mask
            const int32_t nf = n0 - (K - 1) + r0;
            if (walk.pos(nf, cu, n_docs, seqlen, N) >= K - 1 && nf + T <= walk.e)
                body(sl, r0, std::true_type{}, std::false_type{});
            else
                body(sl, r0, std::true_type{}, std::true_type{});
        } else {
            body(sl, r0, std::false_type{}, std::true_type{});
        }
    }
    if (k_fail >= 0 && lane == 0)                    // let the copies already issued land
        for (int k = k_fail; k < min(nch, k_fail + Q); ++k) mbar_wait_drain(&bars[k % Q], (uint32_t)(k / Q) & 1u);
}

// ---- channel-first layout: u, y, g, du are [batch * C, seqlen] rows (tokens contiguous) ----
// A warp takes a window of kCfW tokens t0 .. t0 + kCfW - 1 of one sequence b and up to kCfCPW
// channel rows of one head q; lane l takes tokens t0 + 8 l .. t0 + 8 l + 7, whose filter taps (masked
// for the segment) stay in registers across the channels.  The rows come CH at a time through a
// TMA ring in shared memory: the window (box {kCfW, CH}) and 8 tokens beside it (box {8, CH}:
// before the window for u, after it for g), so each lane finds its K - 1 <= 3
// neighbours in its row of the chunk.  seqlen is a multiple of 8, so a lane's 8 tokens are all
// inside the sequence or all past its end (rows past the end read zero).
constexpr int kCfW = 256;                          // tokens per window (8 per lane)
constexpr int kCfFwdCH = 2, kCfBwdCH = 4;          // channel rows per chunk (CH)
constexpr int kCfQ = 4;                            // ring slots (chunks)
constexpr int kCfCPW = 64;                         // channel rows per warp
// Chunk layouts (every TMA destination on a 128-byte boundary): forward u window, u 8 before;
// backward g window, g 8 after, u window, u 8 before.
constexpr uint32_t kCfFwdUh = kCfFwdCH * 2 * kCfW, kCfFwdChunk = al128(kCfFwdUh + kCfFwdCH * 16);
constexpr uint32_t kCfBwdGa = kCfBwdCH * 2 * kCfW, kCfBwdU = al128(kCfBwdGa + kCfBwdCH * 16);
constexpr uint32_t kCfBwdUh = kCfBwdU + kCfBwdCH * 2 * kCfW, kCfBwdChunk = al128(kCfBwdUh + kCfBwdCH * 16);
static_assert(kCfFwdUh % 128 == 0 && kCfFwdChunk % 128 == 0 && kCfBwdGa % 128 == 0 && kCfBwdU % 128 == 0 &&
                  kCfBwdUh % 128 == 0 && kCfBwdChunk % 128 == 0,
              "TMA destinations in shared memory start on 128-byte boundaries");

// 8 bf16 of a row as floats / the 4 before them, from shared memory.
__device__ __forceinline__ void lds8(const uint8_t* p, float (&f)[8]) { unpack8(*reinterpret_cast<const uint4*>(p), f); }
__device__ __forceinline__ void lds4(const uint8_t* p, float (&f)[4]) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    f[0] = bf16_lo(v.x);
    f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y);
    f[3] = bf16_hi(v.y);
}

// y[c, t] = u[c, t] + sum_{j <= t - s(t)} wh[t, q K + j] u[c, t - j]  (the same FMA order as the
// token-major kernel, so both layouts give the same bits).  Blocks: (b, window, head, part).
template <int K>
__global__ void __launch_bounds__(32, 24) hw_conv_fwd_cf_kernel(const __grid_constant__ CUtensorMap tm_u,
                                                                const __grid_constant__ CUtensorMap tm_uh,
                                                                const __nv_bfloat16* __restrict__ wh, int R, int hd,
                                                                int64_t C, int64_t T, int64_t tps, int parts, int H,
                                                                const int32_t* __restrict__ cu, int64_t n_docs,
                                                                __nv_bfloat16* __restrict__ y, uint32_t* err) {
    extern __shared__ __align__(128) uint8_t hw_smem[];
    __shared__ uint64_t bars[kCfQ];
    __shared__ int abort_flag;
    const int lane = threadIdx.x;
    if (lane == 0) {
        for (int s = 0; s < kCfQ; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        abort_flag = 0;
        tma_prefetch(&tm_u);
        tma_prefetch(&tm_uh);
    }
    __syncwarp();
    pdl_trigger();
    pdl_wait();
    int64_t unit = blockIdx.x;
    const int part = (int)(unit % parts);
    unit /= parts;
    const int q = (int)(unit % H);
    unit /= H;
    const int64_t win = unit % tps, b = unit / tps;
    const int64_t t0 = win * kCfW, t = t0 + 8 * lane;
    const bool live = t < T;
    const int c_begin = q * hd + part * kCfCPW, nrows = min(kCfCPW, hd - part * kCfCPW);
    const int nch = (nrows + kCfFwdCH - 1) / kCfFwdCH;
    const int64_t n0 = b * T + t;
    float wm[8][K];                                  // taps of the lane's tokens, masked for the segment
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (live) {
            load_taps<K>(wh + (n0 + i) * R + q * K, wm[i]);
            const int64_t pos = n0 + i - seg_start(n0 + i, cu, n_docs, T);
#pragma unroll
            for (int j = 0; j < K; ++j) wm[i][j] = j <= pos ? wm[i][j] : 0.f;
        } else {
#pragma unroll
            for (int j = 0; j < K; ++j) wm[i][j] = 0.f;
        }
    }
    auto issue = [&](int k) {                        // lane 0
        if (k >= nch) return;
        uint8_t* sl = hw_smem + (uint32_t)(k % kCfQ) * kCfFwdChunk;
        uint64_t* bar = &bars[k % kCfQ];
        const int32_t row0 = (int32_t)(b * C + c_begin + k * kCfFwdCH);
        mbar_arrive_expect_tx(bar, kCfFwdCH * (2 * kCfW + 16));
        tma_load_2d(sl, &tm_u, bar, (int32_t)t0, row0);
        tma_load_2d(sl + kCfFwdUh, &tm_uh, bar, (int32_t)t0 - 8, row0);
    };
    if (lane == 0)
        for (int k = 0; k < kCfQ - 1; ++k) issue(k);
    int k_fail = -1;
    for (int k = 0; k < nch; ++k) {
        __syncwarp();                                // slot k - 1, which chunk k + kCfQ - 1 refills, is read
        if (lane == 0) {
            fence_async_smem();
            issue(k + kCfQ - 1);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bars[k % kCfQ], (uint32_t)(k / kCfQ) & 1u, &abort_flag, err))) {
            k_fail = k;
            break;
        }
        const uint8_t* sl = hw_smem + (uint32_t)(k % kCfQ) * kCfFwdChunk;
#pragma unroll
        for (int r = 0; r < kCfFwdCH; ++r) {
            if (k * kCfFwdCH + r >= nrows) break;
            const uint8_t* row = sl + r * 2 * kCfW;
            float x[8], xp[4];                       // tokens t .. t + 7 and t - 4 .. t - 1
            lds8(row + 16 * lane, x);
            lds4(lane > 0 ? row + 16 * lane - 8 : sl + kCfFwdUh + r * 16 + 8, xp);
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                acc[i] = x[i];
#pragma unroll
                for (int j = 0; j < K; ++j) acc[i] = fmaf(wm[i][j], i - j >= 0 ? x[i - j] : xp[4 + i - j], acc[i]);
            }
            if (live) {
                const int64_t c = c_begin + k * kCfFwdCH + r;
                *reinterpret_cast<uint4*>(y + (b * C + c) * T + t) = pack8(acc);
            }
        }
    }
    if (k_fail >= 0 && lane == 0)                    // let the copies already issued land
        for (int k = k_fail; k < min(nch, k_fail + kCfQ); ++k)
            mbar_wait_drain(&bars[k % kCfQ], (uint32_t)(k / kCfQ) & 1u);
}

// du[c, t] = g[c, t] + sum_{j < e(t) - t} wh[t + j, q K + j] g[c, t + j]; dwh[t, q K + j] =
// sum_{c in q} [j <= t - s(t)] g[c, t] u[c, t - j].  A block is (b, window, head): warp w streams
// the head's channel rows w kCfCPW .. w kCfCPW + kCfCPW - 1, sums its dwh terms over them in
// order, then the block sums the warps' partials in order (no atomics).
template <int K>
__global__ void __launch_bounds__(256) hw_conv_bwd_cf_kernel(const __grid_constant__ CUtensorMap tm_g,
                                                             const __grid_constant__ CUtensorMap tm_ga,
                                                             const __grid_constant__ CUtensorMap tm_u,
                                                             const __grid_constant__ CUtensorMap tm_uh,
                                                             const __nv_bfloat16* __restrict__ wh, int R, int hd,
                                                             int64_t N, int64_t C, int64_t T, int64_t tps, int H,
                                                             const int32_t* __restrict__ cu, int64_t n_docs,
                                                             __nv_bfloat16* __restrict__ du,
                                                             __nv_bfloat16* __restrict__ dwh, uint32_t* err) {
    extern __shared__ __align__(128) uint8_t hw_smem[];
    __shared__ uint64_t bars[8][kCfQ];
    __shared__ int abort_flag;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    if (lane == 0) {
        for (int s = 0; s < kCfQ; ++s) mbar_init(&bars[warp][s], 1);
        fence_mbar_init();
    }
    if (threadIdx.x == 0) {
        abort_flag = 0;
        tma_prefetch(&tm_g);
        tma_prefetch(&tm_ga);
        tma_prefetch(&tm_u);
        tma_prefetch(&tm_uh);
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();
    const int q = (int)(blockIdx.x % H);
    const int64_t rest = blockIdx.x / H, win = rest % tps, b = rest / tps;
    const int64_t t0 = win * kCfW, t = t0 + 8 * lane;
    const bool live = t < T;
    const int c_begin = q * hd + warp * kCfCPW, nrows = max(0, min(kCfCPW, hd - warp * kCfCPW));
    const int nch = (nrows + kCfBwdCH - 1) / kCfBwdCH;
    const int64_t n0 = b * T + t;
    uint8_t* ring = hw_smem + (uint32_t)warp * kCfQ * kCfBwdChunk;
    // dm[i][j]: tap j of the filter of token t + i + j for du[t + i], zero past the segment end
    float dm[8][K];
    {
        float wf[8 + K - 1][K];
#pragma unroll
        for (int i = 0; i < 8 + K - 1; ++i) {
            if (live && t + i < T) load_taps<K>(wh + (n0 + i) * R + q * K, wf[i]);
            else
#pragma unroll
                for (int j = 0; j < K; ++j) wf[i][j] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int64_t sb = 0, eb = 0;
            if (live) seg_bounds(n0 + i, cu, n_docs, T, N, sb, eb);
            const int64_t epos = eb - 1 - (n0 + i);
#pragma unroll
            for (int j = 0; j < K; ++j) dm[i][j] = (live && j <= epos) ? wf[i + j][j] : 0.f;
        }
    }
    float dacc[8][K];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j) dacc[i][j] = 0.f;
    constexpr uint32_t kGa = kCfBwdGa, kU = kCfBwdU, kUh = kCfBwdUh;
    auto issue = [&](int k) {                        // lane 0
        if (k >= nch) return;
        uint8_t* sl = ring + (uint32_t)(k % kCfQ) * kCfBwdChunk;
        uint64_t* bar = &bars[warp][k % kCfQ];
        const int32_t row0 = (int32_t)(b * C + c_begin + k * kCfBwdCH);
        mbar_arrive_expect_tx(bar, 2 * kCfBwdCH * (2 * kCfW + 16));
        tma_load_2d(sl, &tm_g, bar, (int32_t)t0, row0);
        tma_load_2d(sl + kGa, &tm_ga, bar, (int32_t)t0 + kCfW, row0);
        tma_load_2d(sl + kU, &tm_u, bar, (int32_t)t0, row0);
        tma_load_2d(sl + kUh, &tm_uh, bar, (int32_t)t0 - 8, row0);
    };
    if (lane == 0)
        for (int k = 0; k < kCfQ - 1; ++k) issue(k);
    int k_fail = -1;
    for (int k = 0; k < nch; ++k) {
        __syncwarp();                                // slot k - 1, which chunk k + kCfQ - 1 refills, is read
        if (lane == 0) {
            fence_async_smem();
            issue(k + kCfQ - 1);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bars[warp][k % kCfQ], (uint32_t)(k / kCfQ) & 1u, &abort_flag, err))) {
            k_fail = k;
            break;
        }
        const uint8_t* sl = ring + (uint32_t)(k % kCfQ) * kCfBwdChunk;
#pragma unroll
        for (int r = 0; r < kCfBwdCH; ++r) {
            if (k * kCfBwdCH + r >= nrows) break;
            const uint8_t* grow = sl + r * 2 * kCfW;
            const uint8_t* urow = sl + kU + r * 2 * kCfW;
            float gx[8], gn[4], ux[8], up[4];        // g at t .. t + 7, t + 8 .. t + 11; u at t .. t + 7, t - 4 .. t - 1
            lds8(grow + 16 * lane, gx);
            lds4(lane < 31 ? grow + 16 * lane + 16 : sl + kGa + r * 16, gn);
            lds8(urow + 16 * lane, ux);
            lds4(lane > 0 ? urow + 16 * lane - 8 : sl + kUh + r * 16 + 8, up);
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                acc[i] = gx[i];
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    acc[i] = fmaf(dm[i][j], i + j < 8 ? gx[i + j] : gn[i + j - 8], acc[i]);
                    dacc[i][j] = fmaf(gx[i], i - j >= 0 ? ux[i - j] : up[4 + i - j], dacc[i][j]);
                }
            }
            if (live) {
                const int64_t c = c_begin + k * kCfBwdCH + r;
                *reinterpret_cast<uint4*>(du + (b * C + c) * T + t) = pack8(acc);
            }
        }
    }
    if (k_fail >= 0 && lane == 0)                    // let the copies already issued land
        for (int k = k_fail; k < min(nch, k_fail + kCfQ); ++k)
            mbar_wait_drain(&bars[warp][k % kCfQ], (uint32_t)(k / kCfQ) & 1u);
    // the warps' dwh partials, summed over the warps in order (the rings are free now)
    __syncthreads();
    float* red = reinterpret_cast<float*>(hw_smem);  // [nw][kCfW][K]
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j) red[((size_t)warp * kCfW + 8 * lane + i) * K + j] = dacc[i][j];
    __syncthreads();
    for (int e = threadIdx.x; e < kCfW * K; e += blockDim.x) {
        const int tk = e / K, j = e - tk * K;
        const int64_t tt = t0 + tk;
        if (tt >= T) continue;
        float sum = 0.f;
        for (int w = 0; w < nw; ++w) sum += red[((size_t)w * kCfW + tk) * K + j];
        const int64_t n = b * T + tt;
        const int64_t ps = n - seg_start(n, cu, n_docs, T);
        dwh[n * R + q * K + j] = __float2bfloat16_rn(j <= ps ? sum : 0.f);
    }
}

// gr[n, c] = (R^T g)[n, c] for the rotated channels c < rope_n and g[n, c] for rope_n <= c < gr_w
// (bf16, token-major, rows gr_w wide: whole 256-channel blocks), blocks striding over tokens.
__global__ void __launch_bounds__(128) rope_rows_kernel(const __nv_bfloat16* __restrict__ g, int64_t C,
                                                        __nv_bfloat16* __restrict__ gr, int gr_w, int64_t N,
                                                        int rope_n, int rope_hd, int rope_max,
                                                        const float* __restrict__ cs, const int32_t* __restrict__ cu,
                                                        int64_t n_docs, int64_t seqlen) {
    pdl_trigger();
    pdl_wait();
    rope_rows_bf16(g, C, gr, gr_w, N, (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5),
                   (int64_t)gridDim.x * (blockDim.x / 32), rope_n, rope_hd, rope_max, cs, cu, n_docs, seqlen, true);
}

inline size_t al256(size_t x) { return (x + 255) / 256 * 256; }

// Width of the R^T g rows the token-major backward reads: the rotated channels rounded up to
// whole 256-channel blocks (the channels past rope_n copied), so a block reads g from one tensor.
inline int64_t hw_gr_width(const Prob& p) { return std::min<int64_t>(p.C, (p.rope_n + 255) / 256 * 256); }

// Columns of a block's taps box in wh [N, R]: the K taps of each of its heads, from the first
// one rounded down to a multiple of 8 columns (TMA copies start on 16-byte boundaries).
inline int hw_taps_box(const Prob& p) {
    const int heads = (int)std::max<int64_t>(1, 256 / p.hd);
    return ((int)p.K * heads + 7 + 7) / 8 * 8;
}

// Rows of the RoPE table as an int (at least 1; positions are clamped below it).
inline int rope_rows(const Prob& p) { return (int)std::max<int64_t>(1, std::min<int64_t>(p.rope_max, INT32_MAX)); }

}  // namespace


TcHwLayout tc_hw_layout(const Prob& p) {
    TcHwLayout L{};
    size_t off = 0;
    L.wh = off;     off = al256(off + (size_t)p.N * p.R * 2);
    L.dwh = off;    off = al256(off + (size_t)p.N * p.R * 2);
    L.dpart = off;  off = al256(off + (size_t)gen_bwd_splits(p.N, p.d, (int)p.R) * p.d * p.R * 4);
    L.gr = off;     off = al256(off + (size_t)p.N * (p.rope_n > 0 ? hw_gr_width(p) : 0) * 2);  // RoPE: R^T g
    L.total = off;
    return L;
}

bool tc_headwise_supported(const Prob& p) {
    if (p.dtype != 1 || p.kind != 1) return false;
    if (p.R > 128 || p.R % 8 != 0 || p.d % 8 != 0) return false;
    if (p.K < 1 || p.K > 4) return false;
    if (p.layout == 1) return cf_tiles_ok(p) && p.hd <= 8 * kCfCPW && p.batch * ((p.seqlen + kCfW - 1) / kCfW) * p.H *
                                                                 ((p.hd + kCfCPW - 1) / kCfCPW) < (int64_t(1) << 31);
    if (p.hd < 8 || p.hd > 256 || (p.hd & (p.hd - 1)) != 0) return false;
    if (p.rope_n > 0 && p.rope_hd > kHwMaxRopeHd) return false;   // one table row per slot
    // one block per (run, 256-channel block), 32-bit token indices
    return p.C % 256 == 0 && p.N < (int64_t(1) << 31) - 2 * std::max(kHwRunFwd, kHwRunBwd) &&
           (p.N / std::min(kHwRunFwd, kHwRunBwd) + 1) * (p.C / 256) < (int64_t(1) << 31);
}


template <int K>
static cudaError_t launch_hw_fwd(const Prob& p, const void* u, const void* wh, void* y, uint32_t* err,
                                 cudaStream_t st) {
    cudaError_t e;
    if (p.layout == 1) {
        const int64_t tps = (p.seqlen + kCfW - 1) / kCfW;
        const int parts = (int)((p.hd + kCfCPW - 1) / kCfCPW);
        const int smem = kCfQ * kCfFwdChunk;
        e = cudaFuncSetAttribute(hw_conv_fwd_cf_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        CUtensorMap tu, tuh;
        if (!make_tmap_2d(&tu, u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.seqlen, p.batch * p.C, p.us * 2, kCfW, kCfFwdCH, false) ||
            !make_tmap_2d(&tuh, u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.seqlen, p.batch * p.C, p.us * 2, 8, kCfFwdCH, false))
            return cudaErrorInvalidValue;
        const dim3 grid((unsigned)(p.batch * tps * p.H * parts));
        DC_LAUNCH(kTcHeadwiseFwd, st, e = launch_pdl(hw_conv_fwd_cf_kernel<K>, grid, dim3(32), smem, st, tu, tuh,
            static_cast<const __nv_bfloat16*>(wh), (int)p.R, (int)p.hd, p.C, p.seqlen, tps, parts, (int)p.H, p.cu,
            p.n_docs, static_cast<__nv_bfloat16*>(y), err));
        return e;
    }
    const int n_cblk = (int)(p.C / 256);
    const dim3 grid((unsigned)(n_cblk * ((p.N + kHwRunFwd - 1) / kHwRunFwd)));
    const bool rope = p.rope_n > 0;
    const int box = hw_taps_box(p);
    constexpr uint32_t T = HwTile<K>::T, Q = HwTile<K>::Q;
    const uint32_t roff = al128(T * 512u) + al128(T * (uint32_t)box * 2u);
    const int smem = (int)(Q * al128(roff + (rope ? T * (uint32_t)p.rope_hd * 4u : 0u)));
    e = cudaFuncSetAttribute(hw_conv_fwd_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    CUtensorMap tu, tw;
    if (!make_tmap_2d(&tu, u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.C, p.N, p.us * 2, 256, T, false) ||
        !make_tmap_2d(&tw, wh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.R, p.N, p.R * 2, box, T, false))
        return cudaErrorInvalidValue;
    DC_LAUNCH(kTcHeadwiseFwd, st, e = launch_pdl(hw_conv_fwd_kernel<K>, grid, dim3(32), smem, st, tu, tw, (int)p.hd,
        (int32_t)p.N, p.C, (int32_t)p.seqlen, p.cu, (int32_t)p.n_docs, n_cblk, static_cast<__nv_bfloat16*>(y),
        rope ? p.rope_cs : nullptr,
        (int)p.rope_n, rope ? (int)p.rope_hd : 8, rope_rows(p), kHwRunFwd, box, err));
    return e;
}

template <int K>
static cudaError_t launch_hw_bwd(const Prob& p, const void* g, const void* u, const void* wh, void* du, void* dwh,
                                 const void* gr, uint32_t* err, cudaStream_t st) {
    cudaError_t e;
    if (p.layout == 1) {
        const int64_t tps = (p.seqlen + kCfW - 1) / kCfW;
        const int nw = (int)((p.hd + kCfCPW - 1) / kCfCPW);
        const int smem = nw * kCfQ * kCfBwdChunk;
        e = cudaFuncSetAttribute(hw_conv_bwd_cf_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        const uint64_t rows = p.batch * p.C;
        CUtensorMap tg, tga, tu, tuh;
        if (!make_tmap_2d(&tg, g, BF, p.seqlen, rows, p.seqlen * 2, kCfW, kCfBwdCH, false) ||
            !make_tmap_2d(&tga, g, BF, p.seqlen, rows, p.seqlen * 2, 8, kCfBwdCH, false) ||
            !make_tmap_2d(&tu, u, BF, p.seqlen, rows, p.us * 2, kCfW, kCfBwdCH, false) ||
            !make_tmap_2d(&tuh, u, BF, p.seqlen, rows, p.us * 2, 8, kCfBwdCH, false))
            return cudaErrorInvalidValue;
        const dim3 grid((unsigned)(p.batch * tps * p.H));
        DC_LAUNCH(kTcHeadwiseBwd, st, e = launch_pdl(hw_conv_bwd_cf_kernel<K>, grid, dim3(32 * nw), smem, st, tg, tga,
            tu, tuh, static_cast<const __nv_bfloat16*>(wh), (int)p.R, (int)p.hd, p.N, p.C, p.seqlen, tps, (int)p.H,
            p.cu, p.n_docs, static_cast<__nv_bfloat16*>(du), static_cast<__nv_bfloat16*>(dwh), err));
        return e;
    }
    const int n_cblk = (int)(p.C / 256);
    const dim3 grid((unsigned)(n_cblk * ((p.N + kHwRunBwd - 1) / kHwRunBwd)));
    const int box = hw_taps_box(p);
    constexpr uint32_t T = HwTile<K>::T, Q = HwTile<K>::Q;
    const int smem = (int)(Q * al128(T * 1024u + T * (uint32_t)box * 2u));
    e = cudaFuncSetAttribute(hw_conv_bwd_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    CUtensorMap tg, tgr, tu, tw;
    if (!make_tmap_2d(&tg, g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.C, p.N, p.C * 2, 256, T, false) ||
        !make_tmap_2d(&tu, u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.C, p.N, p.us * 2, 256, T, false) ||
        !make_tmap_2d(&tw, wh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.R, p.N, p.R * 2, box, T, false))
        return cudaErrorInvalidValue;
    tgr = tg;
    if (gr) {
        const int64_t w = hw_gr_width(p);
        if (!make_tmap_2d(&tgr, gr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, p.N, w * 2, 256, T, false))
            return cudaErrorInvalidValue;
    }
    DC_LAUNCH(kTcHeadwiseBwd, st, e = launch_pdl(hw_conv_bwd_kernel<K>, grid, dim3(32), smem, st, tg, tgr, tu, tw,
        (int)p.R, (int)p.hd, (int32_t)p.N, p.C, (int32_t)p.seqlen, p.cu, (int32_t)p.n_docs, n_cblk,
        static_cast<__nv_bfloat16*>(du),
        static_cast<__nv_bfloat16*>(dwh), gr ? (int)p.rope_n : 0, kHwRunBwd, box, err));
    return e;
}

cudaError_t tc_headwise_forward(const Prob& p, const void* u, const void* h, const void* W, void* y, void* z_save,
                                char* tcws, uint32_t* err, cudaStream_t st) {
    const TcHwLayout L = tc_hw_layout(p);
    void* wh = z_save ? z_save : static_cast<void*>(tcws + L.wh);
    cudaError_t e = tc_gen_launch(h, p.hs, W, p.N, p.d, (int)p.R, wh, p.R, err, st);
    if (e != cudaSuccess) return e;
    switch (p.K) {
        case 1: return launch_hw_fwd<1>(p, u, wh, y, err, st);
        case 2: return launch_hw_fwd<2>(p, u, wh, y, err, st);
        case 3: return launch_hw_fwd<3>(p, u, wh, y, err, st);
        default: return launch_hw_fwd<4>(p, u, wh, y, err, st);
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
                                              static_cast<__nv_bfloat16*>(gr), (int)hw_gr_width(p), p.N,
                                              (int)p.rope_n, (int)p.rope_hd,
                                              rope_rows(p), p.rope_cs, p.cu, p.n_docs, p.seqlen));
        if (e != cudaSuccess) return e;
    }
    switch (p.K) {
        case 1: e = launch_hw_bwd<1>(p, g, u, wh, du, dwh, gr, err, st); break;
        case 2: e = launch_hw_bwd<2>(p, g, u, wh, du, dwh, gr, err, st); break;
        case 3: e = launch_hw_bwd<3>(p, g, u, wh, du, dwh, gr, err, st); break;
        default: e = launch_hw_bwd<4>(p, g, u, wh, du, dwh, gr, err, st); break;
    }
    if (e != cudaSuccess) return e;
    return tc_gen_backward(dwh, (int)p.R, h, p.hs, W, p.N, p.d, dh, dW, reinterpret_cast<float*>(tcws + L.dpart),
                           err, st);
}

}  // namespace dynconv
