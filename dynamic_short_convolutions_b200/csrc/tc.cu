// tc.cu -- tensor-core (tcgen05 + TMA) kernels for bf16 dynamic short convolutions.
//
// Forward, low-rank ("Dynamic Short Convolutions Improve Transformers",
// gist.science technical summary: "Parameterization" 1 and the "Fused Low-Rank
// Kernel" paragraph of "Efficient Training Implementation"):
//   gen_kernel         z = h A                        (M = 128 tokens, N = r, K = d)
//                      (the same launch writes Bp, the tap-major copy of B)
//   lowrank_fwd_kernel per (128-token tile, 64-channel chunk):
//                      W = z Bp_chunk -> TMEM        (M = 128, N = 64 K, K = r)
//                      y = u + sum_j W[:, 64 j + c] u[t - j, c]  (epilogue, CUDA cores)
//                      the [N, C, K] filter lives only in TMEM and registers.
//
// Every kernel here is warp-specialised: warp 0 issues TMA loads, warp 1 issues
// tcgen05.mma (one thread; in gen_kernel the whole warp runs the issue loop and an elected lane
// issues) and owns the tensor memory, the remaining warps
// are the epilogue (thread = token row = TMEM lane).  Shared-memory stages and TMEM
// accumulators are handed over with mbarriers; every wait is bounded.
#include <algorithm>
#include <cstdio>

#include "common.cuh"
#include "internal.h"
#include "prof.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace dynconv {
namespace {

using namespace tc;

constexpr int kEpiWarps = 8;                       // two warps per TMEM lane quarter
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kTcThreads = 64 + kEpiThreads;       // warp 0 TMA, warp 1 MMA, warps 2.. epilogue

// =====================================================================================
// gen_kernel: X[N, R] = h[N, d] . P[d, R]   (z = h A; bf16 out), R <= 256.
//   A operand: h tile [128 tokens][64 of d], K-major (TMA box {64, 128}).
//   B operand: P tile [64 rows of d][64 of R] per 64-wide atom, MN-major (box {64, 64}).
//   A ring of up to kGenMaxStages shared stages keeps most of a tile's d-loop in flight.
// =====================================================================================
constexpr int kGenMaxStages = 8;
constexpr uint32_t kGenSmemBudget = 196608;

struct GenArgs {
    int64_t N, d;
    int R, NB, NMMA;   // output width, P atoms per stage, MMA N
    int stages;
    int64_t out_ld;
    uint32_t* err;
    const __nv_bfloat16* pB;   // optional side job: Bp[k, j C + c] = B[k, c K + j]
    __nv_bfloat16* pBp;
    int pr, pC, pK;
};

template <typename OutT>
__global__ void __launch_bounds__(kTcThreads, 1) gen_kernel(const __grid_constant__ CUtensorMap tm_h,
                                                            const __grid_constant__ CUtensorMap tm_p,
                                                            OutT* __restrict__ out, GenArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    const uint32_t stage_bytes = 16384u + a.NB * 8192u;
    const int S = a.stages;
    __shared__ uint64_t full[kGenMaxStages], empty[kGenMaxStages], tfull[2], tempty[2];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_tiles = (a.N + 127) / 128;
    const int nk = (int)((a.d + 63) / 64);
    const uint32_t tcols = tmem_cols_for(2 * a.NMMA);
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
        }
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch(&tm_h);
        tma_prefetch(&tm_p);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base;
    pdl_trigger();
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
            uint32_t it = 0;
            for (int64_t tile = blockIdx.x; tile < n_tiles && !abort_flag; tile += gridDim.x) {
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1;
                    if (!mbar_wait(&empty[s], ph ^ 1, &abort_flag, a.err)) break;
                    uint8_t* st = sm + s * stage_bytes;
                    mbar_arrive_expect_tx(&full[s], stage_bytes);
                    tma_load_2d_hint(st, &tm_h, &full[s], 64 * kb, (int32_t)(tile * 128), stream);
                    for (int b = 0; b < a.NB; ++b)
                        tma_load_2d_hint(st + 16384 + b * 8192, &tm_p, &full[s], 64 * b, 64 * kb, keep);
                }
            }
        }
    } else if (warp == 1) {
        // the whole warp runs the loop (warp-uniform descriptor arithmetic); one elected lane issues
        const uint32_t idesc = idesc_bf16(128, a.NMMA, false, true);
        uint32_t it = 0, t = 0;
        for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++t) {
            if (__any_sync(0xffffffffu, abort_flag != 0)) break;      // the lanes leave together
            const int b = t & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&tempty[b], ((t >> 1) & 1) ^ 1, &abort_flag, a.err))) break;
            tc_fence_after();
            const uint32_t dcol = tbase + b * a.NMMA;
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, &abort_flag, a.err))) { ok = false; break; }
                tc_fence_after();
                const uint32_t st = smem_u32(sm + s * stage_bytes);
                uint64_t da[4], db[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    da[k] = kmajor_desc(st, k);
                    db[k] = mnmajor_desc(st + 16384, 8192, 16 * k);
                }
                if (elect_one()) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) umma_bf16(dcol, da[k], db[k], idesc, (kb | k) != 0);
                    umma_commit(&empty[s]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (elect_one()) umma_commit(&tfull[b]);
            __syncwarp();
        }
    } else {
        if (a.pB) {                              // the side job, before the first accumulator is ready
            // (k, c) pairs in grid-stride order, consecutive threads on consecutive channels: a warp
            // reads 32 K-element groups of one row of B (contiguous) and writes K runs of 32 channels
            const int C = a.pC, Kt = a.pK;
            const int64_t total = (int64_t)a.pr * C, nthr = (int64_t)gridDim.x * kEpiThreads;
            const int64_t e0 = (int64_t)blockIdx.x * kEpiThreads + (threadIdx.x - 64);
            const int dk = (int)(nthr / C), dc = (int)(nthr - (int64_t)dk * C);
            int k = (int)(e0 / C), c = (int)(e0 - (int64_t)k * C);
            for (int64_t e = e0; e < total; e += nthr) {
                const __nv_bfloat16* src = a.pB + ((int64_t)k * C + c) * Kt;
                __nv_bfloat16* dst = a.pBp + (int64_t)k * Kt * C + c;
                for (int j = 0; j < Kt; ++j) dst[(int64_t)j * C] = src[j];
                c += dc;
                k += dk;
                if (c >= C) {
                    c -= C;
                    ++k;
                }
            }
        }
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int half = (warp - 2) >> 2;        // which columns of the row this warp converts
        const int row = q * 32 + lane;
        uint32_t t = 0;
        for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++t) {
            const int b = t & 1;
            if (!mbar_wait(&tfull[b], (t >> 1) & 1, &abort_flag, a.err)) break;
            tc_fence_after();
            const int64_t n = tile * 128 + row;
            const uint32_t taddr = tbase + (uint32_t(q * 32) << 16) + b * a.NMMA;
            for (int c = 8 * half; c < a.R; c += 16) {
                uint32_t v[8];
                tmem_ld8(taddr + c, v);
                tmem_wait_ld();
                if (n < a.N) {
                    if constexpr (sizeof(OutT) == 2) {
                        uint4 pk;
                        pk.x = pack_bf16(__uint_as_float(v[0]), __uint_as_float(v[1]));
                        pk.y = pack_bf16(__uint_as_float(v[2]), __uint_as_float(v[3]));
                        pk.z = pack_bf16(__uint_as_float(v[4]), __uint_as_float(v[5]));
                        pk.w = pack_bf16(__uint_as_float(v[6]), __uint_as_float(v[7]));
                        *reinterpret_cast<uint4*>(out + n * a.out_ld + c) = pk;
                    } else {
                        float4* o = reinterpret_cast<float4*>(out + n * a.out_ld + c);
                        o[0] = make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]),
                                           __uint_as_float(v[3]));
                        o[1] = make_float4(__uint_as_float(v[4]), __uint_as_float(v[5]), __uint_as_float(v[6]),
                                           __uint_as_float(v[7]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, tcols);
    }
}

// =====================================================================================
// lowrank_fwd_kernel<K>: work items (128-token tile m0, 64-channel chunk c0) in contiguous
// chunk-major runs, one run per CTA, so the chunk's B stays in shared memory.
//   rings:      u tiles [136 rows = m0-8 .. m0+127][64 channels] (kFwdU slots) and z tiles
//               [128][64] (K-major A, kFwdZ slots)
//   resident:   the chunk's slice of the tap-major Bp (Bp[k, j C + c] = B[k, c K + j], written by
//               the generator launch) as K atoms [64 r-rows][64] (MN-major B), reloaded when the
//               chunk changes
//   TMEM: W[128 tokens][64 K] fp32, column 64 j + c = w[m0 + row, c0 + c, j]; two buffers.
//   warps: 0 TMA loads, 1 MMA, 2 TMA stores, 3.. epilogue (FwdEpi<K>::warps in two teams taking
//   alternate items; each warp a TMEM lane quarter and a share of the channels):
//   y[t, c] = u[t, c] + sum_{j <= t - s(t)} W[t, 64 j + c] u[t - j, c]
//   -> bf16 staging (128-byte swizzled) -> TMA store by warp 2.
// CF (channel-first u and y, [batch * C, seqlen]): the u tile is a [64 channels][136 tokens]
// box (272-byte rows, no swizzle), y is staged [64 channels][128 tokens]; token tiles stay
// inside one sequence (tps tiles per sequence), the z tile starts at the tile's first token.
// =====================================================================================
struct FwdArgs {
    int64_t N, C, seqlen, n_docs;
    const int32_t* cu;
    uint32_t* err;
    int64_t per_cta;         // work items per CTA (contiguous run)
    int ksteps;              // 16-wide K steps of the filter MMA: r / 16 rounded up
    int64_t n_tiles, tps;    // token tiles; tiles per sequence (channel-first)
    const float* rope_cs;    // RoPE table [rope_max][rope_hd] (cos, sin pairs) or nullptr
    int rope_n, rope_hd;     // rotated channels [0, rope_n), channels per rotary head
    int rope_max;            // table rows (positions are clamped below it)
};

// u tiles (DRAM, the epilogue's operand) and z tiles (L2-resident, the MMA's operand) have rings of
// their own: the u ring is the deeper one (the loads in flight per SM set the forward's throughput;
// one shared ring of 4 stages left each u load ~3 us of queueing), and the producer issues each z
// load kFwdZLag items after the u load of the same item.
constexpr int kFwdU = 6, kFwdZ = 3, kFwdZLag = 2;
constexpr uint32_t kZBytes = 16384, kUBytes = 136 * 128, kYBytes = 16384;
constexpr uint32_t kCfUPitch = 136 * 2, kCfYPitch = 128 * 2;   // channel-first tile rows (bytes)
// Epilogue of lowrank_fwd_kernel<K>: 16 warps in two teams of 8 that take alternate items
// (ping-pong: one team's arithmetic overlaps the other's TMEM and shared-memory loads; measured
// 46 -> 42 us at the 150M QKV layer, 343 -> 279 us at the packed workload, against all 16 warps on
// every item); in a team, two warps per TMEM lane quarter, four 8-channel groups each; K = 4
// takes one group per TMEM wait to stay within the registers of 16 warps.
template <int K>
struct FwdEpi {
    static constexpr int warps = 16;
    static constexpr int teams = 2;
    static constexpr int team_warps = warps / teams;
    static constexpr int groups = 8 / (team_warps / 4);   // 8-channel groups per warp and item
    static constexpr int per_pass = K <= 3 ? 2 : 1;       // groups per TMEM wait
    static constexpr int threads = 96 + 32 * warps;       // producer, MMA, store warps + epilogue
};

template <int K>
struct FwdSmem {
    static constexpr uint32_t u0 = 0;
    static constexpr uint32_t z0 = u0 + kFwdU * kUBytes;
    static constexpr uint32_t bres = z0 + kFwdZ * kZBytes;
    static constexpr uint32_t ys = bres + K * 8192;
    static constexpr uint32_t total = ys + 2 * kYBytes + 1024;
    static_assert(z0 % 1024 == 0 && bres % 1024 == 0, "swizzled tiles start on 1024-byte boundaries");
};

// y for 8 channels of one row: wv[j][c] = W_j[t, 8 g + c] (fp32 bits), uj[j] = u[t - j, 8 g .. 8 g + 7].
// Channel pairs go through the packed fp32 FMA (conv8f: the fp32 values, before the bf16 rounding).
template <int K>
__device__ __forceinline__ void conv8f(const uint32_t (*wv)[8], const uint4* uj, int32_t pos, float (&acc)[8]) {
    const uint32_t* u0 = reinterpret_cast<const uint32_t*>(&uj[0]);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        acc[2 * p] = bf16_lo(u0[p]);
        acc[2 * p + 1] = bf16_hi(u0[p]);
    }
#pragma unroll
    for (int j = 0; j < K; ++j) {
        if (j <= pos) {
            const uint32_t* uu = reinterpret_cast<const uint32_t*>(&uj[j]);
#pragma unroll
            for (int p = 0; p < 4; ++p)
                ffma2(acc[2 * p], acc[2 * p + 1], __uint_as_float(wv[j][2 * p]), __uint_as_float(wv[j][2 * p + 1]),
                      bf16_lo(uu[p]), bf16_hi(uu[p]));
        }
    }
}
__device__ __forceinline__ uint4 pack8f(const float (&acc)[8]) {
    return make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]), pack_bf16(acc[4], acc[5]),
                      pack_bf16(acc[6], acc[7]));
}

template <int K>
__device__ __forceinline__ uint4 conv8(const uint32_t (*wv)[8], const uint4* uj, int32_t pos) {
    float acc[8];
    const uint32_t* u0 = reinterpret_cast<const uint32_t*>(&uj[0]);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        acc[2 * p] = bf16_lo(u0[p]);
        acc[2 * p + 1] = bf16_hi(u0[p]);
    }
#pragma unroll
    for (int j = 0; j < K; ++j) {
        if (j <= pos) {
            const uint32_t* uu = reinterpret_cast<const uint32_t*>(&uj[j]);
#pragma unroll
            for (int p = 0; p < 4; ++p)
                ffma2(acc[2 * p], acc[2 * p + 1], __uint_as_float(wv[j][2 * p]), __uint_as_float(wv[j][2 * p + 1]),
                      bf16_lo(uu[p]), bf16_hi(uu[p]));
        }
    }
    uint4 pk;
    pk.x = pack_bf16(acc[0], acc[1]);
    pk.y = pack_bf16(acc[2], acc[3]);
    pk.z = pack_bf16(acc[4], acc[5]);
    pk.w = pack_bf16(acc[6], acc[7]);
    return pk;
}

template <int K, bool CF, bool ROPE>
__global__ void __launch_bounds__(FwdEpi<K>::threads, 1) lowrank_fwd_kernel(const __grid_constant__ CUtensorMap tm_z,
                                                                     const __grid_constant__ CUtensorMap tm_b,
                                                                     const __grid_constant__ CUtensorMap tm_u,
                                                                     const __grid_constant__ CUtensorMap tm_y,
                                                                     FwdArgs a) {
    using S = FwdSmem<K>;
    constexpr int NMMA = 64 * K;
    constexpr int kFwdGroups = FwdEpi<K>::groups;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    __shared__ uint64_t ufull[kFwdU], uempty[kFwdU], zfull[kFwdZ], zempty[kFwdZ], bfull, bempty, tfull[2], tempty[2],
        yfull[2], yempty[2];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_tiles = a.n_tiles, n_items = n_tiles * (a.C / 64);
    const int64_t i0 = (int64_t)blockIdx.x * a.per_cta, i1 = min(i0 + a.per_cta, n_items);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kFwdU; ++s) {
            mbar_init(&ufull[s], 1);
            mbar_init(&uempty[s], FwdEpi<K>::team_warps);   // the team of the item read u
        }
        for (int s = 0; s < kFwdZ; ++s) {
            mbar_init(&zfull[s], 1);
            mbar_init(&zempty[s], 1);                        // the MMA read z
        }
        mbar_init(&bfull, 1);
        mbar_init(&bempty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], FwdEpi<K>::team_warps);
            mbar_init(&yfull[b], FwdEpi<K>::team_warps);
            mbar_init(&yempty[b], 1);
        }
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch(&tm_z);
        tma_prefetch(&tm_b);
        tma_prefetch(&tm_u);
        tma_prefetch(&tm_y);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base;
    pdl_trigger();
    pdl_wait();

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
            int64_t prev = -1;
            uint32_t cc = 0;
            const uint32_t nit = i1 > i0 ? (uint32_t)(i1 - i0) : 0u;
            ItemPos upos(i0, n_tiles), zpos(i0, n_tiles);
            // step k: the u tile of item k, then the z tile (and at a chunk start the Bp slice) of item
            // k - kFwdZLag
            for (uint32_t k = 0; k < nit + kFwdZLag && !abort_flag; ++k) {
                if (k < nit) {
                    const int s = k % kFwdU;
                    if (!mbar_wait(&uempty[s], ((k / kFwdU) & 1) ^ 1, &abort_flag, a.err)) break;
                    const TileAt ta = tile_at<CF>(upos.tile, (int32_t)(upos.chunk * 64), a.tps, a.seqlen, a.C);
                    uint8_t* ut = sm + S::u0 + s * kUBytes;
                    mbar_arrive_expect_tx(&ufull[s], kUBytes);
                    if (CF) tma_load_2d_hint(ut, &tm_u, &ufull[s], ta.x - 8, ta.y, stream);
                    else tma_load_2d_hint(ut, &tm_u, &ufull[s], ta.x, ta.y - 8, stream);
                    upos.next();
                }
                if (k >= (uint32_t)kFwdZLag) {
                    const uint32_t it = k - kFwdZLag;
                    const int64_t chunk = zpos.chunk;
                    const int32_t c0 = (int32_t)(chunk * 64);
                    if (chunk != prev) {
                        if (!mbar_wait(&bempty, (cc & 1) ^ 1, &abort_flag, a.err)) break;
                        mbar_arrive_expect_tx(&bfull, K * 8192);
                        for (int j = 0; j < K; ++j)
                            tma_load_2d_hint(sm + S::bres + j * 8192, &tm_b, &bfull, (int32_t)(j * a.C) + c0, 0,
                                             keep);
                        ++cc;
                        prev = chunk;
                    }
                    const int s = it % kFwdZ;
                    if (!mbar_wait(&zempty[s], ((it / kFwdZ) & 1) ^ 1, &abort_flag, a.err)) break;
                    const TileAt ta = tile_at<CF>(zpos.tile, c0, a.tps, a.seqlen, a.C);
                    mbar_arrive_expect_tx(&zfull[s], kZBytes);
                    tma_load_2d_hint(sm + S::z0 + s * kZBytes, &tm_z, &zfull[s], 0, ta.m0, keep);
                    zpos.next();
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, NMMA, false, true);
            const uint32_t b0 = smem_u32(sm + S::bres);
            int64_t prev = -1;
            uint32_t cc = 0, it = 0;
            ItemPos ipos(i0, n_tiles);
            for (int64_t item = i0; item < i1 && !abort_flag; ++item, ++it, ipos.next()) {
                const int64_t chunk = ipos.chunk;
                const bool last = (item + 1 == i1) || ipos.last_of_chunk();
                if (chunk != prev) {
                    if (!mbar_wait(&bfull, cc & 1, &abort_flag, a.err)) break;
                    ++cc;
                    prev = chunk;
                }
                const int s = it % kFwdZ, b = it & 1;
                if (!mbar_wait(&tempty[b], ((it >> 1) & 1) ^ 1, &abort_flag, a.err)) break;
                if (!mbar_wait(&zfull[s], (it / kFwdZ) & 1, &abort_flag, a.err)) break;
                tc_fence_after();
                const uint32_t st = smem_u32(sm + S::z0 + s * kZBytes);
#pragma unroll
                for (int k = 0; k < 4; ++k)      // ksteps = r / 16 rounded up, at most 4
                    if (k < a.ksteps)
                        umma_bf16(tbase + b * 256, kmajor_desc(st, k), mnmajor_desc(b0, 8192, 16 * k), idesc, k != 0);
                umma_commit(&tfull[b]);
                umma_commit(&zempty[s]);
                if (last) umma_commit(&bempty);
            }
        }
    } else if (warp == 2) {
        if (lane == 0) {
            uint32_t it = 0;
            ItemPos ipos(i0, n_tiles);
            for (int64_t item = i0; item < i1; ++item, ++it, ipos.next()) {
                const int64_t chunk = ipos.chunk, tile = ipos.tile;
                const int b = it & 1;
                if (!mbar_wait(&yfull[b], (it >> 1) & 1, &abort_flag, a.err)) break;
                const TileAt ta = tile_at<CF>(tile, (int32_t)(chunk * 64), a.tps, a.seqlen, a.C);
                tma_store_2d_hint(&tm_y, sm + S::ys + b * kYBytes, ta.x, ta.y, l2_evict_first());
                tma_store_commit();
                asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                mbar_arrive(&yempty[b]);
            }
            tma_store_wait_all();
        }
    } else {
        // team t takes items t, t + 2, ... of the run, so it always uses TMEM buffer and y buffer t
        const int q = warp & 3;
        const int team = (warp - 3) / FwdEpi<K>::team_warps;
        const int half = ((warp - 3) % FwdEpi<K>::team_warps) >> 2;   // channel groups kFwdGroups*half ..
        const int row = q * 32 + lane;
        static_assert(FwdEpi<K>::teams == 2, "each team steps its item position twice per item");
        uint32_t it = team;
        ItemPos ipos(i0 + team, n_tiles);
        for (int64_t item = i0 + team; item < i1;
             item += FwdEpi<K>::teams, it += FwdEpi<K>::teams, ipos.next(), ipos.next()) {
            const int64_t tile = ipos.tile;
            const int s = it % kFwdU, b = it & 1;
            const int32_t n = tile_at<CF>(tile, 0, a.tps, a.seqlen, a.C).m0 + row;
            const int32_t pos = n < a.N ? n - seg_start32(n, a.cu, (int32_t)a.n_docs, (int32_t)a.seqlen) : 0;
            // RoPE: this row's table entries for the thread's channel groups (32 bytes each, at the
            // group's offset within its rotary head), fetched before the waits below so that their
            // latency overlaps them; a chunk lies wholly inside or outside the rotated channels
            constexpr int kRopeG = ROPE ? kFwdGroups : 1;
            float4 rcs[kRopeG][2];
            bool rot = false;
            if constexpr (ROPE) {
                const int c0 = (int)ipos.chunk * 64 + 8 * kFwdGroups * half;   // the thread's first channel
                rot = c0 < a.rope_n;
                if (rot) {
                    const float* crow = a.rope_cs + (int64_t)min(pos, a.rope_max - 1) * a.rope_hd;
#pragma unroll
                    for (int x = 0; x < kRopeG; ++x) {
                        const float4* t4 = reinterpret_cast<const float4*>(crow + (c0 + 8 * x) % a.rope_hd);
                        rcs[x][0] = __ldg(t4);
                        rcs[x][1] = __ldg(t4 + 1);
                    }
                }
            }
            // each warp goes at its own pace (no barrier among the epilogue warps): a failed
            // wait sets the abort flag, and every other wait then gives up too
            const bool ok = mbar_wait(&tfull[b], (it >> 1) & 1, &abort_flag, a.err) &&
                            mbar_wait(&ufull[s], (it / kFwdU) & 1, &abort_flag, a.err) &&
                            mbar_wait(&yempty[b], ((it >> 1) & 1) ^ 1, &abort_flag, a.err);
            if (!ok) break;
            tc_fence_after();
            const uint8_t* us = sm + S::u0 + s * kUBytes;
            uint8_t* ys = sm + S::ys + b * kYBytes;
            const uint32_t taddr = tbase + (uint32_t(q * 32) << 16) + b * 256;
            // NG 8-channel groups per pass: every TMEM and shared-memory load first, then one wait,
            // then the arithmetic (channel-first: one group, its 8 K column loads are enough in flight)
            constexpr int NG = (CF || ROPE) ? 1 : FwdEpi<K>::per_pass;
#pragma unroll
            for (int pass = 0; pass < kFwdGroups / NG; ++pass) {
                const int g0 = kFwdGroups * half + NG * pass;
                uint32_t wv[NG][K][8];
#pragma unroll
                for (int x = 0; x < NG; ++x)
#pragma unroll
                    for (int j = 0; j < K; ++j) tmem_ld8(taddr + 64 * j + 8 * (g0 + x), wv[x][j]);
                uint4 uj[NG][K];
#pragma unroll
                for (int x = 0; x < NG; ++x)
#pragma unroll
                    for (int j = 0; j < K; ++j)
                        uj[x][j] = CF ? cf_gather8(us, kCfUPitch, g0 + x, row + 8 - j)
                                      : *reinterpret_cast<const uint4*>(us + sw128_off(row + 8 - j, g0 + x));
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < NG; ++x) {
                    uint4 yv;
                    if constexpr (ROPE) {
                        float acc[8];
                        conv8f<K>(wv[x], uj[x], pos, acc);
                        if (rot) rope_pairs8v(acc, rcs[NG * pass + x][0], rcs[NG * pass + x][1], false);
                        yv = pack8f(acc);
                    } else {
                        yv = conv8<K>(wv[x], uj[x], pos);
                    }
                    if (CF) cf_scatter8(ys, kCfYPitch, g0 + x, row, yv);
                    else *reinterpret_cast<uint4*>(ys + sw128_off(row, g0 + x)) = yv;
                }
            }
            tc_fence_before();
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&tempty[b]);
                mbar_arrive(&uempty[s]);
                mbar_arrive(&yfull[b]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

template <int K, bool CF, bool ROPE>
cudaError_t launch_lowrank_fwd(const CUtensorMap& tz, const CUtensorMap& tb, const CUtensorMap& tu,
                               const CUtensorMap& ty, FwdArgs fa, int64_t items, cudaStream_t st) {
    constexpr uint32_t smem = FwdSmem<K>::total;
    cudaError_t e =
        cudaFuncSetAttribute(lowrank_fwd_kernel<K, CF, ROPE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    fa.per_cta = (items + num_sms() - 1) / num_sms();
    const unsigned grid = (unsigned)((items + fa.per_cta - 1) / fa.per_cta);
    DC_LAUNCH(kTcLowrankFwd, st, e = launch_pdl(lowrank_fwd_kernel<K, CF, ROPE>, dim3(grid), dim3(FwdEpi<K>::threads),
                                                smem, st, tz, tb, tu, ty, fa));
    return e;
}

template <int K>
cudaError_t launch_lowrank_fwd_l(bool cf, const CUtensorMap& tz, const CUtensorMap& tb, const CUtensorMap& tu,
                                 const CUtensorMap& ty, FwdArgs fa, int64_t items, cudaStream_t st) {
    if (cf) return launch_lowrank_fwd<K, true, false>(tz, tb, tu, ty, fa, items, st);   // RoPE: token-major only
    return fa.rope_cs ? launch_lowrank_fwd<K, false, true>(tz, tb, tu, ty, fa, items, st)
                      : launch_lowrank_fwd<K, false, false>(tz, tb, tu, ty, fa, items, st);
}

}  // namespace

cudaError_t tc_gen_launch(const void* h, int64_t hs, const void* P, int64_t N, int64_t d, int R, void* out,
                          int64_t out_ld, uint32_t* err, cudaStream_t st, BPermute perm) {
    CUtensorMap th, tp;
    if (!make_tmap_bf16(&th, h, d, N, hs, 64, 128) || !make_tmap_bf16(&tp, P, R, d, R, 64, 64))
        return cudaErrorInvalidValue;
    const int NB = (R + 63) / 64;
    const int stage_bytes = 16384 + NB * 8192;
    const int stages = std::max(2, std::min<int>(kGenMaxStages, (int)(kGenSmemBudget / stage_bytes)));
    GenArgs ga{N, d, R, NB, (R + 15) / 16 * 16, stages, out_ld, err, static_cast<const __nv_bfloat16*>(perm.B),
               static_cast<__nv_bfloat16*>(perm.Bp), perm.r, perm.C, perm.K};
    const int smem = 1024 + stages * stage_bytes;
    cudaError_t e = cudaFuncSetAttribute(gen_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int64_t n_tiles = (N + 127) / 128;
    const unsigned grid = (unsigned)std::min<int64_t>(n_tiles, num_sms());
    DC_LAUNCH(kTcGen, st, e = launch_pdl(gen_kernel<__nv_bfloat16>, dim3(grid), dim3(kTcThreads), (size_t)smem, st, th, tp,
                                         static_cast<__nv_bfloat16*>(out), ga));
    return e;
}


bool tc_headwise_supported(const Prob& p);
cudaError_t tc_headwise_forward(const Prob& p, const void* u, const void* h, const void* W, void* y, void* z_save,
                                char* tcws, uint32_t* err, cudaStream_t st);
cudaError_t tc_headwise_backward(const Prob& p, const void* g, const void* u, const void* h, const void* W,
                                 const void* z_saved, void* du, void* dh, float* dW, char* tcws, uint32_t* err,
                                 cudaStream_t st);
cudaError_t tc_lowrank_backward(const Prob& p, const void* g, const void* u, const void* h, const void* A,
                                const void* B, const void* z_saved, void* du, void* dh, float* dA, float* dB,
                                char* tcws, uint32_t* err, cudaStream_t st);

// Why the tensor-core kernels do not take a problem (nullptr: they do).
const char* tc_unsupported_reason(const Prob& p, bool bwd) {
    if (p.dtype != 1) return "fp32 storage runs the CUDA-core kernels (no tensor-core rounding of fp32 inputs)";
    if (tensor_map_encoder() == nullptr) return "the driver entry point cuTensorMapEncodeTiled is unavailable";
    if (p.kind == 1) {
        if (p.rope_n > 0 && (p.layout == 1 || p.rope_hd % 8 != 0 || p.rope_hd > 256))
            return "head-wise RoPE on the tensor cores needs the token-major layout and rope_head_dim % 8 == 0, "
                   "at most 256";
        if (!tc_headwise_supported(p))
            return "head-wise tensor-core kernels need H*K a multiple of 8 up to 128, d a multiple of 8, and "
                   "(token-major) head_dim a power of two in [8, 256] with channels a multiple of 256, or "
                   "(channel-first) seqlen and u_row_stride multiples of 8 and head_dim at most 512";
        return nullptr;
    }
    if (p.r % 8 != 0 || p.r > 64) return "low-rank tensor-core kernels need the rank a multiple of 8 up to 64";
    if (p.C % 64 != 0 || p.d % 8 != 0) return "low-rank tensor-core kernels need channels % 64 == 0 and d % 8 == 0";
    if (p.K < 1 || p.K > 4) return "ksize outside 1..4";
    if (p.N >= (int64_t(1) << 31) || p.r * p.C * p.K >= (int64_t(1) << 31)) return "sizes beyond 32-bit indexing";
    if (p.layout == 1 && !cf_tiles_ok(p))
        return "channel-first tensor-core kernels need seqlen and u_row_stride multiples of 8";
    if (p.rope_n > 0 && p.layout == 1) return "RoPE with the channel-first layout runs the CUDA-core kernels";
    if (p.rope_n > 0 && (p.rope_hd % 8 != 0 || p.rope_n % 64 != 0))
        return "RoPE on the low-rank tensor-core kernels needs rope_head_dim % 8 == 0 and rope_channels % 64 == 0";
    // The low-rank backward adds dz over channel chunks with bulk fp32 reductions (order not
    // fixed), so its deterministic mode runs the CUDA-core kernels; the head-wise backward has
    // no float atomics (warp-shuffle and fixed-order split reductions).
    if (bwd && p.deterministic) return "the deterministic low-rank backward runs the CUDA-core kernels";
    return nullptr;
}

bool tc_supported(const Prob& p) { return tc_unsupported_reason(p, false) == nullptr; }

bool tc_supported_bwd(const Prob& p) { return tc_unsupported_reason(p, true) == nullptr; }

size_t tc_workspace_bytes(const Prob& p) { return p.kind == 1 ? tc_hw_layout(p).total : tc_bwd_layout(p).total; }

cudaError_t tc_forward_scratch(const Prob& p, const void* u, const void* h, const void* A, const void* BW, void* y,
                               void* z, void* bp, uint32_t* err, cudaStream_t st);

cudaError_t tc_forward(const Prob& p, const void* u, const void* h, const void* A, const void* BW, void* y,
                       void* z_save, void* ws, cudaStream_t st) {
    const WsLayout L = ws_layout(p);
    uint32_t* err = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + L.err);
    if (p.kind == 1) return tc_headwise_forward(p, u, h, BW, y, z_save, static_cast<char*>(ws) + L.tc, err, st);
    const TcBwdLayout TL = tc_bwd_layout(p);
    char* tcws = static_cast<char*>(ws) + L.tc;
    void* z = z_save ? z_save : static_cast<void*>(tcws + TL.zs);
    return tc_forward_scratch(p, u, h, A, BW, y, z, tcws + TL.bp, err, st);
}

// Low-rank forward on the tensor cores with caller-chosen scratch: z (bf16 [N, r]), Bp
// (bf16 [r, K C]) and the device error word.
cudaError_t tc_forward_scratch(const Prob& p, const void* u, const void* h, const void* A, const void* BW, void* y,
                               void* z, void* bp, uint32_t* err, cudaStream_t st) {
    cudaError_t e = tc_gen_launch(h, p.hs, A, p.N, p.d, (int)p.r, z, p.r, err, st,
                                  BPermute{BW, bp, (int)p.r, (int)p.C, (int)p.K});
    if (e != cudaSuccess) return e;
    const bool cf = p.layout == 1;
    CUtensorMap tz, tb, tu, ty;
    if (!make_tmap_bf16(&tz, z, p.r, p.N, p.r, 64, 128) || !make_tmap_bf16(&tb, bp, p.C * p.K, p.r, p.C * p.K, 64, 64))
        return cudaErrorInvalidValue;
    if (cf ? !(make_tmap_2d(&tu, u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.seqlen, p.batch * p.C, p.us * 2, 136, 64, false) &&
               make_tmap_2d(&ty, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.seqlen, p.batch * p.C, p.seqlen * 2, 128, 64,
                            false))
           : !(make_tmap_bf16(&tu, u, p.C, p.N, p.us, 64, 136) && make_tmap_bf16(&ty, y, p.C, p.N, p.C, 64, 128)))
        return cudaErrorInvalidValue;
    const int64_t tps = (p.seqlen + 127) / 128;
    const int64_t n_tiles = cf ? p.batch * tps : (p.N + 127) / 128;
    FwdArgs fa{p.N, p.C, p.seqlen, p.n_docs, p.cu, err, 0, (int)((p.r + 15) / 16), n_tiles, tps,
               p.rope_n > 0 ? p.rope_cs : nullptr, (int)p.rope_n, p.rope_n > 0 ? (int)p.rope_hd : 1,
               (int)std::max<int64_t>(1, std::min<int64_t>(p.rope_max, INT32_MAX))};
    const int64_t items = n_tiles * (p.C / 64);
    switch (p.K) {
        case 1: return launch_lowrank_fwd_l<1>(cf, tz, tb, tu, ty, fa, items, st);
        case 2: return launch_lowrank_fwd_l<2>(cf, tz, tb, tu, ty, fa, items, st);
        case 3: return launch_lowrank_fwd_l<3>(cf, tz, tb, tu, ty, fa, items, st);
        default: return launch_lowrank_fwd_l<4>(cf, tz, tb, tu, ty, fa, items, st);
    }
}

cudaError_t tc_backward(const Prob& p, const void* g, const void* u, const void* h, const void* A, const void* BW,
                        const void* z_saved, void* du, void* dh, float* dA, float* dBW, void* ws, cudaStream_t st) {
    const WsLayout L = ws_layout(p);
    uint32_t* err = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + L.err);
    if (p.kind == 1)
        return tc_headwise_backward(p, g, u, h, BW, z_saved, du, dh, dBW, static_cast<char*>(ws) + L.tc, err, st);
    return tc_lowrank_backward(p, g, u, h, A, BW, z_saved, du, dh, dA, dBW, static_cast<char*>(ws) + L.tc, err, st);
}

}  // namespace dynconv
