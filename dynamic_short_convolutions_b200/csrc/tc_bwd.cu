// tc_bwd.cu -- tensor-core (tcgen05 + TMA) backward of the low-rank dynamic short
// convolution, bf16 storage, fp32 accumulation.
//
// The adjoint of y[t,c] = u[t,c] + sum_{j<K, t-j >= s(t)} w[t,c,j] u[t-j,c] with
// w[t,c,j] = sum_k z[t,k] B[k,c K + j] and z = h A ("Dynamic Short Convolutions
// Improve Transformers", gist.science technical summary, "Dynamic Short
// Convolutions": Mechanism, Parameterization 1, Placement), for upstream g = dL/dy:
//   du[t,c]    = g[t,c] + sum_{j<K, t+j < e(t)} w[t+j,c,j] g[t+j,c]
//   dw[t,c,j]  = g[t,c] u[t-j,c]                      (t-j >= s(t), else 0)
//   dz[t,k]    = sum_{c,j} dw[t,c,j] B[k,c K + j]
//   dB[k,cK+j] = sum_t z[t,k] dw[t,c,j]
//   dA = h^T dz,  dh = dz A^T
// where s(t) / e(t) are the first / one-past-last token of t's sequence or document.
//
// Kernels
//   bwd_prep_kernel    zeroes the dz accumulator and writes Bp [r, K C], the tap-major copy of B
//                      (Bp[k, j C + c] = B[k, c K + j]).
//   lowrank_bwd_kernel one CTA per contiguous run of (64-channel chunk, 128-token tile)
//                      work items, chunk-major, so the chunk's Bp stays in shared memory
//                      and dB for the chunk accumulates in TMEM across the run:
//       MMA1  Wd_j[t, c] = sum_k z[t+j, k] Bp[k, j C + c]   (the filter of token t+j:
//             the z tile is loaded with 8 rows of look-ahead and the A operand starts
//             j rows into it), so du needs no exchange between threads; issued by its own
//             warp (the whole warp runs the loop, one elected lane issues);
//       epi A du (-> staged; a warp of its own issues the TMA store) and dw (-> bf16 tile in
//             shared memory, 64 channels per tap; all taps at once for K <= 3, blocks of two
//             taps for K = 4); 16 warps, each paced by mbarriers;
//       MMA2  dz  = dW Bp_chunk^T      (M = 128 tokens, N = r, K = 64 K)
//       MMA3  K <= 3: dB += z^T dW     (M = 128 (r rows used), N = 64 K, K = 128 tokens)
//             K = 4:  dBt += dW^T z    (M = 128 (j, c) rows per block, N = r, K = 128 tokens)
//             MMA2 and MMA3 are issued by a second warp on another scheduler (likewise);
//       epi B dz -> staged fp32 tile (128 or 64 rows at a time), bulk tensor add into a [N, r]
//             buffer (reduction over chunks; fp32 atomics when no tile fits);
//       epi C at the end of the run: dBt -> per-run partial (reduced in order later).
//   bwd_finish_kernel  sums the dB partials of each chunk in run order -> dB [r, C K] fp32, and
//                      converts the fp32 dz to the bf16 operand of the generator backward.
//   gen_bwd_kernel     dh = dz A^T (M = 128 tokens, N = 128 of d, K = r; staged, TMA store) and
//                      dA += h^T dz (M = 128 of d, N = r, K = 128 tokens) per (128-wide d
//                      block, token range); reduce_splits_kernel sums the token ranges.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <type_traits>

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
constexpr int kThreads = 64 + kEpiThreads;         // warp 0 TMA, warp 1 MMA, warps 2.. epilogue
constexpr uint32_t kRowTile = 136 * 128;     // 136-row, 64-column bf16 tile
constexpr uint32_t kAtom128 = 128 * 128;     // 128-row, 64-column bf16 tile

// Backward set-up in one launch.  Blocks [0, r K cb): the tap-major copy Bp[k, j C + c] = B[k, c K + j],
// block (k K + j) cb + x writing channels 8 (256 x + t) .. + 7 of row (k, j) as one 16-byte store;
// the remaining blocks zero the fp32 dz accumulator (float4 stores).
constexpr int kPrepThreads = 256;
// With RoPE, the last nb_rot blocks also write R^T g of the rotated channels (gr [N, rope_n], bf16),
// which the backward kernel reads in place of g for those channels.
struct PrepRope {
    const __nv_bfloat16* g;
    __nv_bfloat16* gr;
    int64_t N, seqlen, n_docs;
    const int32_t* cu;
    const float* cs;
    int rope_n, rope_hd, rope_max, nb_rot;
};
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ B, __nv_bfloat16* __restrict__ Bp, int r, int C,
                                int K, int cb, float4* __restrict__ dz4, int64_t n_dz4, PrepRope rp) {
    pdl_trigger();
    pdl_wait();
    if ((int)blockIdx.x >= (int)gridDim.x - rp.nb_rot) {
        const int b = blockIdx.x - (gridDim.x - rp.nb_rot);
        rope_rows_bf16(rp.g, C, rp.gr, rp.rope_n, rp.N, (int64_t)b * (blockDim.x / 32) + (threadIdx.x >> 5),
                       (int64_t)rp.nb_rot * (blockDim.x / 32), rp.rope_n, rp.rope_hd, rp.rope_max, rp.cs, rp.cu,
                       rp.n_docs, rp.seqlen, true);
        return;
    }
    const int nb_bp = r * K * cb;
    if ((int)blockIdx.x < nb_bp) {
        const int row = blockIdx.x / cb, x = blockIdx.x - row * cb;
        const int k = row / K, j = row - k * K;
        const int c0 = 8 * (kPrepThreads * x + (int)threadIdx.x);
        if (c0 < C) {
            const __nv_bfloat16* src = B + (int64_t)k * C * K + (int64_t)c0 * K + j;
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t lo = *reinterpret_cast<const uint16_t*>(src + (2 * e) * K);
                const uint32_t hi = *reinterpret_cast<const uint16_t*>(src + (2 * e + 1) * K);
                w[e] = lo | (hi << 16);
            }
            *reinterpret_cast<uint4*>(Bp + (int64_t)k * C * K + (int64_t)j * C + c0) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        return;
    }
    const int64_t nthr = (int64_t)(gridDim.x - rp.nb_rot - nb_bp) * kPrepThreads;
    for (int64_t e = (int64_t)(blockIdx.x - nb_bp) * kPrepThreads + threadIdx.x; e < n_dz4; e += nthr)
        dz4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
}

struct BwdArgs {
    int64_t N, C, seqlen, n_docs;
    int64_t tps;              // token tiles per sequence (channel-first)
    const int32_t* cu;
    int r, ndz;               // rank, MMA N for dz / dB (r rounded up to 16)
    int64_t n_tiles, n_items, per_cta;
    int pieces;               // partial slots per chunk
    float* dz_acc;            // [N, r] fp32, zero on entry
    float* dB_part;           // [n_chunks][pieces][r][64 K]
    uint32_t* err;
    int ksteps;               // 16-wide K steps of the filter MMA: r / 16 rounded up
    int dz_tma;               // 1: dz tiles are added with bulk tensor reductions, else fp32 atomics
    int rope_chunks;          // channel chunks whose g is read from R^T g (tm_gr): RoPE's rotated channels / 64
};

constexpr uint32_t kSmemTotal = 232448;              // shared memory per CTA (dynamic + static)

// Shared memory of lowrank_bwd_kernel<K, R64> (R64: rank above 32).  Two g | u slots (each held
// from its TMA load until the du / dw epilogue is done with it) and NZ z slots (held until the dB
// MMA has read z; three when they fit), one dW tile (K tap atoms of 128 tokens x 64 channels,
// handed to the MMAs in 128-row blocks of two atoms), the du tile staged for its TMA store, the
// chunk's Bp slice (rank rounded up to 16 rows per tap), and one fp32 dz box [128 rows][32 ranks]
// staged for its bulk reduction (rank 64: the two boxes in turn); where that does not fit (K = 4
// at rank 64), a box of 64 rows (the four boxes in turn); with neither, dz goes through fp32
// atomics.
template <int K, bool R64>
struct BwdSmem {
    static constexpr uint32_t gu = 2 * kRowTile;
    static constexpr uint32_t bp_tap = R64 ? 8192 : 4096;
    static constexpr uint32_t stat = 512;                                     // static shared memory
    static constexpr uint32_t base2 = 2 * gu + 2 * kRowTile + K * kAtom128 + kAtom128 + K * bp_tap + 1024 + stat;
    static constexpr uint32_t dzst_bytes = base2 + kAtom128 <= kSmemTotal       ? kAtom128
                                           : base2 + kAtom128 / 2 <= kSmemTotal ? kAtom128 / 2
                                                                                : 0;
    static constexpr int dz_rows = dzst_bytes / 128;                             // rows per dz box
    static constexpr int NZ = base2 + kRowTile + dzst_bytes <= kSmemTotal ? 3 : 2;
    static constexpr uint32_t z0 = 2 * gu;
    static constexpr uint32_t dw = z0 + NZ * kRowTile;
    static constexpr uint32_t dust = dw + K * kAtom128;
    static constexpr uint32_t bp = dust + kAtom128;
    static constexpr uint32_t dzst = bp + K * bp_tap;
    static constexpr uint32_t total = dzst + dzst_bytes + 1024;
};

// Warp roles of lowrank_bwd_kernel<K>: 0 TMA loads, 1 filter MMA issue (and TMEM owner), then the
// du / dw epilogue (GA: 16 warps, four per TMEM lane quarter, each a quarter of the channels),
// then 4 warps of dz / dB readout (GB: one TMEM lane quarter each), then the dz / dB MMA issue.  The epilogue is latency-bound
// (two warps per scheduler leave its TMEM / shared-memory round trips exposed), so it takes 16
// warps for every K (measured: 3-5 % faster than 8 at the 150M QKV and 2B all-linear shapes).
template <int K>
struct BwdEpi {
    static constexpr int ga = 16;
    static constexpr int groups = 32 / ga;             // 8-channel groups per GA warp
    static constexpr int per_wait = ga <= 8 ? 2 : 1;   // groups per TMEM wait in A1
    static constexpr int gb0 = 2 + ga;
    static constexpr int mma_d = gb0 + 4;              // the dz / dB MMA warp
    static constexpr int du_store = mma_d + 1;         // the du store warp
    static constexpr int threads = 32 * (du_store + 1);
};
constexpr int kGbWarps = 4, kGa0 = 2;

// dB orientation.  A tcgen05.mma of M = 128, K = 16 issued back to back takes ~28 ns at N = 64,
// ~36 ns at N = 128, ~52 ns at N = 192 and ~70 ns at N = 256 on the B200 (M = 64 costs the same
// as M = 128), so fewer, wider MMAs are cheaper.  K <= 3: dB[r][(j, c)] += z^T dW, one chain of
// 8 MMAs (N = 64 K, K = 128 tokens; A = z^T with the r index on the TMEM lanes, rows r .. 127 unused).  K = 4: dB^T[(j, c)][r] += dW^T z in 128-row
// blocks of two taps, 16 MMAs (N = 64 K = 256 would not leave TMEM for dz).
template <int K>
struct BwdCols {
    static constexpr bool dbt = K <= 3;
    // TMEM columns: Wd taps at 0 (64 K); dB; dz double buffer
    static constexpr uint32_t db = dbt ? 192 : 384;    // dbt: 64 K columns; else two blocks of 64
    static constexpr uint32_t dz = dbt ? 384 : 256;    // two buffers of 64
};

constexpr uint32_t kCfPitch = 136 * 2, kCfStPitch = 128 * 2;   // channel-first tile rows (bytes)

template <int K, bool R64, bool CF>
__global__ void __launch_bounds__(BwdEpi<K>::threads, 1) lowrank_bwd_kernel(const __grid_constant__ CUtensorMap tm_z,
                                                                         const __grid_constant__ CUtensorMap tm_g,
                                                                         const __grid_constant__ CUtensorMap tm_u,
                                                                         const __grid_constant__ CUtensorMap tm_bp,
                                                                         const __grid_constant__ CUtensorMap tm_du,
                                                                         const __grid_constant__ CUtensorMap tm_dz,
                                                                         const __grid_constant__ CUtensorMap tm_gr,
                                                                         BwdArgs a) {
    using S = BwdSmem<K, R64>;
    constexpr int NBLK = (K + 1) / 2;
    constexpr bool kDbt = BwdCols<K>::dbt;
    constexpr uint32_t kColDz = BwdCols<K>::dz, kColDb = BwdCols<K>::db;
    constexpr int kGaWarps = BwdEpi<K>::ga, kGaGroups = BwdEpi<K>::groups, kGaPerWait = BwdEpi<K>::per_wait;
    constexpr int kGb0 = BwdEpi<K>::gb0, kMmaD = BwdEpi<K>::mma_d, kDuSt = BwdEpi<K>::du_store;
    constexpr int NZ = S::NZ;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    // dwready / dwfree: per 128-row block (two tap atoms) of the dW tile, so the MMAs of one
    // block overlap the writing of the next and the next item's first block
    __shared__ uint64_t gufull[2], guempty[2], zfull[NZ], zempty[NZ], bfull, bempty, wfull, wempty, dwready[NBLK],
        dwfree[NBLK], dzfull[2], dzempty[2], dbfree, dustaged, dusfree;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t i0 = (int64_t)blockIdx.x * a.per_cta;
    const int64_t i1 = min(i0 + a.per_cta, a.n_items);
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&gufull[s], 1);
            mbar_init(&guempty[s], kGaWarps);
            mbar_init(&dzfull[s], 1);
            mbar_init(&dzempty[s], kGbWarps);
        }
        for (int s = 0; s < NZ; ++s) {
            mbar_init(&zfull[s], 1);
            mbar_init(&zempty[s], 2);      // the filter and the dB MMAs of the item read z
        }
        for (int bb = 0; bb < NBLK; ++bb) {
            mbar_init(&dwready[bb], kGaWarps);
            mbar_init(&dwfree[bb], 1);
        }
        mbar_init(&bfull, 1);
        mbar_init(&bempty, 2);             // the filter and the dz MMAs read Bp
        mbar_init(&wfull, 1);
        mbar_init(&wempty, kGaWarps);
        mbar_init(&dbfree, kGbWarps);
        mbar_init(&dustaged, kGaWarps);    // every GA warp has staged its du rows
        mbar_init(&dusfree, 1);            // the du store has read the staging tile
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch(&tm_z);
        tma_prefetch(&tm_g);
        tma_prefetch(&tm_u);
        tma_prefetch(&tm_bp);
        tma_prefetch(&tm_du);
        if (a.dz_tma) tma_prefetch(&tm_dz);
        if (a.rope_chunks) tma_prefetch(&tm_gr);
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
        // TMA loads: the whole warp runs the loop (warp-uniform coordinates), the elected lane issues
        const bool leader = elect_one();
        const uint64_t keep = l2_evict_last(), stream = l2_evict_first();
        auto wait_all = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, &abort_flag, a.err));
        };
        int64_t prev = -1;
        uint32_t cc = 0, it = 0;
        ItemPos ipos(i0, a.n_tiles);
        for (int64_t item = i0; item < i1; ++item, ++it, ipos.next()) {
            if (__any_sync(0xffffffffu, abort_flag != 0)) break;      // the lanes leave together
            const int64_t chunk = ipos.chunk, tile = ipos.tile;
            if (chunk != prev) {
                if (!wait_all(&bempty, (cc & 1) ^ 1)) break;
                if (leader) {
                    mbar_arrive_expect_tx(&bfull, K * a.ndz * 128);
                    for (int j = 0; j < K; ++j)
                        tma_load_2d_hint(sm + S::bp + j * S::bp_tap, &tm_bp, &bfull, (int32_t)(j * a.C + chunk * 64),
                                         0, keep);
                }
                ++cc;
                prev = chunk;
            }
            const TileAt ta = tile_at<CF>(tile, (int32_t)(chunk * 64), a.tps, a.seqlen, a.C);
            const int zs = it % NZ, gs = it & 1;
            if (!wait_all(&zempty[zs], ((it / NZ) & 1) ^ 1)) break;
            if (leader) {
                mbar_arrive_expect_tx(&zfull[zs], kRowTile);
                tma_load_2d_hint(sm + S::z0 + zs * kRowTile, &tm_z, &zfull[zs], 0, ta.m0, keep);
            }
            if (!wait_all(&guempty[gs], ((it >> 1) & 1) ^ 1)) break;
            if (leader) {
                uint8_t* gu = sm + gs * S::gu;
                mbar_arrive_expect_tx(&gufull[gs], S::gu);
                // RoPE: the conv backward of a rotated chunk reads R^T g, written by the set-up kernel
                tma_load_2d_hint(gu, chunk < a.rope_chunks ? &tm_gr : &tm_g, &gufull[gs], ta.x, ta.y, stream);
                if (CF) tma_load_2d_hint(gu + kRowTile, &tm_u, &gufull[gs], ta.x - 8, ta.y, stream);
                else tma_load_2d_hint(gu + kRowTile, &tm_u, &gufull[gs], ta.x, ta.y - 8, stream);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // ---- filter MMAs of every item, issued by their own warp (the dz / dB MMAs have another,
        // on another scheduler: one thread issuing both kinds was the kernel's critical path).  The
        // whole warp runs the loop, so the descriptor arithmetic is warp-uniform; the elected lane
        // issues the MMAs and commits.
        const bool leader = elect_one();
        const uint32_t idesc_w = idesc_bf16(128, 64, false, true);
        const uint32_t bp0 = smem_u32(sm + S::bp);
        const uint32_t nit = i1 > i0 ? (uint32_t)(i1 - i0) : 0u;
        uint32_t cc = 0;          // B loads consumed
        // Wd_j = z[j : j+128] . Bp_j (K-major A starting j rows into the z slot), KS 16-wide steps
        // over the rank, unrolled (a loop with a run-time trip count per tap cost ~2.5x the issue time)
        auto filter_mmas = [&](auto ks, uint32_t z0) {
            constexpr int KS = decltype(ks)::value;
#pragma unroll
            for (int j = 0; j < K; ++j)
#pragma unroll
                for (int k = 0; k < KS; ++k) {
                    const uint64_t da = kmajor_desc(z0 + 128u * j, k);
                    const uint64_t db = mnmajor_desc(bp0 + j * S::bp_tap, 8192, 16 * k);
                    if (leader) umma_bf16(tbase + 64 * j, da, db, idesc_w, k != 0);
                }
        };
        auto wait_all = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, &abort_flag, a.err));
        };
        ItemPos ipos(i0, a.n_tiles);
        for (uint32_t it = 0; it < nit; ++it, ipos.next()) {
            if (__any_sync(0xffffffffu, abort_flag != 0)) break;      // the lanes leave together
            const int zs = it % NZ;
            if (it == 0 || ipos.tile == 0) {      // a chunk starts: its Bp slice
                if (!wait_all(&bfull, cc & 1)) break;
                ++cc;
            }
            if (it > 0 && !wait_all(&wempty, (it - 1) & 1)) break;   // Wd read
            if (!wait_all(&zfull[zs], (it / NZ) & 1)) break;
            tc_fence_after();
            const uint32_t z0 = smem_u32(sm + S::z0 + zs * kRowTile);
            // ksteps = ceil(r / 16): 3 or 4 when r > 32, else 1 or 2
            if constexpr (R64) {
                if (a.ksteps == 4) filter_mmas(std::integral_constant<int, 4>{}, z0);
                else filter_mmas(std::integral_constant<int, 3>{}, z0);
            } else {
                if (a.ksteps == 2) filter_mmas(std::integral_constant<int, 2>{}, z0);
                else filter_mmas(std::integral_constant<int, 1>{}, z0);
            }
            if (leader) {
                umma_commit(&wfull);
                umma_commit(&zempty[zs]);
                if (it + 1 < nit && ipos.last_of_chunk()) umma_commit(&bempty);   // B is reloaded next
            }
            __syncwarp();
        }
    } else if (warp == kMmaD) {
        // ---- dz and dB MMAs of every item (the whole warp runs the loop; the elected lane issues)
        const bool leader = elect_one();
        const uint32_t idesc_dz = idesc_bf16(128, a.ndz, false, false);
        const uint32_t idesc_db = kDbt ? idesc_bf16(128, 64 * K, true, true) : idesc_bf16(128, a.ndz, true, true);
        const uint32_t bp0 = smem_u32(sm + S::bp);
        const uint32_t dw0 = smem_u32(sm + S::dw);
        const uint32_t nit = i1 > i0 ? (uint32_t)(i1 - i0) : 0u;
        uint32_t cc = 0;          // B loads consumed
        uint32_t m = 0;           // chunks whose dB accumulation has started
        auto wait_all = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, &abort_flag, a.err));
        };
        ItemPos ipos(i0, a.n_tiles);
        for (uint32_t it = 0; it < nit; ++it, ipos.next()) {
            if (__any_sync(0xffffffffu, abort_flag != 0)) break;      // the lanes leave together
            const bool first = it == 0 || ipos.tile == 0;
            const int zs = it % NZ, b = it & 1;
            if (first) {
                if (!wait_all(&bfull, cc & 1)) break;
                ++cc;
            }
            if (!wait_all(&zfull[zs], (it / NZ) & 1)) break;
            if (!wait_all(&dzempty[b], ((it >> 1) & 1) ^ 1)) break;
            if (first && m > 0 && !wait_all(&dbfree, (m - 1) & 1)) break;
            const uint32_t z0 = smem_u32(sm + S::z0 + zs * kRowTile);
            bool blk_ok = true;
#pragma unroll
            for (int bb = 0; bb < NBLK; ++bb) {
                if (!wait_all(&dwready[bb], it & 1)) {
                    blk_ok = false;
                    break;
                }
                tc_fence_after();
                // dz += dW_j . Bp_j^T for the block's taps (both K-major, K = 64 channels)
#pragma unroll
                for (int j = 2 * bb; j < 2 * bb + 2 && j < K; ++j)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t da = kmajor_desc(dw0 + j * kAtom128, k);
                        const uint64_t db = kmajor_desc(bp0 + j * S::bp_tap, k);
                        if (leader) umma_bf16(tbase + kColDz + 64 * b, da, db, idesc_dz, (j | k) != 0);
                    }
                if constexpr (!kDbt) {
                    // dB^T[blk] += dW^T . z  (both MN-major, K = 128 tokens)
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint64_t da = mnmajor_desc(dw0 + 2 * bb * kAtom128, kAtom128, 16 * ks);
                        const uint64_t db = mnmajor_desc(z0, kRowTile, 16 * ks);
                        if (leader) umma_bf16(tbase + kColDb + 64 * bb, da, db, idesc_db, !(first && ks == 0));
                    }
                    if (leader) umma_commit(&dwfree[bb]);
                }
                __syncwarp();
            }
            if (!blk_ok) break;
            if constexpr (kDbt) {
                // dB += z^T . dW over every tap at once (A: z tile, MN-major, its second 64-row
                // M atom is the next tile and only feeds unused rows; B: the K dW atoms, MN-major)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t da = mnmajor_desc(z0, kRowTile, 16 * ks);
                    const uint64_t db = mnmajor_desc(dw0, kAtom128, 16 * ks);
                    if (leader) umma_bf16(tbase + kColDb, da, db, idesc_db, !(first && ks == 0));
                }
                if (leader)
#pragma unroll
                    for (int bb = 0; bb < NBLK; ++bb) umma_commit(&dwfree[bb]);
            }
            if (first) ++m;
            if (leader) {
                umma_commit(&dzfull[b]);
                umma_commit(&zempty[zs]);
                if (it + 1 < nit && ipos.last_of_chunk()) umma_commit(&bempty);   // B is reloaded next
            }
            __syncwarp();
        }
    } else if (warp < kGb0) {
        // ---- GA: du (A1, staged for a TMA store) and dw (A2) of each item
        const int q = warp & 3;
        const int half = (warp - kGa0) >> 2;   // channel groups kGaGroups*half ..
        const int row = q * 32 + lane;
        const uint32_t lane_base = tbase + (uint32_t(q * 32) << 16);
        uint8_t* dus = sm + S::dust;
        uint8_t* dws = sm + S::dw;
        uint32_t it = 0;
        ItemPos ipos(i0, a.n_tiles);
        for (int64_t item = i0; item < i1; ++item, ++it, ipos.next()) {
            const int64_t chunk = ipos.chunk, tile = ipos.tile;
            const int gs = it & 1;
            // each GA warp goes at its own pace (no barrier among them): a failed wait sets the abort
            // flag, and every other wait in the kernel then gives up too
            bool ok = mbar_wait(&wfull, it & 1, &abort_flag, a.err) &&
                      mbar_wait(&gufull[gs], (it >> 1) & 1, &abort_flag, a.err) &&
                      (it == 0 || mbar_wait(&dusfree, (it - 1) & 1, &abort_flag, a.err));
            if (!ok) break;
            tc_fence_after();
            const TileAt ta = tile_at<CF>(tile, (int32_t)(chunk * 64), a.tps, a.seqlen, a.C);
            const int32_t n = ta.m0 + row;
            int32_t pos = -1, epos = -1;             // valid past / future taps of this row
            if (n < a.N) {
                int32_t sb, eb;
                seg_bounds32(n, a.cu, (int32_t)a.n_docs, (int32_t)a.seqlen, (int32_t)a.N, sb, eb);
                pos = n - sb;
                epos = eb - 1 - n;
            }
            const uint8_t* gt = sm + gs * S::gu;
            const uint8_t* ut = gt + kRowTile;
            // A1: du[t, c] = g[t, c] + sum_{j <= epos} Wd_j[t, c] g[t + j, c], two 8-channel
            // groups per TMEM wait, channel pairs on the packed fp32 FMA; g[t] is kept for A2
            uint4 gv[kGaGroups];
#pragma unroll
            for (int gp = 0; gp < kGaGroups / kGaPerWait; ++gp) {
                const int g0 = kGaGroups * half + kGaPerWait * gp;
                uint32_t wv[kGaPerWait][K][8];
#pragma unroll
                for (int x = 0; x < kGaPerWait; ++x)
#pragma unroll
                    for (int j = 0; j < K; ++j) tmem_ld8(lane_base + 64 * j + 8 * (g0 + x), wv[x][j]);
                uint4 gg[kGaPerWait][K];
#pragma unroll
                for (int x = 0; x < kGaPerWait; ++x)
#pragma unroll
                    for (int j = 0; j < K; ++j)
                        gg[x][j] = CF ? cf_gather8(gt, kCfPitch, g0 + x, row + j)
                                      : *reinterpret_cast<const uint4*>(gt + sw128_off(row + j, g0 + x));
                tmem_wait_ld();
                if (gp + 1 == kGaGroups / kGaPerWait) {   // every Wd value is in registers: the next
                    tc_fence_before();                    // filter MMA may overwrite the TMEM columns
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&wempty);
                }
#pragma unroll
                for (int x = 0; x < kGaPerWait; ++x) {
                    gv[kGaPerWait * gp + x] = gg[x][0];
                    float acc[8];
                    const uint32_t* g0w = reinterpret_cast<const uint32_t*>(&gg[x][0]);
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        acc[2 * p] = bf16_lo(g0w[p]);
                        acc[2 * p + 1] = bf16_hi(g0w[p]);
                    }
#pragma unroll
                    for (int j = 0; j < K; ++j) {
                        if (j <= epos) {
                            const uint32_t* gj = reinterpret_cast<const uint32_t*>(&gg[x][j]);
#pragma unroll
                            for (int p = 0; p < 4; ++p)
                                ffma2(acc[2 * p], acc[2 * p + 1], __uint_as_float(wv[x][j][2 * p]),
                                      __uint_as_float(wv[x][j][2 * p + 1]), bf16_lo(gj[p]), bf16_hi(gj[p]));
                        }
                    }
                    const uint4 dv = make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]),
                                                pack_bf16(acc[4], acc[5]), pack_bf16(acc[6], acc[7]));
                    if (CF) cf_scatter8(dus, kCfStPitch, g0 + x, row, dv);
                    else *reinterpret_cast<uint4*>(dus + sw128_off(row, g0 + x)) = dv;
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&dustaged);
            // A2: dw[t, c, j] = g[t, c] u[t - j, c] (bf16 products, one 64-channel atom per tap).  K <= 3:
            // every tap in one pass (the dB MMA reads every tap, so the blocks are freed together, and
            // each pass costs a barrier and an async-proxy fence); K = 4: block by block (taps 2 bb,
            // 2 bb + 1), each once the MMAs that last read it have finished.
            constexpr int kPasses = kDbt ? 1 : NBLK;
            bool quit = false;
#pragma unroll
            for (int ps = 0; ps < kPasses; ++ps) {
                const int blk0 = kDbt ? 0 : ps, blk1 = kDbt ? NBLK : ps + 1;
                ok = true;
#pragma unroll
                for (int bb = blk0; bb < blk1; ++bb)
                    ok = ok && mbar_wait(&dwfree[bb], (it & 1) ^ 1, &abort_flag, a.err);
                if (!ok) {
                    quit = true;
                    break;
                }
#pragma unroll
                for (int i = 0; i < kGaGroups; ++i) {
                    const int g8 = kGaGroups * half + i;
#pragma unroll
                    for (int j = 2 * blk0; j < 2 * blk1 && j < K; ++j) {
                        const uint4 uu = CF ? cf_gather8(ut, kCfPitch, g8, row + 8 - j)
                                            : *reinterpret_cast<const uint4*>(ut + sw128_off(row + 8 - j, g8));
                        const bool v = j <= pos;
                        uint4 d;
                        d.x = v ? mul_bf16x2(gv[i].x, uu.x) : 0u;
                        d.y = v ? mul_bf16x2(gv[i].y, uu.y) : 0u;
                        d.z = v ? mul_bf16x2(gv[i].z, uu.z) : 0u;
                        d.w = v ? mul_bf16x2(gv[i].w, uu.w) : 0u;
                        *reinterpret_cast<uint4*>(dws + j * kAtom128 + sw128_off(row, g8)) = d;
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int bb = blk0; bb < blk1; ++bb) mbar_arrive(&dwready[bb]);
                }
            }
            if (quit) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&guempty[gs]);
        }
    } else if (warp == kDuSt) {
        // ---- du store: each item's staged du tile, once every GA warp has written its rows
        if (lane == 0) {
            const uint8_t* dus = sm + S::dust;
            uint32_t it = 0;
            ItemPos ipos(i0, a.n_tiles);
            for (int64_t item = i0; item < i1; ++item, ++it, ipos.next()) {
                if (!mbar_wait(&dustaged, it & 1, &abort_flag, a.err)) break;
                const TileAt ta = tile_at<CF>(ipos.tile, (int32_t)(ipos.chunk * 64), a.tps, a.seqlen, a.C);
                tma_store_2d_hint(&tm_du, dus, ta.x, ta.y, l2_evict_first());
                tma_store_commit();
                tma_store_wait_read_all();
                mbar_arrive(&dusfree);
            }
            tma_store_wait_all();
        }
    } else {
        // ---- GB: dz readout (added into the [N, r] fp32 buffer: reduction over chunks) and dB partials
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const bool leader = warp == kGb0 && lane == 0;
        const uint32_t lane_base = tbase + (uint32_t(q * 32) << 16);
        uint8_t* dzs = sm + S::dzst;
        const bool via_tma = S::dzst_bytes > 0 && a.dz_tma;
        uint32_t it = 0;
        ItemPos ipos(i0, a.n_tiles);
        for (int64_t item = i0; item < i1; ++item, ++it, ipos.next()) {
            const int64_t chunk = ipos.chunk, tile = ipos.tile;
            const bool last = (item + 1 == i1) || ipos.last_of_chunk();
            const int b = it & 1;
            const bool ok = mbar_wait(&dzfull[b], (it >> 1) & 1, &abort_flag, a.err);
            if (via_tma && leader) tma_store_wait_read_all();   // the previous reduction has read the tile
            if (named_bar_any<3, 32 * kGbWarps>(!ok)) break;
            tc_fence_after();
            const int32_t m0 = tile_at<CF>(tile, 0, a.tps, a.seqlen, a.C).m0;
            const int32_t n = m0 + row;
            if (via_tma) {
                // one fp32 box [dz_rows rows][32 ranks] at a time through the staging tile, each added
                // into the [N, r] buffer by one bulk tensor reduction; with 64-row boxes the two
                // warps of the box's rows stage it while the other two wait
                constexpr int kDzRows = S::dz_rows > 0 ? S::dz_rows : 128;
                for (int bx = 0; bx * 32 < a.r; ++bx) {
                    for (int rh = 0; rh < 128 / kDzRows; ++rh) {
                        if (bx > 0 || rh > 0) {         // the previous box's reduction has read the tile
                            if (leader) tma_store_wait_read_all();
                            named_bar_any<3, 32 * kGbWarps>(false);
                        }
                        if (row / kDzRows == rh) {
                            const int srow = row - rh * kDzRows;
#pragma unroll
                            for (int c = 0; c < 32; c += 16) {
                                uint32_t v[2][8];
                                tmem_ld8(lane_base + kColDz + 64 * b + 32 * bx + c, v[0]);
                                tmem_ld8(lane_base + kColDz + 64 * b + 32 * bx + c + 8, v[1]);
                                tmem_wait_ld();
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const int qq = (c + 8 * h) >> 2;
                                    *reinterpret_cast<uint4*>(dzs + sw128_off(srow, qq)) =
                                        make_uint4(v[h][0], v[h][1], v[h][2], v[h][3]);
                                    *reinterpret_cast<uint4*>(dzs + sw128_off(srow, qq + 1)) =
                                        make_uint4(v[h][4], v[h][5], v[h][6], v[h][7]);
                                }
                            }
                        }
                        if ((bx + 1) * 32 >= a.r && rh + 1 == 128 / kDzRows) {   // every dz column is read
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&dzempty[b]);
                        }
                        fence_async_smem();
                        named_bar_any<3, 32 * kGbWarps>(false);     // the box's rows are staged
                        if (leader) {
                            tma_reduce_add_2d_hint(&tm_dz, dzs, bx * 32, m0 + rh * kDzRows, l2_evict_last());
                            tma_store_commit();
                        }
                    }
                }
            } else {
                for (int c = 0; c < a.r; c += 16) {
                    uint32_t v[2][8];
                    tmem_ld8(lane_base + kColDz + 64 * b + c, v[0]);
                    if (c + 8 < a.r) tmem_ld8(lane_base + kColDz + 64 * b + c + 8, v[1]);
                    tmem_wait_ld();
                    if (n < a.N) {
                        float4* dst = reinterpret_cast<float4*>(a.dz_acc + (int64_t)n * a.r + c);
                        atomicAdd(dst, make_float4(__uint_as_float(v[0][0]), __uint_as_float(v[0][1]),
                                                   __uint_as_float(v[0][2]), __uint_as_float(v[0][3])));
                        atomicAdd(dst + 1, make_float4(__uint_as_float(v[0][4]), __uint_as_float(v[0][5]),
                                                       __uint_as_float(v[0][6]), __uint_as_float(v[0][7])));
                        if (c + 8 < a.r) {
                            atomicAdd(dst + 2, make_float4(__uint_as_float(v[1][0]), __uint_as_float(v[1][1]),
                                                           __uint_as_float(v[1][2]), __uint_as_float(v[1][3])));
                            atomicAdd(dst + 3, make_float4(__uint_as_float(v[1][4]), __uint_as_float(v[1][5]),
                                                           __uint_as_float(v[1][6]), __uint_as_float(v[1][7])));
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dzempty[b]);
            }
            if (last) {                            // the run for this chunk ends: its dB partial
                // partial [k][m] (m = j * 64 + c): a warp writes 32 consecutive m per k
                const int64_t piece = (int64_t)blockIdx.x - (chunk * a.n_tiles) / a.per_cta;
                float* part = a.dB_part + ((chunk * a.pieces + piece) * a.r) * (64 * K);
                if constexpr (kDbt) {
                    // lane = k (rows below r), columns j * 64 + c: 32 contiguous bytes per load
                    if (q * 32 < a.r) {
                        float* dst = part + (int64_t)row * (64 * K);
                        for (int c = 0; c < 64 * K; c += 8) {
                            uint32_t v[8];
                            tmem_ld8(lane_base + kColDb + c, v);
                            tmem_wait_ld();
                            if (row < a.r) {
                                *reinterpret_cast<float4*>(dst + c) =
                                    make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]),
                                                __uint_as_float(v[3]));
                                *reinterpret_cast<float4*>(dst + c + 4) =
                                    make_float4(__uint_as_float(v[4]), __uint_as_float(v[5]), __uint_as_float(v[6]),
                                                __uint_as_float(v[7]));
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int bb = 0; bb < NBLK; ++bb) {
                        const int mrow = bb * 128 + row;     // (tap, channel) row = j * 64 + c
                        for (int c = 0; c < a.r; c += 8) {
                            uint32_t v[8];
                            tmem_ld8(lane_base + kColDb + 64 * bb + c, v);
                            tmem_wait_ld();
                            if (mrow < 64 * K) {
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    part[(int64_t)(c + i) * (64 * K) + mrow] = __uint_as_float(v[i]);
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dbfree);
            }
        }
        if (via_tma && leader) tma_store_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

// After the backward kernel, in one launch.  Blocks [0, n_chunks r): block chunk r + k sums, for
// each m = j 64 + c (one thread each), the partials of the runs covering the chunk in run order
// -> dB[k, (64 chunk + c) K + j]; the remaining blocks convert the fp32 dz accumulator to the bf16
// operand of the generator backward (four values per thread).
template <int K>
__global__ void __launch_bounds__(64 * K) bwd_finish_kernel(const float* __restrict__ part, float* __restrict__ dB,
                                                            int r, int C, int n_tiles, int per_cta, int pieces,
                                                            const float4* __restrict__ dz4, uint2* __restrict__ dzb,
                                                            int64_t count4) {
    pdl_trigger();
    pdl_wait();
    const int n_chunks = C / 64;
    const int nb = n_chunks * r;
    if ((int)blockIdx.x < nb) {
        const int chunk = blockIdx.x / r, k = blockIdx.x - chunk * r;
        const int m = threadIdx.x, j = m >> 6, c = chunk * 64 + (m & 63);
        const int first = (int)(((int64_t)chunk * n_tiles) / per_cta);
        const int lastc = (int)(((int64_t)(chunk + 1) * n_tiles - 1) / per_cta);
        const float* src = part + ((int64_t)chunk * pieces * r + k) * (64 * K) + m;
        float acc = 0.f;
        for (int p = 0; p <= lastc - first; ++p) acc += src[(int64_t)p * r * (64 * K)];
        dB[(int64_t)k * (C * K) + (int64_t)c * K + j] = acc;
        return;
    }
    const int64_t nthr = (int64_t)(gridDim.x - nb) * blockDim.x;
    for (int64_t i4 = (int64_t)(blockIdx.x - nb) * blockDim.x + threadIdx.x; i4 < count4; i4 += nthr) {
        const float4 v = dz4[i4];
        dzb[i4] = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
    }
}

// out[i] = sum_s part[s][i] for i < count (count a multiple of 4): one thread per 4 outputs, summing
// the splits in order (deterministic).
__global__ void reduce_splits_kernel(const float* __restrict__ part, float* __restrict__ out, int64_t count,
                                     int n_split) {
    pdl_trigger();
    pdl_wait();
    const int64_t i4 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i4 * 4 >= count) return;
    const float4* p = reinterpret_cast<const float4*>(part) + i4;
    const int64_t stride = count / 4;
    float4 acc = p[0];
    for (int s = 1; s < n_split; ++s) {
        const float4 v = p[s * stride];
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    reinterpret_cast<float4*>(out)[i4] = acc;
}

// =====================================================================================
// gen_bwd_kernel<XA>: per (128-wide block db of d, token range), X = dz (low-rank) or the
// head-wise filter gradient dwh, P = A or W, with R = X's width:
//   dh[t, db*128 + i] = sum_k X[t, k] P[db*128 + i, k]
//   dPpart[split][db*128 + i, k] = sum_{t in range} h[t, db*128 + i] X[t, k]
// XA = 64-wide atoms of X (1: R <= 64, 2: R <= 128).
// smem: NS stages of X tile [128 tokens][XA atoms] (K-major A of dh; MN-major B of dP) + h tile
//       [128 tokens][2 atoms] (MN-major A of dP); P block [128 rows of d][XA atoms] resident
//       (K-major B of dh); the bf16 dh tile [128 tokens][2 atoms] staged for its TMA store.
// TMEM: dh [128][128] at column 0, the dP block [128 rows of d][R] at column 128.
// =====================================================================================
struct GenBwdArgs {
    int64_t N, d;
    int R, ndz, ksteps;       // X width, dP MMA N (R rounded up to 16), dh K steps (R / 16 rounded up)
    int64_t hs;
    int n_dblk, n_split;
    int64_t n_tiles;
    int want_dh;
    float* dP_part;           // [n_split][d][R]
    uint32_t* err;
};

template <int XA>
struct GbCfg {
    static constexpr int DB = 128;                          // d columns per CTA
    static constexpr int NS = XA == 1 ? 3 : 2;
    static constexpr uint32_t stage = (XA + 2) * kAtom128;
    static constexpr uint32_t pblk = NS * stage;
    static constexpr uint32_t dhst = pblk + DB * 128 * XA;
    static constexpr uint32_t smem = dhst + 2 * kAtom128 + 1024;
    static constexpr uint32_t col_dp = DB;                  // TMEM column of the dP block
};

template <int XA>
__global__ void __launch_bounds__(kThreads, 1) gen_bwd_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                              const __grid_constant__ CUtensorMap tm_h,
                                                              const __grid_constant__ CUtensorMap tm_p,
                                                              const __grid_constant__ CUtensorMap tm_dh,
                                                              GenBwdArgs a) {
    using G = GbCfg<XA>;
    constexpr int NS = G::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint8_t* pblk = sm + G::pblk;
    uint8_t* dhs = sm + G::dhst;
    __shared__ uint64_t full[NS], empty[NS], pfull, hfull, hempty, dpfull;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int db = blockIdx.x % a.n_dblk, split = blockIdx.x / a.n_dblk;
    const int64_t t0 = (a.n_tiles * split) / a.n_split, t1 = (a.n_tiles * (split + 1)) / a.n_split;
    const bool want_dh = a.want_dh != 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&pfull, 1);
        mbar_init(&hfull, 1);
        mbar_init(&hempty, kEpiWarps);
        mbar_init(&dpfull, 1);
        abort_flag = 0;
        fence_mbar_init();
        tma_prefetch(&tm_x);
        tma_prefetch(&tm_h);
        tma_prefetch(&tm_p);
        if (want_dh) tma_prefetch(&tm_dh);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, 256);
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
            mbar_arrive_expect_tx(&pfull, G::DB * 128 * XA);
            for (int xa = 0; xa < XA; ++xa)
                tma_load_2d_hint(pblk + xa * G::DB * 128, &tm_p, &pfull, 64 * xa, db * G::DB, keep);
            uint32_t it = 0;
            for (int64_t tile = t0; tile < t1 && !abort_flag; ++tile, ++it) {
                const int s = it % NS;
                if (!mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, &abort_flag, a.err)) break;
                uint8_t* st = sm + s * G::stage;
                mbar_arrive_expect_tx(&full[s], G::stage);
                for (int xa = 0; xa < XA; ++xa)
                    tma_load_2d_hint(st + xa * kAtom128, &tm_x, &full[s], 64 * xa, (int32_t)(tile * 128), keep);
                for (int at = 0; at < 2; ++at)
                    tma_load_2d_hint(st + kAtom128 * (XA + at), &tm_h, &full[s], db * G::DB + 64 * at,
                                     (int32_t)(tile * 128), stream);
            }
        }
    } else if (warp == 1) {
        // the whole warp runs the loop (warp-uniform descriptor arithmetic); the elected lane issues
        const bool leader = elect_one();
        const uint32_t idesc_dh = idesc_bf16(128, G::DB, false, false);
        const uint32_t idesc_dp = idesc_bf16(128, a.ndz, true, true);
        const uint32_t p0 = smem_u32(pblk);
        auto wait_all = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, &abort_flag, a.err));
        };
        bool ok = wait_all(&pfull, 0);
        uint32_t it = 0;
        for (int64_t tile = t0; ok && tile < t1; ++tile, ++it) {
            if (__any_sync(0xffffffffu, abort_flag != 0)) break;      // the lanes leave together
            const int s = it % NS;
            if (!wait_all(&full[s], (it / NS) & 1)) break;
            tc_fence_after();
            const uint32_t x0 = smem_u32(sm + s * G::stage), h0 = x0 + XA * kAtom128;
            if (want_dh) {
                if (!wait_all(&hempty, (it & 1) ^ 1)) break;
                tc_fence_after();
                // dh = X . P^T: ksteps (R / 16 rounded up, at most 8) 16-wide steps over R, unrolled
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < a.ksteps) {
                        const uint64_t da = kmajor_desc(x0 + (k >> 2) * kAtom128, k & 3);
                        const uint64_t db = kmajor_desc(p0 + (k >> 2) * G::DB * 128, k & 3);
                        if (leader) umma_bf16(tbase, da, db, idesc_dh, k != 0);
                    }
                if (leader) umma_commit(&hfull);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t da = mnmajor_desc(h0, kAtom128, 16 * ks), db = mnmajor_desc(x0, kAtom128, 16 * ks);
                if (leader) umma_bf16(tbase + G::col_dp, da, db, idesc_dp, !(tile == t0 && ks == 0));
            }
            if (leader) umma_commit(&empty[s]);
            __syncwarp();
        }
        if (leader) umma_commit(&dpfull);     // every dP MMA of this CTA has completed
        __syncwarp();
    } else {
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;      // dh columns 64 half ..; dP columns 8 half + 16 i
        const int row = q * 32 + lane;
        const bool leader = warp == 2 && lane == 0;
        const uint32_t lane_base = tbase + (uint32_t(q * 32) << 16);
        uint32_t it = 0;
        bool ok = true;
        if (want_dh) {
            for (int64_t tile = t0; tile < t1; ++tile, ++it) {
                ok = mbar_wait(&hfull, it & 1, &abort_flag, a.err);
                if (leader) tma_store_wait_read_all();     // the previous dh store has read the staging tile
                if (epi_bar_any<kEpiThreads>(!ok)) break;
                tc_fence_after();
                // columns 64 half .. 64 half + 63 of the block = staging atom `half`
#pragma unroll 1
                for (int c = 0; c < 64; c += 32) {
                    uint32_t v[4][8];
#pragma unroll
                    for (int x = 0; x < 4; ++x) tmem_ld8(lane_base + 64 * half + c + 8 * x, v[x]);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        uint4 pk;
                        pk.x = pack_bf16(__uint_as_float(v[x][0]), __uint_as_float(v[x][1]));
                        pk.y = pack_bf16(__uint_as_float(v[x][2]), __uint_as_float(v[x][3]));
                        pk.z = pack_bf16(__uint_as_float(v[x][4]), __uint_as_float(v[x][5]));
                        pk.w = pack_bf16(__uint_as_float(v[x][6]), __uint_as_float(v[x][7]));
                        *reinterpret_cast<uint4*>(dhs + half * kAtom128 + sw128_off(row, (c >> 3) + x)) = pk;
                    }
                }
                tc_fence_before();
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&hempty);
                epi_bar_any<kEpiThreads>(false);          // every epilogue warp has staged its rows
                if (leader) {
                    for (int at = 0; at < 2; ++at)
                        tma_store_2d_hint(&tm_dh, dhs + at * kAtom128, db * G::DB + 64 * at, (int32_t)(tile * 128),
                                          l2_evict_first());
                    tma_store_commit();
                }
            }
            if (leader) tma_store_wait_all();
        }
        if (ok && t1 > t0) ok = mbar_wait(&dpfull, 0, &abort_flag, a.err);
        if (!epi_bar_any<kEpiThreads>(!ok) && t1 > t0) {
            tc_fence_after();
            float* part = a.dP_part + (int64_t)split * a.d * a.R;
            const int64_t drow = (int64_t)db * G::DB + row;
            for (int c = 8 * half; c < a.R; c += 16) {
                uint32_t v[8];
                tmem_ld8(lane_base + G::col_dp + c, v);
                tmem_wait_ld();
                if (drow < a.d) {
                    float4* dst = reinterpret_cast<float4*>(part + drow * a.R + c);
                    dst[0] = make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]),
                                         __uint_as_float(v[3]));
                    dst[1] = make_float4(__uint_as_float(v[4]), __uint_as_float(v[5]), __uint_as_float(v[6]),
                                         __uint_as_float(v[7]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, 256);
    }
}

template <int K, bool R64, bool CF>
cudaError_t launch_bwd_l(const CUtensorMap& tz, const CUtensorMap& tg, const CUtensorMap& tu, const CUtensorMap& tbp,
                         const CUtensorMap& tdu, const CUtensorMap& tdz, const CUtensorMap& tgr, BwdArgs ba,
                         unsigned grid, cudaStream_t st) {
    using S = BwdSmem<K, R64>;
    static_assert(S::total + S::stat <= kSmemTotal, "shared memory of lowrank_bwd_kernel");
    if (S::dzst_bytes == 0) ba.dz_tma = 0;
    cudaError_t e = cudaFuncSetAttribute(lowrank_bwd_kernel<K, R64, CF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         S::total);
    if (e != cudaSuccess) return e;
    DC_LAUNCH(kTcLowrankBwd, st, e = launch_pdl(lowrank_bwd_kernel<K, R64, CF>, dim3(grid), dim3(BwdEpi<K>::threads),
                                                S::total, st, tz, tg, tu, tbp, tdu, tdz, tgr, ba));
    return e;
}

template <int K, bool R64>
cudaError_t launch_bwd(bool cf, const CUtensorMap& tz, const CUtensorMap& tg, const CUtensorMap& tu,
                       const CUtensorMap& tbp, const CUtensorMap& tdu, const CUtensorMap& tdz, const CUtensorMap& tgr,
                       BwdArgs ba, unsigned grid, cudaStream_t st) {
    return cf ? launch_bwd_l<K, R64, true>(tz, tg, tu, tbp, tdu, tdz, tgr, ba, grid, st)
              : launch_bwd_l<K, R64, false>(tz, tg, tu, tbp, tdu, tdz, tgr, ba, grid, st);
}

}  // namespace

// Generator backward on the tensor cores: dP = h^T X (fp32, overwritten) and, when dh is
// non-null, dh = X P^T (bf16), for X [N, R] bf16 (R <= 128, multiple of 8), P [d, R] bf16.
// dP_part must hold n_split * d * R floats (gen_bwd_splits()).
int gen_bwd_dblk(int64_t d, int R) { return (int)((d + 127) / 128); }
int gen_bwd_splits(int64_t N, int64_t d, int R) {
    const int64_t n_tiles = (N + 127) / 128;
    return (int)std::max<int64_t>(1, std::min<int64_t>(148 / std::max(1, gen_bwd_dblk(d, R)), n_tiles));
}

cudaError_t tc_gen_backward(const void* X, int R, const void* h, int64_t hs, const void* P, int64_t N, int64_t d,
                            void* dh, float* dP, float* dP_part, uint32_t* err, cudaStream_t st) {
    const int n_dblk = gen_bwd_dblk(d, R), n_split = gen_bwd_splits(N, d, R);
    const int XA = R <= 64 ? 1 : 2;
    CUtensorMap tx, th, tp, tdh;
    std::memset(&tdh, 0, sizeof(tdh));                 // unused when dh is not requested
    if (!make_tmap_bf16(&tx, X, R, N, R, 64, 128) || !make_tmap_bf16(&th, h, d, N, hs, 64, 128) ||
        !make_tmap_bf16(&tp, P, R, d, R, 64, 128) || (dh && !make_tmap_bf16(&tdh, dh, d, N, d, 64, 128)))
        return cudaErrorInvalidValue;
    GenBwdArgs ga{N, d, R, (R + 15) / 16 * 16, (R + 15) / 16, hs, n_dblk, n_split, (N + 127) / 128, dh ? 1 : 0,
                  dP_part, err};
    cudaError_t e;
    const dim3 grid(n_dblk * n_split);
    if (XA == 1) {
        e = cudaFuncSetAttribute(gen_bwd_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, GbCfg<1>::smem);
        if (e != cudaSuccess) return e;
        DC_LAUNCH(kTcGenBwd, st, e = launch_pdl(gen_bwd_kernel<1>, grid, dim3(kThreads), GbCfg<1>::smem, st, tx, th, tp,
                                                tdh, ga));
    } else {
        e = cudaFuncSetAttribute(gen_bwd_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, GbCfg<2>::smem);
        if (e != cudaSuccess) return e;
        DC_LAUNCH(kTcGenBwd, st, e = launch_pdl(gen_bwd_kernel<2>, grid, dim3(kThreads), GbCfg<2>::smem, st, tx, th, tp,
                                                tdh, ga));
    }
    if (e != cudaSuccess) return e;
    DC_LAUNCH(kTcReduce, st, e = launch_pdl(reduce_splits_kernel, dim3((unsigned)((d * R / 4 + 255) / 256)), dim3(256), 0, st,
                                            (const float*)dP_part, dP, d * R, n_split));
    return e;
}


static inline size_t al256(size_t x) { return (x + 255) / 256 * 256; }

// Rows of the dz box the backward stages for its bulk reductions (BwdSmem<K, R64>::dz_rows).
static int dz_box_rows(int K, bool r64) {
    switch (K * 2 + (r64 ? 1 : 0)) {
        case 2: return BwdSmem<1, false>::dz_rows;
        case 3: return BwdSmem<1, true>::dz_rows;
        case 4: return BwdSmem<2, false>::dz_rows;
        case 5: return BwdSmem<2, true>::dz_rows;
        case 6: return BwdSmem<3, false>::dz_rows;
        case 7: return BwdSmem<3, true>::dz_rows;
        case 8: return BwdSmem<4, false>::dz_rows;
        default: return BwdSmem<4, true>::dz_rows;
    }
}

TcBwdLayout tc_bwd_layout(const Prob& p) {
    TcBwdLayout L{};
    const int sms = 148;   // sizing only; the launch uses at most this many CTAs
    L.n_tiles = p.layout == 1 ? p.batch * ((p.seqlen + 127) / 128) : (p.N + 127) / 128;
    const int64_t n_chunks = p.C / 64;
    L.n_items = L.n_tiles * n_chunks;
    L.per_cta = std::max<int64_t>(1, (L.n_items + sms - 1) / sms);
    L.grid = (int)((L.n_items + L.per_cta - 1) / L.per_cta);
    L.pieces = (int)(L.n_tiles / L.per_cta + 2);
    L.n_dblk = gen_bwd_dblk(p.d, (int)p.r);
    L.n_split = gen_bwd_splits(p.N, p.d, (int)p.r);
    size_t off = 0;
    L.zs = off;      off = al256(off + (size_t)p.N * p.r * 2);                     // z scratch (bf16)
    L.bp = off;      off = al256(off + (size_t)p.r * p.C * p.K * 2);               // tap-major B
    L.dz = off;      off = al256(off + (size_t)p.N * p.r * 4);                     // dz fp32 accumulator
    L.dzb = off;     off = al256(off + (size_t)p.N * p.r * 2);                     // dz bf16
    L.dbpart = off;  off = al256(off + (size_t)n_chunks * L.pieces * 64 * p.K * p.r * 4);
    L.dpart = off;   off = al256(off + (size_t)L.n_split * p.d * p.r * 4);
    L.gr = off;      off = al256(off + (size_t)p.N * p.rope_n * 2);                // RoPE: R^T g of the rotated channels
    L.total = off;
    return L;
}

cudaError_t tc_lowrank_backward(const Prob& p, const void* g, const void* u, const void* h, const void* A,
                                const void* B, const void* z_saved, void* du, void* dh, float* dA, float* dB,
                                char* tcws, uint32_t* err, cudaStream_t st) {
    const TcBwdLayout L = tc_bwd_layout(p);
    const void* z = z_saved;
    if (!z) {
        void* zs = tcws + L.zs;
        cudaError_t e = tc_gen_launch(h, p.hs, A, p.N, p.d, (int)p.r, zs, p.r, err, st);
        if (e != cudaSuccess) return e;
        z = zs;
    }
    __nv_bfloat16* bp = reinterpret_cast<__nv_bfloat16*>(tcws + L.bp);
    float* dz = reinterpret_cast<float*>(tcws + L.dz);
    __nv_bfloat16* dzb = reinterpret_cast<__nv_bfloat16*>(tcws + L.dzb);
    float* dbpart = reinterpret_cast<float*>(tcws + L.dbpart);
    float* dpart = reinterpret_cast<float*>(tcws + L.dpart);
    cudaError_t e;
    const int cb = (int)((p.C / 8 + kPrepThreads - 1) / kPrepThreads);     // channel blocks per Bp row
    __nv_bfloat16* gr = reinterpret_cast<__nv_bfloat16*>(tcws + L.gr);
    const PrepRope rp{static_cast<const __nv_bfloat16*>(g), gr, p.N, p.seqlen, p.n_docs, p.cu, p.rope_cs,
                      (int)p.rope_n, p.rope_n > 0 ? (int)p.rope_hd : 1,
                      (int)std::max<int64_t>(1, std::min<int64_t>(p.rope_max, INT32_MAX)),
                      p.rope_n > 0 ? (int)std::min<int64_t>(p.N, 148 * 8) : 0};
    const unsigned prep_grid = (unsigned)(p.r * p.K * cb + std::min<int64_t>((p.N * p.r / 4 + 1023) / 1024, 1024) +
                                          rp.nb_rot);
    DC_LAUNCH(kTcPrep, st, e = launch_pdl(bwd_prep_kernel, dim3(prep_grid), dim3(kPrepThreads), 0, st,
        static_cast<const __nv_bfloat16*>(B), bp, (int)p.r, (int)p.C, (int)p.K, cb, reinterpret_cast<float4*>(dz),
        p.N * p.r / 4, rp));
    if (e != cudaSuccess) return e;
    CUtensorMap tz, tg, tu, tbp, tdu, tdz, tgr;
    std::memset(&tdz, 0, sizeof(tdz));                 // unused unless dz goes through bulk reductions
    std::memset(&tgr, 0, sizeof(tgr));                 // unused without RoPE
    if (p.rope_n > 0 && !make_tmap_bf16(&tgr, gr, p.rope_n, p.N, p.rope_n, 64, 136)) return cudaErrorInvalidValue;
    const int dz_rows = dz_box_rows((int)p.K, p.r > 32);
    const bool dz_tma = p.r % 32 == 0 && dz_rows > 0;
    const bool cf = p.layout == 1;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_tmap_bf16(&tz, z, p.r, p.N, p.r, 64, 136) || !make_tmap_bf16(&tbp, bp, p.C * p.K, p.r, p.C * p.K, 64, (uint32_t)((p.r + 15) / 16 * 16)) ||
        (dz_tma && !make_tmap_2d(&tdz, dz, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.r, p.N, p.r * 4, 32,
                                 (uint32_t)dz_rows, true)))
        return cudaErrorInvalidValue;
    if (cf ? !(make_tmap_2d(&tg, g, BF, p.seqlen, p.batch * p.C, p.seqlen * 2, 136, 64, false) &&
               make_tmap_2d(&tu, u, BF, p.seqlen, p.batch * p.C, p.us * 2, 136, 64, false) &&
               make_tmap_2d(&tdu, du, BF, p.seqlen, p.batch * p.C, p.seqlen * 2, 128, 64, false))
           : !(make_tmap_bf16(&tg, g, p.C, p.N, p.C, 64, 136) && make_tmap_bf16(&tu, u, p.C, p.N, p.us, 64, 136) &&
               make_tmap_bf16(&tdu, du, p.C, p.N, p.C, 64, 128)))
        return cudaErrorInvalidValue;
    BwdArgs ba{p.N, p.C, p.seqlen, p.n_docs, (p.seqlen + 127) / 128, p.cu, (int)p.r, (int)((p.r + 15) / 16 * 16),
               L.n_tiles, L.n_items, L.per_cta, L.pieces, dz, dbpart, err, (int)((p.r + 15) / 16), dz_tma ? 1 : 0,
               (int)(p.rope_n / 64)};
    const bool r64 = p.r > 32;
    switch (p.K * 2 + (r64 ? 1 : 0)) {
        case 2: e = launch_bwd<1, false>(cf, tz, tg, tu, tbp, tdu, tdz, tgr, ba, L.grid, st); break;
        case 3: e = launch_bwd<1, true>(cf, tz, tg, tu, tbp, tdu, tdz, tgr, ba, L.grid, st); break;
        case 4: e = launch_bwd<2, false>(cf, tz, tg, tu, tbp, tdu, tdz, tgr, ba, L.grid, st); break;
        case 5: e = launch_bwd<2, true>(cf, tz, tg, tu, tbp, tdu, tdz, tgr, ba, L.grid, st); break;
        case 6: e = launch_bwd<3, false>(cf, tz, tg, tu, tbp, tdu, tdz, tgr, ba, L.grid, st); break;
        case 7: e = launch_bwd<3, true>(cf, tz, tg, tu, tbp, tdu, tdz, tgr, ba, L.grid, st); break;
        case 8: e = launch_bwd<4, false>(cf, tz, tg, tu, tbp, tdu, tdz, tgr, ba, L.grid, st); break;
        default: e = launch_bwd<4, true>(cf, tz, tg, tu, tbp, tdu, tdz, tgr, ba, L.grid, st); break;
    }
    if (e != cudaSuccess) return e;
    switch (p.K) {
#define DC_FINISH(KK)                                                                                             \
    case KK:                                                                                                       \
        DC_LAUNCH(kTcReduce, st, e = launch_pdl(bwd_finish_kernel<KK>,                                              \
                                                dim3((unsigned)(p.C / 64 * p.r + std::min<int64_t>((p.N * p.r / 4 + 64 * KK * 4 - 1) / (64 * KK * 4), 1024))), \
                                                dim3(64 * KK), 0, st, (const float*)dbpart, dB, (int)p.r, (int)p.C,  \
                                                (int)L.n_tiles, (int)L.per_cta, L.pieces,                            \
                                                reinterpret_cast<const float4*>(dz), reinterpret_cast<uint2*>(dzb), \
                                                p.N * p.r / 4));                                                     \
        break;
        DC_FINISH(1)
        DC_FINISH(2)
        DC_FINISH(3)
        DC_FINISH(4)
#undef DC_FINISH
    }
    if (e != cudaSuccess) return e;
    // generator backward: dA = h^T dz, dh = dz A^T
    return tc_gen_backward(dzb, (int)p.r, h, p.hs, A, p.N, p.d, dh, dA, dpart, err, st);
}

}  // namespace dynconv
