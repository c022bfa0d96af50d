// selftest.cu -- self-test of the tensor-core building blocks: one 128-row tile of
// D = A * B^T loaded by TMA (128-byte swizzle) and multiplied by tcgen05.mma with
// the same descriptor helpers the product kernels use, for the operand layouts
// they use.  It exists so that a layout or descriptor mistake shows up as a
// plain wrong number on a small case.
#include <cstdio>

#include "../../include/dynconv.h"
#include "../../include/dynconv_diag.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace dynconv {
namespace {

using namespace tc;

constexpr int kSelftestSmem = 1024 + 49152 + 98304;

// variant 0: A [128][Kd] and B [N][Kd], both K-major, Kd in {64, 128, 192}.
// variant 1: A stored [Kd][128] and B stored [Kd][N], both MN-major, Kd in {16, ..., 128}.
// variant 2: A [128][64] K-major and B stored [64][N] MN-major (Kd = 64).
// variant 3/4: A [136][64] K-major loaded as one 136-row tile, the operand starting
//   `Kd` rows (1..7) into it (D = A[Kd : Kd+128] B^T), B [N][64] K-major; variant 3
//   leaves the descriptor's base-offset field 0, variant 4 sets it from the start address.
__global__ void __launch_bounds__(128) selftest_kernel(const __grid_constant__ CUtensorMap ta,
                                                       const __grid_constant__ CUtensorMap tb, int variant, int N,
                                                       int Kd, float* __restrict__ D, uint32_t* err) {
    extern __shared__ uint8_t raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sa = sm;
    uint8_t* sb = sm + 49152;
    __shared__ uint64_t bar_load, bar_mma;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bar_load, 1);
        mbar_init(&bar_mma, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base;
    bool ok = true;
    if (threadIdx.x == 0) {
        if (variant == 0) {
            const int na = Kd / 64;
            mbar_arrive_expect_tx(&bar_load, uint32_t(na * (128 * 128 + N * 128)));
            for (int a = 0; a < na; ++a) tma_load_2d(sa + a * 16384, &ta, &bar_load, 64 * a, 0);
            for (int a = 0; a < na; ++a) tma_load_2d(sb + a * N * 128, &tb, &bar_load, 64 * a, 0);
        } else if (variant >= 3) {
            mbar_arrive_expect_tx(&bar_load, uint32_t(136 * 128 + N * 128));
            tma_load_2d(sa, &ta, &bar_load, 0, 0);
            tma_load_2d(sb, &tb, &bar_load, 0, 0);
        } else if (variant == 2) {
            const int nb = (N + 63) / 64;
            mbar_arrive_expect_tx(&bar_load, uint32_t(128 * 128 + nb * 64 * 128));
            tma_load_2d(sa, &ta, &bar_load, 0, 0);
            for (int a = 0; a < nb; ++a) tma_load_2d(sb + a * 64 * 128, &tb, &bar_load, 64 * a, 0);
        } else {
            const int nb = (N + 63) / 64;
            mbar_arrive_expect_tx(&bar_load, uint32_t((2 + nb) * Kd * 128));
            for (int a = 0; a < 2; ++a) tma_load_2d(sa + a * Kd * 128, &ta, &bar_load, 64 * a, 0);
            for (int a = 0; a < nb; ++a) tma_load_2d(sb + a * Kd * 128, &tb, &bar_load, 64 * a, 0);
        }
        ok = mbar_wait(&bar_load, 0, &abort_flag, err);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(128, N, variant == 1, variant == 1 || variant == 2);
            const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
            if (variant == 0) {
                for (int kb = 0; kb < Kd / 64; ++kb)
                    for (int k = 0; k < 4; ++k)
                        umma_bf16(tbase, kmajor_desc(a0 + kb * 16384, k), kmajor_desc(b0 + kb * N * 128, k), idesc,
                                  (kb | k) != 0);
            } else if (variant >= 3) {
                const uint32_t start = a0 + 128u * Kd;
                for (int k = 0; k < 4; ++k) {
                    uint64_t da = kmajor_desc(start, k);
                    if (variant == 4) da |= uint64_t(((start + 32u * k) >> 7) & 7u) << 49;
                    umma_bf16(tbase, da, kmajor_desc(b0, k), idesc, k != 0);
                }
            } else if (variant == 2) {
                for (int k = 0; k < 4; ++k)
                    umma_bf16(tbase, kmajor_desc(a0, k), mnmajor_desc(b0, 64 * 128, k * 16), idesc, k != 0);
            } else {
                for (int ks = 0; ks < Kd / 16; ++ks)
                    umma_bf16(tbase, mnmajor_desc(a0, Kd * 128, ks * 16), mnmajor_desc(b0, Kd * 128, ks * 16),
                              idesc, ks != 0);
            }
            umma_commit(&bar_mma);
        }
    }
    __syncwarp();
    if (mbar_wait(&bar_mma, 0, &abort_flag, err)) {
        tc_fence_after();
        const int row = warp * 32 + lane;
        for (int c = 0; c < N; c += 8) {
            uint32_t r[8];
            tmem_ld8(tbase + (uint32_t(warp * 32) << 16) + c, r);
            tmem_wait_ld();
            for (int i = 0; i < 8; ++i) D[row * N + c + i] = __uint_as_float(r[i]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, 256);
    }
}

// A wait that runs out: thread 0 waits, with a limit of limit_ns, on an mbarrier that nothing
// arrives on; thread 32 (another warp) waits on the same barrier with the kernels' own limit and
// must give up as soon as thread 0 has (the abort flag).  out[0], out[1] = 1 if the wait
// returned true, 2 if it gave up; the error word gets kErrWaitTimeout.
__global__ void __launch_bounds__(64) selftest_wait_kernel(uint64_t limit_ns, uint32_t* err, uint32_t* out) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) out[0] = mbar_wait(&bar, 0, &abort_flag, err, limit_ns) ? 1u : 2u;
    if (threadIdx.x == 32) out[1] = mbar_wait(&bar, 0, &abort_flag, err) ? 1u : 2u;
}

}  // namespace
}  // namespace dynconv

using namespace dynconv;

extern "C" DYNCONV_API dynconv_status dynconv_selftest_wait(uint64_t limit_ns, void* err_word, void* out2,
                                                            void* stream) {
    if (!err_word || !out2 || limit_ns == 0 || limit_ns > tc::kWaitNs) return DYNCONV_ERR_INVALID;
    selftest_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, static_cast<uint32_t*>(err_word),
                                                                          static_cast<uint32_t*>(out2));
    return cudaGetLastError() == cudaSuccess ? DYNCONV_OK : DYNCONV_ERR_CUDA;
}

extern "C" DYNCONV_API dynconv_status dynconv_selftest_umma(int variant, const void* A, const void* B, float* D,
                                                            int N, int Kd, void* err_word, void* stream) {
    if (variant == 0 && !(Kd == 64 || Kd == 128 || Kd == 192)) return DYNCONV_ERR_INVALID;
    if (variant == 1 && !(Kd >= 16 && Kd <= 128 && Kd % 16 == 0)) return DYNCONV_ERR_INVALID;
    if (variant == 2 && Kd != 64) return DYNCONV_ERR_INVALID;
    if (variant >= 3 && !(Kd >= 1 && Kd <= 7)) return DYNCONV_ERR_INVALID;
    if (variant < 0 || variant > 4) return DYNCONV_ERR_INVALID;
    if (N < 16 || N > 256 || N % 16) return DYNCONV_ERR_INVALID;
    if (!A || !B || !D || !err_word) return DYNCONV_ERR_INVALID;
    CUtensorMap ta, tb;
    bool ok;
    if (variant == 0)
        ok = make_tmap_bf16(&ta, A, Kd, 128, Kd, 64, 128) && make_tmap_bf16(&tb, B, Kd, N, Kd, 64, N);
    else if (variant == 2)
        ok = make_tmap_bf16(&ta, A, 64, 128, 64, 64, 128) && make_tmap_bf16(&tb, B, N, 64, N, 64, 64);
    else if (variant >= 3)
        ok = make_tmap_bf16(&ta, A, 64, 136, 64, 64, 136) && make_tmap_bf16(&tb, B, 64, N, 64, 64, N);
    else
        ok = make_tmap_bf16(&ta, A, 128, Kd, 128, 64, Kd) && make_tmap_bf16(&tb, B, N, Kd, N, 64, Kd);
    if (!ok) return DYNCONV_ERR_CUDA;
    if (cudaFuncSetAttribute(selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelftestSmem) !=
        cudaSuccess)
        return DYNCONV_ERR_CUDA;
    selftest_kernel<<<1, 128, kSelftestSmem, static_cast<cudaStream_t>(stream)>>>(
        ta, tb, variant, N, Kd, D, static_cast<uint32_t*>(err_word));
    return cudaGetLastError() == cudaSuccess ? DYNCONV_OK : DYNCONV_ERR_CUDA;
}
