// tc_common.cuh -- sm_100a building blocks: mbarriers with bounded waits, TMA tile
// copies, tcgen05 tensor-memory allocation, UMMA issue/commit and TMEM loads, and
// the shared-memory matrix descriptors for 128-byte-swizzled bf16 tiles.
//
// Shared-memory tile convention (what a TMA load with CU_TENSOR_MAP_SWIZZLE_128B
// writes): a tile is a stack of 128-byte rows, 64 bf16 each; within row r the
// 16-byte chunk q is stored at chunk position q ^ (r % 8), the tile base being
// 1024-byte aligned.  Such a tile is a valid UMMA operand either
//   K-major : rows = M (or N) index, the 64 elements = K      (SBO = 1024 B between 8-row groups)
//   MN-major: rows = K index, the 64 elements = M (or N)       (SBO = 1024 B between 8-row K groups,
//                                                               LBO = bytes between 64-wide MN atoms)
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"

namespace dynconv {
namespace tc {

constexpr uint64_t kWaitNs = 2000000000ull;   // bounded waits give up after 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- programmatic dependent launch
// Kernels launched with launch_pdl() may start while the previous kernel on the stream is
// still finishing; each kernel runs its prologue (barriers, TMEM, tensor-map prefetch),
// then pdl_wait() before touching global memory, which returns once the previous grid has
// completed and its writes are visible.  Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase of parity `parity` to complete.  Gives up after limit_ns (kWaitNs
// unless given), or as soon as another thread of the CTA has given up (abort flag): then it
// raises kErrWaitTimeout in the device error word and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* err, uint64_t limit_ns = kWaitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            if (err) atomicOr(err, kErrWaitTimeout);
            return false;
        }
    }
}

// After an abort: waits (at most kWaitNs, raising nothing) for a phase whose copies were
// already issued, so that no copy lands in shared memory after the CTA has exited.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < kWaitNs) {
    }
}

// One lane of a converged warp, the same lane every time the whole warp calls it (elect.sync):
// an MMA-issuing warp runs its loop on every lane, so the descriptor arithmetic is warp-uniform
// (uniform registers), and only the elected lane issues the tcgen05 instructions and commits.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}
// Untiled bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from global to
// shared memory, completing on an mbarrier.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// L2 eviction policies for the TMA copies: evict_last for tiles that many CTAs read again (z, the
// projection, the dz accumulator), evict_first for tensors streamed once (g, u, du, y, h).
__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x, int32_t y,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* map, const void* src, int32_t x, int32_t y,
                                                  uint64_t policy) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y), "l"(policy)
                 : "memory");
}
__device__ __forceinline__ void tma_reduce_add_2d_hint(const CUtensorMap* map, const void* src, int32_t x, int32_t y,
                                                       uint64_t policy) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;"
        ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void tma_store_wait_read_le1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void tma_store_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Element-wise fp32 add of a shared-memory tile into global memory (bulk tensor reduction,
// completed through the bulk async-group like a store).
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int32_t x, int32_t y) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, fp32 accumulate, one CTA.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives once on `bar` when every previously issued tcgen05.mma of this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, dense.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn_major) << 15) | (uint32_t(b_mn_major) << 16) |
           (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled tile (layout type 2).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           (uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major operand: tile base (1024-aligned) of the 64-wide K atom, k16 = which 16-element K step (0..3).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t atom_base, int k16) {
    return sdesc_sw128(atom_base + 32u * k16, 16u, 1024u);
}
// MN-major operand: first 64-wide MN atom at `base`, next atoms `atom_stride` bytes apart;
// the 16 K rows of this step start at row k0 (a multiple of 8).
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, uint32_t atom_stride, int k0) {
    return sdesc_sw128(base + 128u * k0, atom_stride, 1024u);
}

// 32 lanes x 32 bits, N consecutive columns: thread i of the warp gets lane (base lane + i).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Byte offset of 16-byte chunk q of row r inside a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(uint32_t r, uint32_t q) { return r * 128u + ((q ^ (r & 7u)) << 4); }

// Channel-first tiles (TMA boxes of a [batch * C, seqlen] tensor, no swizzle): one row of
// `pitch` bytes per channel, tokens contiguous.  cf_gather8 reads token column i of channels
// 8 c8 .. 8 c8 + 7 and packs them like a 16-byte segment of a token-major row; cf_scatter8
// writes such a segment back as a column.  A warp's lanes take consecutive tokens, so each
// 2-byte access of a warp covers 64 contiguous bytes (no bank conflict).
__device__ __forceinline__ uint4 cf_gather8(const uint8_t* tile, uint32_t pitch, int c8, int i) {
    const uint8_t* p = tile + (uint32_t)(8 * c8) * pitch + 2u * (uint32_t)i;
    uint32_t v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = *reinterpret_cast<const uint16_t*>(p + e * pitch);
    return make_uint4(v[0] | (v[1] << 16), v[2] | (v[3] << 16), v[4] | (v[5] << 16), v[6] | (v[7] << 16));
}
__device__ __forceinline__ void cf_scatter8(uint8_t* tile, uint32_t pitch, int c8, int i, uint4 v) {
    uint8_t* p = tile + (uint32_t)(8 * c8) * pitch + 2u * (uint32_t)i;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        *reinterpret_cast<uint16_t*>(p + (2 * e) * pitch) = (uint16_t)(w[e] & 0xFFFFu);
        *reinterpret_cast<uint16_t*>(p + (2 * e + 1) * pitch) = (uint16_t)(w[e] >> 16);
    }
}

// Token tile `tile` (128 tokens) and 64-channel chunk c0 of a conv-side tensor (u, g, y, du):
// m0 = its first token (the row of z / dz), (x, y) = the TMA coordinates of the tile.
//   token-major   [N, C]:                 x = c0, y = m0
//   channel-first [batch * C, seqlen]:    x = t0 (first token within the sequence), y = b C + c0,
//                 with tps = tiles per sequence, so a tile never spans two sequences
// Position (channel chunk, token tile) of a work item in a CTA's contiguous, chunk-major run,
// stepped item by item (no 64-bit division per item).
struct ItemPos {
    int64_t chunk, tile, n_tiles;
    __device__ __forceinline__ ItemPos(int64_t item, int64_t nt) : chunk(item / nt), tile(item - (item / nt) * nt), n_tiles(nt) {}
    __device__ __forceinline__ void next() {
        if (++tile == n_tiles) {
            tile = 0;
            ++chunk;
        }
    }
    __device__ __forceinline__ bool last_of_chunk() const { return tile + 1 == n_tiles; }
};

struct TileAt {
    int32_t m0, x, y;
};
template <bool CF>
__device__ __forceinline__ TileAt tile_at(int64_t tile, int32_t c0, int64_t tps, int64_t seqlen, int64_t C) {
    if (!CF) return TileAt{(int32_t)(tile * 128), c0, (int32_t)(tile * 128)};
    const int64_t b = tile / tps, t0 = (tile - b * tps) * 128;
    return TileAt{(int32_t)(b * seqlen + t0), (int32_t)t0, (int32_t)(b * C + c0)};
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Two fp32 lanes at once: (d0, d1) += (a0, a1) * (b0, b1), each lane one fused
// multiply-add rounded to nearest (the packed fp32 FMA of sm_100).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
    uint64_t d, a, b;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(d0), "f"(d1));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(d));
}

// Products of two bf16 pairs, each rounded once to bf16.  The exact product of
// two bf16 values fits an fp32 significand, so this equals rounding the fp32
// product to bf16.
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Named barrier 1 over the NT epilogue threads (the warps after the producer
// and MMA warps).
template <int NT>
__device__ __forceinline__ void epi_bar_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); }

// Barrier 2 over the NT epilogue threads that also ORs a predicate across them,
// so that a bounded wait giving up in one warp makes every epilogue warp leave
// its loop at the same point (no thread is left waiting at a named barrier).
template <int NT>
__device__ __forceinline__ bool epi_bar_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, 2, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(pred)), "n"(NT)
        : "memory");
    return r != 0;
}

// Reducing named barrier `ID` over NT threads (same contract as epi_bar_any).
template <int ID, int NT>
__device__ __forceinline__ bool named_bar_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(pred)), "n"(ID), "n"(NT)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__host__ __device__ inline uint32_t tmem_cols_for(int cols) {
    uint32_t c = 32;
    while (c < (uint32_t)cols) c <<= 1;
    return c;
}

}  // namespace tc
}  // namespace dynconv
