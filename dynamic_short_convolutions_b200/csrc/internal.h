// internal.h -- host-side structures shared by the C ABI layer and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dynconv {

// Bits of the device error word kept at the start of the workspace.
enum : uint32_t {
    kErrBadSeqlens = 1u,   // cu_seqlens not 0 ... N, non-decreasing
    kErrWaitTimeout = 2u,  // an mbarrier wait ran out of its iteration limit
    kErrRopePos = 4u,      // a packed document longer than the RoPE table
};

// A validated problem: all sizes resolved, strides filled in.
struct Prob {
    int kind;           // 0 low-rank, 1 head-wise
    int dtype;          // 0 fp32, 1 bf16
    int64_t batch, seqlen, N;
    int64_t d, C, K;
    int64_t r;          // low-rank rank
    int64_t hd, H;      // head-wise head_dim and head count
    int64_t R;          // generator width: r (low-rank) or H*K (head-wise)
    int64_t us, hs;     // u: token-major row stride / channel-first channel stride; h: row stride
    int layout;         // 0 token-major [N, C]; 1 channel-first [batch, C, seqlen] (u, y, g, du)
    const int32_t* cu;  // device cu_seqlens or nullptr (dense batch)
    int64_t n_docs;
    int deterministic;
    int algo;           // requested kernel family (dynconv_algo: 0 auto, 1 CUDA cores, 2 tensor cores)
    // rotary position embedding after the conv (rope_n == 0: none)
    int64_t rope_n, rope_hd, rope_max;
    const float* rope_cs;
};

// Workspace carve-up (byte offsets; every region 256-byte aligned).
struct WsLayout {
    size_t err;         // uint32 device error word
    size_t gen;         // fp32 [N, R]: z (low-rank) or head-wise filters (SIMT path)
    size_t dgen;        // fp32 [N, R]: dz or dwh
    size_t tc;          // start of the tensor-core path's private region
    size_t tc_bytes;
    size_t dec;         // decode step (seqlen == 1): split-d partial generator rows
    size_t rope;        // CUDA-core backward with RoPE: R^T g in the storage dtype [N, C]
    size_t total;
};

// Channel-first problems the tiled kernels take: seqlen and u's channel stride multiples of 8
// elements (16-byte TMA rows and vector loads), TMA coordinates within int32.
inline bool cf_tiles_ok(const Prob& p) {
    return p.seqlen % 8 == 0 && p.us % 8 == 0 && p.batch * p.C < (int64_t(1) << 31) &&
           p.seqlen < (int64_t(1) << 31);
}

// Workspace of the low-rank tensor-core path (inside the tensor-core region), byte offsets.
struct TcBwdLayout {
    size_t zs, bp, dz, dzb, dbpart, dpart, gr, total;
    int64_t per_cta, n_items, n_tiles;
    int pieces, grid, n_dblk, n_split;
};
TcBwdLayout tc_bwd_layout(const Prob& p);
// Workspace of the head-wise tensor-core path (inside the tensor-core region), byte offsets.
struct TcHwLayout {
    size_t wh, dwh, dpart, gr, total;
};
TcHwLayout tc_hw_layout(const Prob& p);

WsLayout ws_layout(const Prob& p);
size_t tc_workspace_bytes(const Prob& p);
bool tc_supported(const Prob& p);      // forward
bool tc_supported_bwd(const Prob& p);  // backward
const char* tc_unsupported_reason(const Prob& p, bool bwd);   // nullptr when the tensor cores take it

// Generic CUDA-core kernels (any shape, fp32 or bf16 storage).
cudaError_t simt_forward(const Prob& p, const void* u, const void* h, const void* A, const void* BW,
                         void* y, void* z_save, void* ws, cudaStream_t st);
cudaError_t simt_backward(const Prob& p, const void* g, const void* u, const void* h, const void* A,
                          const void* BW, const void* z_saved, void* du, void* dh, float* dA, float* dBW,
                          void* ws, cudaStream_t st);

// Generator GEMM out[N, R] = h[N, d] . P[d, R] on the tensor cores (bf16 in and out).
// Optionally the same launch also writes the tap-major copy Bp[k, j C + c] = B[k, c K + j]
// of a low-rank projection (the layout the low-rank conv kernels read), using the
// epilogue threads before the first accumulator is ready.
struct BPermute {
    const void* B = nullptr;
    void* Bp = nullptr;
    int r = 0, C = 0, K = 0;
};
cudaError_t tc_gen_launch(const void* h, int64_t hs, const void* P, int64_t N, int64_t d, int R, void* out,
                          int64_t out_ld, uint32_t* err, cudaStream_t st, BPermute perm = BPermute{});

// tcgen05 / TMA kernels (bf16 storage, shapes accepted by tc_supported).
cudaError_t tc_forward(const Prob& p, const void* u, const void* h, const void* A, const void* BW,
                       void* y, void* z_save, void* ws, cudaStream_t st);
cudaError_t tc_backward(const Prob& p, const void* g, const void* u, const void* h, const void* A,
                        const void* BW, const void* z_saved, void* du, void* dh, float* dA, float* dBW,
                        void* ws, cudaStream_t st);

// Bytes of the decode step's partial generator rows (split-d), for ws_layout.
size_t decode_partial_bytes(const Prob& p);
// One decode step for p.batch sequences (p.seqlen == 1), CUDA-core kernels.
cudaError_t decode_step(const Prob& p, const void* u, const void* h, const void* A, const void* BW, void* state,
                        void* y, void* ws, cudaStream_t st);
cudaError_t launch_check_seqlens(const int32_t* cu, int64_t n_docs, int64_t N, uint32_t* err, cudaStream_t st,
                                 int64_t max_doc_len = 0);
// RoPE on the CUDA-core path: y rotated in place (forward), or out = R^T g (backward), any layout.
cudaError_t simt_rope(const Prob& p, const void* x, void* out, bool inverse, cudaStream_t st);

// Text for the thread-local error message.
void set_error(const char* fmt, ...);

}  // namespace dynconv
