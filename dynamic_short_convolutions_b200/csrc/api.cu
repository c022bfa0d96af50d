// api.cu -- the C ABI: argument validation, workspace sizing, kernel-family dispatch.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/dynconv.h"
#include "internal.h"

namespace dynconv {

namespace {
thread_local char g_err[512] = "";

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool is_device_ptr(const void* ptr) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

dynconv_status check_ptr(const void* ptr, const char* name, bool required) {
    if (ptr == nullptr) {
        if (!required) return DYNCONV_OK;
        set_error("%s is NULL", name);
        return DYNCONV_ERR_INVALID;
    }
    if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) {
        set_error("%s is not 16-byte aligned", name);
        return DYNCONV_ERR_INVALID;
    }
    if (!is_device_ptr(ptr)) {
        set_error("%s is not a device pointer (there is no host path)", name);
        return DYNCONV_ERR_INVALID;
    }
    return DYNCONV_OK;
}

dynconv_status make_prob(const dynconv_desc* d, Prob* p) {
    if (!d) { set_error("desc is NULL"); return DYNCONV_ERR_INVALID; }
    if (d->kind != DYNCONV_LOWRANK && d->kind != DYNCONV_HEADWISE) { set_error("bad kind %d", d->kind); return DYNCONV_ERR_INVALID; }
    if (d->dtype != DYNCONV_F32 && d->dtype != DYNCONV_BF16) { set_error("bad dtype %d", d->dtype); return DYNCONV_ERR_INVALID; }
    if (d->algo < DYNCONV_ALGO_AUTO || d->algo > DYNCONV_ALGO_TC) { set_error("bad algo %d", d->algo); return DYNCONV_ERR_INVALID; }
    if (d->batch < 0 || d->seqlen < 0) { set_error("negative batch/seqlen"); return DYNCONV_ERR_INVALID; }
    if (d->d_model < 1 || d->channels < 1) { set_error("d_model and channels must be >= 1"); return DYNCONV_ERR_INVALID; }
    if (d->ksize < 1) { set_error("ksize must be >= 1"); return DYNCONV_ERR_INVALID; }
    if (d->ksize > 4) { set_error("ksize %lld > 4 is not supported", (long long)d->ksize); return DYNCONV_ERR_UNSUPPORTED; }
    p->kind = d->kind;
    p->dtype = d->dtype;
    p->batch = d->batch;
    p->seqlen = d->seqlen;
    if (__builtin_mul_overflow(d->batch, d->seqlen, &p->N)) {
        set_error("batch * seqlen overflows 64 bits");
        return DYNCONV_ERR_INVALID;
    }
    p->d = d->d_model;
    p->C = d->channels;
    p->K = d->ksize;
    if (d->layout != DYNCONV_TOKEN_MAJOR && d->layout != DYNCONV_CHANNEL_FIRST) {
        set_error("bad layout %d", d->layout);
        return DYNCONV_ERR_INVALID;
    }
    p->layout = d->layout;
    p->hs = d->h_row_stride ? d->h_row_stride : d->d_model;
    const int64_t vec = d->dtype == DYNCONV_BF16 ? 8 : 4;
    if (p->layout == DYNCONV_TOKEN_MAJOR) {
        p->us = d->u_row_stride ? d->u_row_stride : d->channels;
        if (p->us < p->C) { set_error("u row stride below the channel count"); return DYNCONV_ERR_INVALID; }
        if (p->us % vec) { set_error("u row stride must be a multiple of 16 bytes"); return DYNCONV_ERR_INVALID; }
    } else {
        // channel-first: any channel stride >= seqlen (the vectorised kernels check their own alignment)
        p->us = d->u_row_stride ? d->u_row_stride : d->seqlen;
        if (p->us < p->seqlen) { set_error("u channel stride below seqlen"); return DYNCONV_ERR_INVALID; }
        // one token per sequence with unit channel stride: [batch, C, 1] is the memory of [batch, C]
        if (p->seqlen == 1 && p->us == 1 && p->C % vec == 0) {
            p->layout = DYNCONV_TOKEN_MAJOR;
            p->us = p->C;
        }
    }
    if (p->hs < p->d) { set_error("h row stride below d_model"); return DYNCONV_ERR_INVALID; }
    if (p->hs % vec) { set_error("h row stride must be a multiple of 16 bytes"); return DYNCONV_ERR_INVALID; }
    if (d->kind == DYNCONV_LOWRANK) {
        if (d->rank < 1) { set_error("low-rank needs rank >= 1"); return DYNCONV_ERR_INVALID; }
        if (d->rank > 128) { set_error("rank %lld > 128 is not supported", (long long)d->rank); return DYNCONV_ERR_UNSUPPORTED; }
        p->r = d->rank; p->hd = 0; p->H = 0; p->R = p->r;
    } else {
        if (d->head_dim < 1 || d->channels % d->head_dim) { set_error("head_dim must divide channels"); return DYNCONV_ERR_INVALID; }
        p->r = 0; p->hd = d->head_dim; p->H = d->channels / d->head_dim; p->R = p->H * p->K;
    }
    {
        // Every operand's byte count must fit well inside 64 bits: a product that wrapped
        // would turn a huge problem into a small or negative one (and the workspace sum
        // of a few such counts must not wrap either).
        const int64_t kMaxBytes = int64_t(1) << 56;
        auto fits = [&](int64_t a, int64_t b, int64_t c) {
            int64_t t;
            return !__builtin_mul_overflow(a, b, &t) && !__builtin_mul_overflow(t, c, &t) && t <= kMaxBytes;
        };
        const int64_t es = d->dtype == DYNCONV_BF16 ? 2 : 4;
        const int64_t rows = p->layout == DYNCONV_TOKEN_MAJOR ? p->N : (fits(p->batch, p->C, 1) ? p->batch * p->C : -1);
        const bool ok = rows >= 0 && fits(rows, p->us, es)         // u, y, g, du
                        && fits(p->N, p->hs, es)                    // h, dh
                        && fits(p->N, p->R, 4)                      // per-token generator rows (fp32)
                        && fits(p->d, p->R, 4)                      // A or W and their fp32 gradients
                        && fits(p->C, p->K * std::max<int64_t>(p->r, 1), 4);   // B and dB
        if (!ok) {
            set_error("sizes overflow: every operand must stay below 2^56 bytes");
            return DYNCONV_ERR_INVALID;
        }
    }
    p->cu = nullptr;
    p->n_docs = 0;
    p->deterministic = d->deterministic;
    p->algo = d->algo;
    p->rope_n = d->rope_channels;
    p->rope_hd = d->rope_head_dim;
    p->rope_max = d->rope_max_pos;
    p->rope_cs = d->rope_cos_sin;
    if (p->rope_n < 0) { set_error("rope_channels must be >= 0"); return DYNCONV_ERR_INVALID; }
    if (p->rope_n > 0) {
        if (p->rope_hd < 2 || p->rope_hd % 2) { set_error("rope_head_dim must be even and >= 2"); return DYNCONV_ERR_INVALID; }
        if (p->rope_n > p->C || p->rope_n % p->rope_hd) {
            set_error("rope_channels must be a multiple of rope_head_dim and at most channels");
            return DYNCONV_ERR_INVALID;
        }
        if (p->rope_max < 1) { set_error("rope_max_pos must be >= 1"); return DYNCONV_ERR_INVALID; }
        if (p->N > 0 && p->batch > 1 && p->seqlen > p->rope_max) {
            set_error("seqlen %lld exceeds rope_max_pos %lld", (long long)p->seqlen, (long long)p->rope_max);
            return DYNCONV_ERR_INVALID;
        }
    }
    return DYNCONV_OK;
}

// The RoPE table: a device pointer, 16-byte aligned.
dynconv_status check_rope(const Prob& p) {
    if (p.rope_n == 0) return DYNCONV_OK;
    return check_ptr(p.rope_cs, "rope_cos_sin", true);
}

bool use_tc(const Prob& p, int algo) {
    if (algo == DYNCONV_ALGO_SIMT) return false;
    return tc_supported(p);
}

dynconv_status workspace_ok(const Prob& p, void* ws, size_t ws_bytes) {
    const size_t need = ws_layout(p).total;
    if (ws_bytes < need) {
        set_error("workspace %zu bytes, need %zu", ws_bytes, need);
        return DYNCONV_ERR_WORKSPACE;
    }
    return check_ptr(ws, "ws", true);
}

dynconv_status cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return DYNCONV_OK;
    set_error("%s: %s", what, cudaGetErrorString(e));
    return DYNCONV_ERR_CUDA;
}

dynconv_status forward_common(const dynconv_desc* desc, const int32_t* cu, int64_t n_docs, bool varlen,
                              const void* u, const void* h, const void* A, const void* BW, void* y,
                              void* z_save, void* ws, size_t ws_bytes, void* stream) {
    g_err[0] = 0;
    Prob p;
    dynconv_status s = make_prob(desc, &p);
    if (s != DYNCONV_OK) return s;
    if (varlen) {
        if (p.batch != 1) { set_error("varlen needs batch == 1"); return DYNCONV_ERR_INVALID; }
        if (n_docs < 1) { set_error("n_docs must be >= 1"); return DYNCONV_ERR_INVALID; }
        if (p.N > INT32_MAX) { set_error("packed tokens must number below 2^31 (cu_seqlens is int32)"); return DYNCONV_ERR_INVALID; }
        if ((s = check_ptr(cu, "cu_seqlens", true)) != DYNCONV_OK) return s;
        p.cu = cu;
        p.n_docs = n_docs;
    }
    if (desc->algo == DYNCONV_ALGO_TC && !tc_supported(p)) {
        set_error("the tensor-core kernels do not cover this shape/dtype");
        return DYNCONV_ERR_UNSUPPORTED;
    }
    if (p.N == 0) return DYNCONV_OK;
    if (!varlen && p.rope_n > 0 && p.seqlen > p.rope_max) {
        set_error("seqlen %lld exceeds rope_max_pos %lld", (long long)p.seqlen, (long long)p.rope_max);
        return DYNCONV_ERR_INVALID;
    }
    if ((s = check_ptr(u, "u", true)) || (s = check_ptr(h, "h", true)) ||
        (s = check_ptr(A, "A", p.kind == 0)) || (s = check_ptr(BW, p.kind == 0 ? "B" : "W", true)) ||
        (s = check_ptr(y, "y", true)) || (s = check_ptr(z_save, "z_save", false)) || (s = check_rope(p)))
        return s;
    if ((s = workspace_ok(p, ws, ws_bytes)) != DYNCONV_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(p);
    uint32_t* err = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + L.err);
    if (varlen && (s = cuda_status(launch_check_seqlens(cu, n_docs, p.N, err, st, p.rope_n > 0 ? p.rope_max : 0),
                                   "cu_seqlens check")))
        return s;
    cudaError_t e = use_tc(p, desc->algo) ? tc_forward(p, u, h, A, BW, y, z_save, ws, st)
                                          : simt_forward(p, u, h, A, BW, y, z_save, ws, st);
    return cuda_status(e, "forward launch");
}

}  // namespace

dynconv_status validate_desc(const dynconv_desc* d, Prob* p) { return make_prob(d, p); }

dynconv_status validate_ptr(const void* ptr, const char* name, bool required) { return check_ptr(ptr, name, required); }

void set_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

WsLayout ws_layout(const Prob& p) {
    WsLayout L{};
    size_t off = 0;
    L.err = off;
    off += 256;
    L.gen = off;
    off = align_up(off + sizeof(float) * (size_t)(p.N * p.R), 256);
    L.dgen = off;
    off = align_up(off + sizeof(float) * (size_t)(p.N * p.R), 256);
    L.tc = off;
    L.tc_bytes = tc_supported(p) ? tc_workspace_bytes(p) : 0;
    off = align_up(off + L.tc_bytes, 256);
    L.dec = off;
    if (p.seqlen == 1) off = align_up(off + decode_partial_bytes(p), 256);
    L.rope = off;      // R^T g for a backward on the CUDA-core kernels (chosen, or forced by desc->algo)
    if (p.rope_n > 0 && (p.algo == DYNCONV_ALGO_SIMT || !tc_supported_bwd(p)))
        off = align_up(off + (size_t)p.N * p.C * (p.dtype == 0 ? 4 : 2), 256);
    L.total = off;
    return L;
}

}  // namespace dynconv

using namespace dynconv;

extern "C" {

size_t dynconv_workspace_bytes(const dynconv_desc* desc) {
    Prob p;
    if (make_prob(desc, &p) != DYNCONV_OK) return 0;
    return ws_layout(p).total;
}

dynconv_status dynconv_fwd(const dynconv_desc* desc, const void* u, const void* h, const void* A,
                           const void* B_or_W, void* y, void* z_save, void* ws, size_t ws_bytes, void* stream) {
    return forward_common(desc, nullptr, 0, false, u, h, A, B_or_W, y, z_save, ws, ws_bytes, stream);
}

dynconv_status dynconv_fwd_varlen(const dynconv_desc* desc, const int32_t* cu_seqlens, int64_t n_docs,
                                  const void* u, const void* h, const void* A, const void* B_or_W, void* y,
                                  void* z_save, void* ws, size_t ws_bytes, void* stream) {
    return forward_common(desc, cu_seqlens, n_docs, true, u, h, A, B_or_W, y, z_save, ws, ws_bytes, stream);
}

dynconv_status dynconv_bwd(const dynconv_desc* desc, const int32_t* cu_seqlens, int64_t n_docs, const void* g,
                           const void* u, const void* h, const void* A, const void* B_or_W, const void* z_saved,
                           void* du, void* dh, float* dA, float* dB_or_dW, void* ws, size_t ws_bytes,
                           void* stream) {
    g_err[0] = 0;
    Prob p;
    dynconv_status s = make_prob(desc, &p);
    if (s != DYNCONV_OK) return s;
    if (cu_seqlens) {
        if (p.batch != 1) { set_error("varlen needs batch == 1"); return DYNCONV_ERR_INVALID; }
        if (n_docs < 1) { set_error("n_docs must be >= 1"); return DYNCONV_ERR_INVALID; }
        if (p.N > INT32_MAX) { set_error("packed tokens must number below 2^31 (cu_seqlens is int32)"); return DYNCONV_ERR_INVALID; }
        if ((s = check_ptr(cu_seqlens, "cu_seqlens", true)) != DYNCONV_OK) return s;
        p.cu = cu_seqlens;
        p.n_docs = n_docs;
    }
    if (desc->algo == DYNCONV_ALGO_TC && !tc_supported_bwd(p)) {
        set_error("the tensor-core kernels do not cover this shape/dtype/mode");
        return DYNCONV_ERR_UNSUPPORTED;
    }
    if ((s = check_ptr(dA, "dA", p.kind == 0)) || (s = check_ptr(dB_or_dW, "dB_or_dW", true))) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (p.N == 0) {
        // No tokens: the parameter gradients are empty sums.
        if (p.kind == 0 && (s = cuda_status(cudaMemsetAsync(dA, 0, sizeof(float) * p.d * p.r, st), "memset")))
            return s;
        const size_t nbw = p.kind == 0 ? (size_t)(p.r * p.C * p.K) : (size_t)(p.d * p.R);
        return cuda_status(cudaMemsetAsync(dB_or_dW, 0, sizeof(float) * nbw, st), "memset");
    }
    if (!cu_seqlens && p.rope_n > 0 && p.seqlen > p.rope_max) {
        set_error("seqlen %lld exceeds rope_max_pos %lld", (long long)p.seqlen, (long long)p.rope_max);
        return DYNCONV_ERR_INVALID;
    }
    if ((s = check_ptr(g, "g", true)) || (s = check_ptr(u, "u", true)) || (s = check_ptr(h, "h", true)) ||
        (s = check_ptr(A, "A", p.kind == 0)) || (s = check_ptr(B_or_W, p.kind == 0 ? "B" : "W", true)) ||
        (s = check_ptr(z_saved, "z_saved", false)) || (s = check_ptr(du, "du", true)) ||
        (s = check_ptr(dh, "dh", false)) || (s = check_rope(p)))
        return s;
    if ((s = workspace_ok(p, ws, ws_bytes)) != DYNCONV_OK) return s;
    const WsLayout L = ws_layout(p);
    uint32_t* err = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + L.err);
    if (cu_seqlens && (s = cuda_status(launch_check_seqlens(cu_seqlens, n_docs, p.N, err, st,
                                                            p.rope_n > 0 ? p.rope_max : 0),
                                       "cu_seqlens check")))
        return s;
    cudaError_t e = (desc->algo != DYNCONV_ALGO_SIMT && tc_supported_bwd(p))
                        ? tc_backward(p, g, u, h, A, B_or_W, z_saved, du, dh, dA, dB_or_dW, ws, st)
                        : simt_backward(p, g, u, h, A, B_or_W, z_saved, du, dh, dA, dB_or_dW, ws, st);
    return cuda_status(e, "backward launch");
}

dynconv_status dynconv_decode_step(const dynconv_desc* desc, const void* u, const void* h, const void* A,
                                   const void* B_or_W, void* state, void* y, void* ws, size_t ws_bytes,
                                   void* stream) {
    g_err[0] = 0;
    Prob p;
    dynconv_status s = make_prob(desc, &p);
    if (s != DYNCONV_OK) return s;
    if (p.seqlen != 1) {
        set_error("dynconv_decode_step takes one new token per sequence: seqlen must be 1");
        return DYNCONV_ERR_INVALID;
    }
    if (p.rope_n > 0) {
        set_error("dynconv_decode_step does not apply RoPE (rope_channels must be 0)");
        return DYNCONV_ERR_UNSUPPORTED;
    }
    if (p.layout == DYNCONV_CHANNEL_FIRST) {
        // validation already turned [batch, C, 1] with unit channel stride and 16-byte rows into [batch, C]
        set_error("channel-first decode needs u_row_stride 0 or 1 and channels a multiple of 16 bytes");
        return DYNCONV_ERR_UNSUPPORTED;
    }
    if (p.N == 0) return DYNCONV_OK;
    if ((s = check_ptr(u, "u", true)) || (s = check_ptr(h, "h", true)) || (s = check_ptr(A, "A", p.kind == 0)) ||
        (s = check_ptr(B_or_W, p.kind == 0 ? "B" : "W", true)) || (s = check_ptr(state, "state", p.K > 1)) ||
        (s = check_ptr(y, "y", true)))
        return s;
    if ((s = workspace_ok(p, ws, ws_bytes)) != DYNCONV_OK) return s;
    return cuda_status(decode_step(p, u, h, A, B_or_W, state, y, ws, static_cast<cudaStream_t>(stream)),
                       "decode launch");
}

dynconv_status dynconv_device_status(void* ws, size_t ws_bytes, void* stream) {
    g_err[0] = 0;
    if (ws_bytes < 256) { set_error("workspace too small to hold the error word"); return DYNCONV_ERR_WORKSPACE; }
    dynconv_status s = check_ptr(ws, "ws", true);
    if (s != DYNCONV_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if ((s = cuda_status(cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st), "read error word")))
        return s;
    if ((s = cuda_status(cudaStreamSynchronize(st), "stream synchronize"))) return s;
    if (word == 0) return DYNCONV_OK;
    if ((s = cuda_status(cudaMemsetAsync(ws, 0, sizeof(word), st), "clear error word"))) return s;
    if ((s = cuda_status(cudaStreamSynchronize(st), "stream synchronize"))) return s;
    set_error("device check failed:%s%s%s", (word & kErrBadSeqlens) ? " malformed cu_seqlens" : "",
              (word & kErrWaitTimeout) ? " pipeline wait timed out" : "",
              (word & kErrRopePos) ? " a packed document is longer than rope_max_pos" : "");
    return DYNCONV_ERR_DEVICE_CHECK;
}

dynconv_status dynconv_query_family(const dynconv_desc* desc, int32_t* fwd_family, int32_t* bwd_family) {
    g_err[0] = 0;
    Prob p;
    dynconv_status s = make_prob(desc, &p);
    if (s != DYNCONV_OK) return s;
    const char* rf = tc_unsupported_reason(p, false);
    const char* rb = tc_unsupported_reason(p, true);
    if (desc->algo == DYNCONV_ALGO_TC && rb) {
        // the entry points refuse a forced tensor-core run they cannot do (rf implies rb)
        set_error("desc->algo asks for the tensor-core kernels, which %s refuses: %s",
                  rf ? "the forward (and the backward)" : "the backward", rf ? rf : rb);
        return DYNCONV_ERR_UNSUPPORTED;
    }
    const bool simt = desc->algo == DYNCONV_ALGO_SIMT;
    if (fwd_family) *fwd_family = (!simt && !rf) ? DYNCONV_FAMILY_TENSOR_CORE : DYNCONV_FAMILY_CUDA_CORE;
    if (bwd_family) *bwd_family = (!simt && !rb) ? DYNCONV_FAMILY_TENSOR_CORE : DYNCONV_FAMILY_CUDA_CORE;
    if (simt) set_error("desc->algo asks for the CUDA-core kernels");
    else if (rf) set_error("forward and backward on the CUDA-core kernels: %s", rf);
    else if (rb) set_error("backward on the CUDA-core kernels: %s", rb);
    return DYNCONV_OK;
}

const char* dynconv_last_error(void) { return g_err; }

const char* dynconv_status_string(dynconv_status status) {
    switch (status) {
        case DYNCONV_OK: return "DYNCONV_OK";
        case DYNCONV_ERR_INVALID: return "DYNCONV_ERR_INVALID";
        case DYNCONV_ERR_UNSUPPORTED: return "DYNCONV_ERR_UNSUPPORTED";
        case DYNCONV_ERR_WORKSPACE: return "DYNCONV_ERR_WORKSPACE";
        case DYNCONV_ERR_CUDA: return "DYNCONV_ERR_CUDA";
        case DYNCONV_ERR_DEVICE_CHECK: return "DYNCONV_ERR_DEVICE_CHECK";
    }
    return "unknown status";
}

int dynconv_version(void) { return 200; }

}  // extern "C"
