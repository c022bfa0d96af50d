/*
 * dynconv.h -- C ABI of the B200 (sm_100a) dynamic short convolution library.
 *
 * The operation ("Dynamic Short Convolutions Improve Transformers",
 * gist.science technical summary, section "Dynamic Short Convolutions"):
 * every token n generates its own depthwise causal filter of K taps from its
 * hidden state h[n,:] by a learned linear map, factored either
 *
 *   low-rank  (Parameterization 1):  z[n,:] = h[n,:] A            A: [d, r]
 *                                    w[n,c,j] = sum_k z[n,k] B[k, c*K + j]
 *                                                                 B: [r, C*K]
 *   head-wise (Parameterization 2):  w[n,c,j] = sum_i h[n,i] W[i, (c/head_dim)*K + j]
 *                                                                 W: [d, H*K]
 *
 * and applies it with the residual of the "Placement" paragraph
 * (X = X + dynamicShortConv(X)) and the "Mechanism" formula, tap 0 being the
 * current token:
 *
 *   y[n,c] = u[n,c] + sum_{j<K, n-j >= s(n)} w[n,c,j] u[n-j,c]
 *
 * where s(n) is the first token of n's sequence (dense batch) or packed
 * document (cu_seqlens); taps before it read zero.  The filter tensor
 * w [N,C,K] is never written to memory by the tensor-core path.
 *
 * Conventions shared by every entry point
 *   - Layout (default, desc->layout = DYNCONV_TOKEN_MAJOR): token-major,
 *     channels contiguous.  u is [N, C] with row stride
 *     desc->u_row_stride elements (0 means C), so u may be a column slice of
 *     a fused QKV output; h is [N, d] with row stride desc->h_row_stride
 *     (0 means d).  y, g, du are dense [N, C]; dh is dense [N, d]; A is
 *     [d, r]; B is [r, C*K] (column c*K + j); W is [d, H*K] (column q*K + j).
 *     N = batch * seqlen tokens.
 *   - Channel-first layout (desc->layout = DYNCONV_CHANNEL_FIRST), the layout
 *     of the depthwise causal convolutions in linear-RNN blocks (Mamba-2,
 *     Gated DeltaNet), whose static conv the dynamic one replaces (gist.science
 *     technical summary, "Language Modeling", linear RNNs; atlas.scime.ai
 *     summary, "Surprising findings"):
 *     u, y, g and du are [batch, C, seqlen], tokens contiguous; u's channel
 *     rows are desc->u_row_stride elements apart (0 means seqlen) and its
 *     sequences C * u_row_stride apart; y, g, du are dense.  Packed documents
 *     (batch 1) are [C, N].  h, dh and z stay token-major [N, d] / [N, R]: the
 *     generator input is the token's hidden state.  The tensor-core and
 *     vectorised kernels take channel-first problems whose seqlen and
 *     u_row_stride are multiples of 8 elements; other shapes run the generic
 *     kernels (any seqlen, any u_row_stride >= seqlen).
 *   - Storage dtype desc->dtype (fp32 or bf16) for u, h, A, B/W, y, z, g, du,
 *     dh; accumulation is always fp32; parameter gradients dA, dB/dW are fp32
 *     and OVERWRITTEN (not accumulated).
 *   - Ownership: the caller allocates every buffer, including the workspace
 *     (size from dynconv_workspace_bytes).  All pointers are device pointers
 *     (a host pointer is rejected with DYNCONV_ERR_INVALID: there is no CPU
 *     path).  Pointers must be 16-byte aligned and token-major row strides
 *     (u_row_stride, h_row_stride) multiples of 8 elements for bf16 / 4 for
 *     fp32.  The library allocates nothing.
 *   - Stream: `stream` is a cudaStream_t (NULL = legacy default stream).  All
 *     work is enqueued asynchronously on it; nothing synchronises.
 *   - Errors: arguments are validated before any launch (a descriptor whose
 *     operands would pass 2^56 bytes, or whose size products would wrap 64
 *     bits, is DYNCONV_ERR_INVALID); a failed launch returns DYNCONV_ERR_CUDA.  dynconv_last_error() gives a thread-local
 *     message for the last failure.  Nothing traps on the device.
 */
#ifndef DYNCONV_H
#define DYNCONV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DYNCONV_API __attribute__((visibility("default")))
#else
#define DYNCONV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DYNCONV_OK = 0,
    DYNCONV_ERR_INVALID = 1,      /* bad argument: null/host/misaligned pointer, bad shape */
    DYNCONV_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. ksize > 4) */
    DYNCONV_ERR_WORKSPACE = 3,    /* ws_bytes below dynconv_workspace_bytes() */
    DYNCONV_ERR_CUDA = 4,         /* a CUDA runtime/driver call or launch failed */
    DYNCONV_ERR_DEVICE_CHECK = 5  /* a device-side check failed (bad cu_seqlens, barrier timeout) */
} dynconv_status;

typedef enum { DYNCONV_F32 = 0, DYNCONV_BF16 = 1 } dynconv_dtype;
typedef enum { DYNCONV_LOWRANK = 0, DYNCONV_HEADWISE = 1 } dynconv_kind;

/* Kernel family.  AUTO picks the tcgen05/TMA tensor-core kernels for bf16
 * shapes they cover and the generic CUDA-core kernels otherwise (always for
 * fp32, which must not be rounded to a tensor-core input type). */
typedef enum { DYNCONV_ALGO_AUTO = 0, DYNCONV_ALGO_SIMT = 1, DYNCONV_ALGO_TC = 2 } dynconv_algo;

/* Memory layout of u, y, g, du (see "Conventions" above). */
typedef enum { DYNCONV_TOKEN_MAJOR = 0, DYNCONV_CHANNEL_FIRST = 1 } dynconv_layout;

typedef struct {
    int32_t kind;           /* dynconv_kind */
    int32_t dtype;          /* dynconv_dtype */
    int64_t batch;          /* B sequences of seqlen tokens (varlen: 1) */
    int64_t seqlen;         /* T (varlen: total packed tokens N) */
    int64_t d_model;        /* d: width of the hidden state h feeding the generator */
    int64_t channels;       /* C: channels of u being filtered */
    int64_t ksize;          /* K: taps, 1..4 */
    int64_t rank;           /* low-rank r (1..128); head-wise: 0 */
    int64_t head_dim;       /* head-wise channels per head (C % head_dim == 0); low-rank: 0 */
    int64_t u_row_stride;   /* token-major: elements between tokens of u (0 = channels);
                               channel-first: elements between channels of u (0 = seqlen) */
    int64_t h_row_stride;   /* elements between tokens of h; 0 = d_model */
    int32_t deterministic;  /* 1: every reduction in a fixed order, no float atomics.  The
                               low-rank backward then runs the CUDA-core kernels, two to three
                               orders of magnitude slower than the tensor-core backward; the
                               head-wise backward stays on the tensor-core path at full speed */
    int32_t algo;           /* dynconv_algo */
    int32_t layout;         /* dynconv_layout of u, y, g, du */
    /* Rotary position embedding fused after the conv (0 channels = none): see "RoPE" below. */
    int64_t rope_channels;  /* channels [0, rope_channels) of y are rotated (Q and K of a fused QKV) */
    int64_t rope_head_dim;  /* channels per rotary head: even, divides rope_channels */
    int64_t rope_max_pos;   /* rows of rope_cos_sin; every position must be below it */
    const float *rope_cos_sin; /* DEVICE fp32 [rope_max_pos, rope_head_dim]: entries 2i, 2i+1 of row p
                                  are cos and sin of pair i's angle at position p */
} dynconv_desc;

/* RoPE.  The pages apply the conv to Q, K and V "before RoPE"; with
 * rope_channels > 0 the library fuses that rotation into the conv, so that
 *   dynconv_fwd returns y_rot = R(y), y = u + dynamic causal conv(u), and
 *   dynconv_bwd takes g = dL/dy_rot and returns the gradients of L through R:
 *   the conv backward is fed with R^T g.
 * R rotates the consecutive channel pairs (2i, 2i+1) of each head of
 * rope_head_dim channels among the first rope_channels, at the token's
 * position p = n - s(n) in its sequence or packed document, as Su et al.
 * define the rotation (RoFormer, section 3.4.2):
 *   (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos),
 * cos and sin read from rope_cos_sin[p, 2i] and [p, 2i + 1] (the caller's
 * table; RoFormer's angle p * base^(-2i/rope_head_dim) with base 10000 is the
 * usual choice, e.g. dynamic_short_convolutions_b200.ops.rope_table).  Channels
 * from rope_channels on pass unrotated.  Positions are checked against
 * rope_max_pos: a dense batch needs seqlen <= rope_max_pos
 * (DYNCONV_ERR_INVALID otherwise); a packed document longer than that raises
 * the device check (DYNCONV_ERR_DEVICE_CHECK from dynconv_device_status).
 * The tensor-core kernels take RoPE on the token-major layout with
 * rope_head_dim a multiple of 8; other shapes run the CUDA-core kernels.
 * dynconv_decode_step and dynconv_fwd_noalloc reject rope_channels > 0
 * (DYNCONV_ERR_UNSUPPORTED). */

/* Workspace needed by dynconv_fwd / dynconv_fwd_varlen / dynconv_bwd for this
 * descriptor (one size serves all three).  Returns 0 for an invalid desc.
 * Zero the workspace once before its first use (cudaMemset; torch.zeros): its
 * first bytes hold the device error word, which the library clears when it
 * reports it.  One workspace must not be used by two calls that overlap on
 * the device. */
DYNCONV_API size_t dynconv_workspace_bytes(const dynconv_desc *desc);

/* Forward, dense batch: y = u + dynamic causal conv(u), filters from h.
 *   u      [N, C] (u_row_stride), h [N, d] (h_row_stride); channel-first:
 *          u and y are [batch, C, seqlen]
 *   A      [d, r] (low-rank) or NULL (head-wise)
 *   B_or_W [r, C*K] (low-rank) or [d, H*K] (head-wise)
 *   y      [N, C] output, dense
 *   z_save nullable; receives the generator output [N, R] in the storage
 *          dtype, R = r (low-rank: z = h A) or H*K (head-wise: the per-head
 *          filters h W), for the backward pass to reuse. */
DYNCONV_API dynconv_status dynconv_fwd(const dynconv_desc *desc, const void *u, const void *h, const void *A,
                           const void *B_or_W, void *y, void *z_save, void *ws, size_t ws_bytes,
                           void *stream);

/* Forward over packed documents: desc->batch must be 1 and desc->seqlen the
 * total token count N (below 2^31).  cu_seqlens is a DEVICE int32 array [n_docs + 1] with
 * cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_docs] = N; the filter never
 * reaches across a document start.  A malformed cu_seqlens is caught by a
 * device pre-check that raises a flag read by dynconv_device_status(); the
 * results of that call are then undefined, but every access stays inside the
 * tensors (each tap's source index is clamped into the token range). */
DYNCONV_API dynconv_status dynconv_fwd_varlen(const dynconv_desc *desc, const int32_t *cu_seqlens, int64_t n_docs,
                                  const void *u, const void *h, const void *A, const void *B_or_W,
                                  void *y, void *z_save, void *ws, size_t ws_bytes, void *stream);

/* Backward of dynconv_fwd / dynconv_fwd_varlen (cu_seqlens NULL = dense batch):
 * the gradients of the Mechanism formula and of the generator map (the same
 * passages as the forward).  The training kernels of "Efficient Training
 * Implementation" keep the filter tensor on chip; the backward keeps the same
 * rule for w and dw.  With dw[n,c,j] = g[n,c] u[n-j,c] for n-j >= s(n):
 *   du[m,c] = g[m,c] + sum_j w[m+j,c,j] g[m+j,c]   (taps with m >= s(m+j))
 *   low-rank:  dz = dw . B^T  [N, r],  dA = h^T dz,  dB = z^T dw,  dh = dz A^T
 *   head-wise: dwh[n,q,j] = sum_{c in head q} dw[n,c,j],  dW = h^T dwh,  dh = dwh W^T
 * Every sum over tokens or channels is in fp32.  desc->deterministic = 1 fixes
 * every reduction order (the low-rank backward then runs the CUDA-core kernels).
 * Channel-first: g, u and du are [batch, C, seqlen] ([C, N] for packed documents).
 *   g        [N, C] upstream gradient dL/dy, dense
 *   z_saved  nullable: the generator output saved by the forward ([N, r] or
 *            [N, H*K]); NULL recomputes it
 *   du       [N, C] output dL/du, dense
 *   dh       nullable [N, d] output dL/dh, dense
 *   dA       [d, r] fp32 output (low-rank; ignored for head-wise)
 *   dB_or_dW [r, C*K] or [d, H*K] fp32 output */
/* Errors: as dynconv_fwd; with DYNCONV_ALGO_TC, DYNCONV_ERR_UNSUPPORTED where the
 * tensor-core backward does not cover the descriptor. */
DYNCONV_API dynconv_status dynconv_bwd(const dynconv_desc *desc, const int32_t *cu_seqlens, int64_t n_docs,
                           const void *g, const void *u, const void *h, const void *A,
                           const void *B_or_W, const void *z_saved, void *du, void *dh, float *dA,
                           float *dB_or_dW, void *ws, size_t ws_bytes, void *stream);

/* Forward for callers that cannot allocate device memory (no counterpart in
 * the paper: a deployment variant of dynconv_fwd).  Runs the bf16 low-rank
 * tensor-core forward of a dense batch with no workspace argument: its scratch
 * (the tap-major copy of B, bf16 [r, K*C]; z = h A, bf16 [N, r]; the device
 * error word) lives in a buffer built into the library, 8 MiB + 256 bytes held
 * on every GPU that loads the library until the process exits.  It calls no
 * cudaMalloc/cudaFree or other allocating routine.
 *   u, h, A, B, y, z_save: as for dynconv_fwd (z_save nullable; when given, z
 *   is written there instead of the built-in buffer).
 *   Returns DYNCONV_ERR_UNSUPPORTED for shapes outside the tensor-core forward
 *   (fp32, head-wise, rank not a multiple of 8 or above 64, channels not a
 *   multiple of 64) and when the scratch does not fit 8 MiB: rank * channels *
 *   ksize * 2 bytes (rounded up to 256) plus, when z_save is NULL,
 *   N * rank * 2 bytes.
 * The first call with a given device current looks up the buffer's device
 * address (cudaGetSymbolAddress) once for that device and context, and zeroes
 * the error word on `stream`; make that first call before any stream capture.
 * A call that finds another context current than the one of the lookup (after
 * cudaDeviceReset) looks the address up again.  All calls share the buffer,
 * which keeps the last call's contents: each call rewrites Bp and z, and the
 * error word collects the device-side failures (a pipeline wait that ran out
 * of its time limit) of every call until dynconv_noalloc_status reads it.
 * Calls whose work overlaps on the GPU race on the buffer: serialise them. */
DYNCONV_API dynconv_status dynconv_fwd_noalloc(const dynconv_desc *desc, const void *u, const void *h,
                                               const void *A, const void *B, void *y, void *z_save, void *stream);

/* Device-side status of the dynconv_fwd_noalloc calls on the current device
 * (no counterpart in the paper).  Synchronises `stream`, reads the error word
 * of the built-in buffer and clears it: DYNCONV_ERR_DEVICE_CHECK if a call
 * since the last query had a pipeline wait run out of its time limit (its y is
 * then not valid), else DYNCONV_OK; DYNCONV_ERR_CUDA if the read failed.
 * Allocates nothing (a copy of 4 bytes into host stack memory). */
DYNCONV_API dynconv_status dynconv_noalloc_status(void *stream);

/* One decode step: the newest token of each of desc->batch sequences (desc->seqlen
 * must be 1), with the K-1 previous conv inputs of every sequence carried in a
 * rolling state.  The operation is the Mechanism formula of "Dynamic Short
 * Convolutions Improve Transformers" (gist.science technical summary, "Dynamic
 * Short Convolutions") at the last position, with the filter generated from h as
 * in dynconv_fwd and the residual added once:
 *   y[b,c] = u[b,c] + sum_{j<K} w[b,c,j] x_j[b,c],  x_0 = u[b,c], x_j = state[b,j-1,c]
 * after which the state rolls by one token: state[b,j,c] <- x_j[b,c], j = 0..K-2.
 * The pages leave inference unoptimised (atlas.scime.ai summary, "Limitations");
 * this is the step a generation loop calls.  Feeding a sequence token by token
 * from a zero state reproduces dynconv_fwd on that sequence.
 *   u      [batch, C] (row stride desc->u_row_stride): the new token's conv input
 *   h      [batch, d] (row stride desc->h_row_stride): its generator input
 *   A, B_or_W: as for dynconv_fwd
 *   state  [batch, K-1, C] in the storage dtype, read and rewritten in place;
 *          zero it when a sequence starts (taps before the start read zero);
 *          may be NULL when K = 1
 *   y      [batch, C] output, dense
 *   ws     workspace of dynconv_workspace_bytes(desc), zeroed once
 * Always runs the CUDA-core kernels (fp32 accumulation) whatever desc->algo says.
 * desc->layout may be channel-first only with u_row_stride 0 or 1 and channels a
 * multiple of 8 (bf16) / 4 (fp32): u [batch, C, 1] is then the same memory as
 * [batch, C] (every entry point treats such a descriptor as token-major).
 * Errors: as dynconv_fwd, and DYNCONV_ERR_INVALID when seqlen != 1. */
DYNCONV_API dynconv_status dynconv_decode_step(const dynconv_desc *desc, const void *u, const void *h,
                                               const void *A, const void *B_or_W, void *state, void *y,
                                               void *ws, size_t ws_bytes, void *stream);

/* Synchronises `stream` and reports device-side check failures raised by the
 * calls that used this workspace since the last query (then clears them):
 * DYNCONV_ERR_DEVICE_CHECK for a malformed cu_seqlens or a pipeline wait that
 * ran out of its time limit (2 s), else DYNCONV_OK. */
DYNCONV_API dynconv_status dynconv_device_status(void *ws, size_t ws_bytes, void *stream);

/* Kernel families (see dynconv_query_family). */
typedef enum { DYNCONV_FAMILY_TENSOR_CORE = 1, DYNCONV_FAMILY_CUDA_CORE = 2 } dynconv_family;

/* Which kernel family dynconv_fwd / dynconv_fwd_varlen (*fwd_family) and
 * dynconv_bwd (*bwd_family) run for this descriptor (either pointer may be
 * NULL): DYNCONV_FAMILY_TENSOR_CORE (tcgen05/TMA kernels) or
 * DYNCONV_FAMILY_CUDA_CORE (the generic kernels).  With DYNCONV_ALGO_AUTO a
 * descriptor falls to the CUDA-core kernels for fp32 storage, shapes outside
 * the tensor-core kernels' coverage (low-rank rank above 64 or not a multiple
 * of 8, channels not a multiple of 64, ...) and, backward only, the
 * deterministic low-rank mode; dynconv_last_error() then names the reason
 * (else it is "").  Host-only: no device work, no allocation.
 * Returns DYNCONV_ERR_INVALID / _UNSUPPORTED for a descriptor that the entry
 * points would reject: among them, with DYNCONV_ALGO_TC, one that the
 * tensor-core kernels of either pass do not cover (dynconv_last_error() names
 * the pass and the reason). */
DYNCONV_API dynconv_status dynconv_query_family(const dynconv_desc *desc, int32_t *fwd_family,
                                                int32_t *bwd_family);

/* Thread-local text of the last failure in this thread ("" if none). */
DYNCONV_API const char *dynconv_last_error(void);

/* Name of a status code. */
DYNCONV_API const char *dynconv_status_string(dynconv_status status);

/* Per-kernel device timing (tracing).  When enabled, every kernel launch of
 * the library is bracketed by two CUDA events recorded on its launch stream.
 * dynconv_profile_enable returns the previous state.  dynconv_profile_read
 * waits for the recorded events, writes up to max_entries rows (kernel name,
 * launches, summed device milliseconds) for kernels launched since the last
 * reset, and returns how many kernels have rows; reset != 0 clears the sums.
 * Not for use inside CUDA graph capture. */
typedef struct {
    char name[48];
    int64_t launches;
    double total_ms;
} dynconv_profile_entry;

DYNCONV_API int dynconv_profile_enable(int enable);
DYNCONV_API int dynconv_profile_read(dynconv_profile_entry *entries, int max_entries, int reset);

/* Library version, major * 10000 + minor * 100 + patch. */
DYNCONV_API int dynconv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DYNCONV_H */
