// noalloc.cu -- a forward entry point that allocates nothing, for callers that
// cannot call cudaMalloc.
//
// Some callers have no way to obtain device memory for a workspace: code that
// runs where the CUDA allocator must not be entered (inside a framework's
// allocator or memory-pool callbacks, in a runtime whose memory is fully
// pre-partitioned, or in a host process that only receives device pointers
// from elsewhere).  For them dynconv_fwd_noalloc runs the low-rank tensor-core
// forward with its scratch in a buffer that is part of this library's device
// image: the tap-major copy of B (bf16 [r, K C]), the z = h A intermediate
// (bf16 [N, r]) unless the caller passes z_save, and the device error word,
// which dynconv_noalloc_status reads and clears.
//
// The buffer is a file-scope device array of kScratchBytes + 256 bytes; every
// GPU on which the library's kernels are loaded holds it until the process
// exits.  In host code the array's name only stands for the device symbol, so
// its device address is looked up with cudaGetSymbolAddress, once per device
// and context, by the first call made with that device current (that first call
// should come before any stream capture).  The address is kept per device
// together with the context it was looked up in, and looked up again when a
// call finds another context current (after cudaDeviceReset the module is
// loaded anew and the array may move).  Every call shares the one buffer and
// leaves its last contents there: Bp and z are fully rewritten by each call;
// the error word is zeroed once at set-up (on the calling stream) and then
// collects the failures of every call until dynconv_noalloc_status reads and
// clears it.  Two calls whose work overlaps on the GPU (other streams, other
// host threads) race on the buffer.
#include <cuda.h>

#include <mutex>

#include "../../include/dynconv.h"
#include "internal.h"

namespace dynconv {

dynconv_status validate_desc(const dynconv_desc* d, Prob* p);
dynconv_status validate_ptr(const void* ptr, const char* name, bool required);
cudaError_t tc_forward_scratch(const Prob& p, const void* u, const void* h, const void* A, const void* BW, void* y,
                               void* z, void* bp, uint32_t* err, cudaStream_t st);

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;   // room for Bp (r C K 2 bytes) and z (N r 2 bytes)
constexpr size_t kErrBytes = 256;                   // the device error word, padded

static __device__ __align__(256) unsigned char g_noalloc_scratch[kErrBytes + kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct Slot {
    CUcontext ctx = nullptr;   // the context the address was looked up in
    void* addr = nullptr;
};
Slot g_slot[kMaxDevices];

// The calling thread's current driver context (nullptr before the runtime has made one current),
// through the driver entry point, like the tensor-map encoder (no link-time libcuda dependency).
CUcontext current_context() {
    using Fn = CUresult (*)(CUcontext*);
    static Fn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        return (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                   ? reinterpret_cast<Fn>(p)
                   : nullptr;
    }();
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}

// Device address of the scratch array on the current device: looked up on the first call with
// this device current, and again whenever the current context differs from the one it was
// looked up in; each lookup also zeroes the error word on stream st.
dynconv_status scratch_address(void** out, cudaStream_t st) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        set_error("no usable current device: %s", cudaGetErrorString(e));
        return DYNCONV_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    Slot& s = g_slot[dev];
    const CUcontext ctx = current_context();
    if (!s.addr || ctx == nullptr || ctx != s.ctx) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            set_error("cudaGetSymbolAddress of the built-in scratch failed: %s", cudaGetErrorString(e));
            return DYNCONV_ERR_CUDA;
        }
        e = cudaMemsetAsync(ptr, 0, kErrBytes, st);
        if (e != cudaSuccess) {
            set_error("clearing the built-in error word: %s", cudaGetErrorString(e));
            return DYNCONV_ERR_CUDA;
        }
        s.addr = ptr;
        s.ctx = current_context();   // the lookup makes the device's primary context current
    }
    *out = s.addr;
    return DYNCONV_OK;
}

}  // namespace
}  // namespace dynconv

using namespace dynconv;

extern "C" DYNCONV_API dynconv_status dynconv_fwd_noalloc(const dynconv_desc* desc, const void* u, const void* h,
                                                          const void* A, const void* B, void* y, void* z_save,
                                                          void* stream) {
    Prob p;
    dynconv_status s = validate_desc(desc, &p);
    if (s != DYNCONV_OK) return s;
    if (p.rope_n > 0) {
        set_error("dynconv_fwd_noalloc does not apply RoPE (rope_channels must be 0)");
        return DYNCONV_ERR_UNSUPPORTED;
    }
    if (p.kind != 0 || !tc_supported(p)) {
        set_error("dynconv_fwd_noalloc covers the bf16 low-rank tensor-core forward only "
                  "(rank a multiple of 8 up to 64, channels a multiple of 64, d_model a multiple of 8)");
        return DYNCONV_ERR_UNSUPPORTED;
    }
    if (p.N == 0) return DYNCONV_OK;
    const size_t bp_bytes = ((size_t)p.r * p.C * p.K * 2 + 255) / 256 * 256;
    const size_t z_bytes = z_save ? 0 : (size_t)p.N * p.r * 2;
    if (bp_bytes + z_bytes > kScratchBytes) {
        set_error("dynconv_fwd_noalloc needs %zu bytes of scratch (rank * channels * ksize * 2 for the tap-major "
                  "projection, plus N * rank * 2 for z unless z_save is given); the built-in buffer holds %zu bytes: "
                  "use dynconv_fwd with a workspace",
                  bp_bytes + z_bytes, kScratchBytes);
        return DYNCONV_ERR_UNSUPPORTED;
    }
    if ((s = validate_ptr(u, "u", true)) || (s = validate_ptr(h, "h", true)) || (s = validate_ptr(A, "A", true)) ||
        (s = validate_ptr(B, "B", true)) || (s = validate_ptr(y, "y", true)) ||
        (s = validate_ptr(z_save, "z_save", false)))
        return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void* base = nullptr;
    if ((s = scratch_address(&base, st)) != DYNCONV_OK) return s;
    uint32_t* err = static_cast<uint32_t*>(base);
    unsigned char* bp = static_cast<unsigned char*>(base) + kErrBytes;
    void* z = z_save ? z_save : static_cast<void*>(bp + bp_bytes);
    const cudaError_t e = tc_forward_scratch(p, u, h, A, B, y, z, bp, err, st);
    if (e != cudaSuccess) {
        set_error("dynconv_fwd_noalloc launch: %s", cudaGetErrorString(e));
        return DYNCONV_ERR_CUDA;
    }
    return DYNCONV_OK;
}

extern "C" DYNCONV_API dynconv_status dynconv_noalloc_status(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void* base = nullptr;
    dynconv_status s = scratch_address(&base, st);
    if (s != DYNCONV_OK) return s;
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, base, sizeof(word), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && word != 0) {
        e = cudaMemsetAsync(base, 0, sizeof(word), st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    if (e != cudaSuccess) {
        set_error("reading the built-in error word: %s", cudaGetErrorString(e));
        return DYNCONV_ERR_CUDA;
    }
    if (word == 0) return DYNCONV_OK;
    set_error("device check failed in a dynconv_fwd_noalloc call:%s",
              (word & kErrWaitTimeout) ? " pipeline wait timed out" : "");
    return DYNCONV_ERR_DEVICE_CHECK;
}
