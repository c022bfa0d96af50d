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
// (bf16 [N, r]) unless the caller passes z_save, and the device error word.
//
// The buffer is a file-scope device array of kScratchBytes + 256 bytes; every
// GPU on which the library's kernels are loaded holds it until the process
// exits.  In host code the array's name only stands for the device symbol, so
// its device address is looked up with cudaGetSymbolAddress, once per device,
// by the first call made with that device current (that first call should come
// before any stream capture).  Every call shares the one buffer and leaves its
// last contents there: the error word is cleared by each call, Bp and z are
// fully rewritten by each call, and two calls whose work overlaps on the GPU (other
// streams, other host threads) race on it.
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
void* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
dynconv_status scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        set_error("no usable current device: %s", cudaGetErrorString(e));
        return DYNCONV_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_addr[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            set_error("cudaGetSymbolAddress of the built-in scratch failed: %s", cudaGetErrorString(e));
            return DYNCONV_ERR_CUDA;
        }
        g_addr[dev] = ptr;
    }
    *out = g_addr[dev];
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
    void* base = nullptr;
    if ((s = scratch_address(&base)) != DYNCONV_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t* err = static_cast<uint32_t*>(base);
    unsigned char* bp = static_cast<unsigned char*>(base) + kErrBytes;
    void* z = z_save ? z_save : static_cast<void*>(bp + bp_bytes);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(uint32_t), st);
    if (e == cudaSuccess) e = tc_forward_scratch(p, u, h, A, B, y, z, bp, err, st);
    if (e != cudaSuccess) {
        set_error("dynconv_fwd_noalloc launch: %s", cudaGetErrorString(e));
        return DYNCONV_ERR_CUDA;
    }
    return DYNCONV_OK;
}
