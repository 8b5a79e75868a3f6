// mq_noalloc.cu -- mq_linear_w4a4 for callers that cannot allocate device
// memory.
//
// mq_linear_w4a4 needs a workspace (the amax accumulator, alpha_x, the status
// word and the quantized activation).  Some callers have no way to provide
// one: a plugin or custom operator inside a host application that owns all
// device memory through its own pool and gives extensions no allocator, or C
// code that must not call cudaMalloc because cudaMalloc synchronizes the
// device.  For them the library keeps its own scratch: one file-scope device
// array of MQ_NOALLOC_SCRATCH_BYTES, which every GPU that loads this module
// holds until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it
// names a stand-in object), so every call, with the caller's device current,
// looks up the real address with cudaGetSymbolAddress.  The lookup is cheap
// once the module is loaded, and doing it per call rather than caching it
// keeps the address right for the context that is current now: after a
// cudaDeviceReset the array lives at a new address in a new context.  The
// first call on a device loads the module and sets the array up, so it
// should come before any stream capture.  Every call then clears the scratch
// header and runs the normal mq_linear_w4a4 path with the scratch as its
// workspace.

#include "../../include/mq.h"
#include "mq_internal.h"

namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[MQ_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch in the current device's current context.
int scratch_for_current_device(void** addr) {
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return MQ_ERR_CUDA;
    if (!(major == 10 && minor == 0)) return MQ_ERR_ARCH;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MQ_ERR_CUDA;
    *addr = p;
    return MQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

__global__ void k_fill_words(uint32_t* p, int n, uint32_t word) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) p[i] = word;
}

}  // namespace

extern "C" int mq_debug_noalloc_fill_header(uint32_t word, void* stream) {
    void* scratch = nullptr;
    const int st = scratch_for_current_device(&scratch);
    if (st != MQ_OK) return st;
    k_fill_words<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(scratch),
                                                                   (int)(mq::WS_HEADER_BYTES / 4), word);
    return cudaGetLastError() == cudaSuccess ? MQ_OK : MQ_ERR_CUDA;
}

extern "C" int mq_linear_w4a4_noalloc(const void* x, int64_t M, int64_t K, const uint8_t* w_codes,
                                      const uint8_t* w_scales, const float* alpha_w, int64_t N, void* y,
                                      void* stream) {
    // Every synchronous check of mq_linear_w4a4 comes before anything is
    // enqueued (its shape limits too, so the size below cannot overflow).
    if (!x || !w_codes || !w_scales || !alpha_w || !y) return MQ_ERR_INVALID_ARG;
    const int shape = mq::check_linear_shape(M, N, K);
    if (shape != MQ_OK) return shape;
    if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y)) return MQ_ERR_ALIGN;
    const size_t need = mq_linear_w4a4_workspace_bytes(M, K);
    if (need == 0) return MQ_ERR_SHAPE;
    if (need > (size_t)MQ_NOALLOC_SCRATCH_BYTES) return MQ_ERR_WORKSPACE;
    void* scratch = nullptr;
    int st = scratch_for_current_device(&scratch);
    if (st != MQ_OK) return st;
    // The previous call's contents remain: the header (amax accumulator,
    // block counter, status) must start at zero.
    if (cudaMemsetAsync(scratch, 0, mq::WS_HEADER_BYTES, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return MQ_ERR_CUDA;
    return mq_linear_w4a4(x, M, K, w_codes, w_scales, alpha_w, N, y, scratch, (size_t)MQ_NOALLOC_SCRATCH_BYTES,
                          stream);
}
