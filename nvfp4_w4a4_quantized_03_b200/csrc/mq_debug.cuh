// mq_debug.cuh -- bounds checks of the debug build of libmq (libmq_debug.so,
// compiled with -DMQ_DEBUG=1; the release build compiles every check to
// `true` and keeps no counter).
//
// A check guards one global-memory access computed from indices, or one TMA
// coordinate.  When it fails, the translation unit's device counter counts a
// hit and the caller skips the access: no kernel traps or faults, the context
// stays usable, and the host reads the count with mq_debug_bounds_hits.
#pragma once
#include <cstdint>

namespace mq {

#ifdef MQ_DEBUG
static __device__ unsigned long long g_bounds_hits;
__device__ __forceinline__ bool debug_check(bool cond) {
    if (!cond) atomicAdd(&g_bounds_hits, 1ull);
    return cond;
}
#define MQ_CHECK(cond) (::mq::debug_check(cond))
// this translation unit's hits since the last read; the counter is cleared
#define MQ_DEBUG_READER(fn)                                                          \
    unsigned long long fn() {                                                        \
        unsigned long long v = 0, z = 0;                                             \
        if (cudaMemcpyFromSymbol(&v, g_bounds_hits, sizeof v) != cudaSuccess) return ~0ull; \
        cudaMemcpyToSymbol(g_bounds_hits, &z, sizeof z);                             \
        return v;                                                                    \
    }
#else
#define MQ_CHECK(cond) (true)
#define MQ_DEBUG_READER(fn) \
    unsigned long long fn() { return 0; }
#endif

// The TMA rule for tiled copies: the innermost coordinate times the element
// size is a multiple of 16 bytes (an unaligned one faults the context), and a
// store never starts at a negative coordinate.
#define MQ_CHECK_TMA_X(x, elem_bytes) MQ_CHECK(((int64_t)(x) * (elem_bytes)) % 16 == 0)
#define MQ_CHECK_TMA_STORE(x, y, elem_bytes) MQ_CHECK(((int64_t)(x) * (elem_bytes)) % 16 == 0 && (x) >= 0 && (y) >= 0)
// A plain bulk copy: 16-byte aligned address and a size that is a multiple of 16.
#define MQ_CHECK_BULK(ptr, bytes) \
    MQ_CHECK((reinterpret_cast<uintptr_t>(ptr) & 15u) == 0 && ((bytes) & 15u) == 0 && (bytes) > 0)

}  // namespace mq
