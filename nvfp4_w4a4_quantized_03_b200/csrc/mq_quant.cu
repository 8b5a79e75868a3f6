// mq_quant.cu -- the two HBM-bound passes of NVFP4 quantization.
//
//   k_amax                : amax = max |x| over a bf16 tensor, then the
//                           tensor-level scale alpha_x = fl32(amax / (q_max * 448))
//                           = fl32(amax / 2688) (alpha_x = 1 for an all-zero tensor).
//   k_quantize_ws         : per 16-element block along K,
//                             sigma_b = Pi_E4M3(fl32(amax_b / fl32(6 alpha_x)))
//                             q_i     = Pi_E2M1(fl32(x_i * fl32(1 / fl32(alpha_x sigma_b))))
//                           codes packed two per byte (lower K index in the low
//                           nibble), scales written straight into the block-scaled
//                           MMA's layout.
//   k_quantize_onepass_ws : both in one cooperative launch (amax pass, grid
//                           barrier, quantization pass over the data the amax
//                           pass left in L2), for the linear.
//
// The formulas are NVFP4's two-level microscaling as given in
// "Mix-Quant：面向智能体LLM的量化预填充与精确解码" (paper.rainbus.top digest),
// section 方法步骤详情, step (3), and in "Mix-Quant: Quantized Prefilling,
// Precise Decoding for Agentic LLMs" (r9-hu digest), section Method, item 1;
// q_max = 6, blocks of g = 16, round to nearest (ties to even, saturating).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>

#include "mq_debug.cuh"
#include "mq_internal.h"
#include "mq_nvfp4.cuh"

namespace mq {

constexpr int AMAX_THREADS = 512;

// Grid barrier of the one-pass quantizers, taken by one thread per block
// with its block's max |x| (bf16 bit pattern) `w`: the max joins the
// workspace's running max, and the last block to arrive (ticket) writes
// alpha_x, resets the counters and bumps the generation word, which releases
// the others.  The others poll the generation with a growing sleep (32 ns up
// to 256 ns), so their loads do not hold up the counters' atomics; the wait
// gives up after `timeout` cycles (returns false).
__device__ __forceinline__ bool amax_grid_barrier(uint32_t* ws, uint32_t w, uint32_t gen0, float* alpha_out,
                                                  long long timeout) {
    atomicMax(&ws[WS_AMAX_BITS], w);
    __threadfence();
    const uint32_t ticket = atomicAdd(&ws[WS_TICKET], 1u);
    if (ticket == gridDim.x - 1) {
        __threadfence();
        const uint32_t bits = atomicExch(&ws[WS_AMAX_BITS], 0u);
        atomicExch(&ws[WS_TICKET], 0u);
        const float amax = __uint_as_float(bits << 16);
        *alpha_out = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
        __threadfence();
        atomicAdd(&ws[WS_GENERATION], 1u);
        return true;
    }
    const long long t0 = clock64();
    unsigned ns = 32;
    while (ld_acquire_gpu(reinterpret_cast<const int*>(&ws[WS_GENERATION])) == (int)gen0) {
        if (clock64() - t0 > timeout) return false;
        __nanosleep(ns);
        if (ns < 256) ns *= 2;
    }
    return true;
}

// One pass over x (16-byte vectors); every block folds its max into ws with
// one atomic, and the last block to finish turns it into alpha (or, with
// raw_amax, writes max |x| itself) and resets the two counters to zero.
// `clear` (may be null) is zero-filled on the way: the fused linear's
// readiness flags for this call.
__global__ void __launch_bounds__(AMAX_THREADS)
k_amax(const uint4* __restrict__ x, int64_t nvec, const uint16_t* __restrict__ tail, int ntail,
       uint32_t* __restrict__ ws, float* __restrict__ alpha_out, int* __restrict__ clear, int nclear, int raw_amax) {
    pdl_launch_dependents();
    pdl_wait();
    uint32_t m = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t j = i; j < nclear; j += stride) clear[j] = 0;
    // eight independent 16-byte loads in flight per thread on every pass
    for (; i < nvec; i += 8 * stride) {
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = x[min(i + j * stride, nvec - 1)];   // a repeat leaves the max unchanged
#pragma unroll
        for (int j = 0; j < 8; ++j) m = absmax_vec(m, v[j]);
    }
    if (blockIdx.x == 0 && (int)threadIdx.x < ntail) m = absmax2(m, tail[threadIdx.x]);

    uint32_t v = max(m & 0xffffu, m >> 16);
    v = __reduce_max_sync(0xffffffffu, v);
    __shared__ uint32_t red[AMAX_THREADS / 32];
    __shared__ bool last;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < AMAX_THREADS / 32 ? red[lane] : 0u;
        w = __reduce_max_sync(0xffffffffu, w);
        if (lane == 0) {
            atomicMax(&ws[WS_AMAX_BITS], w);
            __threadfence();
            uint32_t ticket = atomicAdd(&ws[WS_TICKET], 1u);
            last = (ticket == gridDim.x - 1);
        }
    }
    __syncthreads();
    if (last && threadIdx.x == 0) {
        __threadfence();
        uint32_t bits = atomicExch(&ws[WS_AMAX_BITS], 0u);
        atomicExch(&ws[WS_TICKET], 0u);
        float amax = __uint_as_float(bits << 16);
        *alpha_out = raw_amax ? amax : ((amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f));
    }
}

// Quantizes the four consecutive 16-element blocks [4q, 4q + 4) of row `row`:
// 128 bytes of x in, 32 code bytes and one 32-bit scale word (the four block
// scales, one word of the MMA layout) out.  Padding rows (row >= rows) get a
// zero scale word.  The 32 code bytes leave in one 256-bit store when the
// codes buffer is 32-byte aligned (every quad then is): one full 32-byte
// sector per request instead of two half-sector writes, which took the
// stand-alone quantizer on 8192 x 12288 from 51 to 45 us (the threads of a
// warp write 32 different rows, so no two stores of a warp share a sector).
__device__ __forceinline__ void quantize_quad(int64_t rows, int64_t K, uint32_t row, uint32_t q, const QuantTab& qt,
                                              uint4* __restrict__ codes, uint8_t* __restrict__ scales,
                                              const uint4 (&v)[8]) {
    uint32_t word = 0;
    if (row < rows) {
        uint32_t c[8];
#pragma unroll
        for (int b = 0; b < 4; ++b) word |= quantize_block16_tab(v[2 * b], v[2 * b + 1], qt, c[2 * b], c[2 * b + 1]) << (8 * b);
        uint4* dst = codes + ((int64_t)row * (K / 64) + q) * 2;      // 32 bytes per quad
        if (!MQ_CHECK(q < (uint32_t)(K / 64))) {
        } else if ((reinterpret_cast<uintptr_t>(codes) & 31) == 0) {
            asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(c[0]), "r"(c[1]),
                         "r"(c[2]), "r"(c[3]), "r"(c[4]), "r"(c[5]), "r"(c[6]), "r"(c[7]) : "memory");
        } else {
            dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
            dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
        }
    }
    if (MQ_CHECK(row < padded_rows(rows) && q < (uint32_t)(K / 64)))
        *reinterpret_cast<uint32_t*>(scales + scale_byte_offset(row, 4 * (int64_t)q, K / 64)) = word;
}

// ---------------------------------------------------------------------------
// The quantizers stream X through shared memory by TMA, 256 rows x 64
// elements (32 KB) per box in the 128-byte swizzle.  Thread t quantizes row t
// of a box (four blocks, one scale word) from its 128-byte row of the box;
// the swizzle puts the 16-byte chunk j of row t at chunk j ^ (t % 8), so the
// eight 16-byte shared-memory reads of a warp are conflict-free.  A ring of
// QT_STAGES boxes per block keeps the loads in flight while earlier boxes are
// quantized; two boxes per block let three blocks share an SM (the same
// 192 KB in flight per SM as three boxes for two blocks, and half again as
// many quantizing warps: the stand-alone quantize pass 2.5-3% faster).
// (Loading the same data with eight 16-byte global loads per thread measured
// the L1 at 90% of its throughput, every warp-wide load touching 32 cache
// lines, and ran 17-23% slower.)
constexpr int QT_THREADS = 256;
constexpr int QT_ROWS = 256;
constexpr int QT_STAGES = 2;
constexpr int QT_BOX_BYTES = QT_ROWS * 128;
constexpr int QT_SMEM = QT_STAGES * QT_BOX_BYTES + 1024;

// ---------------------------------------------------------------------------
// k_quantize_ws: a producer/consumer pipeline (one lane of warp 8 streams
// this block's boxes into the ring as slots free up; warps 0..7 quantize one
// box row per thread and release a slot with one arrival per warp, so no
// warp waits for the slowest one of the block between boxes).  Before a warp releases a slot, each of its threads executes a
// generic-to-async proxy fence: the mbarrier's release/acquire alone does not
// order the threads' shared-memory reads before the next TMA write into the
// slot, and without the fence rows were seen quantized from the next box.
// Every wait is bounded.
constexpr int QW_CONSUMERS = QT_THREADS / 32;
constexpr int QW_THREADS = QT_THREADS + 32;

__global__ void __launch_bounds__(QW_THREADS, 3)
k_quantize_ws(const __grid_constant__ CUtensorMap xmap, int64_t rows, int64_t prows, int64_t K,
              const float* __restrict__ alpha_p, uint4* __restrict__ codes, uint8_t* __restrict__ scales) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[QT_STAGES], empty[QT_STAGES];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t kgroups = K / 64;
    const int64_t ntiles = (prows + QT_ROWS - 1) / QT_ROWS * kgroups;
    const int64_t n = ntiles > blockIdx.x ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;   // boxes of this block
    const long long timeout = 4000000000LL;
    if (threadIdx.x == 0) {
        for (int i = 0; i < QT_STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], QW_CONSUMERS);
        }
        fence_mbar_init();
        prefetch_tmap(&xmap);
    }
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();
    if (warp == QW_CONSUMERS) {
        if (lane == 0) {
            int64_t i = 0;
            for (; i < n; ++i) {
                const int st = (int)(i % QT_STAGES);
                const uint32_t round = (uint32_t)(i / QT_STAGES);
                if (round > 0 && !mbar_wait_bounded(&empty[st], (round - 1) & 1, timeout, nullptr)) break;
                const int64_t t = blockIdx.x + i * gridDim.x;
                mbar_arrive_expect_tx(&full[st], QT_BOX_BYTES);
                if (MQ_CHECK_TMA_X((t % kgroups) * 64, 2))
                    tma_load_2d(base + st * QT_BOX_BYTES, &xmap, &full[st], (int32_t)(t % kgroups) * 64,
                                (int32_t)(t / kgroups) * QT_ROWS);
            }
            // every copy this thread issued lands before the block ends
            for (int64_t j = i > QT_STAGES ? i - QT_STAGES : 0; j < i; ++j)
                mbar_wait_bounded(&full[j % QT_STAGES], (uint32_t)(j / QT_STAGES) & 1, timeout, nullptr);
        }
        return;
    }
    __shared__ float rtab[QW_CONSUMERS][128];       // one table per quantizing warp
    const float alpha = __ldg(alpha_p);
    fill_recip_table(rtab[warp], alpha, lane, 32);
    __syncwarp();
    QuantTab qt;
    qt.d = __fmul_rn(6.0f, alpha);
    qt.rtab = rtab[warp];
    for (int64_t i = 0; i < n; ++i) {
        const int st = (int)(i % QT_STAGES);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[st], (uint32_t)(i / QT_STAGES) & 1, timeout, nullptr)))
            break;
        const uint8_t* src = base + st * QT_BOX_BYTES + threadIdx.x * 128;
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = *reinterpret_cast<const uint4*>(src + ((j ^ (threadIdx.x & 7)) << 4));
        fence_proxy_async_shared();   // the reads are performed before the slot's next TMA load
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);       // this warp is done with the slot
        const int64_t t = blockIdx.x + i * gridDim.x;
        const int64_t row = (t / kgroups) * QT_ROWS + threadIdx.x;
        if (row < prows) quantize_quad(rows, K, (uint32_t)row, (uint32_t)(t % kgroups), qt, codes, scales, v);
    }
}

// ---------------------------------------------------------------------------
// k_quantize_onepass_ws: the same one-pass quantizer as a producer/consumer
// pipeline.  One lane of warp 8 streams the boxes into the ring as soon as a
// slot is free (full/empty mbarriers); warps 0..7 take one box row per thread
// and release a slot with one arrival per warp, so within a phase no warp
// waits for another.  At the phase boundary the warps' maxima meet through an
// mbarrier (one arrival per warp), thread 0 joins the grid barrier, and the
// warps wait for alpha on a second mbarrier.  Every wait is bounded.
__global__ void __launch_bounds__(QW_THREADS, 3)
k_quantize_onepass_ws(const __grid_constant__ CUtensorMap xmap, int64_t rows, int64_t prows, int64_t K,
                      uint32_t* __restrict__ ws, float* __restrict__ alpha_out, uint4* __restrict__ codes,
                      uint8_t* __restrict__ scales, int* __restrict__ status, long long timeout) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[QT_STAGES], empty[QT_STAGES], p1_done, alpha_ready;
    __shared__ uint32_t red[QW_CONSUMERS];
    __shared__ int ok_shared;
    __shared__ float alpha_shared;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t kgroups = K / 64;
    const int64_t ntiles = (prows + QT_ROWS - 1) / QT_ROWS * kgroups;
    const int64_t n = ntiles > blockIdx.x ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;   // boxes of this block
    auto box_of = [&](int64_t item) -> int64_t {   // phase 1: boxes in order; phase 2: the same, reversed
        const int64_t i = item < n ? item : 2 * n - 1 - item;
        return blockIdx.x + i * gridDim.x;
    };
    if (threadIdx.x == 0) {
        for (int i = 0; i < QT_STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], QW_CONSUMERS);
        }
        mbar_init(&p1_done, QW_CONSUMERS);
        mbar_init(&alpha_ready, 1);
        fence_mbar_init();
        prefetch_tmap(&xmap);
        ok_shared = 1;
    }
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();
    if (warp == QW_CONSUMERS) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            int64_t item = 0;
            for (; item < 2 * n; ++item) {
                const int st = (int)(item % QT_STAGES);
                const uint32_t round = (uint32_t)(item / QT_STAGES);
                if (round > 0 && !mbar_wait_bounded(&empty[st], (round - 1) & 1, timeout, nullptr)) break;
                const int64_t t = box_of(item);
                mbar_arrive_expect_tx(&full[st], QT_BOX_BYTES);
                if (MQ_CHECK_TMA_X((t % kgroups) * 64, 2))
                    tma_load_2d(base + st * QT_BOX_BYTES, &xmap, &full[st], (int32_t)(t % kgroups) * 64,
                                (int32_t)(t / kgroups) * QT_ROWS);
            }
            // every copy this thread issued lands before the block ends
            for (int64_t j = item > QT_STAGES ? item - QT_STAGES : 0; j < item; ++j)
                mbar_wait_bounded(&full[j % QT_STAGES], (uint32_t)(j / QT_STAGES) & 1, timeout, nullptr);
        }
        return;
    }
    // -------------------------------------------------------------------- consumers
    const uint32_t gen0 = *reinterpret_cast<volatile uint32_t*>(&ws[WS_GENERATION]);
    uint32_t m = 0;
    float alpha = 0.0f;
    bool ok = true;
    __shared__ float rtab[QW_CONSUMERS][128];       // one table per quantizing warp
    QuantTab qt;
    auto boundary = [&]() {
        const uint32_t v = __reduce_max_sync(0xffffffffu, max(m & 0xffffu, m >> 16));
        if (lane == 0) {
            red[warp] = v;
            mbar_arrive(&p1_done);
        }
        if (threadIdx.x == 0) {
            bool good = mbar_wait_bounded(&p1_done, 0, timeout, nullptr);
            if (good) {
                uint32_t w = 0;
                for (int k = 0; k < QW_CONSUMERS; ++k) w = max(w, red[k]);
                good = amax_grid_barrier(ws, w, gen0, alpha_out, timeout);
            }
            if (!good && status) atomicExch(status, -7 /* MQ_ERR_TIMEOUT */);
            alpha_shared = good ? *reinterpret_cast<volatile float*>(alpha_out) : 0.0f;
            ok_shared = good ? 1 : 0;
            mbar_arrive(&alpha_ready);
        }
        const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(&alpha_ready, 0, timeout, nullptr));
        alpha = alpha_shared;
        fill_recip_table(rtab[warp], alpha, lane, 32);
        __syncwarp();
        qt.d = __fmul_rn(6.0f, alpha);
        qt.rtab = rtab[warp];
        ok = got && ok_shared != 0;
    };
    if (n == 0) boundary();
    for (int64_t item = 0; ok && item < 2 * n; ++item) {
        if (item == n) {
            boundary();
            if (!ok) break;
        }
        const int st = (int)(item % QT_STAGES);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[st], (uint32_t)(item / QT_STAGES) & 1, timeout, nullptr))) {
            if (lane == 0 && status) atomicExch(status, -7);
            break;
        }
        const uint8_t* src = base + st * QT_BOX_BYTES + threadIdx.x * 128;
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = *reinterpret_cast<const uint4*>(src + ((j ^ (threadIdx.x & 7)) << 4));
        fence_proxy_async_shared();   // the reads are performed before the slot's next TMA load
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);       // this warp is done with the slot
        if (item < n) {
#pragma unroll
            for (int j = 0; j < 8; ++j) m = absmax_vec(m, v[j]);
        } else {
            const int64_t t = box_of(item);
            const int64_t row = (t / kgroups) * QT_ROWS + threadIdx.x;
            if (row < prows) quantize_quad(rows, K, (uint32_t)row, (uint32_t)(t % kgroups), qt, codes, scales, v);
        }
    }
}

cudaError_t launch_quantize_onepass(const void* x, int64_t rows, int64_t K, uint32_t* ws_words, float* alpha_out,
                                    uint8_t* codes, uint8_t* scales, int* status, long long timeout_cycles,
                                    cudaStream_t stream) {
    static int per_sm[64] = {};
    static int sms[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int d = dev < 64 ? dev : 63;
    if (!per_sm[d]) {
        cudaError_t e = cudaFuncSetAttribute(k_quantize_onepass_ws, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             QT_SMEM);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm[d], k_quantize_onepass_ws, QW_THREADS, QT_SMEM);
        if (e != cudaSuccess || per_sm[d] <= 0) return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
        cudaDeviceGetAttribute(&sms[d], cudaDevAttrMultiProcessorCount, dev);
    }
    CUtensorMap xmap;
    if (!make_bf16_tile_map(&xmap, x, rows, K, QT_ROWS)) return cudaErrorInvalidValue;
    const int64_t prows = padded_rows(rows);
    // every block resident (the grid barrier needs it: a cooperative launch
    // guarantees it or refuses) and every block owning at least one box
    const int64_t ntiles = (prows + QT_ROWS - 1) / QT_ROWS * (K / 64);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(ntiles, (int64_t)sms[d] * per_sm[d])));
    cfg.blockDim = dim3(QW_THREADS);
    cfg.dynamicSmemBytes = QT_SMEM;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_quantize_onepass_ws, xmap, rows, prows, K, ws_words, alpha_out,
                              reinterpret_cast<uint4*>(codes), scales, status, timeout_cycles);
}

cudaError_t launch_amax(const void* x, int64_t numel, uint32_t* ws_words, float* alpha_out,
                        int num_sms, cudaStream_t stream, int* clear, int nclear, int raw_amax) {
    const int64_t nvec = numel / 8;
    const int ntail = (int)(numel - nvec * 8);
    const uint16_t* tail = reinterpret_cast<const uint16_t*>(x) + nvec * 8;
    int64_t want = (nvec + AMAX_THREADS * 8 - 1) / (AMAX_THREADS * 8);
    int blocks = (int)std::min<int64_t>(std::max<int64_t>(want, 1), (int64_t)num_sms * 4);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    int nattr = 0;
    set_pdl_attr(attr, &nattr);
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(AMAX_THREADS);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = nattr;
    return cudaLaunchKernelEx(&cfg, k_amax, reinterpret_cast<const uint4*>(x), nvec, tail, ntail, ws_words,
                              alpha_out, clear, nclear, raw_amax);
}

// alpha_x = fl32(amax / 2688), or 1 for amax = 0, from a device amax (one thread).
// alpha = fl32(amax / 2688) (1 when amax = 0); `reset`, when given, is
// zeroed after the read (a running maximum ready for the next call).
__global__ void k_alpha_from_amax(const float* amax, float* alpha, uint32_t* reset) {
    pdl_launch_dependents();
    pdl_wait();
    const float a = *amax;
    *alpha = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f);
    if (reset) *reset = 0u;
}

cudaError_t launch_alpha_from_amax(const float* amax, float* alpha, cudaStream_t stream, uint32_t* reset) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    int nattr = 0;
    set_pdl_attr(attr, &nattr);
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(1);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = nattr;
    return cudaLaunchKernelEx(&cfg, k_alpha_from_amax, amax, alpha, reset);
}

cudaError_t launch_quantize(const void* x, int64_t rows, int64_t K, const float* alpha,
                            uint8_t* codes, uint8_t* scales, cudaStream_t stream) {
    static int sms[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int d = dev < 64 ? dev : 63;
    if (!sms[d]) {
        cudaError_t e = cudaFuncSetAttribute(k_quantize_ws, cudaFuncAttributeMaxDynamicSharedMemorySize, QT_SMEM);
        if (e != cudaSuccess) return e;
        cudaDeviceGetAttribute(&sms[d], cudaDevAttrMultiProcessorCount, dev);
    }
    CUtensorMap xmap;
    if (!make_bf16_tile_map(&xmap, x, rows, K, QT_ROWS)) return cudaErrorInvalidValue;
    const int64_t prows = padded_rows(rows);
    const int64_t ntiles = (prows + QT_ROWS - 1) / QT_ROWS * (K / 64);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    int nattr = 0;
    set_pdl_attr(attr, &nattr);
    cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(ntiles, 2 * (int64_t)sms[d])));
    cfg.blockDim = dim3(QW_THREADS);
    cfg.dynamicSmemBytes = QT_SMEM;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = nattr;
    return cudaLaunchKernelEx(&cfg, k_quantize_ws, xmap, rows, prows, K, alpha, reinterpret_cast<uint4*>(codes),
                              scales);
}

MQ_DEBUG_READER(debug_hits_quant)

}  // namespace mq
