// mq_quant.cu -- the two HBM-bound passes of NVFP4 quantization.
//
//   k_amax      : amax = max |x| over a bf16 tensor, then the tensor-level
//                 scale alpha_x = fl32(amax / (q_max * 448)) = fl32(amax / 2688)
//                 (alpha_x = 1 for an all-zero tensor).
//   k_quantize  : per 16-element block along K,
//                   sigma_b = Pi_E4M3(fl32(amax_b / fl32(6 alpha_x)))
//                   q_i     = Pi_E2M1(fl32(x_i * fl32(1 / fl32(alpha_x sigma_b))))
//                 codes packed two per byte (lower K index in the low nibble),
//                 scales written straight into the block-scaled MMA's layout.
//
// The formulas are NVFP4's two-level microscaling as given in
// "Mix-Quant：面向智能体LLM的量化预填充与精确解码" (paper.rainbus.top digest),
// section 方法步骤详情, step (3), and in "Mix-Quant: Quantized Prefilling,
// Precise Decoding for Agentic LLMs" (r9-hu digest), section Method, item 1;
// q_max = 6, blocks of g = 16, round to nearest (ties to even, saturating).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "mq_internal.h"
#include "mq_ptx.cuh"

namespace mq {

// max over the two bf16 halves of |w|, kept packed: clearing the sign bits
// leaves non-negative bf16 patterns, which order like unsigned integers.
__device__ __forceinline__ uint32_t absmax2(uint32_t m, uint32_t w) {
    return __vmaxu2(m, w & 0x7fff7fffu);
}

__device__ __forceinline__ uint32_t absmax_vec(uint32_t m, const uint4& v) {
    m = absmax2(m, v.x);
    m = absmax2(m, v.y);
    m = absmax2(m, v.z);
    return absmax2(m, v.w);
}

constexpr int AMAX_THREADS = 512;

// One pass over x (16-byte vectors); every block folds its max into ws with
// one atomic, and the last block to finish turns it into alpha and resets
// the two counters to zero.
__global__ void __launch_bounds__(AMAX_THREADS)
k_amax(const uint4* __restrict__ x, int64_t nvec, const uint16_t* __restrict__ tail, int ntail,
       uint32_t* __restrict__ ws, float* __restrict__ alpha_out) {
    uint32_t m = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        uint4 a = x[i], b = x[i + stride], c = x[i + 2 * stride], d = x[i + 3 * stride];
        m = absmax_vec(m, a);
        m = absmax_vec(m, b);
        m = absmax_vec(m, c);
        m = absmax_vec(m, d);
    }
    for (; i < nvec; i += stride) m = absmax_vec(m, x[i]);
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
        float alpha = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
        *alpha_out = alpha;
    }
}

constexpr int QUANT_THREADS = 256;

// Byte offset of (row, scale column kb) in the MMA scale layout: atoms of
// 128 rows x 4 columns; inside an atom row r sits at (r % 32) * 16 +
// ((r / 32) % 4) * 4 and column kb at kb % 4.
__device__ __forceinline__ int64_t scale_byte_offset(int64_t row, int64_t kb, int64_t katoms) {
    return ((row >> 7) * katoms + (kb >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (kb & 3);
}

// One thread per 16-element block; threads run over the padded row range so
// the padding rows of the scale buffer are written as zeros.
__global__ void __launch_bounds__(QUANT_THREADS)
k_quantize(const uint4* __restrict__ x, int64_t rows, int64_t prows, int64_t K,
           const float* __restrict__ alpha_p, uint2* __restrict__ codes,
           uint8_t* __restrict__ scales) {
    const int64_t nb = K >> 4;
    const int64_t g = (int64_t)blockIdx.x * QUANT_THREADS + threadIdx.x;
    const int64_t row = g / nb, kb = g - row * nb;
    const bool in_pad = g < prows * nb;
    const bool real = row < rows;
    uint32_t sc = 0;
    if (real) {
        const uint4 v0 = x[2 * g], v1 = x[2 * g + 1];
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t m = absmax_vec(absmax_vec(0u, v0), v1);
        const float amax_b = __uint_as_float(max(m & 0xffffu, m >> 16) << 16);
        const float alpha = __ldg(alpha_p);
        // sigma_b = Pi_E4M3(amax_b / (alpha * q_max))
        const float t = __fdiv_rn(amax_b, __fmul_rn(6.0f, alpha));
        sc = cvt_e4m3x2(0.0f, t) & 0xffu;
        const float sigma = __half2float(__ushort_as_half((uint16_t)(cvt_e4m3x2_to_f16x2((uint16_t)sc) & 0xffffu)));
        uint32_t c0 = 0, c1 = 0;
        if (sigma != 0.0f) {
            // q_i = Pi_E2M1(x_i / (alpha * sigma_b)), one reciprocal per block
            const float r = __frcp_rn(__fmul_rn(alpha, sigma));
            float f[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                f[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), r);
                f[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xffff0000u), r);
            }
            c0 = cvt_e2m1x8(f[0], f[1], f[2], f[3], f[4], f[5], f[6], f[7]);
            c1 = cvt_e2m1x8(f[8], f[9], f[10], f[11], f[12], f[13], f[14], f[15]);
        }
        codes[g] = make_uint2(c0, c1);
    }
    // Four consecutive scale columns of one row form one 32-bit word of the
    // layout; lanes 4j..4j+3 hold them (nb is a multiple of 4).
    const uint32_t lane = threadIdx.x & 31;
    uint32_t word = sc << (8 * (lane & 3));
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    if (in_pad && (lane & 3) == 0)
        *reinterpret_cast<uint32_t*>(scales + scale_byte_offset(row, kb, nb >> 2)) = word;
}

cudaError_t launch_amax(const void* x, int64_t numel, uint32_t* ws_words, float* alpha_out,
                        int num_sms, cudaStream_t stream) {
    const int64_t nvec = numel / 8;
    const int ntail = (int)(numel - nvec * 8);
    const uint16_t* tail = reinterpret_cast<const uint16_t*>(x) + nvec * 8;
    int64_t want = (nvec + AMAX_THREADS * 4 - 1) / (AMAX_THREADS * 4);
    int blocks = (int)std::min<int64_t>(std::max<int64_t>(want, 1), (int64_t)num_sms * 4);
    k_amax<<<blocks, AMAX_THREADS, 0, stream>>>(reinterpret_cast<const uint4*>(x), nvec, tail, ntail,
                                               ws_words, alpha_out);
    return cudaGetLastError();
}

cudaError_t launch_quantize(const void* x, int64_t rows, int64_t K, const float* alpha,
                            uint8_t* codes, uint8_t* scales, cudaStream_t stream) {
    const int64_t prows = padded_rows(rows);
    const int64_t threads = prows * (K / 16);
    const int64_t blocks = (threads + QUANT_THREADS - 1) / QUANT_THREADS;
    k_quantize<<<(unsigned)blocks, QUANT_THREADS, 0, stream>>>(
        reinterpret_cast<const uint4*>(x), rows, prows, K, alpha, reinterpret_cast<uint2*>(codes), scales);
    return cudaGetLastError();
}

}  // namespace mq
