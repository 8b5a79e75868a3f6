// mq_nvfp4.cuh -- device-side NVFP4 block quantization, shared by the
// stand-alone quantizer kernel and the quantizer warps of the fused linear.
//
// Per block b of 16 consecutive bf16 elements along K:
//   sigma_b = Pi_E4M3(fl32(amax_b / fl32(6 alpha)))            (round to nearest even, satfinite)
//   q_i     = Pi_E2M1(fl32(x_i * fl32(1 / fl32(alpha sigma_b))))
//   q_i     = +0 for every element when sigma_b = 0
// (NVFP4 two-level microscaling: "Mix-Quant：面向智能体LLM的量化预填充与精确解码",
// section 方法步骤详情, step (3); "Mix-Quant: Quantized Prefilling, Precise
// Decoding for Agentic LLMs", section Method, item 1; q_max = 6, g = 16.)
#pragma once
#include <cuda_fp16.h>

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

// max(|a|, |b|) per bf16 half (the sign bit of the result is junk).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// fl32(x * r) for the two bf16 values packed in w (low half first), IEEE
// round-to-nearest per lane.
__device__ __forceinline__ void scale_bf16x2(uint32_t w, uint64_t rr, float& lo, float& hi) {
    uint64_t xy, d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(xy) : "r"(w << 16), "r"(w & 0xffff0000u));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(xy), "l"(rr));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
}

// Quantizes one 16-element block held as two 16-byte vectors.  Returns the
// E4M3 scale code; writes the eight code bytes as two words (element 0 in
// the low nibble of byte 0).
__device__ __forceinline__ uint32_t quantize_block16(const uint4& v0, const uint4& v1, float alpha,
                                                     uint32_t& c0, uint32_t& c1) {
    uint32_t m = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(v0.x, v0.y), absmax_bf16x2(v0.z, v0.w)),
                               absmax_bf16x2(absmax_bf16x2(v1.x, v1.y), absmax_bf16x2(v1.z, v1.w)));
    m &= 0x7fff7fffu;     // non-negative bf16 patterns order like unsigned integers
    const float amax_b = __uint_as_float(max(m & 0xffffu, m >> 16) << 16);
    // sigma_b = Pi_E4M3(amax_b / (alpha * q_max))
    const float t = __fdiv_rn(amax_b, __fmul_rn(6.0f, alpha));
    const uint32_t sc = cvt_e4m3x2(0.0f, t) & 0xffu;
    const float sigma = __half2float(__ushort_as_half((uint16_t)(cvt_e4m3x2_to_f16x2((uint16_t)sc) & 0xffffu)));
    c0 = 0;
    c1 = 0;
    if (sigma != 0.0f) {
        // q_i = Pi_E2M1(x_i / (alpha * sigma_b)), one reciprocal per block
        const float r = __frcp_rn(__fmul_rn(alpha, sigma));
        uint64_t rr;
        asm("mov.b64 %0, {%1, %1};" : "=l"(rr) : "f"(r));
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float f[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) scale_bf16x2(w[i], rr, f[2 * i], f[2 * i + 1]);
        c0 = cvt_e2m1x8(f[0], f[1], f[2], f[3], f[4], f[5], f[6], f[7]);
        c1 = cvt_e2m1x8(f[8], f[9], f[10], f[11], f[12], f[13], f[14], f[15]);
    }
    return sc;
}

// The per-tensor constants of the table-driven form below, set once alpha
// is known: d = fl32(6 alpha), and rtab[c] = RN(1 / fl32(alpha sigma(c)))
// for every E4M3 code c (entry 0 unused) -- the same operations
// quantize_block16 performs per block, so both forms give the same bits.
struct QuantTab {
    float d;
    const float* rtab;
};

// Fills rtab (128 floats, shared memory) with thread `i` of `n` threads.
__device__ __forceinline__ void fill_recip_table(float* rtab, float alpha, int i, int n) {
    for (int c = i; c < 128; c += n) {
        const float sigma = __half2float(__ushort_as_half((uint16_t)(cvt_e4m3x2_to_f16x2((uint16_t)c) & 0xffffu)));
        rtab[c] = c == 0 ? 0.0f : __frcp_rn(__fmul_rn(alpha, sigma));
    }
}

// quantize_block16 with the same results, fewer instructions: the
// reciprocal of fl32(alpha sigma_b) read from the table instead of computed
// per block, and d = fl32(6 alpha) computed once.
__device__ __forceinline__ uint32_t quantize_block16_tab(const uint4& v0, const uint4& v1, const QuantTab& qt,
                                                         uint32_t& c0, uint32_t& c1) {
    uint32_t m = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(v0.x, v0.y), absmax_bf16x2(v0.z, v0.w)),
                               absmax_bf16x2(absmax_bf16x2(v1.x, v1.y), absmax_bf16x2(v1.z, v1.w)));
    m &= 0x7fff7fffu;
    const float amax_b = __uint_as_float(max(m & 0xffffu, m >> 16) << 16);
    const float t = __fdiv_rn(amax_b, qt.d);
    const uint32_t sc = cvt_e4m3x2(0.0f, t) & 0xffu;
    c0 = 0;
    c1 = 0;
    if (sc != 0) {
        const float r = qt.rtab[sc];
        uint64_t rr;
        asm("mov.b64 %0, {%1, %1};" : "=l"(rr) : "f"(r));
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float f[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) scale_bf16x2(w[i], rr, f[2 * i], f[2 * i + 1]);
        c0 = cvt_e2m1x8(f[0], f[1], f[2], f[3], f[4], f[5], f[6], f[7]);
        c1 = cvt_e2m1x8(f[8], f[9], f[10], f[11], f[12], f[13], f[14], f[15]);
    }
    return sc;
}

// Byte offset of (row, scale column kb) in the MMA scale layout: atoms of
// 128 rows x 4 columns, ordered row-tile major; inside an atom row r sits at
// (r % 32) * 16 + ((r / 32) % 4) * 4 and column kb at kb % 4.
__device__ __forceinline__ int64_t scale_byte_offset(int64_t row, int64_t kb, int64_t katoms) {
    return ((row >> 7) * katoms + (kb >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (kb & 3);
}

}  // namespace mq
