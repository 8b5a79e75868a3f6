// mq_gemm.cu -- block-scaled FP4 GEMM for sm_100a.
//
//   Y[m, n] = bf16( fl32(alpha_a * alpha_b) * sum_k (sigma_a q_a)[m, k] (sigma_b q_b)[n, k] )
//
// i.e. the product of the two dequantized NVFP4 operands xhat = alpha sigma q
// ("Mix-Quant：面向智能体LLM的量化预填充与精确解码", section 方法步骤详情,
// step (3); both weights and activations quantized, W4A4), accumulated in
// fp32 by the tensor cores.  A is [M, K] and B is [N, K], both K-major (the
// nn.Linear layout), codes packed two per byte, scales in the MMA layout.
//
// Design: persistent warp-specialised kernel, one CTA per SM, in two forms.
//   PAIR = 1   one CTA computes a 128 x 256 output tile (cta_group::1 MMA).
//   PAIR = 2   a cluster of two CTAs computes a 256 x 256 tile: each CTA
//              stages its own 128 rows of A and its own 128 rows of B, the
//              even CTA issues cta_group::2 MMAs that read both CTAs' shared
//              memory and accumulate 128 rows in each CTA's TMEM.  Per SM
//              this halves B's shared-memory reads and cuts L2 traffic by a
//              third against PAIR = 1.
// Warp roles (both forms):
//   warp 0      producer: per stage, the A/B code tiles (TMA, 128-byte
//               swizzle; in the pair form both CTAs' copies complete on CTA
//               0's `ready` barrier), then the block-scale slices as TMA boxes
//               of the scale array viewed as 64-bit words (A's slice, and B's
//               two slices in one 2-row box), completing on this CTA's
//               sf_full: four copies per stage.
//   warp 1      allocates TMEM; in the (even) CTA the whole warp runs the
//               MMA loop and an elected lane issues tcgen05.mma (K = 64 per
//               instruction, 4 per stage, back to back) and tcgen05.commit
//               to release stages and to publish a tile.
//   warps 2..3  fused linear only (QUANT): quantizer warps.  They quantize the
//               bf16 activation X into A's codes and scales (mq_nvfp4.cuh),
//               32 rows x one K stage at a time, in the order the tile raster
//               consumes them, and publish each 128-row x stage block with a
//               release-add on a global flag; the producer acquires the flag
//               before loading that block, so X is quantized once, inside the
//               GEMM, with HBM bandwidth the GEMM leaves idle.
//   warps 4..7  scale writers: move each stage's block scales from shared
//               memory into that stage's TMEM scale columns with tcgen05.st
//               and arrive on CTA 0's `ready` barrier (one barrier per stage
//               is all the MMA thread waits on),
//               one warp per 32-lane TMEM sub-partition (the MMA reads the
//               scales replicated in all four).  Done off the MMA thread this
//               costs the tensor pipe nothing, where tcgen05.cp issued by the
//               MMA thread measured ~45 cycles per copy, serialised with the
//               MMAs.
//   warps 8..15 epilogue: drain the CTA's 128 x 256 fp32 accumulator into
//               registers (scaled by alpha_a * alpha_b, rounded to bf16),
//               release it to the MMA thread, then store.
// SwiGLU form (pair tiles, mq_nvfp4_gemm_swiglu): B is a [2 inter, K]
// gate/up weight; CTA 0 stages 128 gate rows and CTA 1 the matching 128 up
// rows, so each accumulator holds the gate and up products of the same 128
// output columns; the epilogue rounds both to bf16, applies SwiGLU, writes H
// and raises the running max|h|.
// Every wait on an mbarrier is bounded; on a timeout the kernel records
// MQ_ERR_TIMEOUT in the status word, unwinds every role, waits (bounded) for
// its own copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "../../include/mq.h"
#include "mq_debug.cuh"
#include "mq_internal.h"
#include "mq_nvfp4.cuh"
#include "mq_ptx.cuh"

namespace mq {
namespace gemm {

constexpr int BM = 128;               // A rows per CTA (TMEM lanes)
constexpr int BN = 256;               // accumulator columns (N of one MMA)
constexpr int MMA_K = 64;             // K elements per tcgen05.mma (kind::mxf4nvf4)
constexpr int QUANT_WARPS = 2;
constexpr int SF_WARPS = 4;
constexpr int EPI_WARPS = 8;
constexpr int FIRST_Q_WARP = 2;
constexpr int FIRST_SF_WARP = FIRST_Q_WARP + QUANT_WARPS;     // a warpgroup: one warp per TMEM sub-partition
constexpr int FIRST_EPI_WARP = FIRST_SF_WARP + SF_WARPS;
constexpr int THREADS = (FIRST_EPI_WARP + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t SF_COL = BN;                     // stage st: SF_COL + st * SF_COLS_PER_STAGE
constexpr int GROUP_M = 32;                         // tile raster: at most this many M-blocks per group
constexpr int64_t RASTER_A_BYTES = 18ll << 20;      // ... and at most this much of A (codes and scales)
constexpr int MAX_STAGES = 10;
constexpr int BARRIER_BYTES = 512;
constexpr int SMEM_LIMIT = 232448;                  // dynamic shared memory per block on sm_100

constexpr int BK = 256;                             // K elements per pipeline stage

// PAIR: CTAs per output tile (1 or 2).
template <int PAIR>
struct Cfg {
    static constexpr int NKB = BK / MMA_K;                    // MMAs per stage
    static constexpr int ROW_BYTES = BK / 2;                  // bytes of one code row per stage (the 128-byte swizzle)
    static constexpr int A_BYTES = BM * ROW_BYTES;
    static constexpr int B_ROWS = BN / PAIR;                  // B rows staged by one CTA
    static constexpr int B_BYTES = B_ROWS * ROW_BYTES;
    static constexpr int SFA_BYTES = BM * BK / 16;
    static constexpr int SFB_BYTES = BN * BK / 16;            // scales of all 256 B rows
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr uint32_t SF_COLS_PER_STAGE = 12 * NKB;   // per MMA: A 4 columns, B 8 columns
    static constexpr uint32_t SFB_OFF = 4 * NKB;              // B scales after the A scales of a stage
    // In the pair form Y leaves through shared memory: one 32-row x 64-column
    // bf16 box (4 KB, 128-byte swizzle) per epilogue warp, written out by the
    // warp's own stores (the SwiGLU form's H by TMA stores)
    static constexpr bool TMA_STORE = PAIR == 2;
    static constexpr int EPI_BOX_BYTES = 32 * 64 * 2;
    static constexpr int EPI_BYTES = TMA_STORE ? EPI_WARPS * EPI_BOX_BYTES : 0;
    static constexpr int SMEM_STAGES = (SMEM_LIMIT - 1024 - BARRIER_BYTES - EPI_BYTES) / STAGE_BYTES;
    static constexpr int TMEM_STAGES = (TMEM_COLS - SF_COL) / SF_COLS_PER_STAGE;
    static constexpr int STAGES = SMEM_STAGES < TMEM_STAGES ? (SMEM_STAGES < MAX_STAGES ? SMEM_STAGES : MAX_STAGES)
                                                            : (TMEM_STAGES < MAX_STAGES ? TMEM_STAGES : MAX_STAGES);
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 /*align*/ + BARRIER_BYTES;
    static constexpr int TILE_M = BM * PAIR;
    static constexpr uint32_t SWIZZLE = 2;                            // descriptor layout: 128-byte swizzle
    static constexpr uint32_t SBO = 8 * ROW_BYTES;                    // 8-row swizzle atom
    // Instruction descriptor of kind::mxf4nvf4: E2M1 x E2M1, UE4M3 scales,
    // K-major A and B, M = TILE_M, N = 256, dense K = 64.
    static constexpr uint32_t IDESC = (1u << 7)            // A format E2M1
                                    | (1u << 10)           // B format E2M1
                                    | ((uint32_t)(BN >> 3) << 17)
                                    | (0u << 23)           // scale format UE4M3
                                    | ((uint32_t)(TILE_M >> 4) << 24);
    static_assert(NKB == 4 && ROW_BYTES == 128, "stage depth: four MMAs, 128-byte code rows");
    static_assert(STAGES >= 2 && STAGES <= MAX_STAGES, "stage count");
    static_assert(SF_COL + STAGES * SF_COLS_PER_STAGE <= TMEM_COLS, "TMEM budget");
    static_assert(STAGE_BYTES % 1024 == 0, "stage alignment for the swizzle atoms");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory");
};

struct Params {
    const uint8_t* a_scales;
    const uint8_t* b_scales;
    const float* alpha_a;
    const float* alpha_b;
    __nv_bfloat16* y;
    int M, N, K;
    int m_blocks, n_blocks, tiles, k_stages, kblocks, katoms, a_row_tiles, b_row_tiles;
    int* status;
    long long timeout;
    int fault_skip_first_load;
    int y_tma;               // pair form: Y leaves through staged boxes (tmap_y is valid; needs N % 8 == 0)
    int group_m;             // tile raster: M-blocks per group (tiles walk N inside a group)
    int stages;              // pipeline stages in use (2 .. Cfg::STAGES)
    const uint16_t* x;       // fused linear: bf16 activation [M, K]
    uint8_t* x_codes;        // fused linear: where A's codes are written
    uint8_t* x_scales;       // fused linear: where A's scales are written
    int* flags;              // fused linear: [a_row_tiles][k_stages] slab counts
    int inter;               // SwiGLU form: gate rows [0, inter), up rows [inter, 2 inter) of B
    uint32_t* h_amax;        // SwiGLU form: running max of |h| (binary32 bits)
};

struct Smem {
    // ready[s] (used in CTA 0): the stage's A and B codes landed in both CTAs
    // (TMA bytes) and every scale writer put its scales into TMEM (arrivals)
    uint64_t ready[MAX_STAGES];
    uint64_t sf_full[MAX_STAGES];    // this CTA's block scales of a stage landed
    uint64_t empty[MAX_STAGES];      // the stage's MMAs completed
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

// SwiGLU of the MLP (gate/up product -> the down projection's input), on
// the bf16 values the plain GEMM would write:
//   h = bf16(fl32(silu(g) u)),  silu(g) = fl32(g / fl32(1 + e(-g))),
// e(x) the binary32 exponential by Cody and Waite's range reduction
// (x = k ln2 + r with ln2 split into a 16-bit head and a tail, |r| <= ln2/2)
// and the Taylor polynomial of e^r to degree 7, each step one IEEE binary32
// operation; +inf above 88, 0 below -87 (2^k stays a normal number).
// Two lanes at once: the binary32 pair instructions (fma.rn.f32x2,
// mul.rn.f32x2) round each lane exactly as the scalar ones do, so the pair
// form gives the same bits as the step-by-step definition above.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
    return v;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// e(x0), e(x1): x clamped to [-87, 88] for the arithmetic (2^k normal, k an
// exact small integer), the out-of-range lanes then set to +inf / 0
__device__ __forceinline__ void exp_cw2(float x0, float x1, float& e0, float& e1) {
    const float c0 = fminf(fmaxf(x0, -87.0f), 88.0f), c1 = fminf(fmaxf(x1, -87.0f), 88.0f);
    float t0, t1;
    f2_split(f2_mul(f2(c0, c1), f2(0x1.715476p+0f, 0x1.715476p+0f)), t0, t1);
    const float k0 = rintf(t0), k1 = rintf(t1);
    const uint64_t nk = f2(-k0, -k1);
    uint64_t r = f2_fma(nk, f2(0x1.62e4p-1f, 0x1.62e4p-1f), f2(c0, c1));
    r = f2_fma(nk, f2(0x1.7f7d1cp-20f, 0x1.7f7d1cp-20f), r);
    uint64_t e = f2(0x1.a01a02p-13f, 0x1.a01a02p-13f);
    e = f2_fma(e, r, f2(0x1.6c16c2p-10f, 0x1.6c16c2p-10f));
    e = f2_fma(e, r, f2(0x1.111112p-7f, 0x1.111112p-7f));
    e = f2_fma(e, r, f2(0x1.555556p-5f, 0x1.555556p-5f));
    e = f2_fma(e, r, f2(0x1.555556p-3f, 0x1.555556p-3f));
    e = f2_fma(e, r, f2(0.5f, 0.5f));
    e = f2_fma(e, r, f2(1.0f, 1.0f));
    e = f2_fma(e, r, f2(1.0f, 1.0f));
    e = f2_mul(e, f2(__int_as_float(((int)k0 + 127) << 23), __int_as_float(((int)k1 + 127) << 23)));
    f2_split(e, e0, e1);
    if (x0 > 88.0f) e0 = __int_as_float(0x7f800000);
    if (x0 < -87.0f) e0 = 0.0f;
    if (x1 > 88.0f) e1 = __int_as_float(0x7f800000);
    if (x1 < -87.0f) e1 = 0.0f;
}

// two bf16 pairs (g, u packed as bf16x2) -> h packed as bf16x2
__device__ __forceinline__ uint32_t swiglu_bf16x2(uint32_t g2, uint32_t u2) {
    const float g0 = __uint_as_float(g2 << 16), g1 = __uint_as_float(g2 & 0xffff0000u);
    float e0, e1, d0, d1;
    exp_cw2(-g0, -g1, e0, e1);
    f2_split(f2_fma(f2(e0, e1), f2(1.0f, 1.0f), f2(1.0f, 1.0f)), d0, d1);     // 1 + e, one rounding each
    const uint64_t s = f2(__fdiv_rn(g0, d0), __fdiv_rn(g1, d1));
    float h0, h1;
    f2_split(f2_mul(s, f2(__uint_as_float(u2 << 16), __uint_as_float(u2 & 0xffff0000u))), h0, h1);
    return cvt_bf16x2(h1, h0);
}

__device__ __forceinline__ void tile_coords(int tile, const Params& p, int& mb, int& nb) {
    const int group = p.group_m * p.n_blocks;
    const int first_m = (tile / group) * p.group_m;
    const int gm = min(p.group_m, p.m_blocks - first_m);
    const int in = tile % group;
    mb = first_m + in % gm;
    nb = in / gm;
}

__device__ __forceinline__ void raise_abort(Smem* s, const Params& p) {
    *(volatile int*)&s->abort_flag = 1;
    if (p.status) atomicExch(p.status, -7 /* MQ_ERR_TIMEOUT */);
}

// Arrive on a barrier of the even CTA of the pair (or on the local one).
template <int PAIR>
__device__ __forceinline__ void arrive_leader(uint64_t* bar) {
    if (PAIR == 2) mbar_arrive_remote(mapa_shared(smem_u32(bar), 0));
    else mbar_arrive(bar);
}

template <int PAIR>
__device__ __forceinline__ void commit_to_all(uint64_t* bar) {
    if (PAIR == 2) mma_commit_pair_mc(bar, 0x3);
    else mma_commit(bar);
}

template <int PAIR, bool QUANT, bool SWIGLU>
__global__ void __launch_bounds__(THREADS, 1)
k_gemm(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
       const __grid_constant__ CUtensorMap tmap_y, const __grid_constant__ CUtensorMap tmap_sfb,
       const __grid_constant__ CUtensorMap tmap_sfa, Params p) {
    using C = Cfg<PAIR>;
    constexpr int NKB = C::NKB;
    constexpr int A_BYTES = C::A_BYTES;
    constexpr int SFA_BYTES = C::SFA_BYTES;
    constexpr int SFB_BYTES = C::SFB_BYTES;
    constexpr uint32_t SF_COLS_PER_STAGE = C::SF_COLS_PER_STAGE;
    constexpr uint32_t SFB_OFF = C::SFB_OFF;
    static_assert(sizeof(Smem) <= BARRIER_BYTES, "barrier area");
    static_assert(!SWIGLU || (PAIR == 2 && !QUANT && C::B_ROWS == 128), "SwiGLU form: pair tiles, gate | up halves");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* epi_stage = base + C::STAGES * C::STAGE_BYTES;          // 1024-byte aligned
    Smem* s = reinterpret_cast<Smem*>(epi_stage + C::EPI_BYTES);
    auto stage_a = [&](int st) { return base + st * C::STAGE_BYTES; };
    auto stage_b = [&](int st) { return base + st * C::STAGE_BYTES + A_BYTES; };
    auto stage_sfa = [&](int st) { return base + st * C::STAGE_BYTES + A_BYTES + C::B_BYTES; };
    auto stage_sfb = [&](int st) { return base + st * C::STAGE_BYTES + A_BYTES + C::B_BYTES + SFA_BYTES; };

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = PAIR == 2 ? cluster_ctarank() : 0;     // 0: the CTA that issues MMAs
    const int unit = blockIdx.x / PAIR;                         // tile-processing unit (CTA or pair)
    const int units = gridDim.x / PAIR;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::STAGES; ++i) {
            mbar_init(&s->ready[i], 1 + SF_WARPS * PAIR);   // producer of CTA 0 + scale writers
            mbar_init(&s->sf_full[i], 1);
            mbar_init(&s->empty[i], 1);
        }
        mbar_init(&s->acc_full, 1);
        mbar_init(&s->acc_empty, EPI_WARPS * PAIR);
        mbar_init(&s->drain, 1);
        s->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        if (C::TMA_STORE && p.y_tma) prefetch_tmap(&tmap_y);
        prefetch_tmap(&tmap_sfb);
        prefetch_tmap(&tmap_sfa);
    }
    if (warp == 1) {
        if (PAIR == 2) {
            tmem_alloc_pair(&s->tmem_base, TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&s->tmem_base, TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR == 2) cluster_sync();      // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = s->tmem_base;
    const volatile int* abort_flag = &s->abort_flag;
    // the next grid may start its set-up; this one touches global memory only
    // once the grids before it are done
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int st = 0;
            uint32_t phase = 0;
            uint32_t pending = 0;           // stages with a load in flight
            uint32_t pending_phase = 0;     // parity of that load's phase
            bool skip = p.fault_skip_first_load != 0;
            for (int tile = unit; tile < p.tiles && !*abort_flag; tile += units) {
                int mb, nb;
                tile_coords(tile, p, mb, nb);
                const int arow = mb * C::TILE_M + (int)rank * BM;          // this CTA's A rows
                // this CTA's B rows (SwiGLU form: CTA 0 the gate rows, CTA 1 the matching up rows)
                const int brow = SWIGLU ? (int)rank * p.inter + nb * 128 : nb * BN + (int)rank * C::B_ROWS;
                // scale rows past the padded end feed only discarded outputs
                const int64_t at = min(arow / 128, p.a_row_tiles - 1);
                for (int kt = 0; kt < p.k_stages; ++kt) {
                    if (!mbar_wait_bounded(&s->empty[st], phase ^ 1, p.timeout, abort_flag)) {
                        raise_abort(s, p);
                        break;
                    }
                    pending &= ~(1u << st);
                    if (skip || !MQ_CHECK_TMA_X(kt * C::ROW_BYTES, 1) || !MQ_CHECK_TMA_X(kt * NKB * 64, 8)) {
                        // failure-detection test hook (or, in the debug build, a
                        // coordinate the TMA would refuse): never complete this stage
                        skip = false;
                    } else {
                        const int64_t ka = (int64_t)kt * NKB;              // first k-atom of the stage
                        // The code tiles first: they take longest to land (the
                        // scales need less than half as long, copy and TMEM
                        // store included).
                        uint32_t bar0 = 0;
                        if (PAIR == 2) {
                            // both CTAs' code tiles complete on CTA 0's barrier
                            if (rank == 0) mbar_arrive_expect_tx(&s->ready[st], 2 * (A_BYTES + C::B_BYTES));
                            bar0 = mapa_shared(smem_u32(&s->ready[st]), 0);
                            tma_load_2d_pair(stage_b(st), &tmap_b, bar0, kt * C::ROW_BYTES, brow);
                            if (!QUANT) tma_load_2d_pair(stage_a(st), &tmap_a, bar0, kt * C::ROW_BYTES, arow);
                        } else {
                            mbar_arrive_expect_tx(&s->ready[st], A_BYTES + C::B_BYTES);
                            tma_load_2d(stage_b(st), &tmap_b, &s->ready[st], kt * C::ROW_BYTES, brow);
                            if (!QUANT) tma_load_2d(stage_a(st), &tmap_a, &s->ready[st], kt * C::ROW_BYTES, arow);
                        }
                        // the scale slices: B's two 128-row slices in one box
                        // (rows nb*2, nb*2+1 of the [row tile][k atom] array;
                        // SwiGLU form: the gate slice and the matching up
                        // slice in one box of a 3-D view), then A's slice; the
                        // boxes always land whole, zero past the ends
                        mbar_arrive_expect_tx(&s->sf_full[st], SFB_BYTES + SFA_BYTES);
                        if (SWIGLU)
                            tma_load_3d(stage_sfb(st), &tmap_sfb, &s->sf_full[st], (int)(ka * 64), nb, 0);
                        else
                            tma_load_2d(stage_sfb(st), &tmap_sfb, &s->sf_full[st], (int)(ka * 64), nb * 2);
                        if (QUANT && arow / 128 < p.a_row_tiles) {
                            // A's block (arow, kt) is written by quantizer warps (of any CTA)
                            const int* f = p.flags + (int64_t)(arow / 128) * p.k_stages + kt;
                            if (ld_acquire_gpu(f) < 4) {
                                const long long t0 = clock64();
                                while (ld_acquire_gpu(f) < 4) {
                                    if (*abort_flag || clock64() - t0 > p.timeout) { raise_abort(s, p); break; }
                                }
                            }
                            fence_proxy_async_global();
                        }
                        tma_load_2d(stage_sfa(st), &tmap_sfa, &s->sf_full[st], (int)(ka * 64), (int)at);
                        if (QUANT) {
                            if (PAIR == 2) tma_load_2d_pair(stage_a(st), &tmap_a, bar0, kt * C::ROW_BYTES, arow);
                            else tma_load_2d(stage_a(st), &tmap_a, &s->ready[st], kt * C::ROW_BYTES, arow);
                        }
                        pending |= 1u << st;
                        pending_phase = (pending_phase & ~(1u << st)) | (phase << st);
                    }
                    if (++st == p.stages) { st = 0; phase ^= 1; }
                }
            }
            if (*abort_flag) {
                // Let the copies this thread issued land before the CTA
                // releases its shared memory: a stage's scale copies complete
                // its sf_full barrier by themselves; its code tiles were
                // issued right after them and get a short grace period (their
                // `ready` barrier also needs scale-writer arrivals that an
                // aborted pipeline no longer makes).
                for (int i = 0; i < C::STAGES; ++i)
                    if (pending & (1u << i))
                        mbar_wait_bounded(&s->sf_full[i], (pending_phase >> i) & 1, p.timeout, nullptr);
                const long long t0 = clock64();
                while (clock64() - t0 < 200000) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop, so its state (stage, phase, the
        // operands) is warp-uniform; one elected lane issues the MMAs and the
        // commits.  With a single lane running it alone, the per-stage issue
        // took ~360 SM cycles instead of ~200 (clock64 traces): the
        // operands had to be moved into place before every MMA.
        const bool leader = elect_one();
        if (rank == 0) {
            int st = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int tile = unit; tile < p.tiles && !*abort_flag; tile += units) {
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s->acc_empty, acc_phase ^ 1, p.timeout, abort_flag))) {
                    if (leader) raise_abort(s, p);
                    break;
                }
                tc_fence_after();
                // Per stage: wait for the stage (its codes in shared memory,
                // its scales in TMEM), then its MMAs back to back, then the
                // commit that frees the stage.  Any other instruction between
                // two MMAs -- even a branch not taken, let alone a barrier
                // poll or operand arithmetic -- costs the tensor pipe 30-60
                // cycles per MMA (clock64 traces: 773 SM cycles per 4-MMA
                // stage with the next stage's wait placed before the last MMA,
                // 700 with the wait at the boundary, 656 with the operands
                // computed ahead, ~590 issued by the whole warp, where the
                // per-SM load intake becomes the limit), so the waits sit only
                // at stage boundaries and the next stage's operands are
                // computed while the current stage's MMAs run.
                bool ok = true;
                // operands of a stage: both descriptors and both scale addresses of each MMA
                uint64_t opa[NKB], opb[NKB];
                uint32_t osa[NKB], osb[NKB];
                auto prep = [&](int stg) {
                    const uint64_t ad0 = smem_desc(smem_u32(stage_a(stg)), 16, C::SBO, C::SWIZZLE);
                    const uint64_t bd0 = smem_desc(smem_u32(stage_b(stg)), 16, C::SBO, C::SWIZZLE);
                    const uint32_t sf = tmem + SF_COL + stg * SF_COLS_PER_STAGE;
#pragma unroll
                    for (int kb = 0; kb < NKB; ++kb) {
                        opa[kb] = ad0 + (uint64_t)(kb * (MMA_K / 2) >> 4);
                        opb[kb] = bd0 + (uint64_t)(kb * (MMA_K / 2) >> 4);
                        osa[kb] = sf + kb * 4;
                        osb[kb] = sf + SFB_OFF + kb * 8;
                    }
                };
                auto mma = [&](int kb, uint32_t acc) {
                    if (PAIR == 2)
                        mma_mxf4nvf4_pair(tmem + ACC_COL, opa[kb], opb[kb], C::IDESC, osa[kb], osb[kb], acc);
                    else
                        mma_mxf4nvf4(tmem + ACC_COL, opa[kb], opb[kb], C::IDESC, osa[kb], osb[kb], acc);
                };
                prep(st);
                const int full_stages = p.kblocks / NKB;        // stages with all NKB MMAs
                for (int kt = 0; kt < p.k_stages; ++kt) {
                    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s->ready[st], phase, p.timeout, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (leader) {
                        if (kt < full_stages) {
                            mma(0, kt != 0);
                            mma(1, 1u);
                            mma(2, 1u);
                            mma(3, 1u);
                        } else {
                            const int nkb = p.kblocks - kt * NKB;
#pragma unroll
                            for (int kb = 0; kb < NKB; ++kb)
                                if (kb < nkb) mma(kb, (kt | kb) != 0);
                        }
                        commit_to_all<PAIR>(&s->empty[st]);
                    }
                    __syncwarp();
                    st = st + 1 == p.stages ? 0 : st + 1;
                    phase = st == 0 ? phase ^ 1 : phase;
                    prep(st);
                }
                if (!ok) {
                    if (leader) raise_abort(s, p);
                    break;
                }
                if (leader) commit_to_all<PAIR>(&s->acc_full);
                __syncwarp();
                acc_phase ^= 1;
            }
            // no MMA may still be running when TMEM is released
            if (leader) {
                if (PAIR == 2) mma_commit_pair_mc(&s->drain, 0x1);
                else mma_commit(&s->drain);
            }
            __syncwarp();
            mbar_wait_bounded(&s->drain, 0, p.timeout, nullptr);
        }
    } else if (warp < FIRST_SF_WARP) {
        // ------------------------------------------------------------ quantizer warps (fused linear)
        if constexpr (QUANT) {
            // A unit is 32 rows x one K stage (BK elements, BK / 16 blocks per
            // row).  Units are numbered in the order the tile raster consumes
            // them: raster group of group_m tile rows, then K stage, then
            // 32-row slab; unit u goes to quantizer warp u mod (all warps).
            static_assert(BK == 256, "the fused quantizer maps one lane to each of a row's 16 blocks");
            const int qw = blockIdx.x * QUANT_WARPS + (warp - FIRST_Q_WARP);
            const int nqw = gridDim.x * QUANT_WARPS;
            const int slabs = p.a_row_tiles * 4;
            const int slabs_per_group = p.group_m * C::TILE_M / 32;
            const int64_t per_group = (int64_t)slabs_per_group * p.k_stages;
            const int64_t units = (int64_t)slabs * p.k_stages;
            const float alpha = *p.alpha_a;
            const int nblk = p.K / 16;
            const int half = lane >> 4;             // which of the two rows of an iteration
            const int kbl = lane & 15;              // block column within the stage
            for (int64_t u = qw; u < units; u += nqw) {
                if (*abort_flag) break;
                const int g = (int)(u / per_group);
                const int first = g * slabs_per_group;
                const int ns = min(slabs_per_group, slabs - first);
                const int64_t ul = u - (int64_t)g * per_group;
                const int kt = (int)(ul / ns);
                const int slab = first + (int)(ul % ns);
                const int kb = kt * (BK / 16) + kbl;
                const bool col_ok = kb < nblk;
#pragma unroll 1
                for (int batch = 0; batch < 2; ++batch) {
                    uint4 v[8][2];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int row = slab * 32 + (batch * 8 + j) * 2 + half;
                        if (row < p.M && col_ok && MQ_CHECK((int64_t)row * p.K + kb * 16 + 16 <= (int64_t)p.M * p.K)) {
                            const uint4* src = reinterpret_cast<const uint4*>(p.x + (int64_t)row * p.K + kb * 16);
                            v[j][0] = src[0];
                            v[j][1] = src[1];
                        } else {
                            v[j][0] = make_uint4(0, 0, 0, 0);
                            v[j][1] = make_uint4(0, 0, 0, 0);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int row = slab * 32 + (batch * 8 + j) * 2 + half;
                        uint32_t c0 = 0, c1 = 0, sc = 0;
                        if (row < p.M && col_ok) {
                            sc = quantize_block16(v[j][0], v[j][1], alpha, c0, c1);
                            if (MQ_CHECK((int64_t)row * (p.K / 2) + kb * 8 + 8 <= (int64_t)p.M * (p.K / 2)))
                                *reinterpret_cast<uint2*>(p.x_codes + (int64_t)row * (p.K / 2) + kb * 8) =
                                    make_uint2(c0, c1);
                        }
                        // four consecutive block columns form one 32-bit scale word
                        uint32_t word = sc << (8 * (kbl & 3));
                        word |= __shfl_xor_sync(0xffffffffu, word, 1);
                        word |= __shfl_xor_sync(0xffffffffu, word, 2);
                        if ((kbl & 3) == 0 && col_ok &&
                            MQ_CHECK(row < p.a_row_tiles * 128 && kb / 4 < p.katoms))
                            *reinterpret_cast<uint32_t*>(p.x_scales + scale_byte_offset(row, kb, p.katoms)) = word;
                    }
                }
                __threadfence();
                __syncwarp();
                if (lane == 0) red_release_gpu_add(p.flags + (int64_t)(slab / 4) * p.k_stages + kt, 1);
            }
        }
    } else if (warp < FIRST_EPI_WARP) {
        // ------------------------------------------------------------ scale writers
        // Lane l of the warp owning TMEM sub-partition q writes row l of each
        // 512-byte scale atom (16 bytes: rows l, l+32, l+64, l+96 of the tile,
        // 4 scales each) into 4 consecutive columns of TMEM lane 32q + l.
        const int quad = warp & 3;
        int st = 0;
        uint32_t phase = 0;
        for (int tile = unit; tile < p.tiles; tile += units) {
            bool ok = true;
            for (int kt = 0; kt < p.k_stages; ++kt) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s->sf_full[st], phase, p.timeout, abort_flag));
                if (!ok) break;
                const uint8_t* sfa = stage_sfa(st) + lane * 16;
                const uint8_t* sfb = stage_sfb(st) + lane * 16;
                const uint32_t t = tmem + ((uint32_t)(quad * 32) << 16) + SF_COL + st * SF_COLS_PER_STAGE;
                // The stage's 12 NKB scale columns are contiguous in TMEM: A's
                // (4 per MMA), then B's (8 per MMA).  All shared-memory reads
                // first, then one store per operand.  In a K-tail stage the
                // columns past the last MMA get the boxes' zero fill, which
                // nothing reads.
                uint32_t va[4 * NKB], vb[8 * NKB];
#pragma unroll
                for (int kb = 0; kb < NKB; ++kb) {
                    const uint4 a4 = *reinterpret_cast<const uint4*>(sfa + kb * 512);
                    const uint4 b0 = *reinterpret_cast<const uint4*>(sfb + kb * 512);
                    const uint4 b1 = *reinterpret_cast<const uint4*>(sfb + SFB_BYTES / 2 + kb * 512);
                    va[4 * kb] = a4.x; va[4 * kb + 1] = a4.y; va[4 * kb + 2] = a4.z; va[4 * kb + 3] = a4.w;
                    vb[8 * kb] = b0.x; vb[8 * kb + 1] = b0.y; vb[8 * kb + 2] = b0.z; vb[8 * kb + 3] = b0.w;
                    vb[8 * kb + 4] = b1.x; vb[8 * kb + 5] = b1.y; vb[8 * kb + 6] = b1.z; vb[8 * kb + 7] = b1.w;
                }
                tmem_st_32x32b_x16(t, va);
                tmem_st_32x32b_x32(t + SFB_OFF, vb);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive_leader<PAIR>(&s->ready[st]);
                if (++st == p.stages) { st = 0; phase ^= 1; }
            }
            if (!ok) {
                if (lane == 0) raise_abort(s, p);
                break;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quad = warp & 3;                          // TMEM lanes this warp may read
        const int half = (warp - FIRST_EPI_WARP) / 4;       // which 128 accumulator columns
        const float ab = __fmul_rn(__ldg(p.alpha_a), __ldg(p.alpha_b));
        const bool vec_ok = (p.N % 8) == 0;
        uint32_t acc_phase = 0;
        for (int tile = unit; tile < p.tiles; tile += units) {
            // warp-uniform decisions: tcgen05.ld below is .sync.aligned
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            int mb, nb;
            tile_coords(tile, p, mb, nb);
            const bool ok = mbar_wait_bounded(&s->acc_full, acc_phase, p.timeout, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) raise_abort(s, p);
                break;
            }
            tc_fence_after();
            const int row = mb * C::TILE_M + (int)rank * BM + quad * 32 + lane;
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + ACC_COL + half * 128;
            const int colh = nb * BN + half * 128;
            if constexpr (SWIGLU) {
                // Gate columns [64 half, 64 half + 64) of the accumulator and
                // the up columns 128 above them, for this warp's 32 rows: G and
                // U are rounded to bf16 as the plain GEMM would write them,
                // TMEM goes back to the MMA thread once the four 32-column
                // loads have landed, then h = SwiGLU(G, U) leaves as one
                // 32 x 64 box of H [M, inter] (columns 128 nb + 64 half) and
                // max|h| joins the tensor's running maximum.
                uint8_t* box = epi_stage + (warp - FIRST_EPI_WARP) * C::EPI_BOX_BYTES;
                const uint32_t box_row = smem_u32(box) + lane * 128;
                const int row0 = mb * C::TILE_M + (int)rank * BM + quad * 32;
                const uint32_t tg = tmem + ((uint32_t)(quad * 32) << 16) + ACC_COL + half * 64;
                const uint32_t tu = tg + 128;
                auto convert = [&](const uint32_t (&r)[32], uint32_t (&pk)[16]) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pk[j] = cvt_bf16x2(__fmul_rn(__uint_as_float(r[2 * j + 1]), ab),
                                           __fmul_rn(__uint_as_float(r[2 * j]), ab));
                };
                if (lane == 0) bulk_wait_group_read0();         // the previous tile's box has been read
                __syncwarp();
                uint32_t ra[32], rb[32], gq[2][16], uq[2][16];
                tmem_ld_32x32b_x32(tg, ra);
                tmem_ld_wait_regs(ra);
                tmem_ld_32x32b_x32(tu, rb);
                convert(ra, gq[0]);
                tmem_ld_wait_regs(rb);
                tmem_ld_32x32b_x32(tg + 32, ra);
                convert(rb, uq[0]);
                tmem_ld_wait_regs(ra);
                tmem_ld_32x32b_x32(tu + 32, rb);
                convert(ra, gq[1]);
                tmem_ld_wait_regs(rb);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive_leader<PAIR>(&s->acc_empty);
                convert(rb, uq[1]);
                uint32_t hmax = 0;                              // max |h| as a bf16 bit pattern
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t hq[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        hq[j] = swiglu_bf16x2(gq[c][j], uq[c][j]);
                        hmax = max(hmax, max(hq[j] & 0x7fffu, (hq[j] >> 16) & 0x7fffu));
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        st_shared_v4(box_row + (((c * 4 + q) ^ (lane & 7)) << 4), hq[4 * q], hq[4 * q + 1],
                                     hq[4 * q + 2], hq[4 * q + 3]);
                }
                fence_proxy_async_shared();
                __syncwarp();
                const int hcol = nb * 128 + half * 64;
                if (lane == 0 && row0 < p.M && MQ_CHECK_TMA_STORE(hcol, row0, 2)) {
                    tma_store_2d(&tmap_y, box, hcol, row0);
                    bulk_commit_group();
                }
                // rows past M hold h = 0 (A reads as zero there)
                hmax = __reduce_max_sync(0xffffffffu, hmax);
                if (lane == 0 && hmax != 0) atomicMax(p.h_amax, hmax << 16);
            } else if (C::TMA_STORE && p.y_tma) {
                // This warp's 32 x 128 block of the accumulator leaves as two
                // 32 x 64 bf16 boxes through the warp's staging buffer.  The
                // four 32-column TMEM loads are double-buffered (chunk c + 1
                // loads while chunk c is scaled, rounded and staged); TMEM goes
                // back to the MMA thread as soon as the last load has landed.
                // A staged box leaves through the warp's own 16-byte global
                // stores, 8 lanes per 128-byte row and 4 rows per instruction
                // (rows >= M and columns >= N skipped), not through a TMA
                // store: the SM's TMA unit also issues the producer's loads,
                // and 16 store boxes per CTA and tile queued in it delayed the
                // next tile's first stages (the launch 2.5% faster; leaving
                // Y out altogether, a timing-only copy, gained 4%).
                // Every CTA pair reaches its tile boundary at about the same
                // time, so, except on the CTA's last tile (where a delay would
                // only lengthen the launch), the epilogue warps also space
                // their stores over the next tile's first microseconds: warp
                // w's first box after w x 200 ns, its second 1.6 us later
                // (+2.6% on the four 8192-token projections with TMA stores,
                // medians of 31 interleaved rounds; gate/up +4%).
                const bool pace = tile + units < p.tiles;
                uint8_t* box = epi_stage + (warp - FIRST_EPI_WARP) * C::EPI_BOX_BYTES;
                const uint32_t box_row = smem_u32(box) + lane * 128;
                const int row0 = mb * C::TILE_M + (int)rank * BM + quad * 32;
                // 16-byte chunk j of a 128-byte box row sits at chunk j ^ (row % 8)
                auto stage_chunk = [&](int j, const uint32_t* v) {
                    st_shared_v4(box_row + ((j ^ (lane & 7)) << 4), v[0], v[1], v[2], v[3]);
                };
                auto issue = [&](int h) {
                    __syncwarp();                               // the box is staged
                    const int col = colh + h * 64 + (lane & 7) * 8;
#pragma unroll
                    for (int it = 0; it < 8; ++it) {
                        const int r = it * 4 + (lane >> 3);
                        const uint4 v = ld_shared_v4(smem_u32(box) + r * 128 + (((lane & 7) ^ (r & 7)) << 4));
                        const int grow = row0 + r;
                        if (grow < p.M && col < p.N && MQ_CHECK((int64_t)grow * p.N + col + 8 <= (int64_t)p.M * p.N))
                            *reinterpret_cast<uint4*>(p.y + (int64_t)grow * p.N + col) = v;
                    }
                    __syncwarp();                               // the box may be staged again
                };
                auto convert = [&](const uint32_t (&r)[32], uint32_t (&pk)[16]) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pk[j] = cvt_bf16x2(__fmul_rn(__uint_as_float(r[2 * j + 1]), ab),
                                           __fmul_rn(__uint_as_float(r[2 * j]), ab));
                };
                uint32_t ra[32], rb[32], pk[16], hi[2][16];
                tmem_ld_32x32b_x32(taddr, ra);
                tmem_ld_wait_regs(ra);
                tmem_ld_32x32b_x32(taddr + 32, rb);
                convert(ra, pk);
#pragma unroll
                for (int q = 0; q < 4; ++q) stage_chunk(q, pk + 4 * q);
                tmem_ld_wait_regs(rb);
                tmem_ld_32x32b_x32(taddr + 64, ra);
                convert(rb, pk);
#pragma unroll
                for (int q = 0; q < 4; ++q) stage_chunk(4 + q, pk + 4 * q);
                tmem_ld_wait_regs(ra);
                tmem_ld_32x32b_x32(taddr + 96, rb);
                convert(ra, hi[0]);
                tmem_ld_wait_regs(rb);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive_leader<PAIR>(&s->acc_empty);
                convert(rb, hi[1]);
                if (pace && warp > FIRST_EPI_WARP) __nanosleep(200u * (uint32_t)(warp - FIRST_EPI_WARP));
                __syncwarp();
                issue(0);
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int q = 0; q < 4; ++q) stage_chunk(c * 4 + q, hi[c] + 4 * q);
                if (pace) __nanosleep(1600u);
                __syncwarp();
                issue(1);
            } else if (!C::TMA_STORE && vec_ok && nb * BN + BN <= p.N) {
                // Whole tile inside Y: drain this warp's 32 x 128 block of the
                // accumulator (scaled and rounded to bf16 on the way), hand TMEM
                // back so the next tile's MMAs overlap the stores, then store.
                uint32_t packed[4][16];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        packed[c][j] = cvt_bf16x2(__fmul_rn(__uint_as_float(r[2 * j + 1]), ab),
                                                  __fmul_rn(__uint_as_float(r[2 * j]), ab));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive_leader<PAIR>(&s->acc_empty);
                if (row < p.M && MQ_CHECK((int64_t)row * p.N + colh + 128 <= (int64_t)p.M * p.N)) {
                    uint4* d4 = reinterpret_cast<uint4*>(p.y + (int64_t)row * p.N + colh);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            d4[c * 4 + j] = make_uint4(packed[c][4 * j], packed[c][4 * j + 1],
                                                       packed[c][4 * j + 2], packed[c][4 * j + 3]);
                }
            } else {
                // Ragged right edge (or N not a multiple of 8): one 32-column
                // chunk at a time, element stores.
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, r);
                    tmem_ld_wait();
                    if (c == 3) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) arrive_leader<PAIR>(&s->acc_empty);
                    }
                    const int col0 = colh + c * 32;
                    if (row >= p.M || col0 >= p.N) continue;
                    uint16_t* d16 = reinterpret_cast<uint16_t*>(p.y + (int64_t)row * p.N + col0);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (col0 + j < p.N && MQ_CHECK((int64_t)row * p.N + col0 + j < (int64_t)p.M * p.N)) {
                            const uint32_t two = cvt_bf16x2(0.0f, __fmul_rn(__uint_as_float(r[j]), ab));
                            d16[j] = (uint16_t)(two & 0xffffu);
                        }
                    }
                }
            }
            acc_phase ^= 1;
        }
    }

    if (C::TMA_STORE && warp >= FIRST_EPI_WARP && lane == 0) bulk_wait_group0();
    __syncwarp();   // reconverge the single-lane roles before the block barrier
    tc_fence_before();
    __syncthreads();
    if (PAIR == 2) cluster_sync();      // the peer's MMAs and arrivals are finished
    if (warp == 1) {
        tc_fence_after();
        if (PAIR == 2) tmem_dealloc_pair(tmem, TMEM_COLS);
        else tmem_dealloc(tmem, TMEM_COLS);
    }
}

MQ_DEBUG_READER(debug_hits_gemm)

}  // namespace gemm

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D byte tensor [rows, K/2] with a box of `box_rows` rows x `box_bytes`
// bytes (128 or 64) in the matching 128- or 64-byte swizzle.
static bool make_code_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, int box_rows,
                          int box_bytes) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE,
               box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_fp4_code_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, int box_rows) {
    return make_code_map(map, codes, rows, K, box_rows, 128);
}

bool make_bf16_tile_map(CUtensorMap* map, const void* x, int64_t rows, int64_t K, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K * 2)};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The block scales of a [rows, K] operand as a 2-D array of 64-bit words:
// [row tile][k atom x 64 words] (one 512-byte atom per 128 rows x 64 K);
// a box is `box_rows` row tiles x `atoms` atoms, unswizzled.
static bool make_scale_map(CUtensorMap* map, const uint8_t* scales, int64_t row_tiles, int64_t katoms,
                           int box_rows, int atoms) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || (reinterpret_cast<uintptr_t>(scales) & 15u)) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(katoms * 64), (cuuint64_t)row_tiles};
    cuuint64_t strides[1] = {(cuuint64_t)(katoms * 512)};
    cuuint32_t box[2] = {(cuuint32_t)(atoms * 64), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(scales), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The scales of a [2 inter, K] gate/up operand as a 3-D array of 64-bit
// words [half][row tile][k atom x 64 words]: one box (`atoms` atoms x 1 row
// tile x 2 halves) brings a gate slice and the matching up slice.
static bool make_gate_up_scale_map(CUtensorMap* map, const uint8_t* scales, int64_t inter, int64_t katoms,
                                   int atoms) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || inter % 128 != 0 || (reinterpret_cast<uintptr_t>(scales) & 15u)) return false;
    cuuint64_t dims[3] = {(cuuint64_t)(katoms * 64), (cuuint64_t)(inter / 128), 2};
    cuuint64_t strides[2] = {(cuuint64_t)(katoms * 512), (cuuint64_t)(inter / 128 * katoms * 512)};
    cuuint32_t box[3] = {(cuuint32_t)(atoms * 64), 1, 2};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<uint8_t*>(scales), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor [M, N] for the epilogue's TMA stores: 32-row x 64-column
// boxes in the 128-byte swizzle.  Needs N % 8 == 0 (16-byte row pitch).
static bool make_y_map(CUtensorMap* map, void* y, int64_t M, int64_t N) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || N % 8 != 0 || (reinterpret_cast<uintptr_t>(y) & 15u)) return false;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)(N * 2)};
    cuuint32_t box[2] = {64, 32};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

struct FormState {
    bool attr_set = false;
    int max_units = 0;      // co-resident CTAs (PAIR 1) or clusters (PAIR 2)
};
FormState g_form[64][3][2][2];

template <int PAIR, bool QUANT, bool SWIGLU = false>
cudaError_t launch_form(const GemmArgs& a, int num_sms, cudaStream_t stream) {
    using namespace gemm;
    using C = Cfg<PAIR>;
    int dev = 0;
    cudaGetDevice(&dev);
    FormState& fs = g_form[dev < 64 ? dev : 63][PAIR][QUANT][SWIGLU];
    auto kernel = k_gemm<PAIR, QUANT, SWIGLU>;
    if (!fs.attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        fs.max_units = num_sms / PAIR;
        if (PAIR == 2) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(2 * fs.max_units);
            cfg.blockDim = dim3(THREADS);
            cfg.dynamicSmemBytes = C::SMEM_BYTES;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) == cudaSuccess && clusters > 0)
                fs.max_units = std::min(fs.max_units, clusters);
            cudaGetLastError();
        }
        fs.attr_set = true;
    }
    CUtensorMap ma, mb, my, msfb, msfa;
    if (!make_code_map(&ma, a.a_codes, a.M, a.K, BM, C::ROW_BYTES) ||
        !make_code_map(&mb, a.b_codes, a.N, a.K, C::B_ROWS, C::ROW_BYTES))
        return cudaErrorInvalidValue;
    memset(&my, 0, sizeof(my));
    memset(&msfb, 0, sizeof(msfb));
    memset(&msfa, 0, sizeof(msfa));
    // the SwiGLU form writes H [M, inter] (inter = N / 2) by TMA stores
    const int64_t n_out = SWIGLU ? a.swiglu_inter : a.N;
    // pair form: Y by TMA stores when its rows are 16-byte multiples, else
    // the element stores of the ragged path
    const bool y_tma = C::TMA_STORE && make_y_map(&my, a.y, a.M, n_out);
    if (SWIGLU) {
        if (!y_tma || a.N != 2 * a.swiglu_inter || !a.h_amax ||
            !make_gate_up_scale_map(&msfb, a.b_scales, a.swiglu_inter, scale_atom_cols(a.K), C::NKB))
            return cudaErrorInvalidValue;
    } else if (!make_scale_map(&msfb, a.b_scales, padded_rows(a.N) / 128, scale_atom_cols(a.K), 2, C::NKB)) {
        return cudaErrorInvalidValue;
    }
    if (!make_scale_map(&msfa, a.a_scales, padded_rows(a.M) / 128, scale_atom_cols(a.K), 1, C::NKB))
        return cudaErrorInvalidValue;
    Params p{};
    p.a_scales = a.a_scales;
    p.b_scales = a.b_scales;
    p.alpha_a = a.alpha_a;
    p.alpha_b = a.alpha_b;
    p.y = reinterpret_cast<__nv_bfloat16*>(a.y);
    p.M = (int)a.M;
    p.N = (int)n_out;
    p.K = (int)a.K;
    p.m_blocks = (int)((a.M + C::TILE_M - 1) / C::TILE_M);
    p.n_blocks = SWIGLU ? (int)(a.swiglu_inter / 128) : (int)((a.N + BN - 1) / BN);
    p.inter = (int)a.swiglu_inter;
    p.h_amax = a.h_amax;
    p.tiles = p.m_blocks * p.n_blocks;
    p.kblocks = (int)(a.K / MMA_K);
    p.k_stages = (p.kblocks + C::NKB - 1) / C::NKB;
    p.katoms = (int)scale_atom_cols(a.K);
    p.a_row_tiles = (int)(padded_rows(a.M) / 128);
    p.b_row_tiles = (int)(padded_rows(a.N) / 128);
    p.status = a.status;
    p.timeout = a.timeout_cycles;
    p.fault_skip_first_load = a.fault_skip_first_load;
    p.y_tma = y_tma ? 1 : 0;
    const int group_m = switch_value(MQ_SWITCH_GEMM_GROUP_M), stages = switch_value(MQ_SWITCH_GEMM_STAGES);
    if (group_m > 0) {
        p.group_m = group_m;
    } else {
        // Tiles walk N inside a group of M-blocks, so a group's rows of A are
        // read from DRAM once if they stay in L2 while the group sweeps B, and
        // B once per group.  32 M-blocks at K <= 4096 (the 8192-token set's
        // whole A, 18 MB); at K = 12288 a group of 32 holds 54 MB of A, which
        // was read ~2.3x from DRAM, so the group is cut to RASTER_A_BYTES
        // (10 M-blocks there: DRAM reads 134 MB instead of 187 MB against
        // 85 MB of A and B, and the launch no slower).
        const int64_t a_block = (int64_t)C::TILE_M * (a.K / 2 + a.K / 16);
        p.group_m = (int)std::max<int64_t>(4, std::min<int64_t>(GROUP_M, RASTER_A_BYTES / a_block));
    }
    p.stages = stages > 0 ? std::min(stages, C::STAGES) : C::STAGES;
    p.x = static_cast<const uint16_t*>(a.x);
    p.x_codes = const_cast<uint8_t*>(a.a_codes);
    p.x_scales = const_cast<uint8_t*>(a.a_scales);
    p.flags = a.flags;
    const int units = std::min(p.tiles, fs.max_units);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[3];
    int nattr = 0;
    if (PAIR == 2) {
        attr[nattr].id = cudaLaunchAttributeClusterDimension;
        attr[nattr].val.clusterDim.x = 2;
        attr[nattr].val.clusterDim.y = 1;
        attr[nattr].val.clusterDim.z = 1;
        ++nattr;
    }
    if (QUANT) {
        // producers wait on quantizer warps of other CTAs: every CTA must be
        // resident at once, which a cooperative launch guarantees (or refuses)
        attr[nattr].id = cudaLaunchAttributeCooperative;
        attr[nattr].val.cooperative = 1;
        ++nattr;
    } else {
        set_pdl_attr(attr, &nattr);
    }
    cfg.gridDim = dim3(PAIR * units);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = nattr;
    return cudaLaunchKernelEx(&cfg, kernel, ma, mb, my, msfb, msfa, p);
}

}  // namespace

int64_t fused_flag_count(int64_t M, int64_t K) {
    using C = gemm::Cfg<2>;
    return padded_rows(M) / 128 * ((K / gemm::MMA_K + C::NKB - 1) / C::NKB);
}

// The 2-CTA form for M > 128, the 1-CTA form otherwise; the decode form for
// M <= 64 (unfused).  MQ_SWITCH_GEMM_FORM = 1 | 2 forces a prefill form and
// MQ_SWITCH_GEMM_DECODE = 0 keeps small M on the prefill kernel (the tests
// compare the forms on the same shapes).
cudaError_t launch_gemm(const GemmArgs& a, int num_sms, cudaStream_t stream) {
    if (a.swiglu_inter > 0) return launch_form<2, false, true>(a, num_sms, stream);
    const int forced = switch_value(MQ_SWITCH_GEMM_FORM);
    if (switch_value(MQ_SWITCH_GEMM_DECODE) == 1 && forced == 0 && !a.x && a.M <= 64) {
        const cudaError_t e = launch_gemm_decode(a, num_sms, stream);
        if (e != cudaErrorNotSupported) return e;
    }
    const int form = forced != 0 ? forced : (a.M > gemm::BM ? 2 : 1);
    if (a.x) return form == 2 ? launch_form<2, true>(a, num_sms, stream) : launch_form<1, true>(a, num_sms, stream);
    return form == 2 ? launch_form<2, false>(a, num_sms, stream) : launch_form<1, false>(a, num_sms, stream);
}

}  // namespace mq
