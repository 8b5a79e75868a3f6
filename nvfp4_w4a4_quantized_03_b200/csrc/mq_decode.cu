// mq_decode.cu -- the block-scaled FP4 GEMM for few rows of A (decode-shaped:
// M <= 64 tokens), the same product as k_gemm,
//
//   Y[m, n] = bf16( fl32(alpha_a * alpha_b) * sum_k (sigma_a q_a)[m, k] (sigma_b q_b)[n, k] )
//
// (W4A4: "Mix-Quant：面向智能体LLM的量化预填充与精确解码", section 方法步骤详情,
// step (3); decoding quantized as well is the pages' P16D4 variant).  With M
// this small the GEMM is a stream over the weight B [N, K]: 0.5625 bytes per
// weight element against 2 M flops, so the design is about keeping every SM
// reading B:
//   - roles swapped: 128 rows of B are the MMA's M = 128 operand (A of the
//     instruction), the M tokens (padded to a multiple of 16) its N;
//   - split-K: the K stages of one 128-row slice of B are shared by a
//     cluster of S CTAs (S <= 8); each accumulates its part in TMEM, the
//     partials (fp32, 128 x MP) go to shared memory, and each CTA of the
//     cluster adds, for a share of the tokens, all partials in rank order
//     through distributed shared memory, then scales, rounds and writes Y:
//     one launch, no workspace, a fixed summation order.
// Roles per CTA: warp 0 producer (TMA for the B and A code tiles, bulk copies
// for their scale slices, 256 K per stage), warp 1 TMEM allocation and the
// MMA thread, warps 2..5 scale writers (tcgen05.st, one warp per TMEM
// sub-partition) and, after the main loop, the epilogue.  Every mbarrier wait
// is bounded; a timeout is written to the status word.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "../../include/mq.h"
#include "mq_debug.cuh"
#include "mq_internal.h"
#include "mq_ptx.cuh"

namespace mq {
namespace decode {

// A cluster barrier that orders no memory accesses: every CTA has reached
// it, nothing more, so a CTA does not wait here for its own global stores to
// drain.
__device__ __forceinline__ void cluster_sync_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

constexpr int ROWS = 128;            // B rows per CTA (the MMA's M)
constexpr int MP_MAX = 64;           // tokens per launch (the MMA's N, padded to 16)
constexpr int STAGES = 3;
constexpr int NKB = 4;               // MMAs (K = 64 each) per 256-K stage
constexpr int W_BYTES = ROWS * 128;              // B codes of a stage
constexpr int X_BYTES = MP_MAX * 128;            // A codes of a stage (room for MP_MAX rows)
constexpr int SF_BYTES = 2048;                   // one 128-row x 256-K scale slice
constexpr int STAGE_BYTES = W_BYTES + X_BYTES + 2 * SF_BYTES;   // 28 KB, a multiple of 1024
constexpr int PART_BYTES = ROWS * MP_MAX * 4;    // fp32 partial, reuses the stage memory
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
constexpr int THREADS = 6 * 32;
constexpr int FIRST_SF_WARP = 2;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t SF_COL = 64;                  // stage st: SF_COL + 32 st (A-side 16, B-side 16)
static_assert(PART_BYTES <= STAGES * STAGE_BYTES, "partial fits the stage memory");
static_assert(SF_COL + STAGES * 32 <= TMEM_COLS, "TMEM budget");

struct Params {
    const uint8_t* w_scales;     // B scales (the weight)
    const uint8_t* x_scales;     // A scales (the tokens)
    const float* alpha_a;
    const float* alpha_b;
    __nv_bfloat16* y;
    int M, N, K, MP;
    int kblocks, k_stages, katoms, w_row_tiles, split;
    int* status;
    long long timeout;
    int fault_skip_first_load;   // failure-detection test hook: withhold the first stage's copies
};

struct Smem {
    uint64_t ready[STAGES];      // codes landed and the scale writers stored the scales
    uint64_t sf_full[STAGES];    // the stage's scale slices landed
    uint64_t empty[STAGES];      // the stage's MMAs completed
    uint64_t acc_full;
    uint32_t tmem_base;
    int abort_flag;
};

__global__ void __launch_bounds__(THREADS, 1)
k_gemm_decode(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x, Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ Smem sm;
    Smem* s = &sm;
    auto stage_w = [&](int st) { return base + st * STAGE_BYTES; };
    auto stage_x = [&](int st) { return base + st * STAGE_BYTES + W_BYTES; };
    auto stage_sfw = [&](int st) { return base + st * STAGE_BYTES + W_BYTES + X_BYTES; };
    auto stage_sfx = [&](int st) { return base + st * STAGE_BYTES + W_BYTES + X_BYTES + SF_BYTES; };
    float* part = reinterpret_cast<float*>(base);     // [MP][ROWS] after the main loop

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();
    const int tile = blockIdx.x / p.split;              // 128-row slice of B
    const int n0 = tile * ROWS;
    // this CTA's K stages
    const int kt0 = (int)((int64_t)p.k_stages * rank / p.split);
    const int kt1 = (int)((int64_t)p.k_stages * (rank + 1) / p.split);
    const uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(p.MP >> 3) << 17) | ((uint32_t)(ROWS >> 4) << 24);

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&s->ready[i], 1 + 4);
            mbar_init(&s->sf_full[i], 1);
            mbar_init(&s->empty[i], 1);
        }
        mbar_init(&s->acc_full, 1);
        s->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_x);
        // This CTA's weight codes and scales start toward L2 before the wait
        // for the previous grid: a prefetch leaves nothing visible (L2 is the
        // point of coherence, later writes by that grid still win), and the
        // weight stream overlaps the previous kernel's tail.
        const int64_t wt = min(n0 / ROWS, p.w_row_tiles - 1);
        for (int kt = kt0; kt < kt1; ++kt) {
            tma_prefetch_2d(&tmap_w, kt * 128, n0);
            const int nkb = min(NKB, p.kblocks - kt * NKB);
            bulk_prefetch_l2(p.w_scales + (wt * p.katoms + (int64_t)kt * NKB) * 512, nkb * 512);
        }
    }
    if (warp == 1) {
        tmem_alloc(&s->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s->tmem_base;
    const volatile int* abort_flag = &s->abort_flag;
    pdl_launch_dependents();     // set-up of the next grid may overlap this one
    pdl_wait();                  // the grids before this one are done
    auto raise = [&]() {
        *(volatile int*)&s->abort_flag = 1;
        if (p.status) atomicExch(p.status, -7 /* MQ_ERR_TIMEOUT */);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int64_t wt = min(n0 / ROWS, p.w_row_tiles - 1);
            int st = 0;
            uint32_t phase = 0;
            uint32_t pending = 0, pending_phase = 0;     // stages with copies in flight, and their parity
            bool skip = p.fault_skip_first_load != 0;
            for (int kt = kt0; kt < kt1; ++kt) {
                if (!mbar_wait_bounded(&s->empty[st], phase ^ 1, p.timeout, abort_flag)) { raise(); break; }
                pending &= ~(1u << st);
                const int nkb = min(NKB, p.kblocks - kt * NKB);
                const int64_t ka = (int64_t)kt * NKB;
                if (skip || !MQ_CHECK_TMA_X(kt * 128, 1) || !MQ_CHECK(ka + nkb <= p.katoms && wt < p.w_row_tiles) ||
                    !MQ_CHECK_BULK(p.w_scales + (wt * p.katoms + ka) * 512, nkb * 512) ||
                    !MQ_CHECK_BULK(p.x_scales + ka * 512, nkb * 512)) {
                    // failure-detection test hook (or, in the debug build, a copy
                    // that would leave the operands): this stage never completes,
                    // every wait on it runs out
                    skip = false;
                } else {
                    // the scale slices first: their path (copy, scale writers,
                    // TMEM store) is the longer one to the stage's barrier
                    // (decode figures 0.6-1.6% faster than codes first)
                    mbar_arrive_expect_tx(&s->sf_full[st], 2 * nkb * 512);
                    bulk_load(stage_sfw(st), p.w_scales + (wt * p.katoms + ka) * 512, nkb * 512, &s->sf_full[st]);
                    bulk_load(stage_sfx(st), p.x_scales + ka * 512, nkb * 512, &s->sf_full[st]);
                    mbar_arrive_expect_tx(&s->ready[st], W_BYTES + p.MP * 128);
                    tma_load_2d(stage_w(st), &tmap_w, &s->ready[st], kt * 128, n0);
                    tma_load_2d(stage_x(st), &tmap_x, &s->ready[st], kt * 128, 0);
                    pending |= 1u << st;
                    pending_phase = (pending_phase & ~(1u << st)) | (phase << st);
                }
                if (++st == STAGES) { st = 0; phase ^= 1; }
            }
            if (*abort_flag) {
                // the copies this thread issued land before the CTA releases
                // its shared memory: a stage's scale copies complete its
                // sf_full barrier by themselves, its code tiles (issued just
                // after them) get a short grace period
                for (int i = 0; i < STAGES; ++i)
                    if (pending & (1u << i))
                        mbar_wait_bounded(&s->sf_full[i], (pending_phase >> i) & 1, p.timeout, nullptr);
                const long long t0 = clock64();
                while (clock64() - t0 < 200000) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop (its state stays warp-uniform) and one
        // elected lane issues; a full stage's four MMAs go out as
        // straight-line code with their operands computed first (as in
        // k_gemm, where a lone lane in a divergent branch took ~360 cycles
        // per stage to issue instead of ~140).
        const bool leader = elect_one();
        int st = 0;
        uint32_t phase = 0;
        for (int kt = kt0; kt < kt1; ++kt) {
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s->ready[st], phase, p.timeout, abort_flag))) {
                if (leader) raise();
                break;
            }
            tc_fence_after();
            const int nkb = min(NKB, p.kblocks - kt * NKB);
            const uint64_t wd = smem_desc(smem_u32(stage_w(st)), 16, 1024, 2);
            const uint64_t xd = smem_desc(smem_u32(stage_x(st)), 16, 1024, 2);
            const uint32_t sf = tmem + SF_COL + st * 32;
            const uint32_t acc0 = kt != kt0 ? 1u : 0u;
            if (leader) {
                if (nkb == NKB) {
                    mma_mxf4nvf4(tmem, wd, xd, IDESC, sf, sf + 16, acc0);
                    mma_mxf4nvf4(tmem, wd + 2, xd + 2, IDESC, sf + 4, sf + 20, 1u);
                    mma_mxf4nvf4(tmem, wd + 4, xd + 4, IDESC, sf + 8, sf + 24, 1u);
                    mma_mxf4nvf4(tmem, wd + 6, xd + 6, IDESC, sf + 12, sf + 28, 1u);
                } else {
                    for (int kb = 0; kb < nkb; ++kb) {
                        const uint64_t step = (uint64_t)(kb * 32 >> 4);
                        mma_mxf4nvf4(tmem, wd + step, xd + step, IDESC, sf + kb * 4, sf + 16 + kb * 4,
                                     kb != 0 ? 1u : acc0);
                    }
                }
                mma_commit(&s->empty[st]);
            }
            __syncwarp();
            if (++st == STAGES) { st = 0; phase ^= 1; }
        }
        // the epilogue waits for this; after an abort it still arrives, once
        // the MMAs issued so far are done
        if (leader) mma_commit(&s->acc_full);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ scale writers
        const int quad = warp & 3;
        int st = 0;
        uint32_t phase = 0;
        for (int kt = kt0; kt < kt1; ++kt) {
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s->sf_full[st], phase, p.timeout, abort_flag));
            if (!ok) {
                if (lane == 0) raise();
                break;
            }
            const uint8_t* sfw = stage_sfw(st) + lane * 16;
            const uint8_t* sfx = stage_sfx(st) + lane * 16;
            uint32_t vw[16], vx[16];
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb) {
                const uint4 a = *reinterpret_cast<const uint4*>(sfw + kb * 512);
                const uint4 b = *reinterpret_cast<const uint4*>(sfx + kb * 512);
                vw[4 * kb] = a.x; vw[4 * kb + 1] = a.y; vw[4 * kb + 2] = a.z; vw[4 * kb + 3] = a.w;
                vx[4 * kb] = b.x; vx[4 * kb + 1] = b.y; vx[4 * kb + 2] = b.z; vx[4 * kb + 3] = b.w;
            }
            const uint32_t t = tmem + ((uint32_t)(quad * 32) << 16) + SF_COL + st * 32;
            tmem_st_32x32b_x16(t, vw);
            tmem_st_32x32b_x16(t + 16, vx);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s->ready[st]);
            if (++st == STAGES) { st = 0; phase ^= 1; }
        }
        // ------------------------------------------------------------ epilogue
        // this CTA's partial, 128 B rows x MP tokens in fp32, into shared
        // memory as [token][row] (the stage memory: every copy has landed and
        // every MMA reading it has completed once acc_full arrives)
        const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(&s->acc_full, 0, p.timeout, nullptr));
        tc_fence_after();
        if (got) {
            const uint32_t r = quad * 32 + lane;
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16);
            for (int c = 0; c < p.MP; c += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(taddr + c, v);
                tmem_ld_wait_regs16(v);
#pragma unroll
                for (int j = 0; j < 16; ++j) part[(c + j) * ROWS + r] = __uint_as_float(v[j]);
            }
        } else if (lane == 0) {
            raise();
        }
        tc_fence_before();
    }
    __syncwarp();
    __syncthreads();
    cluster_sync();     // every CTA's partial is in its shared memory
    if (warp >= FIRST_SF_WARP && !*abort_flag) {
        // every CTA of the cluster finishes a share of the tokens (m = rank,
        // rank + split, ...): the partials of all CTAs added in rank order,
        // scaled, rounded to bf16, written to Y
        const uint32_t r = (warp & 3) * 32 + lane;
        const int n = n0 + (int)r;
        const float ab = __fmul_rn(__ldg(p.alpha_a), __ldg(p.alpha_b));
        const float* peer[8];
        for (int q = 0; q < p.split; ++q) peer[q] = map_shared_rank(part, (uint32_t)q);
        if (n < p.N) {
            for (int m = (int)rank; m < p.M; m += p.split) {
                float acc = peer[0][m * ROWS + r];
                for (int q = 1; q < p.split; ++q) acc += peer[q][m * ROWS + r];
                if (MQ_CHECK((int64_t)m * p.N + n < (int64_t)p.M * p.N))
                    p.y[(int64_t)m * p.N + n] = __float2bfloat16_rn(__fmul_rn(acc, ab));
            }
        }
    }
    __syncthreads();
    // every CTA keeps its shared memory until all have read it; the reads
    // have completed (their values went into Y), so the barrier needs no
    // memory ordering and does not wait for the Y stores
    cluster_sync_relaxed();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

MQ_DEBUG_READER(debug_hits_decode)

}  // namespace decode

// ---------------------------------------------------------------- host side
cudaError_t launch_gemm_decode(const GemmArgs& a, int num_sms, cudaStream_t stream) {
    using namespace decode;
    if (a.x || a.M < 1 || a.M > MP_MAX) return cudaErrorNotSupported;
    const int MP = (int)((a.M + 15) / 16 * 16);
    CUtensorMap mw, mx;
    if (!make_fp4_code_map(&mw, a.b_codes, a.N, a.K, ROWS) || !make_fp4_code_map(&mx, a.a_codes, a.M, a.K, MP))
        return cudaErrorNotSupported;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    const int d = dev < 64 ? dev : 63;
    if (!attr_set[d]) {
        cudaError_t e = cudaFuncSetAttribute(k_gemm_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[d] = true;
    }
    Params p{};
    p.w_scales = a.b_scales;
    p.x_scales = a.a_scales;
    p.alpha_a = a.alpha_a;
    p.alpha_b = a.alpha_b;
    p.y = reinterpret_cast<__nv_bfloat16*>(a.y);
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.MP = MP;
    p.kblocks = (int)(a.K / 64);
    p.k_stages = (p.kblocks + NKB - 1) / NKB;
    p.katoms = (int)scale_atom_cols(a.K);
    p.w_row_tiles = (int)(padded_rows(a.N) / 128);
    p.status = a.status;
    p.timeout = a.timeout_cycles;
    p.fault_skip_first_load = a.fault_skip_first_load;
    const int tiles = (int)((a.N + ROWS - 1) / ROWS);
    // split-K: the largest power of two (<= 8) that keeps the grid within one
    // wave of two CTAs per SM and gives every CTA at least 4 K stages (a
    // partial second wave, or CTAs of 1-2 stages whose set-up and cluster
    // reduction outweigh their loads, measured slower on every Qwen3-8B
    // projection)
    int split = 1;
    while (split < 8 && (int64_t)tiles * split * 2 <= 2 * (int64_t)num_sms && p.k_stages >= 4 * split * 2) split *= 2;
    const int forced = switch_value(MQ_SWITCH_DECODE_SPLIT);
    if (forced > 0 && forced <= p.k_stages) split = forced;
    p.split = split;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    int nattr = 1;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(tiles * split);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    set_pdl_attr(attr, &nattr);
    cfg.attrs = attr;
    cfg.numAttrs = nattr;
    return cudaLaunchKernelEx(&cfg, k_gemm_decode, mw, mx, p);
}

}  // namespace mq
