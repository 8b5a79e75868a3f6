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
// Design (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: A/B code tiles (128-byte swizzle) and the two
//               scale tiles (plain bulk copies) into a 4-stage ring.
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (K = 64 per
//               instruction, 4 per stage) and tcgen05.commit to release
//               stages and to publish a finished tile.
//   warps 2..5  scale writers: move each stage's block scales from shared
//               memory into that stage's TMEM scale columns with tcgen05.st,
//               one warp per 32-lane TMEM sub-partition (the MMA reads the
//               scales replicated in all four).  Done off the MMA thread,
//               this costs the tensor pipe nothing, where tcgen05.cp from the
//               MMA thread measured ~45 cycles per copy, serialised with the
//               MMAs.
//   warps 6..13 epilogue: drain the 128 x 256 fp32 accumulator from TMEM into
//               registers, release it to the MMA warp, then scale by
//               alpha_a * alpha_b, round to bf16 and store.
#include <cuda_bf16.h>

#include "mq_internal.h"
#include "mq_ptx.cuh"

namespace mq {
namespace gemm {

constexpr int BM = 128;               // rows of A per tile (TMEM lanes)
constexpr int BN = 256;               // rows of B per tile (accumulator columns)
constexpr int BK = 256;               // K elements per pipeline stage
constexpr int MMA_K = 64;             // K elements per tcgen05.mma (kind::mxf4nvf4)
constexpr int NKB = BK / MMA_K;       // MMAs per stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK / 2;          // 16 KiB
constexpr int B_BYTES = BN * BK / 2;          // 32 KiB
constexpr int SFA_BYTES = BM * BK / 16;       // 2 KiB
constexpr int SFB_BYTES = BN * BK / 16;       // 4 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int SF_WARPS = 4;
constexpr int EPI_WARPS = 8;
constexpr int FIRST_SF_WARP = 2;
constexpr int FIRST_EPI_WARP = FIRST_SF_WARP + SF_WARPS;
constexpr int THREADS = (FIRST_EPI_WARP + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t SF_COLS_PER_STAGE = 12 * NKB;    // per MMA: A 4 columns, B 8 columns
constexpr uint32_t SF_COL = BN;                     // stage st: SF_COL + st * SF_COLS_PER_STAGE
constexpr uint32_t SFB_OFF = 4 * NKB;               // B scales after the A scales of a stage
constexpr int GROUP_M = 16;                         // tile raster: M-blocks per group
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;

static_assert(SF_COL + STAGES * SF_COLS_PER_STAGE <= TMEM_COLS, "TMEM budget");
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment for the 128-byte swizzle");

// Instruction descriptor of kind::mxf4nvf4: E2M1 x E2M1, UE4M3 scales,
// K-major A and B, M = 128, N = 256, dense K = 64.
constexpr uint32_t IDESC = (1u << 7)              // A format E2M1
                         | (1u << 10)             // B format E2M1
                         | ((uint32_t)(BN >> 3) << 17)
                         | (0u << 23)             // scale format UE4M3
                         | ((uint32_t)(BM >> 4) << 24);

struct Params {
    const uint8_t* a_scales;
    const uint8_t* b_scales;
    const float* alpha_a;
    const float* alpha_b;
    __nv_bfloat16* y;
    int M, N, K;
    int m_blocks, n_blocks, tiles, k_stages, kblocks, katoms, b_row_tiles;
    int* status;
    long long timeout;
    int fault_skip_first_load;
};

struct Smem {
    uint64_t full[STAGES];       // TMA bytes of a stage landed
    uint64_t sf_ready[STAGES];   // the stage's scales are in TMEM
    uint64_t empty[STAGES];      // the stage's MMAs completed
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ void tile_coords(int tile, const Params& p, int& mb, int& nb) {
    const int group = GROUP_M * p.n_blocks;
    const int first_m = (tile / group) * GROUP_M;
    const int gm = min(GROUP_M, p.m_blocks - first_m);
    const int in = tile % group;
    mb = first_m + in % gm;
    nb = in / gm;
}

__device__ __forceinline__ void raise_abort(Smem* s, const Params& p) {
    *(volatile int*)&s->abort_flag = 1;
    if (p.status) atomicExch(p.status, -7 /* MQ_ERR_TIMEOUT */);
}

__global__ void __launch_bounds__(THREADS, 1)
k_gemm(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b, Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Smem* s = reinterpret_cast<Smem*>(base + STAGES * STAGE_BYTES);
    auto stage_a = [&](int st) { return base + st * STAGE_BYTES; };
    auto stage_b = [&](int st) { return base + st * STAGE_BYTES + A_BYTES; };
    auto stage_sfa = [&](int st) { return base + st * STAGE_BYTES + A_BYTES + B_BYTES; };
    auto stage_sfb = [&](int st) { return base + st * STAGE_BYTES + A_BYTES + B_BYTES + SFA_BYTES; };

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&s->full[i], 1);
            mbar_init(&s->sf_ready[i], SF_WARPS);
            mbar_init(&s->empty[i], 1);
        }
        mbar_init(&s->acc_full, 1);
        mbar_init(&s->acc_empty, EPI_WARPS);
        mbar_init(&s->drain, 1);
        s->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
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

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int st = 0;
            uint32_t phase = 0;
            uint32_t pending = 0;           // stages with a load in flight
            uint32_t pending_phase = 0;     // parity of that load's phase
            bool skip = p.fault_skip_first_load != 0;
            for (int tile = blockIdx.x; tile < p.tiles && !*abort_flag; tile += gridDim.x) {
                int mb, nb;
                tile_coords(tile, p, mb, nb);
                for (int kt = 0; kt < p.k_stages; ++kt) {
                    if (!mbar_wait_bounded(&s->empty[st], phase ^ 1, p.timeout, abort_flag)) {
                        raise_abort(s, p);
                        break;
                    }
                    pending &= ~(1u << st);
                    const int nkb = min(NKB, p.kblocks - kt * NKB);
                    const uint32_t sf_a = nkb * 512;
                    if (skip) {     // test hook: never complete this stage
                        skip = false;
                    } else {
                        mbar_arrive_expect_tx(&s->full[st], A_BYTES + B_BYTES + 3 * sf_a);
                        tma_load_2d(stage_a(st), &tmap_a, &s->full[st], kt * (BK / 2), mb * BM);
                        tma_load_2d(stage_b(st), &tmap_b, &s->full[st], kt * (BK / 2), nb * BN);
                        const int64_t ka = (int64_t)kt * NKB;   // first k-atom of the stage
                        bulk_load(stage_sfa(st), p.a_scales + ((int64_t)mb * p.katoms + ka) * 512, sf_a, &s->full[st]);
                        for (int rt = 0; rt < 2; ++rt) {
                            // rows past the padded end of B feed only discarded columns
                            const int64_t bt = min(nb * 2 + rt, p.b_row_tiles - 1);
                            bulk_load(stage_sfb(st) + rt * (SFB_BYTES / 2),
                                      p.b_scales + (bt * p.katoms + ka) * 512, sf_a, &s->full[st]);
                        }
                        pending |= 1u << st;
                        pending_phase = (pending_phase & ~(1u << st)) | (phase << st);
                    }
                    if (++st == STAGES) { st = 0; phase ^= 1; }
                }
            }
            if (*abort_flag) {
                // let the copies this thread issued land before the CTA exits
                for (int i = 0; i < STAGES; ++i)
                    if (pending & (1u << i))
                        mbar_wait_bounded(&s->full[i], (pending_phase >> i) & 1, p.timeout, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int st = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int tile = blockIdx.x; tile < p.tiles && !*abort_flag; tile += gridDim.x) {
                if (!mbar_wait_bounded(&s->acc_empty, acc_phase ^ 1, p.timeout, abort_flag)) {
                    raise_abort(s, p);
                    break;
                }
                tc_fence_after();
                bool ok = true;
                for (int kt = 0; kt < p.k_stages; ++kt) {
                    // the stage's data is in shared memory and its scales in TMEM
                    if (!mbar_wait_bounded(&s->sf_ready[st], phase, p.timeout, abort_flag)) {
                        raise_abort(s, p);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nkb = min(NKB, p.kblocks - kt * NKB);
                    const uint32_t a0 = smem_u32(stage_a(st)), b0 = smem_u32(stage_b(st));
                    const uint32_t sf = tmem + SF_COL + st * SF_COLS_PER_STAGE;
                    for (int kb = 0; kb < nkb; ++kb) {
                        const uint64_t ad = smem_desc(a0 + kb * (MMA_K / 2), 16, 1024, 2);
                        const uint64_t bd = smem_desc(b0 + kb * (MMA_K / 2), 16, 1024, 2);
                        mma_mxf4nvf4(tmem + ACC_COL, ad, bd, IDESC, sf + kb * 4, sf + SFB_OFF + kb * 8,
                                     (kt | kb) != 0);
                    }
                    mma_commit(&s->empty[st]);
                    if (++st == STAGES) { st = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(&s->acc_full);
                acc_phase ^= 1;
            }
            // no MMA may still be running when TMEM is released
            mma_commit(&s->drain);
            mbar_wait_bounded(&s->drain, 0, p.timeout, nullptr);
        }
    } else if (warp < FIRST_EPI_WARP) {
        // ------------------------------------------------------------ scale writers
        // Lane l of the warp owning TMEM sub-partition q writes row l of each
        // 512-byte scale atom (16 bytes: rows l, l+32, l+64, l+96 of the tile,
        // 4 scales each) into 4 consecutive columns of TMEM lane 32q + l.
        const int quad = warp & 3;
        int st = 0;
        uint32_t phase = 0;
        for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x) {
            bool ok = true;
            for (int kt = 0; kt < p.k_stages; ++kt) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s->full[st], phase, p.timeout, abort_flag));
                if (!ok) break;
                const int nkb = min(NKB, p.kblocks - kt * NKB);
                const uint8_t* sfa = stage_sfa(st) + lane * 16;
                const uint8_t* sfb = stage_sfb(st) + lane * 16;
                const uint32_t t = tmem + ((uint32_t)(quad * 32) << 16) + SF_COL + st * SF_COLS_PER_STAGE;
                for (int kb = 0; kb < nkb; ++kb) {
                    tmem_st_32x32b_x4(t + kb * 4, *reinterpret_cast<const uint4*>(sfa + kb * 512));
                    tmem_st_32x32b_x4(t + SFB_OFF + kb * 8, *reinterpret_cast<const uint4*>(sfb + kb * 512));
                    tmem_st_32x32b_x4(t + SFB_OFF + kb * 8 + 4,
                                      *reinterpret_cast<const uint4*>(sfb + SFB_BYTES / 2 + kb * 512));
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s->sf_ready[st]);
                if (++st == STAGES) { st = 0; phase ^= 1; }
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
        for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x) {
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
            const int row = mb * BM + quad * 32 + lane;
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + ACC_COL + half * 128;
            const int colh = nb * BN + half * 128;
            if (vec_ok && nb * BN + BN <= p.N) {
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
                if (lane == 0) mbar_arrive(&s->acc_empty);
                if (row < p.M) {
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
                // chunk at a time, element stores past the last full chunk.
                for (int c = 0; c < 4; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, r);
                    tmem_ld_wait();
                    if (c == 3) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&s->acc_empty);
                    }
                    const int col0 = colh + c * 32;
                    if (row >= p.M || col0 >= p.N) continue;
                    uint16_t* d16 = reinterpret_cast<uint16_t*>(p.y + (int64_t)row * p.N + col0);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (col0 + j < p.N) {
                            const uint32_t two = cvt_bf16x2(0.0f, __fmul_rn(__uint_as_float(r[j]), ab));
                            d16[j] = (uint16_t)(two & 0xffffu);
                        }
                    }
                }
            }
            acc_phase ^= 1;
        }
    }

    __syncwarp();   // reconverge the single-lane roles before the block barrier
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

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

// 2-D byte tensor [rows, K/2] with a box of `box_rows` x 128 bytes, 128-byte swizzle.
static bool make_code_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {(cuuint32_t)(gemm::BK / 2), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_gemm(const GemmArgs& a, int num_sms, cudaStream_t stream) {
    using namespace gemm;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    CUtensorMap ma, mb;
    if (!make_code_map(&ma, a.a_codes, a.M, a.K, BM) || !make_code_map(&mb, a.b_codes, a.N, a.K, BN))
        return cudaErrorInvalidValue;
    Params p{};
    p.a_scales = a.a_scales;
    p.b_scales = a.b_scales;
    p.alpha_a = a.alpha_a;
    p.alpha_b = a.alpha_b;
    p.y = reinterpret_cast<__nv_bfloat16*>(a.y);
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.m_blocks = (int)((a.M + BM - 1) / BM);
    p.n_blocks = (int)((a.N + BN - 1) / BN);
    p.tiles = p.m_blocks * p.n_blocks;
    p.kblocks = (int)(a.K / MMA_K);
    p.k_stages = (p.kblocks + NKB - 1) / NKB;
    p.katoms = (int)scale_atom_cols(a.K);
    p.b_row_tiles = (int)(padded_rows(a.N) / 128);
    p.status = a.status;
    p.timeout = a.timeout_cycles;
    p.fault_skip_first_load = a.fault_skip_first_load;
    const int grid = std::min(p.tiles, num_sms);
    k_gemm<<<grid, THREADS, SMEM_BYTES, stream>>>(ma, mb, p);
    return cudaGetLastError();
}

}  // namespace mq
