// mq_internal.h -- declarations shared by the CUDA translation units of
// libmq.so (not part of the public C ABI, which is include/mq.h).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace mq {

// Workspace header, in 32-bit words.  Every kernel that uses it leaves the
// counters at zero when it finishes, so a zero-filled header stays valid.
enum WsWord : int {
    WS_AMAX_BITS = 0,   // running max of |x| as a bf16 bit pattern (u32)
    WS_TICKET = 1,      // blocks of the amax pass that have finished
    WS_STATUS = 2,      // device-side status (0 = ok, else an mq_status code)
    WS_ALPHA = 3,       // alpha_x written by the amax pass of mq_linear_w4a4
    WS_H_AMAX = 5,      // mq_mlp_w4a4: running max of |h| (binary32 bits), zeroed once read
    WS_H_ALPHA = 6,     // mq_mlp_w4a4: alpha_h of the down projection's input
    WS_GENERATION = 32, // grid-barrier generation of the one-pass quantizer (only grows); a 128-byte
                        // line of its own, so the blocks polling it do not queue the counters' atomics
};
constexpr size_t WS_HEADER_BYTES = 256;

// Scale storage: atoms of 128 rows x 4 scale columns (512 bytes), ordered
// row-tile major, k-tile minor (the order the block-scaled MMA reads).
__host__ __device__ inline int64_t scale_atom_cols(int64_t K) { return (K / 16 + 3) / 4; }
__host__ __device__ inline int64_t padded_rows(int64_t rows) { return (rows + 127) / 128 * 128; }

// Tensor map of a bf16 [rows, K] tensor for TMA loads of box_rows x 64-element
// boxes in the 128-byte swizzle (rows past the end read as zero).
bool make_bf16_tile_map(CUtensorMap* map, const void* x, int64_t rows, int64_t K, int box_rows);

// Tensor map of packed E2M1 codes [rows, K/2 bytes] for TMA loads of
// box_rows x 128-byte boxes (256 K-elements) in the 128-byte swizzle.
bool make_fp4_code_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, int box_rows);

// The shape checks of mq_linear_w4a4 (rows M and N against K): MQ_OK or
// MQ_ERR_SHAPE.
int check_linear_shape(int64_t M, int64_t N, int64_t K);

// The selectable alternatives of include/mq.h (MQ_SWITCH_*): the current
// process-wide value of switch `which` (set from the environment on first use).
int switch_value(int which);

// Programmatic dependent launch: each kernel lets the next grid on the
// stream launch early and waits (griddepcontrol.wait) before its first access
// to global memory.  Launches carry the attribute unless MQ_SWITCH_PDL is 0.
bool pdl_enabled();
void set_pdl_attr(cudaLaunchAttribute* attr, int* nattr);

// Launchers (enqueue on `stream`, no synchronisation).
cudaError_t launch_amax(const void* x, int64_t numel, uint32_t* ws_words, float* alpha_out,
                        int num_sms, cudaStream_t stream, int* clear = nullptr, int nclear = 0, int raw_amax = 0);
cudaError_t launch_alpha_from_amax(const float* amax, float* alpha, cudaStream_t stream,
                                   uint32_t* reset = nullptr);
cudaError_t launch_quantize(const void* x, int64_t rows, int64_t K, const float* alpha,
                            uint8_t* codes, uint8_t* scales, cudaStream_t stream);
// alpha_x and the NVFP4 codes/scales of x in one cooperative launch (amax
// pass, grid barrier, quantization pass over recently read data).
cudaError_t launch_quantize_onepass(const void* x, int64_t rows, int64_t K, uint32_t* ws_words, float* alpha_out,
                                    uint8_t* codes, uint8_t* scales, int* status, long long timeout_cycles,
                                    cudaStream_t stream);

struct GemmArgs {
    const uint8_t* a_codes;
    const uint8_t* a_scales;
    const float* alpha_a;
    const uint8_t* b_codes;
    const uint8_t* b_scales;
    const float* alpha_b;
    void* y;
    int64_t M, N, K;
    int* status;            // may be null
    long long timeout_cycles;
    int fault_skip_first_load;   // failure-detection tests only
    // Fused activation quantization (mq_linear_w4a4): when x is set, the
    // kernel's quantizer warps write A (a_codes / a_scales) from bf16 x with
    // alpha_a, publishing each 128-row x (stage) block through `flags`.
    const void* x = nullptr;
    int* flags = nullptr;
    // The MLP's gate/up GEMM with SwiGLU in the epilogue: B is [2 inter, K]
    // (gate rows, then up rows; inter % 128 == 0, N = 2 inter), y receives
    // H = SwiGLU(G, U) as bf16 [M, inter] and h_amax the running max of |h|
    // (binary32 bits, atomically raised).
    int64_t swiglu_inter = 0;
    uint32_t* h_amax = nullptr;
};

// Debug build (MQ_DEBUG): bounds-check hits of each translation unit since
// its last read (0 in the release build).
unsigned long long debug_hits_quant();
namespace gemm { unsigned long long debug_hits_gemm(); }
namespace decode { unsigned long long debug_hits_decode(); }

// Readiness flags of the fused linear: one int per (128-row block, K stage).
int64_t fused_flag_count(int64_t M, int64_t K);
cudaError_t launch_gemm(const GemmArgs& a, int num_sms, cudaStream_t stream);
// Small-M form of the block-scaled GEMM (decode-shaped, M <= 64): W as the
// MMA's 128-row operand, split-K over a cluster, partials summed through
// distributed shared memory.  Returns cudaErrorNotSupported for shapes it
// does not take.
cudaError_t launch_gemm_decode(const GemmArgs& a, int num_sms, cudaStream_t stream);

}  // namespace mq
