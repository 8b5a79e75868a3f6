/*
 * mq.h -- C ABI of libmq.so: NVFP4 W4A4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The method (NVFP4 two-level microscaling, weights and activations both in
 * 4-bit E2M1, W4A4) is the one stated in
 *   "Mix-Quant：面向智能体LLM的量化预填充与精确解码" (paper.rainbus.top digest),
 *   section 方法步骤详情, step (3), and section NVFP4 微缩放量化; and
 *   "Mix-Quant: Quantized Prefilling, Precise Decoding for Agentic LLMs"
 *   (r9-hu paper digest), section Method, item 1:
 *
 *     sigma_b = Pi_E4M3( max_{i in b} |x_i| / (alpha_x * q_max) )   (block scale)
 *     q_i     = Pi_FP4 ( x_i / (alpha_x * sigma_b(i)) )            (element code)
 *     xhat_i  = alpha_x * sigma_b(i) * q_i                          (dequantized value)
 *
 * with blocks b of 16 consecutive elements along K, q_max = 6, round to
 * nearest.  The arithmetic the kernels use where the pages leave it open:
 *     alpha_x = fl32(amax / 2688)      (amax = max |x| over the tensor; 1 if amax = 0)
 *     sigma_b = RNE_E4M3_satfinite( fl32( amax_b / fl32(6 * alpha_x) ) )
 *     q_i     = RNE_E2M1_satfinite( fl32( x_i * fl32( 1 / fl32(alpha_x * sigma_b) ) ) )
 *     q_i     = +0 for every element of a block whose sigma_b is 0
 *     Y       = bf16_RNE( fl32(alpha_a * alpha_b) * fp32 tensor-core sum_k (sigma q)_a (sigma q)_b )
 *
 * Data layout (all row-major, K contiguous; the nn.Linear layout W[N, K]):
 *   bf16 tensors : [rows, K], 2 bytes per element.
 *   codes        : [rows, K/2] bytes; element 2j in the low nibble of byte j,
 *                  E2M1 code = sign(bit 3) | exponent(bits 2..1) | mantissa(bit 0).
 *   scales       : E4M3 (OCP E4M3FN) bytes in the order the Blackwell
 *                  block-scaled MMA reads: atoms of 128 rows x 4 scale columns
 *                  (512 bytes), atom (row/128, kblock/4) at byte
 *                  ((row/128) * ceil(K/64) + kblock/4) * 512; inside an atom
 *                  (row, kblock) sits at (row%32)*16 + ((row/32)%4)*4 + kblock%4.
 *                  Rows are padded to a multiple of 128 (padding bytes are 0).
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers unless stated otherwise; the caller owns
 *     every buffer.  The library never allocates or frees memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls only
 *     enqueue work; they return before it runs.
 *   - The return value is an mq_status.  A synchronous error (bad argument,
 *     shape, alignment, device) enqueues nothing.  Errors found on the device
 *     (a bounded wait that expired) are written to the workspace status word,
 *     read back with mq_read_status.
 *   - Shapes: rows, M, N >= 1; K >= 64 and K % 64 == 0.  Base pointers must be
 *     16-byte aligned.  Inputs are finite bf16: NaN/Inf are outside the
 *     contract (alpha becomes NaN, nothing else is guaranteed).
 *   - Device: compute capability 10.0 (B200), else MQ_ERR_ARCH.
 */
#ifndef MQ_H
#define MQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mq_status {
    MQ_OK = 0,
    MQ_ERR_INVALID_ARG = -1,   /* null pointer or bad size argument            */
    MQ_ERR_SHAPE = -2,         /* K not a positive multiple of 64, M/N <= 0      */
    MQ_ERR_ALIGN = -3,         /* a base pointer is not 16-byte aligned          */
    MQ_ERR_ARCH = -4,          /* current device is not compute capability 10.0  */
    MQ_ERR_WORKSPACE = -5,     /* workspace missing or smaller than required     */
    MQ_ERR_CUDA = -6,          /* a CUDA runtime call failed                     */
    MQ_ERR_TIMEOUT = -7        /* device side: a bounded wait expired            */
} mq_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *mq_status_string(int status);

/* Bytes of packed E2M1 codes for a [rows, K] tensor: rows * K / 2. */
size_t mq_nvfp4_codes_bytes(int64_t rows, int64_t K);

/* Bytes of the block-scale buffer for a [rows, K] tensor in the MMA order:
 * ceil(rows/128)*128 * ceil(K/64)*4. */
size_t mq_nvfp4_scales_bytes(int64_t rows, int64_t K);

/* Bytes of workspace mq_tensor_scale and mq_nvfp4_gemm use (a 256-byte header
 * holding the amax accumulator, a block counter and the status word). */
size_t mq_workspace_bytes(void);

/* Bytes of workspace mq_linear_w4a4 needs for an [M, K] activation: the
 * header plus room for the quantized activation (codes and scales). */
size_t mq_linear_w4a4_workspace_bytes(int64_t M, int64_t K);

/*
 * Tensor-level scale alpha_x of a bf16 tensor ("张量级尺度", section NVFP4
 * 微缩放量化 of the paper.rainbus.top digest; alpha_x in the r9-hu digest,
 * section Method, item 1):  *alpha = fl32(max|x| / 2688), or 1 if max|x| = 0.
 *   x      : device, numel bf16 values (16-byte aligned)
 *   alpha  : device, 1 float, written
 *   ws     : device workspace of >= mq_workspace_bytes() bytes, zero-filled
 *            before its first use; every call leaves its counters at zero.
 *            Calls that share a workspace must not overlap on the GPU.
 */
int mq_tensor_scale(const void *x, int64_t numel, float *alpha, void *ws, size_t ws_bytes, void *stream);

/*
 * max |x| of a bf16 tensor, as fp32 (exact: the largest magnitude of bf16
 * values), for callers that shard a tensor's rows across devices: the
 * tensor-level scale of the whole tensor ("张量级尺度", section NVFP4 微缩放量化
 * of the paper.rainbus.top digest) is alpha_x = fl32(max over shards / 2688),
 * so the shards' amax values are reduced (max, e.g. an NCCL all-reduce of
 * these 4 bytes) and turned into alpha with mq_alpha_from_amax; quantizing
 * every shard with that alpha gives the codes and scales of the unsharded
 * tensor, row for row.
 *   x      : device, numel bf16 values (16-byte aligned)
 *   amax   : device, 1 float, written
 *   ws     : as for mq_tensor_scale
 */
int mq_tensor_amax(const void *x, int64_t numel, float *amax, void *ws, size_t ws_bytes, void *stream);

/*
 * alpha_x = fl32(amax / 2688), or 1 if amax = 0 (the tensor-level scale of
 * mq_tensor_scale, from a given amax).  amax and alpha: device, 1 float each.
 */
int mq_alpha_from_amax(const float *amax, float *alpha, void *stream);

/*
 * NVFP4 quantization of a bf16 [rows, K] tensor with a given alpha_x
 * (block scale sigma_b and element codes q_i as above; section 方法步骤详情,
 * step (3); section Method, item 1).
 *   x      : device bf16 [rows, K]
 *   alpha  : device, 1 float (e.g. written by mq_tensor_scale)
 *   codes  : device, mq_nvfp4_codes_bytes(rows, K) bytes, written (16-byte
 *            aligned; at 32-byte alignment each thread's 32 code bytes leave
 *            in one 256-bit store, ~13% faster on large tensors)
 *   scales : device, mq_nvfp4_scales_bytes(rows, K) bytes, written (padding = 0)
 */
int mq_nvfp4_quantize(const void *x, int64_t rows, int64_t K, const float *alpha,
                      uint8_t *codes, uint8_t *scales, void *stream);

/*
 * Block-scaled FP4 GEMM on two quantized operands (W4A4: both sides NVFP4,
 * section 方法步骤详情, step (3)):
 *   y[m, n] = bf16( fl32(alpha_a * alpha_b) * sum_k (sigma q)_a[m, k] (sigma q)_b[n, k] )
 *   a_codes/a_scales : A = [M, K] (activations), alpha_a device float
 *   b_codes/b_scales : B = [N, K] (weights, nn.Linear layout), alpha_b device float
 *   y                : device bf16 [M, N], written
 *   ws               : optional (may be NULL) workspace of >= mq_workspace_bytes()
 *                      bytes; when given, a timeout is reported in its status word.
 * Tensor cores accumulate in fp32; the result matches the exact product of
 * the dequantized operands rounded to bf16 to within about 1e-3 relative
 * Frobenius error.
 */
int mq_nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales, const float *alpha_a,
                  const uint8_t *b_codes, const uint8_t *b_scales, const float *alpha_b,
                  int64_t M, int64_t N, int64_t K, void *y, void *ws, size_t ws_bytes, void *stream);

/*
 * The W4A4 linear layer of the FP4 prefill path: Y = X W^T with X quantized
 * on the fly (alpha_x from X, then codes and scales) and W quantized offline
 * (mq_tensor_scale + mq_nvfp4_quantize on W).
 *   x        : device bf16 [M, K]
 *   w_codes, w_scales, alpha_w : quantized W [N, K]
 *   y        : device bf16 [M, N], written
 *   ws       : device workspace of >= mq_linear_w4a4_workspace_bytes(M, K)
 *              bytes, zero-filled before its first use; calls sharing it
 *              must not overlap on the GPU.
 * Y equals mq_nvfp4_gemm applied to (mq_tensor_scale, mq_nvfp4_quantize)(X)
 * and W bit for bit.
 */
int mq_linear_w4a4(const void *x, int64_t M, int64_t K,
                   const uint8_t *w_codes, const uint8_t *w_scales, const float *alpha_w, int64_t N,
                   void *y, void *ws, size_t ws_bytes, void *stream);

/*
 * The MLP's two W4A4 linears with the gated activation between them, for a
 * decoder MLP whose gate and up projections are quantized as one weight
 * (both linears NVFP4 W4A4 as in section 方法步骤详情, step (3); the pages give
 * the activation no numerics, so its binary32 form is this library's):
 *   G = bf16 gate product, U = bf16 up product (as mq_nvfp4_gemm writes them)
 *   h = bf16( fl32( silu(G) * U ) ),  silu(g) = fl32( g / fl32(1 + e(-g)) )
 * with e(x) the binary32 exponential by Cody and Waite's range reduction
 * (ln 2 split into 0x1.62e4p-1 and 0x1.7f7d1cp-20) and the Taylor polynomial
 * of e^r to degree 7, evaluated in Horner form with fused multiply-adds,
 * times 2^k; e(x) = +inf for x > 88 and 0 for x < -87.  Every step is one
 * IEEE binary32 operation, so H is fully determined by G and U.
 *
 * mq_nvfp4_gemm_swiglu: the gate/up GEMM with the activation in its epilogue.
 *   a_codes/a_scales, alpha_a : A = [M, K] (activations)
 *   b_codes/b_scales, alpha_b : B = [2 inter, K], rows [0, inter) the gate
 *                               weight, rows [inter, 2 inter) the up weight,
 *                               quantized as one tensor (one alpha)
 *   inter    : intermediate size, a multiple of 128
 *   h        : device bf16 [M, inter], written with H
 *   h_amax   : device float, raised to max(*h_amax, max |h|) (set it to 0
 *              before the first GEMM of a tensor; atomics, any order)
 *   ws       : optional workspace as for mq_nvfp4_gemm (timeout status)
 *
 * mq_mlp_w4a4: y = (SwiGLU(x Wg^T, x Wu^T) quantized) Wd^T in one call:
 *   x's tensor scale and NVFP4 form (as mq_linear_w4a4), the gate/up GEMM
 *   above into a workspace H, alpha_h = fl32(max|h| / 2688) (1 if 0), H's
 *   NVFP4 form, then the down GEMM.
 *   x        : device bf16 [M, K]
 *   wgu_*    : quantized [2 inter, K] gate/up weight as above
 *   wd_*     : quantized down weight [N, inter]
 *   y        : device bf16 [M, N], written
 *   ws       : >= mq_mlp_w4a4_workspace_bytes(M, K, inter) bytes, 256-byte
 *              aligned, zero-filled before first use (it is left that way);
 *              calls sharing it must not overlap on the GPU.
 * y equals mq_nvfp4_gemm on (mq_nvfp4_quantize with alpha_h)(H) and Wd bit for
 * bit, with H and alpha_h as mq_nvfp4_gemm_swiglu and mq_alpha_from_amax
 * give them.
 */
int mq_nvfp4_gemm_swiglu(const uint8_t *a_codes, const uint8_t *a_scales, const float *alpha_a,
                         const uint8_t *b_codes, const uint8_t *b_scales, const float *alpha_b,
                         int64_t M, int64_t inter, int64_t K, void *h, float *h_amax,
                         void *ws, size_t ws_bytes, void *stream);
size_t mq_mlp_w4a4_workspace_bytes(int64_t M, int64_t K, int64_t inter);
int mq_mlp_w4a4(const void *x, int64_t M, int64_t K,
                const uint8_t *wgu_codes, const uint8_t *wgu_scales, const float *alpha_gu, int64_t inter,
                const uint8_t *wd_codes, const uint8_t *wd_scales, const float *alpha_d, int64_t N,
                void *y, void *ws, size_t ws_bytes, void *stream);

/*
 * mq_linear_w4a4 for callers that cannot allocate device memory -- for
 * example a plugin inside a host application that owns all device memory and
 * hands extensions no allocator, or C code that must not call cudaMalloc
 * because it synchronizes the device.  The paper has no counterpart: this is a
 * deployment convenience of this library, not a step of the method.
 *
 * Same arguments and result as mq_linear_w4a4, without the workspace: the
 * library uses its own scratch, one static device array of
 * MQ_NOALLOC_SCRATCH_BYTES (64 MiB) that every GPU loading libmq.so holds
 * until the process exits.  Nothing is allocated or freed by this call.
 *   - Shapes whose mq_linear_w4a4_workspace_bytes(M, K) exceeds
 *     MQ_NOALLOC_SCRATCH_BYTES are refused with MQ_ERR_WORKSPACE (e.g.
 *     M = 8192 with K up to 12288 fits; M = 131072, K = 4096 does not).
 *   - Every call looks up the scratch's device address in the current
 *     device's current context (cudaGetSymbolAddress), so the address stays
 *     right after a cudaDeviceReset; the reset itself discards the scratch's
 *     contents, which no call relies on.  The first call on a device loads
 *     the library's device code and sets the scratch up: make that first call
 *     before any stream capture.
 *   - Every call shares the one scratch: calls whose GPU work overlaps (other
 *     streams, other host threads) race and corrupt each other's results;
 *     serialize them.  Each call clears the scratch header before use (one
 *     cudaMemsetAsync node ahead of the quantizer, which also keeps the next
 *     call's quantizer from overlapping the previous call's GEMM tail).
 *   - Device-side timeouts land in the scratch's status word, which the caller
 *     cannot read; use mq_linear_w4a4 with a workspace to observe them.
 */
#define MQ_NOALLOC_SCRATCH_BYTES (64u << 20)
int mq_linear_w4a4_noalloc(const void *x, int64_t M, int64_t K,
                           const uint8_t *w_codes, const uint8_t *w_scales, const float *alpha_w, int64_t N,
                           void *y, void *stream);

/*
 * The debug build of the library (libmq_debug.so, the same sources compiled
 * with MQ_DEBUG=1) checks, before it is made, every global-memory access
 * that a kernel computes from indices (quantizer code and scale stores, the
 * fused quantizer's loads and stores, the epilogues' register stores) and
 * every TMA coordinate and bulk-copy address (the 16-byte rules).  A failed
 * check counts one hit and skips the access -- nothing traps, the context
 * stays usable (a skipped copy then shows as MQ_ERR_TIMEOUT on the waits
 * that expected it).  It stands in for a memory checker on machines where
 * none may run.
 *
 * mq_is_debug_build: 1 in libmq_debug.so, 0 in libmq.so.
 * mq_debug_bounds_hits: synchronizes the current device, then writes the
 *   number of failed checks since the previous call into *hits (a host
 *   pointer) and clears the count; always 0 in the release build.
 */
int mq_is_debug_build(void);
int mq_debug_bounds_hits(int64_t *hits);

/*
 * Synchronizes `stream`, then reads the status word of a workspace into
 * *device_status (MQ_OK or MQ_ERR_TIMEOUT) and clears it.  `ws` is a device
 * pointer, `device_status` a host pointer.
 */
int mq_read_status(void *ws, void *stream, int32_t *device_status);

/*
 * Failure-detection test hook; the paper has no counterpart.  Runs the
 * mq_nvfp4_gemm kernel (the decode form for M <= 64) with the loads of the
 * first pipeline stage withheld
 * and every bounded wait limited to `timeout_cycles` SM clock cycles
 * (1e5 .. 4e9), so the pipeline stalls on purpose: each waiting role gives
 * up, the kernel writes MQ_ERR_TIMEOUT into the workspace status word, lets
 * its own copies land, frees its tensor memory and returns.  No fault, trap
 * or hang is involved; the CUDA context stays usable and mq_read_status(ws)
 * then returns MQ_ERR_TIMEOUT.  Arguments as for mq_nvfp4_gemm; `ws` is
 * required.  y is left undefined.
 */
int mq_debug_gemm_stall(const uint8_t *a_codes, const uint8_t *a_scales, const float *alpha_a,
                        const uint8_t *b_codes, const uint8_t *b_scales, const float *alpha_b,
                        int64_t M, int64_t N, int64_t K, void *y, void *ws, size_t ws_bytes,
                        int64_t timeout_cycles, void *stream);

/*
 * Test hook for the allocation-free entry point; the paper has no
 * counterpart.  Enqueues on `stream` a fill of the header words of the
 * current device's static scratch (its grid-barrier ticket, running max,
 * generation and status words) with the 32-bit `word`, the state that a
 * call ended by MQ_ERR_TIMEOUT can leave behind.  The next
 * mq_linear_w4a4_noalloc call clears the header before its kernels run, so
 * its result does not depend on what this wrote.  Returns MQ_OK or
 * MQ_ERR_CUDA.
 */
int mq_debug_noalloc_fill_header(uint32_t word, void *stream);

/*
 * Selectable alternatives.  Each switch picks among kernels or launch
 * shapes that compute the same result (the tests compare their outputs bit
 * for bit); the defaults are the fastest measured.  A switch is one
 * process-wide value: mq_set_switch takes effect for launches enqueued after
 * it returns, from any thread.  The first call that enqueues work or reads
 * or sets a switch sets every switch from its environment variable (named
 * beside it), once; later changes of the environment have no effect.
 *
 *   MQ_SWITCH_LINEAR_PATH   (MQ_LINEAR_PATH: onepass | split | ingemm, or 0 | 1 | 2)
 *       how mq_linear_w4a4 quantizes X: 0 one cooperative kernel (amax, grid
 *       barrier, quantization; default), 1 the mq_tensor_scale and
 *       mq_nvfp4_quantize kernels, 2 the amax kernel and quantizer warps
 *       inside the GEMM.
 *   MQ_SWITCH_GEMM_FORM     (MQ_GEMM_FORM: 1 | 2)
 *       0 by rule (CTA pairs for M > 128, else one CTA; the decode form for
 *       M <= 64), 1 the one-CTA prefill form, 2 the CTA-pair form.
 *   MQ_SWITCH_GEMM_DECODE   (MQ_GEMM_DECODE: 0 | 1)
 *       1 the split-K decode form for M <= 64 (default), 0 the prefill form.
 *   MQ_SWITCH_DECODE_SPLIT  (MQ_DECODE_SPLIT: 1 | 2 | 4 | 8)
 *       0 split-K of the decode form by rule, else that split (at most the
 *       number of 256-K stages).
 *   MQ_SWITCH_GEMM_STAGES   (MQ_GEMM_STAGES)
 *       0 every pipeline stage the prefill form has room for, else 2.. that
 *       many (fewer than the room are used as is).
 *   MQ_SWITCH_GEMM_GROUP_M  (MQ_GEMM_GROUP_M)
 *       0 the tile raster by rule (groups of at most 32 M-blocks and 18 MiB
 *       of A), else that many M-blocks per group, 1 .. 2^20.
 *   MQ_SWITCH_PDL           (MQ_PDL: 0 | 1)
 *       1 launches carry programmatic dependent launch (default), 0 not.
 *
 * mq_set_switch returns MQ_OK, or MQ_ERR_INVALID_ARG for an unknown switch
 * or a value outside its range (the switch keeps its value).
 * mq_get_switch returns the value, or MQ_ERR_INVALID_ARG for an unknown
 * switch.
 */
enum {
    MQ_SWITCH_LINEAR_PATH = 0,
    MQ_SWITCH_GEMM_FORM = 1,
    MQ_SWITCH_GEMM_DECODE = 2,
    MQ_SWITCH_DECODE_SPLIT = 3,
    MQ_SWITCH_GEMM_STAGES = 4,
    MQ_SWITCH_GEMM_GROUP_M = 5,
    MQ_SWITCH_PDL = 6,
    MQ_SWITCH_COUNT = 7
};
int mq_set_switch(int which, int value);
int mq_get_switch(int which);

#ifdef __cplusplus
}
#endif

#endif /* MQ_H */
