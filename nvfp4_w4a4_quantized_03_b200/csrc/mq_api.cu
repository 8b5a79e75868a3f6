// mq_api.cu -- the extern "C" boundary of libmq.so (declared in include/mq.h):
// argument validation, per-device attribute cache, and the launches.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/mq.h"
#include "mq_internal.h"

namespace {

constexpr long long DEFAULT_TIMEOUT_CYCLES = 4000000000LL;   // ~2-3 s of SM clock
constexpr int MAX_DEVICES = 64;

struct DeviceInfo {
    int checked = 0;
    int ok = 0;
    int num_sms = 0;
};
DeviceInfo g_dev[MAX_DEVICES];
std::mutex g_mu;

int current_device_info(int* num_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return MQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.checked) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MQ_ERR_CUDA;
        d.ok = (major == 10 && minor == 0);
        d.num_sms = sms;
        d.checked = 1;
    }
    if (!d.ok) return MQ_ERR_ARCH;
    *num_sms = d.num_sms;
    return MQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

int check_rows_k(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0 || K % 64 != 0) return MQ_ERR_SHAPE;
    if (rows > (int64_t)1 << 31 || K > (int64_t)1 << 24) return MQ_ERR_SHAPE;
    // the quantizers index 16-element blocks of the (row-padded) tensor in 32 bits
    if ((rows + 127) / 128 * 128 * (K / 16) >= ((int64_t)1 << 31)) return MQ_ERR_SHAPE;
    return MQ_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MQ_OK : MQ_ERR_CUDA; }

}  // namespace

namespace mq {
int check_linear_shape(int64_t M, int64_t N, int64_t K) {
    const int st = check_rows_k(M, K);
    return st != MQ_OK ? st : check_rows_k(N, K);
}

namespace {

// Range of each switch (include/mq.h) and its environment variable.
struct SwitchDef {
    const char* env;
    int lo, hi, dflt;
};
constexpr SwitchDef SWITCH_DEFS[MQ_SWITCH_COUNT] = {
    {"MQ_LINEAR_PATH", 0, 2, 0},        // onepass | split | ingemm
    {"MQ_GEMM_FORM", 0, 2, 0},          // rule | one CTA | CTA pair
    {"MQ_GEMM_DECODE", 0, 1, 1},
    {"MQ_DECODE_SPLIT", 0, 8, 0},       // rule | 1, 2, 4, 8
    {"MQ_GEMM_STAGES", 0, 64, 0},       // every stage | 2 ..
    {"MQ_GEMM_GROUP_M", 0, 1 << 20, 0}, // default raster | 1 ..
    {"MQ_PDL", 0, 1, 1},
};

bool switch_value_ok(int which, int v) {
    const SwitchDef& d = SWITCH_DEFS[which];
    if (v < d.lo || v > d.hi) return false;
    if (which == MQ_SWITCH_DECODE_SPLIT) return v == 0 || v == 1 || v == 2 || v == 4 || v == 8;
    if (which == MQ_SWITCH_GEMM_STAGES) return v == 0 || v >= 2;
    return true;
}

// The environment's value of a switch (its default when unset or invalid).
int switch_from_env(int which) {
    const SwitchDef& d = SWITCH_DEFS[which];
    const char* e = getenv(d.env);
    if (!e || !e[0]) return d.dflt;
    if (which == MQ_SWITCH_LINEAR_PATH && !(e[0] >= '0' && e[0] <= '9'))
        return e[0] == 's' ? 1 : e[0] == 'i' ? 2 : 0;            // onepass | split | ingemm
    const int v = atoi(e);
    return switch_value_ok(which, v) ? v : d.dflt;
}

std::atomic<int> g_switch[MQ_SWITCH_COUNT];
std::once_flag g_switch_once;

void init_switches() {
    std::call_once(g_switch_once, [] {
        for (int i = 0; i < MQ_SWITCH_COUNT; ++i) g_switch[i].store(switch_from_env(i), std::memory_order_relaxed);
    });
}

}  // namespace

int switch_value(int which) {
    init_switches();
    return g_switch[which].load(std::memory_order_relaxed);
}

bool pdl_enabled() { return switch_value(MQ_SWITCH_PDL) == 1; }
void set_pdl_attr(cudaLaunchAttribute* attr, int* nattr) {
    if (!pdl_enabled()) return;
    attr[*nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[*nattr].val.programmaticStreamSerializationAllowed = 1;
    ++*nattr;
}
}  // namespace mq

extern "C" {

const char* mq_status_string(int status) {
    switch (status) {
        case MQ_OK: return "MQ_OK";
        case MQ_ERR_INVALID_ARG: return "MQ_ERR_INVALID_ARG";
        case MQ_ERR_SHAPE: return "MQ_ERR_SHAPE";
        case MQ_ERR_ALIGN: return "MQ_ERR_ALIGN";
        case MQ_ERR_ARCH: return "MQ_ERR_ARCH";
        case MQ_ERR_WORKSPACE: return "MQ_ERR_WORKSPACE";
        case MQ_ERR_CUDA: return "MQ_ERR_CUDA";
        case MQ_ERR_TIMEOUT: return "MQ_ERR_TIMEOUT";
        default: return "MQ_ERR_UNKNOWN";
    }
}

size_t mq_nvfp4_codes_bytes(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0) return 0;
    return (size_t)rows * (size_t)(K / 2);
}

size_t mq_nvfp4_scales_bytes(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0) return 0;
    return (size_t)mq::padded_rows(rows) * (size_t)mq::scale_atom_cols(K) * 4;
}

size_t mq_workspace_bytes(void) { return mq::WS_HEADER_BYTES; }

// Workspace of mq_linear_w4a4: header | readiness flags of the fused kernel |
// codes of X | scales of X.
static size_t linear_flags_bytes(int64_t M, int64_t K) { return round256((size_t)mq::fused_flag_count(M, K) * 4); }

size_t mq_linear_w4a4_workspace_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0) return 0;
    return mq::WS_HEADER_BYTES + linear_flags_bytes(M, K) + round256(mq_nvfp4_codes_bytes(M, K)) +
           round256(mq_nvfp4_scales_bytes(M, K));
}

int mq_tensor_scale(const void* x, int64_t numel, float* alpha, void* ws, size_t ws_bytes, void* stream) {
    if (!x || !alpha || numel <= 0) return MQ_ERR_INVALID_ARG;
    if (!ws || ws_bytes < mq::WS_HEADER_BYTES) return MQ_ERR_WORKSPACE;
    if (!aligned16(x) || !aligned16(ws) || (reinterpret_cast<uintptr_t>(alpha) & 3u)) return MQ_ERR_ALIGN;
    int sms = 0;
    int st = current_device_info(&sms);
    if (st != MQ_OK) return st;
    return cuda_status(mq::launch_amax(x, numel, static_cast<uint32_t*>(ws), alpha, sms,
                                       static_cast<cudaStream_t>(stream)));
}

int mq_tensor_amax(const void* x, int64_t numel, float* amax, void* ws, size_t ws_bytes, void* stream) {
    if (!x || !amax || numel <= 0) return MQ_ERR_INVALID_ARG;
    if (!ws || ws_bytes < mq::WS_HEADER_BYTES) return MQ_ERR_WORKSPACE;
    if (!aligned16(x) || !aligned16(ws) || (reinterpret_cast<uintptr_t>(amax) & 3u)) return MQ_ERR_ALIGN;
    int sms = 0;
    int st = current_device_info(&sms);
    if (st != MQ_OK) return st;
    return cuda_status(mq::launch_amax(x, numel, static_cast<uint32_t*>(ws), amax, sms,
                                       static_cast<cudaStream_t>(stream), nullptr, 0, 1));
}

int mq_alpha_from_amax(const float* amax, float* alpha, void* stream) {
    if (!amax || !alpha) return MQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(amax) & 3u) || (reinterpret_cast<uintptr_t>(alpha) & 3u)) return MQ_ERR_ALIGN;
    int sms = 0;
    int st = current_device_info(&sms);
    if (st != MQ_OK) return st;
    return cuda_status(mq::launch_alpha_from_amax(amax, alpha, static_cast<cudaStream_t>(stream)));
}

int mq_nvfp4_quantize(const void* x, int64_t rows, int64_t K, const float* alpha, uint8_t* codes,
                      uint8_t* scales, void* stream) {
    if (!x || !alpha || !codes || !scales) return MQ_ERR_INVALID_ARG;
    int st = check_rows_k(rows, K);
    if (st != MQ_OK) return st;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (reinterpret_cast<uintptr_t>(alpha) & 3u))
        return MQ_ERR_ALIGN;
    int sms = 0;
    st = current_device_info(&sms);
    if (st != MQ_OK) return st;
    return cuda_status(mq::launch_quantize(x, rows, K, alpha, codes, scales, static_cast<cudaStream_t>(stream)));
}

static int gemm_checked(const uint8_t* a_codes, const uint8_t* a_scales, const float* alpha_a,
                        const uint8_t* b_codes, const uint8_t* b_scales, const float* alpha_b, int64_t M,
                        int64_t N, int64_t K, void* y, int* status, cudaStream_t stream) {
    if (!a_codes || !a_scales || !alpha_a || !b_codes || !b_scales || !alpha_b || !y) return MQ_ERR_INVALID_ARG;
    int st = check_rows_k(M, K);
    if (st != MQ_OK) return st;
    st = check_rows_k(N, K);
    if (st != MQ_OK) return st;
    if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(b_codes) || !aligned16(b_scales) ||
        !aligned16(y))
        return MQ_ERR_ALIGN;
    int sms = 0;
    st = current_device_info(&sms);
    if (st != MQ_OK) return st;
    mq::GemmArgs g{a_codes, a_scales, alpha_a, b_codes, b_scales, alpha_b, y, M, N, K,
                   status, DEFAULT_TIMEOUT_CYCLES, 0};
    return cuda_status(mq::launch_gemm(g, sms, stream));
}

int mq_nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* alpha_a, const uint8_t* b_codes,
                  const uint8_t* b_scales, const float* alpha_b, int64_t M, int64_t N, int64_t K, void* y,
                  void* ws, size_t ws_bytes, void* stream) {
    int* status = nullptr;
    if (ws) {
        if (ws_bytes < mq::WS_HEADER_BYTES) return MQ_ERR_WORKSPACE;
        if (!aligned16(ws)) return MQ_ERR_ALIGN;
        status = static_cast<int*>(ws) + mq::WS_STATUS;
    }
    return gemm_checked(a_codes, a_scales, alpha_a, b_codes, b_scales, alpha_b, M, N, K, y, status,
                        static_cast<cudaStream_t>(stream));
}

int mq_linear_w4a4(const void* x, int64_t M, int64_t K, const uint8_t* w_codes, const uint8_t* w_scales,
                   const float* alpha_w, int64_t N, void* y, void* ws, size_t ws_bytes, void* stream) {
    if (!x || !w_codes || !w_scales || !alpha_w || !y) return MQ_ERR_INVALID_ARG;
    int st = check_rows_k(M, K);
    if (st != MQ_OK) return st;
    st = check_rows_k(N, K);
    if (st != MQ_OK) return st;
    if (!ws || ws_bytes < mq_linear_w4a4_workspace_bytes(M, K)) return MQ_ERR_WORKSPACE;
    if (!aligned16(x) || !aligned256(ws) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y))
        return MQ_ERR_ALIGN;
    int sms = 0;
    st = current_device_info(&sms);
    if (st != MQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* words = static_cast<uint32_t*>(ws);
    float* alpha_x = reinterpret_cast<float*>(words + mq::WS_ALPHA);
    int* flags = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + mq::WS_HEADER_BYTES);
    uint8_t* x_codes = reinterpret_cast<uint8_t*>(flags) + linear_flags_bytes(M, K);
    uint8_t* x_scales = x_codes + round256(mq_nvfp4_codes_bytes(M, K));
    mq::GemmArgs g{x_codes, x_scales, alpha_x, w_codes, w_scales, alpha_w, y, M, N, K,
                   reinterpret_cast<int*>(words + mq::WS_STATUS), DEFAULT_TIMEOUT_CYCLES, 0};
    // MQ_SWITCH_LINEAR_PATH selects how X is quantized (all three give identical Y):
    //   0 (default) one cooperative kernel: amax, grid barrier, quantization
    //               of the data the amax pass left in L2;
    //   1           mq_tensor_scale's and mq_nvfp4_quantize's kernels;
    //   2           amax kernel, then quantizer warps inside the GEMM.
    const int mode = mq::switch_value(MQ_SWITCH_LINEAR_PATH);
    cudaError_t e = cudaSuccess;
    if (mode == 2) {
        // amax (which also clears the readiness flags), then the GEMM with
        // the activation's quantization done by its quantizer warps
        e = mq::launch_amax(x, M * K, words, alpha_x, sms, s, flags, (int)mq::fused_flag_count(M, K));
        g.x = x;
        g.flags = flags;
    } else if (mode == 1) {
        e = mq::launch_amax(x, M * K, words, alpha_x, sms, s);
        if (e == cudaSuccess) e = mq::launch_quantize(x, M, K, alpha_x, x_codes, x_scales, s);
    } else {
        e = mq::launch_quantize_onepass(x, M, K, words, alpha_x, x_codes, x_scales,
                                        reinterpret_cast<int*>(words + mq::WS_STATUS), DEFAULT_TIMEOUT_CYCLES, s);
    }
    if (e != cudaSuccess) return MQ_ERR_CUDA;
    return cuda_status(mq::launch_gemm(g, sms, s));
}

int mq_nvfp4_gemm_swiglu(const uint8_t* a_codes, const uint8_t* a_scales, const float* alpha_a,
                         const uint8_t* b_codes, const uint8_t* b_scales, const float* alpha_b, int64_t M,
                         int64_t inter, int64_t K, void* h, float* h_amax, void* ws, size_t ws_bytes, void* stream) {
    if (!a_codes || !a_scales || !alpha_a || !b_codes || !b_scales || !alpha_b || !h || !h_amax)
        return MQ_ERR_INVALID_ARG;
    if (inter <= 0 || inter % 128 != 0) return MQ_ERR_SHAPE;
    int st = check_rows_k(M, K);
    if (st != MQ_OK) return st;
    st = check_rows_k(2 * inter, K);
    if (st != MQ_OK) return st;
    if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(b_codes) || !aligned16(b_scales) ||
        !aligned16(h) || (reinterpret_cast<uintptr_t>(h_amax) & 3u))
        return MQ_ERR_ALIGN;
    int* status = nullptr;
    if (ws) {
        if (ws_bytes < mq::WS_HEADER_BYTES) return MQ_ERR_WORKSPACE;
        if (!aligned16(ws)) return MQ_ERR_ALIGN;
        status = static_cast<int*>(ws) + mq::WS_STATUS;
    }
    int sms = 0;
    st = current_device_info(&sms);
    if (st != MQ_OK) return st;
    mq::GemmArgs g{a_codes, a_scales, alpha_a, b_codes, b_scales, alpha_b, h, M, 2 * inter, K,
                   status, DEFAULT_TIMEOUT_CYCLES, 0};
    g.swiglu_inter = inter;
    g.h_amax = reinterpret_cast<uint32_t*>(h_amax);
    return cuda_status(mq::launch_gemm(g, sms, static_cast<cudaStream_t>(stream)));
}

// Workspace of mq_mlp_w4a4: the linear's (header, flags, codes and scales of
// X) | H bf16 [M, inter] | codes of H | scales of H.
size_t mq_mlp_w4a4_workspace_bytes(int64_t M, int64_t K, int64_t inter) {
    if (M <= 0 || K <= 0 || inter <= 0) return 0;
    return mq_linear_w4a4_workspace_bytes(M, K) + round256((size_t)M * (size_t)inter * 2) +
           round256(mq_nvfp4_codes_bytes(M, inter)) + round256(mq_nvfp4_scales_bytes(M, inter));
}

int mq_mlp_w4a4(const void* x, int64_t M, int64_t K, const uint8_t* wgu_codes, const uint8_t* wgu_scales,
                const float* alpha_gu, int64_t inter, const uint8_t* wd_codes, const uint8_t* wd_scales,
                const float* alpha_d, int64_t N, void* y, void* ws, size_t ws_bytes, void* stream) {
    if (!x || !wgu_codes || !wgu_scales || !alpha_gu || !wd_codes || !wd_scales || !alpha_d || !y)
        return MQ_ERR_INVALID_ARG;
    if (inter <= 0 || inter % 128 != 0) return MQ_ERR_SHAPE;
    int st = check_rows_k(M, K);
    if (st != MQ_OK) return st;
    if ((st = check_rows_k(2 * inter, K)) != MQ_OK || (st = check_rows_k(M, inter)) != MQ_OK ||
        (st = check_rows_k(N, inter)) != MQ_OK)
        return st;
    if (!ws || ws_bytes < mq_mlp_w4a4_workspace_bytes(M, K, inter)) return MQ_ERR_WORKSPACE;
    if (!aligned16(x) || !aligned256(ws) || !aligned16(wgu_codes) || !aligned16(wgu_scales) ||
        !aligned16(wd_codes) || !aligned16(wd_scales) || !aligned16(y))
        return MQ_ERR_ALIGN;
    int sms = 0;
    st = current_device_info(&sms);
    if (st != MQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* words = static_cast<uint32_t*>(ws);
    int* status = reinterpret_cast<int*>(words + mq::WS_STATUS);
    float* alpha_x = reinterpret_cast<float*>(words + mq::WS_ALPHA);
    float* h_amax = reinterpret_cast<float*>(words + mq::WS_H_AMAX);
    float* alpha_h = reinterpret_cast<float*>(words + mq::WS_H_ALPHA);
    uint8_t* x_codes = static_cast<uint8_t*>(ws) + mq::WS_HEADER_BYTES + linear_flags_bytes(M, K);
    uint8_t* x_scales = x_codes + round256(mq_nvfp4_codes_bytes(M, K));
    uint8_t* h = static_cast<uint8_t*>(ws) + mq_linear_w4a4_workspace_bytes(M, K);
    uint8_t* h_codes = h + round256((size_t)M * (size_t)inter * 2);
    uint8_t* h_scales = h_codes + round256(mq_nvfp4_codes_bytes(M, inter));
    // 1. alpha_x and the NVFP4 form of X
    cudaError_t e = mq::launch_quantize_onepass(x, M, K, words, alpha_x, x_codes, x_scales, status,
                                                DEFAULT_TIMEOUT_CYCLES, s);
    // 2. gate/up GEMM, SwiGLU and max|h| in its epilogue -> H
    mq::GemmArgs gu{x_codes, x_scales, alpha_x, wgu_codes, wgu_scales, alpha_gu, h, M, 2 * inter, K,
                    status, DEFAULT_TIMEOUT_CYCLES, 0};
    gu.swiglu_inter = inter;
    gu.h_amax = reinterpret_cast<uint32_t*>(h_amax);
    if (e == cudaSuccess) e = mq::launch_gemm(gu, sms, s);
    // 3. alpha_h (the running max is zeroed for the next call), NVFP4 form of H
    if (e == cudaSuccess) e = mq::launch_alpha_from_amax(h_amax, alpha_h, s, words + mq::WS_H_AMAX);
    if (e == cudaSuccess) e = mq::launch_quantize(h, M, inter, alpha_h, h_codes, h_scales, s);
    // 4. down projection
    mq::GemmArgs dn{h_codes, h_scales, alpha_h, wd_codes, wd_scales, alpha_d, y, M, N, inter,
                    status, DEFAULT_TIMEOUT_CYCLES, 0};
    if (e == cudaSuccess) e = mq::launch_gemm(dn, sms, s);
    return cuda_status(e);
}

int mq_debug_gemm_stall(const uint8_t* a_codes, const uint8_t* a_scales, const float* alpha_a,
                        const uint8_t* b_codes, const uint8_t* b_scales, const float* alpha_b, int64_t M, int64_t N,
                        int64_t K, void* y, void* ws, size_t ws_bytes, int64_t timeout_cycles, void* stream) {
    if (!ws || ws_bytes < mq::WS_HEADER_BYTES) return MQ_ERR_WORKSPACE;
    if (!aligned16(ws)) return MQ_ERR_ALIGN;
    if (timeout_cycles < 100000 || timeout_cycles > DEFAULT_TIMEOUT_CYCLES) return MQ_ERR_INVALID_ARG;
    if (!a_codes || !a_scales || !alpha_a || !b_codes || !b_scales || !alpha_b || !y) return MQ_ERR_INVALID_ARG;
    int st = check_rows_k(M, K);
    if (st != MQ_OK) return st;
    st = check_rows_k(N, K);
    if (st != MQ_OK) return st;
    if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(b_codes) || !aligned16(b_scales) || !aligned16(y))
        return MQ_ERR_ALIGN;
    int sms = 0;
    st = current_device_info(&sms);
    if (st != MQ_OK) return st;
    mq::GemmArgs g{a_codes, a_scales, alpha_a, b_codes, b_scales, alpha_b, y, M, N, K,
                   static_cast<int*>(ws) + mq::WS_STATUS, (long long)timeout_cycles, 1};
    return cuda_status(mq::launch_gemm(g, sms, static_cast<cudaStream_t>(stream)));
}

int mq_is_debug_build(void) {
#ifdef MQ_DEBUG
    return 1;
#else
    return 0;
#endif
}

int mq_set_switch(int which, int value) {
    if (which < 0 || which >= MQ_SWITCH_COUNT || !mq::switch_value_ok(which, value)) return MQ_ERR_INVALID_ARG;
    mq::init_switches();
    mq::g_switch[which].store(value, std::memory_order_relaxed);
    return MQ_OK;
}

int mq_get_switch(int which) {
    if (which < 0 || which >= MQ_SWITCH_COUNT) return MQ_ERR_INVALID_ARG;
    return mq::switch_value(which);
}

int mq_debug_bounds_hits(int64_t* hits) {
    if (!hits) return MQ_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return MQ_ERR_CUDA;
    const unsigned long long q = mq::debug_hits_quant(), g = mq::gemm::debug_hits_gemm(),
                             d = mq::decode::debug_hits_decode();
    if (q == ~0ull || g == ~0ull || d == ~0ull) return MQ_ERR_CUDA;
    *hits = (int64_t)(q + g + d);
    return MQ_OK;
}

int mq_read_status(void* ws, void* stream, int32_t* device_status) {
    if (!ws || !device_status) return MQ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* word = static_cast<int32_t*>(ws) + mq::WS_STATUS;
    int32_t v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MQ_ERR_CUDA;
    if (cudaMemcpy(&v, word, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MQ_ERR_CUDA;
    if (cudaMemset(word, 0, sizeof v) != cudaSuccess) return MQ_ERR_CUDA;
    *device_status = v;
    return MQ_OK;
}

}  // extern "C"
