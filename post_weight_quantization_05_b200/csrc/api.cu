// C ABI of libgptq (declared in include/gptq.h): host-side validation, the
// per-device status word, and the stream-ordered launches of each stage.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace gptq {

// One status word per device (each device holds its own copy of this
// variable once the module is loaded there).
static __device__ DevStatus g_status;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DevStatus* g_status_ptr[kMaxDevices] = {nullptr};
PFN_encodeTiled g_encode = nullptr;

std::atomic<unsigned long long> g_launches{0};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// Device address of this device's status word (looked up once per device,
// with that device current).
int status_ptr(DevStatus** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return GPTQ_ERR_CUDA;
        g_status_ptr[dev] = static_cast<DevStatus*>(p);
    }
    *out = g_status_ptr[dev];
    return GPTQ_OK;
}

int encode_fn(PFN_encodeTiled* out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return GPTQ_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_encodeTiled>(fn);
        set_tensor_map_encoder(g_encode);
    }
    *out = g_encode;
    return GPTQ_OK;
}

namespace {
inline bool valid_d_in(int64_t d_in) { return d_in >= 128 && d_in <= 32768 && d_in % 128 == 0; }
inline bool valid_bits(int bits) { return bits == 2 || bits == 3 || bits == 4 || bits == 8; }
inline bool valid_group(int g, int64_t d_in) { return g == -1 || (g > 0 && g % 128 == 0 && d_in % g == 0); }

}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int validate_quantize_args(const float* W, int64_t d_out, int64_t d_in, const float* U, int bits, int blocksize,
                           int groupsize, const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros,
                           const float* Q) {
    if (d_out <= 0 || d_out > (int64_t(1) << 24) || !valid_d_in(d_in)) return GPTQ_ERR_INVALID_ARG;
    if (!valid_bits(bits) || !valid_group(groupsize, d_in)) return GPTQ_ERR_INVALID_ARG;
    if (blocksize != 128) return GPTQ_ERR_UNSUPPORTED;
    if (!W || !U || !codes || !scales || !zeros) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(U) || !aligned16(codes) || (Q && !aligned16(Q)) ||
        (reinterpret_cast<uintptr_t>(scales) & 1u) || (reinterpret_cast<uintptr_t>(zeros) & 1u))
        return GPTQ_ERR_INVALID_ARG;
    return GPTQ_OK;
}

}  // namespace gptq

using namespace gptq;

extern "C" {

int gptq_abi_version(void) { return 1; }

uint64_t gptq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* gptq_status_string(int s) {
    switch (s) {
        case GPTQ_OK: return "GPTQ_OK";
        case GPTQ_ERR_INVALID_ARG: return "GPTQ_ERR_INVALID_ARG";
        case GPTQ_ERR_UNSUPPORTED: return "GPTQ_ERR_UNSUPPORTED";
        case GPTQ_ERR_NOT_PD: return "GPTQ_ERR_NOT_PD";
        case GPTQ_ERR_NONFINITE: return "GPTQ_ERR_NONFINITE";
        case GPTQ_ERR_GRID: return "GPTQ_ERR_GRID";
        case GPTQ_ERR_TIMEOUT: return "GPTQ_ERR_TIMEOUT";
        case GPTQ_ERR_CUDA: return "GPTQ_ERR_CUDA";
        default: return "GPTQ_ERR_UNKNOWN";
    }
}

size_t gptq_hessian_workspace_size(int dtype, int64_t n, int64_t d_in) {
    if (dtype != GPTQ_F32 || n <= 0 || d_in <= 0) return 0;
    return size_t(3) * size_t(n) * size_t(d_in) * 2;
}

int gptq_hessian_accumulate(const void* X, int dtype, int64_t n, int64_t d_in, float* H, void* ws,
                            size_t ws_bytes, void* stream) {
    if (dtype != GPTQ_F32 && dtype != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
    if (!valid_d_in(d_in) || n < 0 || n > (int64_t(1) << 31) - 1) return GPTQ_ERR_INVALID_ARG;
    if (n == 0) return GPTQ_OK;
    if (!X || !H || !aligned16(X) || !aligned16(H)) return GPTQ_ERR_INVALID_ARG;
    if (dtype == GPTQ_F32 && (!ws || !aligned16(ws) || ws_bytes < gptq_hessian_workspace_size(dtype, n, d_in)))
        return GPTQ_ERR_INVALID_ARG;
    DevStatus* st = nullptr;
    PFN_encodeTiled enc = nullptr;
    if (status_ptr(&st) || encode_fn(&enc)) return GPTQ_ERR_CUDA;
    return launch_hessian(X, dtype, n, d_in, H, ws, static_cast<cudaStream_t>(stream), st, enc);
}

int gptq_hessian_accumulate_batches(const void* const* X, const int64_t* n, int count, int dtype, int64_t d_in,
                                    float* H, void* ws, size_t ws_bytes, void* stream) {
    if (dtype != GPTQ_F32 && dtype != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
    if (!valid_d_in(d_in) || count < 0 || (count > 0 && (!X || !n))) return GPTQ_ERR_INVALID_ARG;
    if (!H || !aligned16(H)) return GPTQ_ERR_INVALID_ARG;
    int64_t n_max = 0;
    for (int i = 0; i < count; ++i) {
        if (n[i] < 0 || n[i] > (int64_t(1) << 31) - 1) return GPTQ_ERR_INVALID_ARG;
        if (n[i] > 0 && (!X[i] || !aligned16(X[i]))) return GPTQ_ERR_INVALID_ARG;
        n_max = std::max(n_max, n[i]);
    }
    if (n_max == 0) return GPTQ_OK;
    if (dtype == GPTQ_F32 && (!ws || !aligned16(ws) || ws_bytes < gptq_hessian_workspace_size(dtype, n_max, d_in)))
        return GPTQ_ERR_INVALID_ARG;
    DevStatus* st = nullptr;
    PFN_encodeTiled enc = nullptr;
    if (status_ptr(&st) || encode_fn(&enc)) return GPTQ_ERR_CUDA;
    bool launched = false;
    for (int i = 0; i < count; ++i) {
        if (n[i] == 0) continue;
        const int rc = launch_hessian(X[i], dtype, n[i], d_in, H, ws, static_cast<cudaStream_t>(stream), st, enc,
                                      launched);
        if (rc) return rc;
        launched = true;
    }
    return GPTQ_OK;
}

size_t gptq_prepare_hinv_workspace_size(int64_t d_in) {
    if (!valid_d_in(d_in)) return 0;
    return factor_workspace_bytes(d_in);
}

int gptq_prepare_hinv(const float* H, int64_t d_in, float percdamp, float* U, int* info_dev, void* ws,
                      size_t ws_bytes, void* stream) {
    if (!valid_d_in(d_in)) return GPTQ_ERR_INVALID_ARG;
    if (!(percdamp >= 0.0f) || !(percdamp < 1e30f)) return GPTQ_ERR_INVALID_ARG;
    if (!H || !U || !ws || !aligned16(H) || !aligned16(U) || !aligned16(ws)) return GPTQ_ERR_INVALID_ARG;
    if (ws_bytes < factor_workspace_bytes(d_in)) return GPTQ_ERR_INVALID_ARG;
    if (info_dev && (reinterpret_cast<uintptr_t>(info_dev) & 3u)) return GPTQ_ERR_INVALID_ARG;
    DevStatus* st = nullptr;
    PFN_encodeTiled enc = nullptr;
    if (status_ptr(&st) || encode_fn(&enc)) return GPTQ_ERR_CUDA;
    return launch_prepare_hinv(H, d_in, percdamp, U, info_dev, ws, static_cast<cudaStream_t>(stream), st);
}

size_t gptq_quantize_workspace_size(int64_t d_out, int64_t d_in, int blocksize) {
    if (d_out <= 0 || !valid_d_in(d_in) || blocksize != 128) return 0;
    return sweep_workspace_bytes(d_out, d_in);
}

int gptq_quantize_layer(float* W, int64_t d_out, int64_t d_in, const float* U, int bits, int blocksize,
                        int groupsize, uint32_t* codes, uint16_t* scales, uint16_t* zeros, float* Q, void* ws,
                        size_t ws_bytes, void* stream) {
    const int v = validate_quantize_args(W, d_out, d_in, U, bits, blocksize, groupsize, codes, scales, zeros, Q);
    if (v) return v;
    if (!ws || !aligned16(ws) || ws_bytes < sweep_workspace_bytes(d_out, d_in)) return GPTQ_ERR_INVALID_ARG;
    DevStatus* st = nullptr;
    PFN_encodeTiled enc = nullptr;
    if (status_ptr(&st) || encode_fn(&enc)) return GPTQ_ERR_CUDA;
    return launch_quantize(W, d_out, d_in, U, bits, groupsize, codes, scales, zeros, Q, ws,
                           static_cast<cudaStream_t>(stream), st);
}

int gptq_rtn_layer(const float* W, int64_t d_out, int64_t d_in, int bits, int groupsize, uint32_t* codes,
                   uint16_t* scales, uint16_t* zeros, float* Q, void* stream) {
    if (d_out <= 0 || d_out > (int64_t(1) << 24) || !valid_d_in(d_in)) return GPTQ_ERR_INVALID_ARG;
    if (!valid_bits(bits) || !valid_group(groupsize, d_in)) return GPTQ_ERR_INVALID_ARG;
    if (!W || !codes || !scales || !zeros) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(codes) || (Q && !aligned16(Q)) ||
        (reinterpret_cast<uintptr_t>(scales) & 1u) || (reinterpret_cast<uintptr_t>(zeros) & 1u))
        return GPTQ_ERR_INVALID_ARG;
    DevStatus* st = nullptr;
    if (status_ptr(&st)) return GPTQ_ERR_CUDA;
    return launch_rtn(W, d_out, d_in, bits, groupsize, codes, scales, zeros, Q, static_cast<cudaStream_t>(stream),
                      st);
}

int gptq_act_order_perm(const float* H, int64_t d_in, int32_t* perm, void* stream) {
    if (!valid_d_in(d_in) || !H || !perm || !aligned16(H) || (reinterpret_cast<uintptr_t>(perm) & 3u))
        return GPTQ_ERR_INVALID_ARG;
    const uintptr_t h0 = reinterpret_cast<uintptr_t>(H), h1 = h0 + size_t(d_in) * size_t(d_in) * sizeof(float);
    const uintptr_t p0 = reinterpret_cast<uintptr_t>(perm), p1 = p0 + size_t(d_in) * sizeof(int32_t);
    if (p0 < h1 && h0 < p1) return GPTQ_ERR_INVALID_ARG;
    return launch_act_order_perm(H, d_in, perm, static_cast<cudaStream_t>(stream));
}

int gptq_permute_hessian(const float* H, int64_t d_in, const int32_t* perm, float* Hp, void* stream) {
    if (!valid_d_in(d_in) || !H || !perm || !Hp || !aligned16(H) || !aligned16(Hp) ||
        (reinterpret_cast<uintptr_t>(perm) & 3u))
        return GPTQ_ERR_INVALID_ARG;
    const size_t bytes = size_t(d_in) * size_t(d_in) * sizeof(float);
    const uintptr_t h0 = reinterpret_cast<uintptr_t>(H), o0 = reinterpret_cast<uintptr_t>(Hp);
    const uintptr_t p0 = reinterpret_cast<uintptr_t>(perm), p1 = p0 + size_t(d_in) * sizeof(int32_t);
    if ((o0 < h0 + bytes && h0 < o0 + bytes) || (p0 < o0 + bytes && o0 < p1)) return GPTQ_ERR_INVALID_ARG;
    DevStatus* st = nullptr;
    if (status_ptr(&st)) return GPTQ_ERR_CUDA;
    return launch_permute_hessian(H, d_in, perm, Hp, static_cast<cudaStream_t>(stream), st);
}

int gptq_permute_columns(const float* src, int64_t rows, int64_t cols, const int32_t* perm, int inverse,
                         float* dst, void* stream) {
    if (rows < 0 || rows > (int64_t(1) << 24) || !valid_d_in(cols) || (inverse != 0 && inverse != 1))
        return GPTQ_ERR_INVALID_ARG;
    if (rows == 0) return GPTQ_OK;
    if (!src || !dst || !perm || !aligned16(src) || !aligned16(dst) || (reinterpret_cast<uintptr_t>(perm) & 3u))
        return GPTQ_ERR_INVALID_ARG;
    const size_t bytes = size_t(rows) * size_t(cols) * sizeof(float);
    const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), d0 = reinterpret_cast<uintptr_t>(dst);
    const uintptr_t p0 = reinterpret_cast<uintptr_t>(perm), p1 = p0 + size_t(cols) * sizeof(int32_t);
    if (s0 != d0 && s0 < d0 + bytes && d0 < s0 + bytes) return GPTQ_ERR_INVALID_ARG;   // partial overlap
    if (p0 < d0 + bytes && d0 < p1) return GPTQ_ERR_INVALID_ARG;
    DevStatus* st = nullptr;
    if (status_ptr(&st)) return GPTQ_ERR_CUDA;
    return launch_permute_columns(src, rows, cols, perm, inverse != 0, dst, static_cast<cudaStream_t>(stream), st);
}

size_t gptq_dequant_gemv_workspace_size(int64_t m, int64_t d_in, int with_perm) {
    if (m <= 0 || m > 8 || !valid_d_in(d_in)) return 0;
    return gemv_workspace_bytes(m, d_in, with_perm != 0);
}

int gptq_dequant_gemv(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                      int64_t d_in, int bits, int groupsize, const int32_t* perm, const uint16_t* x, int64_t m,
                      float* y, void* ws, size_t ws_bytes, void* stream) {
    if (d_out <= 0 || d_out > (int64_t(1) << 24) || !valid_d_in(d_in)) return GPTQ_ERR_INVALID_ARG;
    if (!valid_bits(bits) || !valid_group(groupsize, d_in) || m < 0 || m > 8) return GPTQ_ERR_INVALID_ARG;
    if (bits != 4) return GPTQ_ERR_UNSUPPORTED;
    if (m == 0) return GPTQ_OK;
    if (!codes || !scales || !zeros || !x || !y) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(x) || (reinterpret_cast<uintptr_t>(y) & 3u) ||
        (reinterpret_cast<uintptr_t>(scales) & 1u) || (reinterpret_cast<uintptr_t>(zeros) & 1u) ||
        (perm && (reinterpret_cast<uintptr_t>(perm) & 3u)))
        return GPTQ_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || ws_bytes < gemv_workspace_bytes(m, d_in, perm != nullptr)) return GPTQ_ERR_INVALID_ARG;
    DevStatus* st = nullptr;
    PFN_encodeTiled enc = nullptr;
    if (status_ptr(&st) || encode_fn(&enc)) return GPTQ_ERR_CUDA;
    return launch_dequant_gemv(codes, scales, zeros, d_out, d_in, groupsize, perm, x, m, y, ws,
                               static_cast<cudaStream_t>(stream), st, enc);
}

int gptq_dequantize(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                    int64_t d_in, int bits, int groupsize, const int32_t* perm, int out_dtype, void* out,
                    void* stream) {
    if (d_out <= 0 || d_out > (int64_t(1) << 24) || !valid_d_in(d_in)) return GPTQ_ERR_INVALID_ARG;
    if (!valid_bits(bits) || !valid_group(groupsize, d_in) || out_dtype < 0 || out_dtype > 2)
        return GPTQ_ERR_INVALID_ARG;
    if (!codes || !scales || !zeros || !out) return GPTQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(codes) & 3u) || !aligned16(out) || (reinterpret_cast<uintptr_t>(scales) & 1u) ||
        (reinterpret_cast<uintptr_t>(zeros) & 1u) || (perm && !aligned16(perm)))
        return GPTQ_ERR_INVALID_ARG;
    DevStatus* st = nullptr;
    if (status_ptr(&st)) return GPTQ_ERR_CUDA;
    return launch_dequantize(codes, scales, zeros, d_out, d_in, bits, groupsize, perm, out_dtype, out,
                             static_cast<cudaStream_t>(stream), st);
}

int gptq_widen_bf16(const uint16_t* src, float* dst, int64_t count, void* stream) {
    if (count < 0) return GPTQ_ERR_INVALID_ARG;
    if (count == 0) return GPTQ_OK;
    if (!src || !dst || (reinterpret_cast<uintptr_t>(src) & 1u) || (reinterpret_cast<uintptr_t>(dst) & 3u))
        return GPTQ_ERR_INVALID_ARG;
    return launch_widen_bf16(src, dst, count, static_cast<cudaStream_t>(stream));
}

int gptq_fill_f32(float* p, int64_t count, float value, void* stream) {
    if (count < 0) return GPTQ_ERR_INVALID_ARG;
    if (count == 0) return GPTQ_OK;
    if (!p || (reinterpret_cast<uintptr_t>(p) & 3u)) return GPTQ_ERR_INVALID_ARG;
    return launch_fill(p, count, value, static_cast<cudaStream_t>(stream));
}

int gptq_get_status(void* stream, int* detail_out) {
    DevStatus* st = nullptr;
    if (status_ptr(&st)) return GPTQ_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return GPTQ_ERR_CUDA;
    DevStatus h{0, 0};
    if (cudaMemcpy(&h, st, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (h.code != 0) {
        const DevStatus zero{0, 0};
        if (cudaMemcpy(st, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return GPTQ_ERR_CUDA;
    }
    if (detail_out) *detail_out = h.detail;
    return h.code;
}

}  // extern "C"
