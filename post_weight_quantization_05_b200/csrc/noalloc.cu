// gptq_quantize_layer_noalloc: the blocked sweep of gptq_quantize_layer with
// its scratch in a fixed array inside this library instead of a caller
// workspace.
//
// Who needs it: code that must not allocate device memory at the point where
// it quantizes -- for example a host framework whose memory pool owns every
// device buffer and hands out only inputs and outputs, or a serving process
// that reserves its memory budget at start-up and may not call cudaMalloc
// later (the call can fail once the budget is taken, and it synchronizes the
// device).  Such a caller passes W, U and the outputs and nothing else.
//
// The scratch is one file-scope device array of kNoAllocScratchBytes, held
// by every GPU that loads this library until the process exits.  It holds the
// super-block error matrix E [d_out, min(d_in, 1024)] fp32 and U^T [d_in, d_in] fp32, the
// same two pieces gptq_quantize_layer keeps in its workspace.  Host code may
// not use the array's name as a device pointer, so its device address is
// looked up once per device (cudaGetSymbolAddress, with that device current)
// on the first call made on the device.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(40) << 20;   // 40 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

int noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return GPTQ_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return GPTQ_OK;
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" int gptq_quantize_layer_noalloc(float* W, int64_t d_out, int64_t d_in, const float* U, int bits,
                                           int blocksize, int groupsize, uint32_t* codes, uint16_t* scales,
                                           uint16_t* zeros, float* Q, void* stream) {
    const int v = validate_quantize_args(W, d_out, d_in, U, bits, blocksize, groupsize, codes, scales, zeros, Q);
    if (v) return v;
    if (sweep_workspace_bytes(d_out, d_in) > kNoAllocScratchBytes) return GPTQ_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    DevStatus* st = nullptr;
    PFN_encodeTiled enc = nullptr;
    if (noalloc_scratch(&scratch) || status_ptr(&st) || encode_fn(&enc)) return GPTQ_ERR_CUDA;
    // Nothing in the scratch has to start at zero: every call writes E and the
    // part of U^T it reads before reading them.
    return launch_quantize(W, d_out, d_in, U, bits, groupsize, codes, scales, zeros, Q, scratch,
                           static_cast<cudaStream_t>(stream), st);
}
