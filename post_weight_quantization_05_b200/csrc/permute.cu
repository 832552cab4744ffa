// Act-order (itwiki "GPTQ", section "실무 변형": the columns are processed in
// the order of decreasing Hessian diagonal, so that the columns whose inputs
// carry the most energy are quantized while the most freedom is left).
//
// Three stream-ordered kernels:
//   order_rank_kernel     perm = column indices by descending diag(H), ties by
//                         index, NaN last (a stable descending sort, computed
//                         as ranks: every rank is unique, so perm is always a
//                         permutation)
//   permute_sym_kernel    Hp[a][b] = H[perm[a]][perm[b]] of the symmetric H,
//                         read from H's upper triangle
//   permute_cols_kernel   dst[r][k] = src[r][perm[k]]  (into processing order)
//                         dst[r][perm[k]] = src[r][k]  (back to the original
//                         order); in place when src == dst
// All three are bound by HBM (or L2) traffic, not arithmetic.
#include <atomic>
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace perm {

constexpr int RANK_LANES = 32;   // i values per block (one per lane)
constexpr int RANK_PARTS = 32;   // j ranges per block (one per warp)
constexpr int ROW_THREADS = 256;

// Key whose ascending order is the processing order: larger diagonal first,
// -0 and +0 equal, every NaN after every number (and equal to each other).
__device__ __forceinline__ uint32_t order_key(float x) {
    if (x != x) return 0xFFFFFFFFu;
    const uint32_t u = __float_as_uint(x + 0.0f);   // -0 -> +0
    const uint32_t asc = (u & 0x80000000u) ? ~u : (u | 0x80000000u);   // ascending in x
    return ~asc;   // descending in x; a number never maps to 0xFFFFFFFF
}

// Block (RANK_PARTS warps x RANK_LANES lanes): lane l owns i = i0 + l, warp p
// counts the j of its range that come before i; the counts are summed and
// perm[rank(i)] = i.
__global__ void __launch_bounds__(RANK_LANES * RANK_PARTS)
    order_rank_kernel(const float* __restrict__ H, int d, int32_t* __restrict__ perm) {
    extern __shared__ uint32_t keys[];   // [d]
    __shared__ int partial[RANK_PARTS][RANK_LANES + 1];
    const int t = threadIdx.x;
    for (int j = t; j < d; j += blockDim.x) keys[j] = order_key(H[size_t(j) * d + j]);
    __syncthreads();
    const int lane = t % RANK_LANES, part = t / RANK_LANES;
    const int i = blockIdx.x * RANK_LANES + lane;
    int count = 0;
    if (i < d) {
        const uint32_t ki = keys[i];
        const int span = (d + RANK_PARTS - 1) / RANK_PARTS;
        const int j0 = part * span, j1 = min(d, j0 + span);
        for (int j = j0; j < j1; ++j) {
            const uint32_t kj = keys[j];
            count += (kj < ki) | ((kj == ki) & (j < i));
        }
    }
    partial[part][lane] = count;
    __syncthreads();
    if (part == 0 && i < d) {
        int rank = 0;
#pragma unroll 8
        for (int p = 0; p < RANK_PARTS; ++p) rank += partial[p][lane];
        perm[rank] = i;
    }
}

// One block per output row a: stage row perm[a] of the symmetric H in shared
// memory (the part right of the diagonal from row perm[a], the part left of
// it from column perm[a]), then write Hp[a][b] = row[perm[b]] coalesced.  An
// index outside [0, d) is reported and its outputs are NaN.
__global__ void __launch_bounds__(ROW_THREADS)
    permute_sym_kernel(const float* __restrict__ H, int d, const int32_t* __restrict__ perm,
                       float* __restrict__ Hp, DevStatus* st) {
    extern __shared__ float row[];   // [d]
    const int a = blockIdx.x;
    const int pa = perm[a];
    float* out = Hp + size_t(a) * d;
    if (pa < 0 || pa >= d) {
        if (threadIdx.x == 0) record_error(st, GPTQ_ERR_INVALID_ARG, a);
        for (int b = threadIdx.x; b < d; b += blockDim.x) out[b] = __int_as_float(0x7fc00000);
        return;
    }
    for (int c = threadIdx.x; c < d; c += blockDim.x)
        row[c] = c >= pa ? H[size_t(pa) * d + c] : H[size_t(c) * d + pa];
    __syncthreads();
    for (int b = threadIdx.x; b < d; b += blockDim.x) {
        const int pb = perm[b];
        float v = __int_as_float(0x7fc00000);
        if (pb >= 0 && pb < d) v = row[pb];
        else if (a == 0) record_error(st, GPTQ_ERR_INVALID_ARG, b);
        out[b] = v;
    }
}

// One block per row.  The row is read whole into shared memory before any of
// it is written, so src == dst is safe.  Forward: dst[k] = src[perm[k]];
// inverse: dst[perm[k]] = src[k] (slots that no index reaches stay NaN).
__global__ void __launch_bounds__(ROW_THREADS)
    permute_cols_kernel(const float* src, float* dst, int cols, const int32_t* __restrict__ perm, int inverse,
                        DevStatus* st) {
    extern __shared__ float row[];   // [cols]
    const size_t base = size_t(blockIdx.x) * cols;
    const float4* s4 = reinterpret_cast<const float4*>(src + base);
    float4* r4 = reinterpret_cast<float4*>(row);
    const float qnan = __int_as_float(0x7fc00000);
    const int n4 = cols / 4;
    if (!inverse) {
        for (int k = threadIdx.x; k < n4; k += blockDim.x) r4[k] = s4[k];
    } else {
        for (int k = threadIdx.x; k < n4; k += blockDim.x) r4[k] = make_float4(qnan, qnan, qnan, qnan);
    }
    __syncthreads();
    if (!inverse) {
        for (int k = threadIdx.x; k < cols; k += blockDim.x) {
            const int p = perm[k];
            float v = qnan;
            if (p >= 0 && p < cols) v = row[p];
            else if (blockIdx.x == 0) record_error(st, GPTQ_ERR_INVALID_ARG, k);
            dst[base + k] = v;
        }
    } else {
        // Read this thread's values before the barrier that precedes any write.
        for (int k = threadIdx.x; k < cols; k += blockDim.x) {
            const int p = perm[k];
            if (p >= 0 && p < cols) row[p] = src[base + k];
            else if (blockIdx.x == 0) record_error(st, GPTQ_ERR_INVALID_ARG, k);
        }
        __syncthreads();
        float4* d4 = reinterpret_cast<float4*>(dst + base);
        for (int k = threadIdx.x; k < n4; k += blockDim.x) d4[k] = r4[k];
    }
}

// Opt each kernel in to the largest row it can be given (32768 floats) once
// per device.
constexpr size_t MAX_ROW_SMEM = 32768 * sizeof(float);

int allow_big_rows(const void* fn, int slot) {
    static std::atomic<bool> done[64][3];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (dev >= 0 && dev < 64 && done[dev][slot]) return GPTQ_OK;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(MAX_ROW_SMEM)) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    if (dev >= 0 && dev < 64) done[dev][slot] = true;
    return GPTQ_OK;
}

}  // namespace perm

int launch_act_order_perm(const float* H, int64_t d, int32_t* out, cudaStream_t stream) {
    using namespace perm;
    const size_t smem = size_t(d) * sizeof(uint32_t);
    if (allow_big_rows(reinterpret_cast<const void*>(order_rank_kernel), 0)) return GPTQ_ERR_CUDA;
    const unsigned blocks = unsigned((d + RANK_LANES - 1) / RANK_LANES);
    order_rank_kernel<<<blocks, RANK_LANES * RANK_PARTS, smem, stream>>>(H, int(d), out);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

int launch_permute_hessian(const float* H, int64_t d, const int32_t* p, float* Hp, cudaStream_t stream,
                           DevStatus* st) {
    using namespace perm;
    const size_t smem = size_t(d) * sizeof(float);
    if (allow_big_rows(reinterpret_cast<const void*>(permute_sym_kernel), 1)) return GPTQ_ERR_CUDA;
    permute_sym_kernel<<<unsigned(d), ROW_THREADS, smem, stream>>>(H, int(d), p, Hp, st);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

int launch_permute_columns(const float* src, int64_t rows, int64_t cols, const int32_t* p, bool inverse,
                           float* dst, cudaStream_t stream, DevStatus* st) {
    using namespace perm;
    const size_t smem = size_t(cols) * sizeof(float);
    if (allow_big_rows(reinterpret_cast<const void*>(permute_cols_kernel), 2)) return GPTQ_ERR_CUDA;
    permute_cols_kernel<<<unsigned(rows), ROW_THREADS, smem, stream>>>(src, dst, int(cols), p, inverse ? 1 : 0,
                                                                        st);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
