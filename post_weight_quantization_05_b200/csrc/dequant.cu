// The weights rebuilt from the stored form (note "Model Quantization",
// section "주요 양자화 기법", the GPTQ entry: at inference the INT4 weights are
// restored to FP16 for the computation; blog "GPTQ를 밑바닥부터 구현하며 배운
// 것들", section 5: codes stored, dequantized for use):
//
//   Wq[r][perm[k]] = s[r][g(k)] (c[r][k] - z[r][g(k)])
//
// for codes of 2, 3, 4 or 8 bits in the packed little-endian stream, groups in
// processing order, and the act-order permutation undone (perm = NULL: the
// natural order).  fp32 output is exact (an fp16 scale times a small integer);
// fp16 / bf16 outputs are rounded to nearest even.
//
// Without a permutation one thread decodes a 32-code unit (`bits` words) and
// writes its 32 outputs directly.  With one, a block takes a row: the codes
// are decoded into shared memory at their original columns, then written out
// coalesced.  Bound by HBM: bits / 8 bytes per weight in, 2 or 4 out.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace dq {

constexpr int THREADS = 1024;   // the permuted path: one row per block

template <int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[BITS], int i) {
    if constexpr (BITS == 3) {
        const int bit = 3 * i, j = bit >> 5, sh = bit & 31;
        const uint64_t pair = uint64_t(w[j]) | (j + 1 < 3 ? uint64_t(w[j + 1]) << 32 : 0ull);
        return uint32_t(pair >> sh) & 7u;
    } else {
        constexpr int PER = 32 / BITS;
        return (w[i / PER] >> ((i % PER) * BITS)) & ((1u << BITS) - 1u);
    }
}

// Shared-memory slot of column k: one pad float per 32 columns, so that a
// warp whose threads each write 32 consecutive columns hits 32 banks.
__device__ __forceinline__ int slot(int k) { return k + (k >> 5); }

template <int BITS>
__global__ void __launch_bounds__(THREADS)
    dequant_rows_kernel(const uint32_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                        const uint16_t* __restrict__ zeros, int d_in, int group, int n_groups,
                        const int32_t* __restrict__ perm, int out_dtype, void* out, DevStatus* st) {
    extern __shared__ float row[];   // [d_in + d_in / 32], original column order, padded
    const int r = blockIdx.x;
    const uint32_t* crow = codes + size_t(r) * (size_t(d_in) * BITS / 32);
    const uint16_t* srow = scales + size_t(r) * n_groups;
    const uint16_t* zrow = zeros + size_t(r) * n_groups;
    if (perm) {   // a column that no entry reaches (a duplicate entry) stays NaN
        for (int k = threadIdx.x; k < d_in; k += THREADS) row[slot(k)] = __int_as_float(0x7fc00000);
        __syncthreads();
    }
    for (int u = threadIdx.x; u < d_in / 32; u += THREADS) {
        uint32_t w[BITS];
#pragma unroll
        for (int j = 0; j < BITS; ++j) w[j] = crow[u * BITS + j];
        const int gi = (u * 32) / group;                  // a group is a multiple of 128 columns
        const float s = __half2float(__ushort_as_half(srow[gi]));
        const float z = __half2float(__ushort_as_half(zrow[gi]));
        int dst[32];
        if (perm) {
            const int4* p4 = reinterpret_cast<const int4*>(perm + u * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int4 v = p4[j];
                dst[4 * j] = v.x; dst[4 * j + 1] = v.y; dst[4 * j + 2] = v.z; dst[4 * j + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) dst[i] = u * 32 + i;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float v = s * (float(code_at<BITS>(w, i)) - z);
            if (dst[i] >= 0 && dst[i] < d_in) row[slot(dst[i])] = v;
            else if (r == 0) record_error(st, GPTQ_ERR_INVALID_ARG, u * 32 + i);
        }
    }
    __syncthreads();
    if (out_dtype == 0) {
        float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + size_t(r) * d_in);
        for (int i = threadIdx.x; i < d_in / 4; i += THREADS)
            o[i] = make_float4(row[slot(4 * i)], row[slot(4 * i + 1)], row[slot(4 * i + 2)], row[slot(4 * i + 3)]);
    } else {
        uint2* o = reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + size_t(r) * d_in);
        for (int i = threadIdx.x; i < d_in / 4; i += THREADS) {
            uint16_t h[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float v = row[slot(4 * i + e)];
                h[e] = out_dtype == 1 ? __bfloat16_as_ushort(__float2bfloat16_rn(v)) : __half_as_ushort(__float2half_rn(v));
            }
            o[i] = make_uint2(uint32_t(h[0]) | (uint32_t(h[1]) << 16), uint32_t(h[2]) | (uint32_t(h[3]) << 16));
        }
    }
}

// Without a permutation: one thread per 32-code unit anywhere in the matrix,
// writing its 32 outputs straight to global memory (a warp covers 32
// consecutive units of a row: contiguous, coalesced stores).
template <int BITS>
__global__ void __launch_bounds__(256)
    dequant_direct_kernel(const uint32_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                          const uint16_t* __restrict__ zeros, int64_t d_out, int d_in, int group, int n_groups,
                          int out_dtype, void* out) {
    const int upr = d_in / 32;
    const int64_t units = d_out * upr;
    for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < units; e += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = e / upr;
        const int u = int(e - r * upr);
        uint32_t w[BITS];
        const uint32_t* src = codes + size_t(e) * BITS;       // unit e of the row-major stream
#pragma unroll
        for (int j = 0; j < BITS; ++j) w[j] = src[j];
        const size_t gsel = size_t(r) * n_groups + (u * 32) / group;
        const float s = __half2float(__ushort_as_half(scales[gsel]));
        const float z = __half2float(__ushort_as_half(zeros[gsel]));
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = s * (float(code_at<BITS>(w, i)) - z);
        if (out_dtype == 0) {
            float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + size_t(e) * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else {
            uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + size_t(e) * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t h[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float a = v[8 * i + 2 * j], b = v[8 * i + 2 * j + 1];
                    h[j] = out_dtype == 1 ? (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(a))) |
                                             (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(b))) << 16))
                                          : (uint32_t(__half_as_ushort(__float2half_rn(a))) |
                                             (uint32_t(__half_as_ushort(__float2half_rn(b))) << 16));
                }
                o[i] = make_uint4(h[0], h[1], h[2], h[3]);
            }
        }
    }
}

}  // namespace dq

int launch_dequantize(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                      int64_t d_in, int bits, int groupsize, const int32_t* perm, int out_dtype, void* out,
                      cudaStream_t stream, DevStatus* st) {
    using namespace dq;
    const int group = groupsize > 0 ? groupsize : int(d_in);
    const int n_groups = int(d_in / group);
    const size_t smem = size_t(d_in + d_in / 32) * sizeof(float);
    static bool attr_done[64][4] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
    const int which = bits == 2 ? 0 : bits == 3 ? 1 : bits == 4 ? 2 : 3;
    const void* fn = bits == 2   ? reinterpret_cast<const void*>(dequant_rows_kernel<2>)
                     : bits == 3 ? reinterpret_cast<const void*>(dequant_rows_kernel<3>)
                     : bits == 4 ? reinterpret_cast<const void*>(dequant_rows_kernel<4>)
                                 : reinterpret_cast<const void*>(dequant_rows_kernel<8>);
    if (dev < 0 || dev >= 64 || !attr_done[dev][which]) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (32768 + 1024) * 4) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        if (dev >= 0 && dev < 64) attr_done[dev][which] = true;
    }
    if (!perm) {
        const int64_t units = d_out * (d_in / 32);
        const unsigned blocks = unsigned(std::min<int64_t>((units + 255) / 256, 148 * 16));
        switch (bits) {
            case 2: dequant_direct_kernel<2><<<blocks, 256, 0, stream>>>(codes, scales, zeros, d_out, int(d_in), group, n_groups, out_dtype, out); break;
            case 3: dequant_direct_kernel<3><<<blocks, 256, 0, stream>>>(codes, scales, zeros, d_out, int(d_in), group, n_groups, out_dtype, out); break;
            case 4: dequant_direct_kernel<4><<<blocks, 256, 0, stream>>>(codes, scales, zeros, d_out, int(d_in), group, n_groups, out_dtype, out); break;
            case 8: dequant_direct_kernel<8><<<blocks, 256, 0, stream>>>(codes, scales, zeros, d_out, int(d_in), group, n_groups, out_dtype, out); break;
            default: return GPTQ_ERR_UNSUPPORTED;
        }
        count_launch();
        return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
    }
    const dim3 grid{unsigned(d_out)}, block{unsigned(THREADS)};
    switch (bits) {
        case 2: dequant_rows_kernel<2><<<grid, block, smem, stream>>>(codes, scales, zeros, int(d_in), group, n_groups, perm, out_dtype, out, st); break;
        case 3: dequant_rows_kernel<3><<<grid, block, smem, stream>>>(codes, scales, zeros, int(d_in), group, n_groups, perm, out_dtype, out, st); break;
        case 4: dequant_rows_kernel<4><<<grid, block, smem, stream>>>(codes, scales, zeros, int(d_in), group, n_groups, perm, out_dtype, out, st); break;
        case 8: dequant_rows_kernel<8><<<grid, block, smem, stream>>>(codes, scales, zeros, int(d_in), group, n_groups, perm, out_dtype, out, st); break;
        default: return GPTQ_ERR_UNSUPPORTED;
    }
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
