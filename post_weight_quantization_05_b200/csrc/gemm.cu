// fp32 SIMT GEMM used by the factorization (panel solve, trailing SYRK,
// triangular inverse) and by the sweep's lazy trailing update.  These
// products need fp32 accuracy: a single bf16 or tf32 tensor-core product
// changes GPTQ codes, so they run on the fp32 FMA pipes.
//
// C[M,N] = alpha * A[M,K] * op(B)[K,N] + beta * C_in, row-major.
// 128 x 128 output tile per CTA, K step 8, 256 threads with an 8 x 8
// register tile each (two 4-row x two 4-column sub-blocks so that shared-
// memory reads are broadcasts / conflict-free), register-prefetched double
// buffering of the shared-memory tiles.
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace gemm {

constexpr int TM = 128, TN = 128, TK = 8, PAD = 4, THREADS = 256;

template <bool TRANS_B>
__device__ __forceinline__ void load_tiles(const float* __restrict__ A, int lda, const float* __restrict__ B,
                                           int ldb, int M, int N, int K, int m0, int n0, int k0, float (&ra)[4],
                                           float (&rb)[4]) {
    const int t = threadIdx.x;
    {   // A tile: row t/2, k offset (t%2)*4
        const int m = m0 + (t >> 1), k = k0 + (t & 1) * 4;
        if (m < M && k + 3 < K) {
            const float4 v = *reinterpret_cast<const float4*>(A + size_t(m) * lda + k);
            ra[0] = v.x; ra[1] = v.y; ra[2] = v.z; ra[3] = v.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) ra[i] = (m < M && k + i < K) ? A[size_t(m) * lda + k + i] : 0.0f;
        }
    }
    if (!TRANS_B) {   // B tile: k = t/32, n offset (t%32)*4
        const int k = k0 + (t >> 5), n = n0 + (t & 31) * 4;
        if (k < K && n + 3 < N) {
            const float4 v = *reinterpret_cast<const float4*>(B + size_t(k) * ldb + n);
            rb[0] = v.x; rb[1] = v.y; rb[2] = v.z; rb[3] = v.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) rb[i] = (k < K && n + i < N) ? B[size_t(k) * ldb + n + i] : 0.0f;
        }
    } else {          // B^T tile: n = t/2, k offset (t%2)*4
        const int n = n0 + (t >> 1), k = k0 + (t & 1) * 4;
        if (n < N && k + 3 < K) {
            const float4 v = *reinterpret_cast<const float4*>(B + size_t(n) * ldb + k);
            rb[0] = v.x; rb[1] = v.y; rb[2] = v.z; rb[3] = v.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) rb[i] = (n < N && k + i < K) ? B[size_t(n) * ldb + k + i] : 0.0f;
        }
    }
}

template <bool TRANS_B>
__device__ __forceinline__ void store_tiles(float (*As)[TM + PAD], float (*Bs)[TN + PAD], const float (&ra)[4],
                                            const float (&rb)[4]) {
    const int t = threadIdx.x;
#pragma unroll
    for (int i = 0; i < 4; ++i) As[(t & 1) * 4 + i][t >> 1] = ra[i];
    if (!TRANS_B) {
        *reinterpret_cast<float4*>(&Bs[t >> 5][(t & 31) * 4]) = make_float4(rb[0], rb[1], rb[2], rb[3]);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) Bs[(t & 1) * 4 + i][t >> 1] = rb[i];
    }
}

template <bool TRANS_B>
__global__ void __launch_bounds__(THREADS, 2)
    sgemm_kernel(int M, int N, int K, float alpha, const float* __restrict__ A, int lda, const float* __restrict__ B,
                 int ldb, float beta, const float* C_in, float* C_out, int ldc, int lower_only) {
    __shared__ __align__(16) float As[2][TK][TM + PAD];
    __shared__ __align__(16) float Bs[2][TK][TN + PAD];
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    if (lower_only && n0 > m0 + TM - 1) return;
    const int t = threadIdx.x, ty = t >> 4, tx = t & 15;

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

    float ra[4], rb[4];
    load_tiles<TRANS_B>(A, lda, B, ldb, M, N, K, m0, n0, 0, ra, rb);
    store_tiles<TRANS_B>(As[0], Bs[0], ra, rb);
    __syncthreads();

    int buf = 0;
    for (int k0 = 0; k0 < K; k0 += TK) {
        const bool more = k0 + TK < K;
        if (more) load_tiles<TRANS_B>(A, lda, B, ldb, M, N, K, m0, n0, k0 + TK, ra, rb);
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        if (more) {
            store_tiles<TRANS_B>(As[buf ^ 1], Bs[buf ^ 1], ra, rb);
            __syncthreads();
            buf ^= 1;
        }
    }

#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
        if (m >= M) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int n = n0 + h * 64 + tx * 4;
            if (n + 3 < N) {
                float4 r;
                const float* a4 = &acc[i][h * 4];
                if (beta != 0.0f) {
                    const float4 c = *reinterpret_cast<const float4*>(C_in + size_t(m) * ldc + n);
                    r = make_float4(fmaf(alpha, a4[0], beta * c.x), fmaf(alpha, a4[1], beta * c.y),
                                    fmaf(alpha, a4[2], beta * c.z), fmaf(alpha, a4[3], beta * c.w));
                } else {
                    r = make_float4(alpha * a4[0], alpha * a4[1], alpha * a4[2], alpha * a4[3]);
                }
                *reinterpret_cast<float4*>(C_out + size_t(m) * ldc + n) = r;
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (n + j < N) {
                        const float c = beta != 0.0f ? beta * C_in[size_t(m) * ldc + n + j] : 0.0f;
                        C_out[size_t(m) * ldc + n + j] = fmaf(alpha, acc[i][h * 4 + j], c);
                    }
                }
            }
        }
    }
}

}  // namespace gemm

int launch_sgemm(int M, int N, int K, float alpha, const float* A, int lda, const float* B, int ldb, bool trans_b,
                 float beta, const float* C_in, float* C_out, int ldc, bool lower_only, cudaStream_t stream) {
    using namespace gemm;
    if (M <= 0 || N <= 0) return GPTQ_OK;
    dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
    if (trans_b)
        sgemm_kernel<true><<<grid, THREADS, 0, stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C_in, C_out, ldc,
                                                         lower_only ? 1 : 0);
    else
        sgemm_kernel<false><<<grid, THREADS, 0, stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C_in, C_out, ldc,
                                                          lower_only ? 1 : 0);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
