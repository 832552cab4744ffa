// Stage 2: dampening and U = upper Cholesky factor of (H + lambda I)^-1.
//
// Source: itwiki "GPTQ", "GPTQ의 세 가지 변경" row 3 (dampening by 1% of the
// mean diagonal; the rows of the Cholesky form of H^-1 are all the sweep
// needs, so it is computed once up front), "알고리즘" and "최소 구현" (the
// chain chol -> cholesky_inverse -> chol(upper)).
//
// Route taken here (same U, fewer flops): with P the index reversal,
// H + lambda I = U^-1 U^-T and P U^-1 P is lower triangular with a positive
// diagonal, so it is L' = chol(P (H + lambda I) P) and U = P L'^-1 P.  That is
// one Cholesky (d^3/3 flops) plus one triangular inverse (d^3/3) instead of
// the chain's chol + inverse + chol.
//
// All arithmetic is fp32.  Blocked right-looking, block nb = 128:
//   per diagonal block: one CTA factors it in shared memory and inverts the
//   factor (potrf_diag_kernel); the panel below is solved against it with an
//   SGEMM by the inverse; the trailing lower triangle gets a SYRK-shaped
//   SGEMM.  The inverse L'^-1 is then built block row by block row
//   (right-looking forward substitution on the identity), and U is written
//   by reversing both indices.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace factor {

constexpr int NB = 128;
constexpr int LD = NB + 1;   // padded shared-memory row (column accesses conflict-free)
constexpr int LDY = NB + 4;  // inverse rows: 16-byte aligned for vector access
constexpr int DIAG_THREADS = 256;
constexpr size_t DIAG_SMEM = size_t(NB) * (LD + LDY) * sizeof(float);

struct Layout {
    size_t a_off, y_off, dinv_off, scal_off, total;
};

__host__ __device__ inline Layout layout(int64_t d) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    Layout L;
    L.a_off = 0;
    L.y_off = up(L.a_off + size_t(d) * d * sizeof(float));
    L.dinv_off = up(L.y_off + size_t(d) * d * sizeof(float));
    L.scal_off = up(L.dinv_off + size_t(d) * NB * sizeof(float));
    L.total = L.scal_off + 256;
    return L;
}

// lambda = percdamp * mean(diag H); also resets *info.
__global__ void damp_lambda_kernel(const float* __restrict__ H, int d, float percdamp, float* lam, int* info,
                                   DevStatus* st) {
    __shared__ double part[32];
    double s = 0.0;
    for (int i = threadIdx.x; i < d; i += blockDim.x) s += double(H[size_t(i) * d + i]);
    for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double tot = 0.0;
        for (int w = 0; w < int(blockDim.x >> 5); ++w) tot += part[w];
        const float l = float(double(percdamp) * (tot / double(d)));
        *lam = l;
        *info = 0;
        if (!isfinite(l)) record_error(st, GPTQ_ERR_NONFINITE, -1);
    }
}

// A[i][j] = H[d-1-i][d-1-j] (+ lambda on the diagonal) for j <= i: the lower
// triangle of P (H + lambda I) P, read from the upper triangle of H.
__global__ void reverse_damp_kernel(const float* __restrict__ H, int d, const float* __restrict__ lam,
                                    float* __restrict__ A) {
    const float l = *lam;
    const size_t total = size_t(d) * d;
    for (size_t idx = size_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += size_t(gridDim.x) * blockDim.x) {
        const int i = int(idx / d), j = int(idx % d);
        if (j > i) continue;
        float v = H[size_t(d - 1 - i) * d + (d - 1 - j)];
        if (i == j) v += l;
        A[idx] = v;
    }
}

// ---------------------------------------------------------------------------
// One 128 x 128 diagonal block: L L^T = A_kk (in place, lower) and L^-1.
// The block is cut into 4 x 4 sub-blocks of 32.  For each sub-block column:
// one warp factors the 32 x 32 diagonal sub-block in registers (lane = row,
// column broadcasts by shuffles) and inverts it; all 8 warps then solve the
// sub-blocks below against it and update the trailing sub-blocks.  Finally
// the off-diagonal sub-blocks of L^-1 are formed from the diagonal ones.
// ---------------------------------------------------------------------------
constexpr int SB = 32;
constexpr unsigned FULL = 0xffffffffu;

// The 32 x 32 pieces are written as template recursions so that every
// register index is a compile-time constant (a rolled or partly unrolled loop
// would put the row in local memory).

// One row a[] (32 values) solved against L (32 x 32 lower, in shared memory
// with row stride LD):  a <- a L^-T  (right-looking, invd[c] = 1/L[c][c]).
template <int C>
struct Trsm32 {
    __device__ __forceinline__ static void run(float (&a)[SB], const float* __restrict__ L,
                                               const float* __restrict__ invd) {
        const float xc = a[C] * invd[C];
        a[C] = xc;
#pragma unroll
        for (int j = C + 1; j < SB; ++j) a[j] = fmaf(-xc, L[j * LD + C], a[j]);
        if constexpr (C + 1 < SB) Trsm32<C + 1>::run(a, L, invd);
    }
};

// Column-oriented Cholesky of a 32 x 32 block by one warp: lane j holds
// column j (col[r] = A[r][j]; entries above the diagonal are ignored).  At
// step C lane C finalizes its column and publishes it through `buf` (shared
// memory); every later lane then updates its own column with one broadcast
// read per row -- no shuffles, one short dependency chain per column.
template <int C>
struct ColChol32 {
    __device__ __forceinline__ static void run(float (&col)[SB], int lane, float* __restrict__ buf, int& bad,
                                               float& badpiv) {
        if (lane == C) {
            const float piv = col[C];
            if (bad < 0 && (!(piv > 0.0f) || !isfinite(piv))) { bad = C; badpiv = piv; }
            const float inv = rsqrtf(piv);
            col[C] = piv * inv;
#pragma unroll
            for (int r = C + 1; r < SB; ++r) col[r] *= inv;
#pragma unroll
            for (int r = (C / 4) * 4; r < SB; r += 4)      // whole 16-byte groups; entries < C unused
                *reinterpret_cast<float4*>(buf + r) = make_float4(col[r], col[r + 1], col[r + 2], col[r + 3]);
        }
        __syncwarp();
        if (lane > C) {
            const float ljc = buf[lane];                  // L[lane][C]
#pragma unroll
            for (int r4 = ((C + 1) / 4) * 4; r4 < SB; r4 += 4) {
                const float4 b = *reinterpret_cast<const float4*>(buf + r4);
                if (r4 + 0 > C) col[r4 + 0] = fmaf(-b.x, ljc, col[r4 + 0]);
                if (r4 + 1 > C) col[r4 + 1] = fmaf(-b.y, ljc, col[r4 + 1]);
                if (r4 + 2 > C) col[r4 + 2] = fmaf(-b.z, ljc, col[r4 + 2]);
                if (r4 + 3 > C) col[r4 + 3] = fmaf(-b.w, ljc, col[r4 + 3]);
            }
        }
        __syncwarp();
        if constexpr (C + 1 < SB) ColChol32<C + 1>::run(col, lane, buf, bad, badpiv);
    }
};

// Column-oriented inverse of a 32 x 32 lower-triangular L held in shared
// memory (row stride LD, 1/L[i][i] in invd): lane j computes column j of
// L^-1 (y[i] for i >= j) by forward substitution, reading L by broadcast.
template <int I>
struct ColInv32 {
    __device__ __forceinline__ static void run(float (&y)[SB], const float* __restrict__ L,
                                               const float* __restrict__ invd, int lane) {
        const float yi = y[I] * invd[I];
        y[I] = yi;
#pragma unroll
        for (int r = I + 1; r < SB; ++r) y[r] = fmaf(-L[r * LD + I], yi, y[r]);
        if constexpr (I + 1 < SB) ColInv32<I + 1>::run(y, L, invd, lane);
    }
};

// Factor the diagonal block A[k0:k0+NB, k0:k0+NB] = L L^T in place (lower) and
// write its inverse L^-1 to Dinv (NB x NB, row-major).  A non-positive or
// non-finite pivot sets *info = k0 + c + 1 (first failure only).
__global__ void __launch_bounds__(DIAG_THREADS)
    potrf_diag_kernel(float* __restrict__ A, int d, int k0, float* __restrict__ Dinv, int* info, DevStatus* st) {
    extern __shared__ float sm[];
    float* S = sm;             // [NB][LD] factor (upper part used as scratch)
    float* Y = sm + NB * LD;   // [NB][LDY] inverse (NB * LD is a multiple of 4: 16-byte aligned)
    __shared__ float invd[NB];
    __shared__ __align__(16) float colbuf[SB];
    __shared__ int failed;
    if (*info != 0) return;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
#pragma unroll 4
    for (int idx = 4 * t; idx < NB * NB; idx += 4 * DIAG_THREADS) {
        const int r = idx / NB, c = idx % NB;
        const float4 v = *reinterpret_cast<const float4*>(A + size_t(k0 + r) * d + k0 + c);
        S[r * LD + c] = (c <= r) ? v.x : 0.0f;
        S[r * LD + c + 1] = (c + 1 <= r) ? v.y : 0.0f;
        S[r * LD + c + 2] = (c + 2 <= r) ? v.z : 0.0f;
        S[r * LD + c + 3] = (c + 3 <= r) ? v.w : 0.0f;
    }
    for (int idx = t; idx < NB * LDY; idx += DIAG_THREADS) Y[idx] = 0.0f;
    if (t == 0) failed = 0;
    __syncthreads();

    for (int kb = 0; kb < NB / SB; ++kb) {
        const int o = kb * SB;
        if (warp == 0) {
            float col[SB];
#pragma unroll
            for (int r = 0; r < SB; ++r) col[r] = (r >= lane) ? S[(o + r) * LD + o + lane] : 0.0f;
            int bad = -1;
            float badpiv = 0.0f;
            ColChol32<0>::run(col, lane, colbuf, bad, badpiv);
#pragma unroll
            for (int r = 0; r < SB; ++r)
                if (r >= lane) S[(o + r) * LD + o + lane] = col[r];
            __syncwarp();
            invd[o + lane] = 1.0f / S[(o + lane) * LD + o + lane];
            bad = __reduce_min_sync(FULL, bad < 0 ? SB : bad);
            const float p = __shfl_sync(FULL, badpiv, bad < SB ? bad : 0);   // the failing pivot's value
            if (bad < SB && lane == 0) {
                failed = 1;
                if (atomicCAS(info, 0, k0 + o + bad + 1) == 0)
                    record_error(st, isfinite(p) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE, k0 + o + bad + 1);
            }
        }
        __syncthreads();
        if (failed) return;
        const int below = NB - o - SB;
        if (below == 0) break;
        // solve the rows below against this sub-block: S[r][o..o+32) <- S[r][o..o+32) L_kk^-T
        if (t < below) {
            const int r = o + SB + t;
            float a[SB];
#pragma unroll
            for (int k = 0; k < SB; ++k) a[k] = S[r * LD + o + k];
            Trsm32<0>::run(a, S + o * LD + o, invd + o);
#pragma unroll
            for (int k = 0; k < SB; ++k) S[r * LD + o + k] = a[k];
        }
        __syncthreads();
        // trailing update of the sub-blocks (bi, bj), kb < bj <= bi
        {
            const int i = t >> 3, j4 = (t & 7) * 4;
            for (int bi = kb + 1; bi < NB / SB; ++bi) {
                for (int bj = kb + 1; bj <= bi; ++bj) {
                    const int r = bi * SB + i;
                    float acc[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[q] = S[r * LD + bj * SB + j4 + q];
#pragma unroll 8
                    for (int k = 0; k < SB; ++k) {
                        const float av = S[r * LD + o + k];
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[q] = fmaf(-av, S[(bj * SB + j4 + q) * LD + o + k], acc[q]);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) S[r * LD + bj * SB + j4 + q] = acc[q];
                }
            }
        }
        __syncthreads();
    }

    // inverse: the four diagonal sub-blocks in parallel (warps 0..3), one
    // column of L^-1 per lane ...
    if (warp < NB / SB) {
        const int o = warp * SB;
        float y[SB];
#pragma unroll
        for (int r = 0; r < SB; ++r) y[r] = (r == lane) ? 1.0f : 0.0f;
        ColInv32<0>::run(y, S + o * LD + o, invd + o, lane);
#pragma unroll
        for (int r = 0; r < SB; ++r) Y[(o + r) * LDY + o + lane] = (r >= lane) ? y[r] : 0.0f;
    }
    __syncthreads();

    // ... then the off-diagonal ones:  Y[bi][bj] = -Y[bi][bi] * sum_{k=bj}^{bi-1} L[bi][k] Y[k][bj]
    // T[bj] is kept in the (unused) strictly upper sub-blocks (0, 1 + bj) of S.
    {
        const int i = t >> 3, j4 = (t & 7) * 4;
        for (int bi = 1; bi < NB / SB; ++bi) {
            // one pass over k serves every bj (independent accumulators)
            float4 acc[NB / SB - 1];
#pragma unroll
            for (int bj = 0; bj < NB / SB - 1; ++bj) acc[bj] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            const float* lrow = S + (bi * SB + i) * LD;
#pragma unroll 4
            for (int k = 0; k < bi * SB; ++k) {
                const float l = lrow[k];
#pragma unroll
                for (int bj = 0; bj < NB / SB - 1; ++bj) {
                    if (bj < bi && k >= bj * SB) {
                        const float4 y = *reinterpret_cast<const float4*>(Y + k * LDY + bj * SB + j4);
                        acc[bj].x = fmaf(l, y.x, acc[bj].x); acc[bj].y = fmaf(l, y.y, acc[bj].y);
                        acc[bj].z = fmaf(l, y.z, acc[bj].z); acc[bj].w = fmaf(l, y.w, acc[bj].w);
                    }
                }
            }
#pragma unroll
            for (int bj = 0; bj < NB / SB - 1; ++bj) {
                if (bj < bi) {
                    float* trow = S + i * LD + (1 + bj) * SB + j4;
                    trow[0] = acc[bj].x; trow[1] = acc[bj].y; trow[2] = acc[bj].z; trow[3] = acc[bj].w;
                }
            }
            __syncthreads();
            for (int bj = 0; bj < bi; ++bj) {
                float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                const float* yrow = Y + (bi * SB + i) * LDY + bi * SB;
                for (int k = 0; k <= i; ++k) {
                    const float y = yrow[k];
                    const float* trow = S + k * LD + (1 + bj) * SB + j4;
                    acc.x = fmaf(y, trow[0], acc.x); acc.y = fmaf(y, trow[1], acc.y);
                    acc.z = fmaf(y, trow[2], acc.z); acc.w = fmaf(y, trow[3], acc.w);
                }
                *reinterpret_cast<float4*>(Y + (bi * SB + i) * LDY + bj * SB + j4) =
                    make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
            }
            __syncthreads();
        }
    }

#pragma unroll 4
    for (int idx = 4 * t; idx < NB * NB; idx += 4 * DIAG_THREADS) {
        const int r = idx / NB, c = idx % NB;
        float* arow = A + size_t(k0 + r) * d + k0 + c;
        if (c + 3 <= r) {
            *reinterpret_cast<float4*>(arow) =
                make_float4(S[r * LD + c], S[r * LD + c + 1], S[r * LD + c + 2], S[r * LD + c + 3]);
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (c + q <= r) arow[q] = S[r * LD + c + q];
        }
        const float4 yv = *reinterpret_cast<const float4*>(Y + r * LDY + c);
        *reinterpret_cast<float4*>(Dinv + idx) =
            make_float4((c <= r) ? yv.x : 0.0f, (c + 1 <= r) ? yv.y : 0.0f, (c + 2 <= r) ? yv.z : 0.0f,
                        (c + 3 <= r) ? yv.w : 0.0f);
    }
}

// Z[k*NB + c][k*NB + r] = Dinv_k[r][c]: diagonal block k of Z = L^-T,
// transposed through shared memory (coalesced on both sides).
__global__ void place_diag_inverse_t_kernel(const float* __restrict__ Dinv_k, int d, int k, float* __restrict__ Z) {
    extern __shared__ float tile[];   // [NB][LD]
    for (int idx = 4 * threadIdx.x; idx < NB * NB; idx += 4 * blockDim.x) {
        const int r = idx / NB, c = idx % NB;
        const float4 v = *reinterpret_cast<const float4*>(Dinv_k + idx);
        tile[r * LD + c] = v.x; tile[r * LD + c + 1] = v.y; tile[r * LD + c + 2] = v.z; tile[r * LD + c + 3] = v.w;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
        const int c = idx / NB, r = idx % NB;
        Z[size_t(k * NB + c) * d + k * NB + r] = tile[r * LD + c];
    }
}

// Three internal streams and a few events per device (created on first use).
// The factorization's critical chain runs on a high-priority stream; the
// inverse's block steps run on another, each as soon as the factorization has
// finished the block column it needs; the trailing update beyond the next
// block column runs on a low-priority stream, so that the next diagonal block
// is factored while it proceeds (look-ahead) and gets the SMs first.
struct AuxStream {
    cudaStream_t main = nullptr;    // the factorization's critical chain (highest priority)
    cudaStream_t s = nullptr;       // inverse steps
    cudaStream_t side = nullptr;    // trailing updates beyond the next block column
    cudaEvent_t fork = nullptr, step = nullptr, rest = nullptr, join = nullptr, join_side = nullptr;
};

static int aux_stream(AuxStream** out) {
    static std::mutex mu;
    static AuxStream per_dev[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    AuxStream& a = per_dev[dev];
    if (!a.s) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&a.main, cudaStreamNonBlocking, greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&a.s, cudaStreamNonBlocking, greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&a.side, cudaStreamNonBlocking, least) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.step, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.rest, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.join_side, cudaEventDisableTiming) != cudaSuccess)
            return GPTQ_ERR_CUDA;
    }
    *out = &a;
    return GPTQ_OK;
}

// U[r][c] = Z[d-1-c][d-1-r] for r <= c (U = P L'^-1 P = P Z^T P), 0 below the
// diagonal; NaN everywhere if the factorization failed.  32 x 32 tiles are
// transposed through shared memory so that both sides stay coalesced.
__global__ void write_u_kernel(const float* __restrict__ Z, int d, const int* __restrict__ info,
                               float* __restrict__ U) {
    __shared__ float tile[32][33];
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    const bool bad = *info != 0;
    const bool below = c0 + 31 < r0;    // tile entirely in the strict lower triangle
    if (!below && !bad) {
        for (int cc = threadIdx.y; cc < 32; cc += blockDim.y)
            tile[cc][threadIdx.x] = Z[size_t(d - 1 - (c0 + cc)) * d + (d - 1 - (r0 + threadIdx.x))];
    }
    __syncthreads();
    for (int rr = threadIdx.y; rr < 32; rr += blockDim.y) {
        const int r = r0 + rr, c = c0 + threadIdx.x;
        float v = (!below && c >= r) ? tile[threadIdx.x][rr] : 0.0f;
        if (bad) v = __int_as_float(0x7fc00000);
        U[size_t(r) * d + c] = v;
    }
}

}  // namespace factor

size_t factor_workspace_bytes(int64_t d) { return factor::layout(d).total; }

int launch_prepare_hinv(const float* H, int64_t d64, float percdamp, float* U, int* info_user, void* ws,
                        cudaStream_t stream, DevStatus* st) {
    using namespace factor;
    const int d = int(d64);
    const Layout L = layout(d64);
    uint8_t* base = static_cast<uint8_t*>(ws);
    float* A = reinterpret_cast<float*>(base + L.a_off);
    float* Z = reinterpret_cast<float*>(base + L.y_off);
    float* Dinv = reinterpret_cast<float*>(base + L.dinv_off);
    float* lam = reinterpret_cast<float*>(base + L.scal_off);
    int* info = info_user ? info_user : reinterpret_cast<int*>(base + L.scal_off + 64);
    const int nblk = d / NB;
    const int ew_blocks = int(std::min<int64_t>((int64_t(d) * d + 255) / 256, 148 * 32));

    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(potrf_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(DIAG_SMEM)) !=
                cudaSuccess ||
            cudaFuncSetAttribute(place_diag_inverse_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(NB * LD * sizeof(float))) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        attr_set[dev] = true;
    }

    // One call enqueues at a time (per process): the auxiliary stream and its
    // events are shared by every call on a device.
    static std::mutex enqueue_mu;
    std::lock_guard<std::mutex> enqueue_lock(enqueue_mu);
    AuxStream* aux = nullptr;
    if (aux_stream(&aux)) return GPTQ_ERR_CUDA;
    const cudaStream_t as = aux->s;
    const cudaStream_t caller = stream;
    stream = aux->main;
    if (cudaEventRecord(aux->fork, caller) != cudaSuccess || cudaStreamWaitEvent(stream, aux->fork, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;

    damp_lambda_kernel<<<1, 1024, 0, stream>>>(H, d, percdamp, lam, info, st); count_launch();
    reverse_damp_kernel<<<ew_blocks, 256, 0, stream>>>(H, d, lam, A); count_launch();
    // fork: the inverse (stream `as`) starts from a zeroed Z; `ss` takes the
    // trailing updates beyond the next block column
    const cudaStream_t ss = aux->side;
    if (cudaEventRecord(aux->fork, stream) != cudaSuccess || cudaStreamWaitEvent(as, aux->fork, 0) != cudaSuccess ||
        cudaStreamWaitEvent(ss, aux->fork, 0) != cudaSuccess || cudaEventRecord(aux->rest, ss) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    {
        const int rc = launch_fill(Z, int64_t(d) * d, 0.0f, as);
        if (rc) return rc;
    }

    // Cholesky of A (lower), blocked right-looking, products on the tensor
    // cores.  Step k on `stream`: factor the diagonal block, solve the panel,
    // update the next block column (after the previous step's far update on
    // `ss` is done); the rest of the trailing update goes to `ss`.
    // Z = L^-T (upper) on `as`: block step i needs only L's block column i and
    // Dinv_i, so it runs as soon as the factorization has them:
    //   Z[i][i] = Dinv_i^T;  Z[0:i0, i] <- Z[0:i0, i] Dinv_i^T;
    //   Z[0:i0+NB, i0+NB:] -= Z[0:i0+NB, i] L[i0+NB:, i]^T
    // (the transpose of the block forward substitution Y = L^-1; working on Z
    // keeps every tensor-core operand K-major).
    for (int k = 0; k < nblk; ++k) {
        const int k0 = k * NB;
        float* dk = Dinv + size_t(k) * NB * NB;
        potrf_diag_kernel<<<1, DIAG_THREADS, DIAG_SMEM, stream>>>(A, d, k0, dk, info, st); count_launch();
        const int rest = d - k0 - NB;
        float* panel = A + size_t(k0 + NB) * d + k0;
        int rc;
        if (rest > 0) {
            // panel <- panel * Dinv_k^T.  In place is safe: N = NB is one output
            // tile column, so each CTA reads only the rows it writes, all before
            // its epilogue.
            rc = launch_tgemm(rest, NB, NB, 1.0f, panel, nullptr, d, dk, nullptr, NB, false, panel, d, false, stream, st);
            if (rc) return rc;
        }
        if (cudaEventRecord(aux->step, stream) != cudaSuccess || cudaStreamWaitEvent(as, aux->step, 0) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        if (rest > 0) {
            // next block column (it holds the next diagonal block) on `stream` ...
            if (cudaStreamWaitEvent(stream, aux->rest, 0) != cudaSuccess) return GPTQ_ERR_CUDA;
            float* next = A + size_t(k0 + NB) * d + k0 + NB;
            rc = launch_tgemm(rest, NB, NB, -1.0f, panel, nullptr, d, panel, nullptr, d, true, next, d, true, stream, st);
            if (rc) return rc;
            // ... the columns after it on `ss`
            if (rest > NB) {
                if (cudaStreamWaitEvent(ss, aux->step, 0) != cudaSuccess) return GPTQ_ERR_CUDA;
                float* far = A + size_t(k0 + 2 * NB) * d + k0 + 2 * NB;
                const float* prow = panel + size_t(NB) * d;
                rc = launch_tgemm(rest - NB, rest - NB, NB, -1.0f, prow, nullptr, d, prow, nullptr, d, true, far, d, true,
                                  ss, st);
                if (rc) return rc;
                if (cudaEventRecord(aux->rest, ss) != cudaSuccess) return GPTQ_ERR_CUDA;
            }
        }
        // inverse block step k on the auxiliary stream
        place_diag_inverse_t_kernel<<<1, 512, NB * LD * sizeof(float), as>>>(dk, d, k, Z); count_launch();
        if (k > 0) {
            float* zi = Z + k0;   // in place is safe for the same reason as the panel
            rc = launch_tgemm(k0, NB, NB, 1.0f, zi, nullptr, d, dk, nullptr, NB, false, zi, d, false, as, st);
            if (rc) return rc;
        }
        if (rest > 0) {
            float* zc = Z + k0 + NB;
            rc = launch_tgemm(k0 + NB, rest, NB, -1.0f, Z + k0, nullptr, d, panel, nullptr, d, true, zc, d, false, as, st);
            if (rc) return rc;
        }
    }
    // join both auxiliary streams
    if (cudaEventRecord(aux->join, as) != cudaSuccess || cudaStreamWaitEvent(stream, aux->join, 0) != cudaSuccess ||
        cudaEventRecord(aux->join_side, ss) != cudaSuccess ||
        cudaStreamWaitEvent(stream, aux->join_side, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    write_u_kernel<<<dim3(d / 32, d / 32), dim3(32, 8), 0, stream>>>(Z, d, info, U); count_launch();
    // back to the caller's stream
    if (cudaEventRecord(aux->join, stream) != cudaSuccess || cudaStreamWaitEvent(caller, aux->join, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
