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
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace factor {

constexpr int NB = 128;
constexpr int LD = NB + 1;  // padded shared-memory row
constexpr int DIAG_THREADS = 512;
constexpr size_t DIAG_SMEM = size_t(2) * NB * LD * sizeof(float);

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

// Factor the diagonal block A[k0:k0+NB, k0:k0+NB] = L L^T in place (lower) and
// write its inverse L^-1 to Dinv (NB x NB, row-major).  A non-positive or
// non-finite pivot sets *info = k0 + c + 1 (first failure only).
__global__ void __launch_bounds__(DIAG_THREADS)
    potrf_diag_kernel(float* __restrict__ A, int d, int k0, float* __restrict__ Dinv, int* info, DevStatus* st) {
    extern __shared__ float sm[];
    float* S = sm;             // [NB][LD] factor
    float* Y = sm + NB * LD;   // [NB][LD] inverse
    __shared__ int failed;
    if (*info != 0) return;
    const int t = threadIdx.x, ty = t >> 5, tx = t & 31;
    constexpr int NY = DIAG_THREADS / 32;
    for (int idx = t; idx < NB * NB; idx += DIAG_THREADS) {
        const int r = idx / NB, c = idx % NB;
        S[r * LD + c] = (c <= r) ? A[size_t(k0 + r) * d + k0 + c] : 0.0f;
        Y[r * LD + c] = (r == c) ? 1.0f : 0.0f;
    }
    if (t == 0) failed = 0;
    __syncthreads();

    for (int c = 0; c < NB; ++c) {
        if (t == 0) {
            const float p = S[c * LD + c];
            if (!(p > 0.0f) || !isfinite(p)) {
                failed = 1;
                if (atomicCAS(info, 0, k0 + c + 1) == 0)
                    record_error(st, isfinite(p) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE, k0 + c + 1);
            }
            S[c * LD + c] = sqrtf(p);
        }
        __syncthreads();
        if (failed) break;
        const float lcc = S[c * LD + c];
        for (int r = c + 1 + t; r < NB; r += DIAG_THREADS) S[r * LD + c] = __fdiv_rn(S[r * LD + c], lcc);
        __syncthreads();
        for (int r = c + 1 + ty; r < NB; r += NY) {
            const float lrc = S[r * LD + c];
            for (int j = c + 1 + tx; j <= r; j += 32) S[r * LD + j] = fmaf(-lrc, S[j * LD + c], S[r * LD + j]);
        }
        __syncthreads();
    }
    if (failed) return;

    // L^-1 by forward substitution on the identity, one pivot row at a time.
    for (int i = 0; i < NB; ++i) {
        const float lii = S[i * LD + i];
        for (int j = t; j <= i; j += DIAG_THREADS) Y[i * LD + j] = __fdiv_rn(Y[i * LD + j], lii);
        __syncthreads();
        for (int r = i + 1 + ty; r < NB; r += NY) {
            const float lri = S[r * LD + i];
            for (int j = tx; j <= i; j += 32) Y[r * LD + j] = fmaf(-lri, Y[i * LD + j], Y[r * LD + j]);
        }
        __syncthreads();
    }

    for (int idx = t; idx < NB * NB; idx += DIAG_THREADS) {
        const int r = idx / NB, c = idx % NB;
        if (c <= r) A[size_t(k0 + r) * d + k0 + c] = S[r * LD + c];
        Dinv[idx] = Y[r * LD + c];
    }
}

// Y[k*NB + r][k*NB + c] = Dinv_k[r][c] for every diagonal block k.
__global__ void place_diag_inverses_kernel(const float* __restrict__ Dinv, int d, float* __restrict__ Y) {
    const int k = blockIdx.x;
    for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
        const int r = idx / NB, c = idx % NB;
        Y[size_t(k * NB + r) * d + k * NB + c] = Dinv[size_t(k) * NB * NB + idx];
    }
}

// U[r][c] = Y[d-1-r][d-1-c] for r <= c, 0 below the diagonal; NaN everywhere
// if the factorization failed.
__global__ void write_u_kernel(const float* __restrict__ Y, int d, const int* __restrict__ info, float* __restrict__ U) {
    const bool bad = *info != 0;
    const size_t total = size_t(d) * d;
    for (size_t idx = size_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += size_t(gridDim.x) * blockDim.x) {
        const int r = int(idx / d), c = int(idx % d);
        float v = (c >= r) ? Y[size_t(d - 1 - r) * d + (d - 1 - c)] : 0.0f;
        if (bad) v = __int_as_float(0x7fc00000);
        U[idx] = v;
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
    float* Y = reinterpret_cast<float*>(base + L.y_off);
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
            cudaSuccess)
            return GPTQ_ERR_CUDA;
        attr_set[dev] = true;
    }

    damp_lambda_kernel<<<1, 1024, 0, stream>>>(H, d, percdamp, lam, info, st); count_launch();
    reverse_damp_kernel<<<ew_blocks, 256, 0, stream>>>(H, d, lam, A); count_launch();

    // Cholesky of A (lower), blocked right-looking.
    for (int k = 0; k < nblk; ++k) {
        const int k0 = k * NB;
        potrf_diag_kernel<<<1, DIAG_THREADS, DIAG_SMEM, stream>>>(A, d, k0, Dinv + size_t(k) * NB * NB, info, st); count_launch();
        const int rest = d - k0 - NB;
        if (rest <= 0) break;
        float* panel = A + size_t(k0 + NB) * d + k0;
        // panel <- panel * Dinv_k^T.  In place is safe: N = NB is one output
        // tile column, so each CTA reads only the rows it writes.
        int rc = launch_sgemm(rest, NB, NB, 1.0f, panel, d, Dinv + size_t(k) * NB * NB, NB, true, 0.0f, panel,
                              panel, d, false, stream);
        if (rc) return rc;
        float* trail = A + size_t(k0 + NB) * d + k0 + NB;
        rc = launch_sgemm(rest, rest, NB, -1.0f, panel, d, panel, d, true, 1.0f, trail, trail, d, true, stream);
        if (rc) return rc;
    }

    // Y = L^-1, right-looking block forward substitution on the identity.
    {
        const int rc = launch_fill(Y, int64_t(d) * d, 0.0f, stream);
        if (rc) return rc;
    }
    place_diag_inverses_kernel<<<nblk, 256, 0, stream>>>(Dinv, d, Y); count_launch();
    for (int i = 0; i < nblk; ++i) {
        const int i0 = i * NB;
        int rc;
        if (i > 0) {
            // Y[i, 0:i0] <- Dinv_i * Y[i, 0:i0].  In place is safe: M = NB is one
            // output tile row, so each CTA reads only the columns it writes.
            float* yi = Y + size_t(i0) * d;
            rc = launch_sgemm(NB, i0, NB, 1.0f, Dinv + size_t(i) * NB * NB, NB, yi, d, false, 0.0f, yi, yi, d,
                              false, stream);
            if (rc) return rc;
        }
        const int below = d - i0 - NB;
        if (below > 0) {
            // Y[i0+NB:, 0:i0+NB] -= L[i0+NB:, i0:i0+NB] * Y[i0:i0+NB, 0:i0+NB]
            float* yb = Y + size_t(i0 + NB) * d;
            rc = launch_sgemm(below, i0 + NB, NB, -1.0f, A + size_t(i0 + NB) * d + i0, d, Y + size_t(i0) * d, d,
                              false, 1.0f, yb, yb, d, false, stream);
            if (rc) return rc;
        }
    }
    write_u_kernel<<<ew_blocks, 256, 0, stream>>>(Y, d, info, U); count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
