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
//   factor (potrf_diag_kernel); the panel below is solved against it with a
//   GEMM by the inverse; the trailing lower triangle gets a SYRK-shaped GEMM
//   (both on the tensor cores, tgemm).  Z = L'^-T is built block column by
//   block column alongside (right-looking forward substitution on the
//   identity, transposed), and U is written by reversing both indices.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace factor {

constexpr int NB = 128;
// Block columns per super-panel.  Inside a super-panel the factorization is
// right-looking by 128-column blocks; the columns beyond it get the
// super-panel's whole update at once, as one product SUPER * 128 deep.  A
// build-time tuning knob.
#ifndef GPTQ_FACTOR_SUPER
#define GPTQ_FACTOR_SUPER 8
#endif
constexpr int SUPER = GPTQ_FACTOR_SUPER;
static_assert(SUPER >= 1 && SUPER * 128 <= 8192, "super-panel width");

// Workspace: A (the reversed damped H, then L'), Z (= L'^-T), the diagonal
// blocks' inverses, and the operands of the once-per-super-panel products
// pre-split into tf32 parts and remainders: a super-panel's block columns of
// L' (two buffers, so that one super-panel's can be written while the
// previous one's are still read) and of Z, each [d, min(d, SUPER * NB)] fp32.
struct Layout {
    size_t a_off, y_off, dinv_off, ls_off, zs_off, scal_off, total;
    size_t sp_elems;   // elements of one pre-split array
};

__host__ __device__ inline Layout layout(int64_t d) {
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    Layout L;
    L.sp_elems = size_t(d) * size_t(d < SUPER * NB ? d : SUPER * NB);
    L.a_off = 0;
    L.y_off = up(L.a_off + size_t(d) * d * sizeof(float));
    L.dinv_off = up(L.y_off + size_t(d) * d * sizeof(float));
    L.ls_off = up(L.dinv_off + size_t(d) * NB * sizeof(float));          // [2 buffers][hi, lo]
    L.zs_off = up(L.ls_off + 4 * L.sp_elems * sizeof(float));             // [hi, lo]
    L.scal_off = up(L.zs_off + 2 * L.sp_elems * sizeof(float));
    L.total = L.scal_off + 256;
    return L;
}

// hi[r][c] + lo[r][c] = src[r * ld + c] (tf32 part and remainder), r < rows,
// c < cols (a multiple of 4); hi and lo are dense [rows, cols].
__global__ void split_cols_kernel(const float* __restrict__ src, int ld, int rows, int cols, float* __restrict__ hi,
                                  float* __restrict__ lo) {
    const int c4 = cols / 4;
    const size_t n = size_t(rows) * c4;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += size_t(gridDim.x) * blockDim.x) {
        const int r = int(i / c4), c = int(i % c4) * 4;
        const float4 v = *reinterpret_cast<const float4*>(src + size_t(r) * ld + c);
        float4 h, l;
        split_tf32(v.x, h.x, l.x); split_tf32(v.y, h.y, l.y);
        split_tf32(v.z, h.z, l.z); split_tf32(v.w, h.w, l.w);
        *reinterpret_cast<float4*>(hi + size_t(r) * cols + c) = h;
        *reinterpret_cast<float4*>(lo + size_t(r) * cols + c) = l;
    }
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
// triangle of P (H + lambda I) P, read from the upper triangle of H.  One
// block per row i; each thread moves four columns, read as one reversed
// float4 of H's row d-1-i (d is a multiple of 128, so both sides stay
// aligned).  The float4 that holds the diagonal also writes up to three
// entries above it, which nothing reads.
__global__ void __launch_bounds__(256)
    reverse_damp_kernel(const float* __restrict__ H, int d, const float* __restrict__ lam, float* __restrict__ A) {
    const int i = blockIdx.x;
    const float l = *lam;
    const float* src = H + size_t(d - 1 - i) * d;
    float4* dst = reinterpret_cast<float4*>(A + size_t(i) * d);
    for (int j4 = threadIdx.x; 4 * j4 <= i; j4 += blockDim.x) {
        const float4 h = *reinterpret_cast<const float4*>(src + (d - 4 - 4 * j4));   // columns d-4-4j4 .. d-1-4j4
        float4 v = make_float4(h.w, h.z, h.y, h.x);
        const int k = i - 4 * j4;                                                      // the diagonal's place, if < 4
        if (k == 0) v.x += l;
        else if (k == 1) v.y += l;
        else if (k == 2) v.z += l;
        else if (k == 3) v.w += l;
        dst[j4] = v;
    }
}

// ---------------------------------------------------------------------------
// One 128 x 128 diagonal block: L L^T = A_kk and L^-1, in one CTA of 12 warps.
// The block is cut into 4 x 4 sub-blocks of 32.  Step kb (o = 32 kb):
//   A: warp 0 (the leader) runs the Cholesky of the diagonal sub-block
//      (kb, kb) in registers, lane = row, and publishes each column of L_kk
//      and 1 / L[c][c] in shared memory, in groups of columns.  Followers
//      trail it group by group: warp w in 1 .. 3-kb solves rows o + 32 w +
//      lane of the panel below against L_kk^T, and warp YW builds column
//      `lane` of L_kk^-1 (forward substitution on e_lane).  Meanwhile the
//      other warps (not those sharing the leader's scheduler) apply step
//      kb-1's update to block column kb+1 and to the inverse's rows of
//      block kb.
//   C: step kb's update of block column kb+1 (what step kb+1 needs first),
//      step kb of the inverse's block solve, and the rest of step kb-1's
//      updates (the blocks that phase A of step kb+1 does not read).
// Every block receives its updates in the same order on every run.
// The inverse Y = L^-1 is built right-looking on the identity (Y = X after
//   X_k <- L_kk^-1 X_k;  X_i -= L_ik X_k  (i > k)  for k = 0..3)
// and kept transposed (Yt = Y^T = L^-T) so that every product reads both of
// its operands along rows, four at a time.  Row strides of 132 floats make
// those float4 reads and the scattered scalar writes free of bank conflicts.
// ---------------------------------------------------------------------------
constexpr int SB = 32;
constexpr int LDS = NB + 4;              // S and Yt row stride (floats)
constexpr int LDI = SB + 4;              // Lr and Lp row stride
constexpr int DIAG_THREADS = 384;        // 12 warps
constexpr int YW = 5;                    // the follower that builds L_kk^-1 (not on the leader's scheduler)
static_assert(NB / SB == 4, "the diagonal kernel's task lists are written for 4 x 4 sub-blocks");
constexpr size_t DIAG_SMEM = (size_t(2) * NB * LDS + size_t(2) * SB * LDI + 2 * SB) * sizeof(float);

// The leader's columns are published in groups of GROUP steps; group g of
// sub-block kb completes mbarrier 4 kb + g (each used once, so every wait is
// for phase 0).  Followers sleep in the barrier's bounded wait instead of
// polling shared memory beside the leader.
constexpr int GROUP = 8;
constexpr int NGROUPS = (NB / SB) * (SB / GROUP);

// Leader step C (template recursion keeps every register index a
// compile-time constant).  a[] holds row `lane` of the sub-block (entries
// right of the diagonal are don't-care); piv is entry (C, C) after the steps
// before C.  Column C is scaled to L's (l = a[C] / sqrt(piv)), published as
// row C of Lp (Lp[C][j] = L[j][C]) with rs[C] = 1 / L[C][C], and l * L[j][C]
// is subtracted from every a[j], j > C.  The next pivot comes from lane C+1's
// own l by a shuffle, beside the shared-memory round trip.  After every
// GROUP steps lane 0 arrives on the group's barrier (release: the warp's
// published columns become visible to the followers' waits).  The pivots go
// to shared memory and are tested after the last step: tested inside the
// chain, they cost a third of its time.
template <int C>
struct LeadStep {
    __device__ __forceinline__ static void run(float (&a)[SB], float piv, int lane, float* __restrict__ Lp,
                                               float* __restrict__ rs_out, float* __restrict__ piv_out,
                                               uint64_t* grp) {
        piv_out[C] = piv;   // checked once after the last step, off the chain
        const float rs = rsqrtf(piv);
        const float l = a[C] * rs;
        a[C] = l;
        float* col = Lp + C * LDI;
        col[lane] = l;
        rs_out[C] = rs;   // every lane: the same value, one broadcast write, no branch
        if constexpr (C + 1 < SB) {
            const float next = __shfl_sync(0xffffffffu, fmaf(-l, l, a[C + 1]), C + 1);
            __syncwarp();
            if constexpr ((C + 1) % GROUP == 0) {
                if (lane == 0) mbar_arrive(grp + (C + 1) / GROUP - 1);
            }
#pragma unroll
            for (int j4 = ((C + 1) / 4) * 4; j4 < SB; j4 += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(col + j4);
                const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (j4 + q > C) a[j4 + q] = fmaf(-l, v[q], a[j4 + q]);
            }
            LeadStep<C + 1>::run(a, next, lane, Lp, rs_out, piv_out, grp);
        } else {
            __syncwarp();
            if (lane == 0) mbar_arrive(grp + SB / GROUP - 1);
        }
    }
};

// Follower step C: once the leader has published column C, x[C] is scaled by
// 1 / L[C][C] and x[j] -= x[C] L[j][C] for j > C.  With x = a panel row that
// is the solve x <- x L^-T; with x = e_lane it builds column `lane` of L^-1.
// A follower waits once per group of columns.  After a wait that timed out
// (ok == false) the remaining steps run without waiting; the kernel then
// stops at its next barrier.
template <int C>
struct FollowStep {
    __device__ __forceinline__ static void run(float (&x)[SB], const float* __restrict__ Lp,
                                               const float* __restrict__ rs, uint64_t* grp, bool& ok, DevStatus* st) {
        if constexpr (C % GROUP == 0) {
            if (ok) ok = mbar_wait(grp + C / GROUP, 0, st, 0x600 + C);
        }
        const float xc = x[C] * rs[C];
        x[C] = xc;
        if constexpr (C + 1 < SB) {
            const float* col = Lp + C * LDI;
#pragma unroll
            for (int j4 = ((C + 1) / 4) * 4; j4 < SB; j4 += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(col + j4);
                const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (j4 + q > C) x[j4 + q] = fmaf(-xc, v[q], x[j4 + q]);
            }
            FollowStep<C + 1>::run(x, Lp, rs, grp, ok, st);
        }
    }
};

// Out[R_a][C_b] -= sum_m P[R_a][m] Q[C_b][m] over one 32-wide sub-block of m,
// for the 4 x 4 outputs of lane (g, h) = (lane / 4, lane % 4) in one half
// (columns 16 s .. 16 s + 15) of a 32 x 32 output sub-block:
// R_a = r0 + g + 8a, C_b = c0 + 16 s + h + 4b.  P, Q and Out have row stride
// LDS and P, Q point at the first m column.
__device__ __forceinline__ void sub_block_update(const float* __restrict__ P, const float* __restrict__ Q,
                                                 float* __restrict__ Out, int r0, int c0, int s, int lane) {
    const int g = lane >> 2, h = lane & 3;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
#pragma unroll 1
    for (int m = 0; m < SB; m += 4) {
        float4 p[4], q[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) p[a] = *reinterpret_cast<const float4*>(P + (r0 + g + 8 * a) * LDS + m);
#pragma unroll
        for (int b = 0; b < 4; ++b) q[b] = *reinterpret_cast<const float4*>(Q + (c0 + 16 * s + h + 4 * b) * LDS + m);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                acc[a][b] = fmaf(p[a].x, q[b].x, acc[a][b]);
                acc[a][b] = fmaf(p[a].y, q[b].y, acc[a][b]);
                acc[a][b] = fmaf(p[a].z, q[b].z, acc[a][b]);
                acc[a][b] = fmaf(p[a].w, q[b].w, acc[a][b]);
            }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) Out[(r0 + g + 8 * a) * LDS + c0 + 16 * s + h + 4 * b] -= acc[a][b];
}

// Phase A of step kb for the leader: the Cholesky of the diagonal sub-block
// (its factor is not written back: nothing reads L_kk afterwards).  Kept out
// of line, like the followers, so that its registers are allocated on their
// own, away from the rest of the kernel.
__device__ __noinline__ void lead_warp(const float* __restrict__ S, float* __restrict__ Lp, float* __restrict__ rs,
                                       float* __restrict__ pv, uint64_t* grp, int o, int lane, uint32_t* badmask,
                                       uint32_t* nonfinite) {
    float a[SB];
    const float* arow = S + (o + lane) * LDS + o;
#pragma unroll
    for (int j = 0; j < SB; j += 4) {
        const float4 v = *reinterpret_cast<const float4*>(arow + j);
        a[j] = v.x; a[j + 1] = v.y; a[j + 2] = v.z; a[j + 3] = v.w;
    }
    LeadStep<0>::run(a, __shfl_sync(0xffffffffu, a[0], 0), lane, Lp, rs, pv, grp);
    __syncwarp();
    const float piv = pv[lane];   // bit c: pivot c failed
    *badmask = __ballot_sync(0xffffffffu, !(piv > 0.0f && isfinite(piv)));
    *nonfinite = __ballot_sync(0xffffffffu, !isfinite(piv));
}

// Phase A of step kb for a follower: row_group = w >= 1 solves rows
// o + 32 w + lane of the panel in place; row_group = 0 builds column `lane`
// of L_kk^-1 and writes it as Yt row o + lane and into Lr (row-major).
// Returns false if a wait for the leader timed out.
__device__ __noinline__ bool follow_warp(float* __restrict__ S, float* __restrict__ Yt, float* __restrict__ Lr,
                                         const float* __restrict__ Lp, const float* __restrict__ rs, uint64_t* grp,
                                         int o, int row_group, int lane, DevStatus* st) {
    float x[SB];
    float* xrow = S + (o + SB * row_group + lane) * LDS + o;
    if (row_group == 0) {
#pragma unroll
        for (int j = 0; j < SB; ++j) x[j] = (j == lane) ? 1.0f : 0.0f;
    } else {
#pragma unroll
        for (int j = 0; j < SB; j += 4) {
            const float4 v = *reinterpret_cast<const float4*>(xrow + j);
            x[j] = v.x; x[j + 1] = v.y; x[j + 2] = v.z; x[j + 3] = v.w;
        }
    }
    bool ok = true;
    FollowStep<0>::run(x, Lp, rs, grp, ok, st);
    if (row_group == 0) {
#pragma unroll
        for (int r = 0; r < SB; r += 4)
            *reinterpret_cast<float4*>(Yt + (o + lane) * LDS + o + r) = make_float4(x[r], x[r + 1], x[r + 2], x[r + 3]);
#pragma unroll
        for (int r = 0; r < SB; ++r) Lr[r * LDI + lane] = x[r];
    } else {
#pragma unroll
        for (int j = 0; j < SB; j += 4)
            *reinterpret_cast<float4*>(xrow + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
    }
    return ok;
}

// Factor the diagonal block A[k0:k0+NB, k0:k0+NB] = L L^T and write
//   Dinv = L^-1 (NB x NB row-major, zeros above the diagonal) and
//   Z[k0 + c][k0 + r] = L^-1[r][c]  (the diagonal block of Z = L'^-T).
// A's block itself is left as it was (nothing reads L_kk afterwards).  A
// non-positive or non-finite pivot sets *info = k0 + c + 1 (first failure only).
__global__ void __launch_bounds__(DIAG_THREADS, 1)
    potrf_diag_kernel(const float* __restrict__ A, int d, int k0, float* __restrict__ Dinv, float* __restrict__ Z,
                      int* info, DevStatus* st) {
    extern __shared__ __align__(16) float sm[];
    float* S = sm;                     // [NB][LDS] the block, factored in place (lower)
    float* Yt = S + NB * LDS;          // [NB][LDS] X, then Y, transposed (upper)
    float* Lr = Yt + NB * LDS;         // [SB][LDI] L_kk^-1 of the current step, row-major
    float* Lp = Lr + SB * LDI;         // [SB][LDI] the leader's published columns: Lp[c][j] = L_kk[j][c]
    float* rs = Lp + SB * LDI;         // [SB] 1 / L_kk[c][c]
    float* pv = rs + SB;               // [SB] the pivots L_kk[c][c]^2, for the positivity test
    __shared__ int failed;
    __shared__ __align__(8) uint64_t grp_bar[NGROUPS];   // the leader's column groups, one barrier per group
    pdl_wait();
    pdl_trigger();
    if (*info != 0) return;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;

    // lower triangle of the block (zeros above), Yt = 0; every load is issued
    // before the first shared-memory store
    {
        constexpr int PER = (NB * NB / 4 + DIAG_THREADS - 1) / DIAG_THREADS;
        float4 v[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int idx = t + i * DIAG_THREADS;
            const int r = idx / (NB / 4), c = (idx % (NB / 4)) * 4;
            v[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (idx < NB * NB / 4 && c <= r) v[i] = *reinterpret_cast<const float4*>(A + size_t(k0 + r) * d + k0 + c);
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int idx = t + i * DIAG_THREADS;
            if (idx >= NB * NB / 4) break;
            const int r = idx / (NB / 4), c = (idx % (NB / 4)) * 4;
            float4 w = v[i];
            if (c + 1 > r) w.y = 0.0f;
            if (c + 2 > r) w.z = 0.0f;
            if (c + 3 > r) w.w = 0.0f;
            *reinterpret_cast<float4*>(S + r * LDS + c) = w;
            *reinterpret_cast<float4*>(Yt + r * LDS + c) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
    }
    if (t == 0) {
        failed = 0;
        for (int g = 0; g < NGROUPS; ++g) mbar_init(&grp_bar[g], 1);
    }
    __syncthreads();

    for (int kb = 0; kb < NB / SB; ++kb) {
        const int o = kb * SB;
        const int npanel = NB / SB - kb;   // 32-row groups of block column kb
        // ---- A: Cholesky (leader) || panel solve and L_kk^-1 (followers) || rest of step kb-1
        if (warp == 0) {
            uint32_t badmask = 0, nonfinite = 0;   // the same in every lane
            lead_warp(S, Lp, rs, pv, grp_bar + kb * (SB / GROUP), o, lane, &badmask, &nonfinite);
            if (badmask != 0 && lane == 0) {   // the first failing pivot of this sub-block
                const int bad = __ffs(int(badmask)) - 1;
                failed = 1;
                if (atomicCAS(info, 0, k0 + o + bad + 1) == 0)
                    record_error(st, (nonfinite >> bad) & 1u ? GPTQ_ERR_NONFINITE : GPTQ_ERR_NOT_PD, k0 + o + bad + 1);
            }
        } else if (warp < npanel || warp == YW) {
            if (!follow_warp(S, Yt, Lr, Lp, rs, grp_bar + kb * (SB / GROUP), o, warp == YW ? 0 : warp, lane, st))
                failed = 1;
        } else if (kb > 0 && (warp & 3) != 0) {
            // What step kb's phase C needs of step kb-1, on the warps other than YW
            // that do not share the leader's scheduler, in halves of 32 x 32
            // sub-blocks (P = block column kb-1 of L):
            //  - block column kb+1: S[bi][kb+1] -= L_{bi,kb-1} L_{kb+1,kb-1}^T, bi > kb;
            //  - X_{kb,j} -= L_{kb,kb-1} Y_{kb-1,j} for j < kb, transposed:
            //    Yt[j-block][kb-block] -= Yt[j-block][(kb-1)-block] S[kb-block][(kb-1)-block]^T.
            const int w = warp - npanel - (warp > 4) - (warp > YW) - (warp > 8);
            const int nw = DIAG_THREADS / 32 - npanel - 3;
            const int ncol = 2 * (NB / SB - kb - 1);
            const int tasks = ncol + 2 * kb;
            const int po = (kb - 1) * SB;
            for (int task = w; task < tasks; task += nw) {
                if (task < ncol) {
                    const int bi = kb + 1 + (task >> 1);
                    sub_block_update(S + po, S + po, S, bi * SB, (kb + 1) * SB, task & 1, lane);
                } else {
                    const int j = (task - ncol) >> 1;
                    sub_block_update(Yt + po, S + po, Yt, j * SB, kb * SB, (task - ncol) & 1, lane);
                }
            }
        }
        __syncthreads();
        if (failed) return;

        // ---- C: step kb's update of block column kb+1 (what step kb+1 needs first)
        //      || step kb of the inverse's block solve || the rest of step kb-1
        {
            const int n3 = 2 * (NB / SB - kb - 1);     // lookahead: two warps per pair (bi, kb+1)
            const int n5 = kb == 1 ? 2 : 0;            // step kb-1 beyond column kb+1: pair (3, 3), only for kb = 1
            const int n6 = kb >= 1 ? 2 * kb * (NB / SB - kb - 1) : 0;   // X_{i,j}, i > kb, j < kb, of step kb-1
            if (warp < n3) {
                const int bi = kb + 1 + (warp >> 1);
                sub_block_update(S + o, S + o, S, bi * SB, (kb + 1) * SB, warp & 1, lane);
            } else if (warp < n3 + kb) {
                // Y_{kb,j} = L_kk^-1 X_{kb,j} for j < kb: thread = column c of block j,
                // reading X_{kb,j}[., c] as row (j*SB + c) of Yt
                const int u = t - 32 * n3;                     // 0 .. 32 kb - 1
                float* row = Yt + (size_t(u)) * LDS + o;       // j = u / SB, c = u % SB: row j*SB + c = u
                float x[SB];
#pragma unroll
                for (int m = 0; m < SB; m += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(row + m);
                    x[m] = v.x; x[m + 1] = v.y; x[m + 2] = v.z; x[m + 3] = v.w;
                }
#pragma unroll
                for (int r = 0; r < SB; r += 4) {
                    float y4[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float acc = 0.0f;
#pragma unroll
                        for (int m = 0; m < SB; m += 4) {
                            if (m <= r + q) {
                                const float4 l = *reinterpret_cast<const float4*>(Lr + (r + q) * LDI + m);
                                acc = fmaf(l.x, x[m], acc);
                                acc = fmaf(l.y, x[m + 1], acc);
                                acc = fmaf(l.z, x[m + 2], acc);
                                acc = fmaf(l.w, x[m + 3], acc);
                            }
                        }
                        y4[q] = acc;
                    }
                    *reinterpret_cast<float4*>(row + r) = make_float4(y4[0], y4[1], y4[2], y4[3]);
                }
            } else if (warp < n3 + kb + n5 + n6) {
                const int task = warp - n3 - kb, po = (kb - 1) * SB;
                if (task < n5) {
                    // S[3][3] -= L_{3,0} L_{3,0}^T (step 0 beyond column 2)
                    sub_block_update(S + po, S + po, S, 3 * SB, 3 * SB, task & 1, lane);
                } else {
                    // Yt[j-block][i-block] -= Yt[j-block][(kb-1)-block] S[i-block][(kb-1)-block]^T
                    const int blk = (task - n5) >> 1, j = blk % kb, i = kb + 1 + blk / kb;
                    sub_block_update(Yt + po, S + po, Yt, j * SB, i * SB, (task - n5) & 1, lane);
                }
            }
        }
        __syncthreads();
    }

    // Z's diagonal block = Yt, as float4 rows; Dinv = Yt^T, gathered four
    // columns at a time into the factor's (now free) buffer -- column reads
    // and float4 writes both free of bank conflicts -- and written out as
    // float4 rows.
    for (int idx = t; idx < NB * NB / 4; idx += DIAG_THREADS) {
        const int c = idx / (NB / 4), r4 = (idx % (NB / 4)) * 4;
        *reinterpret_cast<float4*>(Z + size_t(k0 + c) * d + k0 + r4) = *reinterpret_cast<const float4*>(Yt + c * LDS + r4);
    }
    float* D = S;   // [NB][LDS]
    for (int idx = t; idx < NB * NB / 4; idx += DIAG_THREADS) {
        const int r = idx % NB, c4 = (idx / NB) * 4;
        *reinterpret_cast<float4*>(D + r * LDS + c4) =
            make_float4(Yt[c4 * LDS + r], Yt[(c4 + 1) * LDS + r], Yt[(c4 + 2) * LDS + r], Yt[(c4 + 3) * LDS + r]);
    }
    __syncthreads();
    for (int idx = t; idx < NB * NB / 4; idx += DIAG_THREADS) {
        const int r = idx / (NB / 4), c4 = (idx % (NB / 4)) * 4;
        *reinterpret_cast<float4*>(Dinv + size_t(r) * NB + c4) = *reinterpret_cast<const float4*>(D + r * LDS + c4);
    }
}

// Three internal streams and a few events per set (created on first use).
// The factorization's critical chain runs on a high-priority stream; the
// inverse's block steps run on another, each as soon as the factorization has
// finished the block column it needs; the update of the columns beyond the
// next super-panel runs on a low-priority stream, beside the next
// super-panel's chain (look-ahead).
// Each device has AUX_SETS sets.  A caller stream keeps the set it was given
// first, so that factorizations called on different streams (independent
// layers) run concurrently; once every set is taken, further caller streams
// share them in turn, and calls on a shared set enqueue one at a time.
constexpr int AUX_SETS = 4;
struct AuxStream {
    cudaStream_t main = nullptr;    // the factorization's critical chain (highest priority)
    cudaStream_t s = nullptr;       // inverse steps
    cudaStream_t side = nullptr;    // updates of the columns beyond the next super-panel
    static constexpr int RING = 4;
    cudaEvent_t fork = nullptr, step = nullptr, join = nullptr, join_side = nullptr, filled = nullptr;
    cudaEvent_t far_done[RING] = {};   // the far update of super-panel p, slot p % RING
    cudaEvent_t zfar_done[2] = {};     // Z's far update of super-panel p, slot p % 2
    std::mutex enqueue;                // one call enqueues on this set at a time
    cudaStream_t owner = nullptr;      // the caller stream the set was given to
    bool taken = false;
};

static int aux_stream(cudaStream_t caller, AuxStream** out) {
    static std::mutex mu;
    static AuxStream per_dev[64][AUX_SETS];
    static int next_shared[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    AuxStream* pick = nullptr;
    for (int i = 0; i < AUX_SETS && !pick; ++i)
        if (per_dev[dev][i].taken && per_dev[dev][i].owner == caller) pick = &per_dev[dev][i];
    for (int i = 0; i < AUX_SETS && !pick; ++i)
        if (!per_dev[dev][i].taken) {
            pick = &per_dev[dev][i];
            pick->taken = true;
            pick->owner = caller;
        }
    if (!pick) pick = &per_dev[dev][next_shared[dev]++ % AUX_SETS];
    AuxStream& a = *pick;
    if (!a.s) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&a.main, cudaStreamNonBlocking, greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&a.s, cudaStreamNonBlocking, greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&a.side, cudaStreamNonBlocking, least) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.step, cudaEventDisableTiming) != cudaSuccess ||

            cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.join_side, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&a.filled, cudaEventDisableTiming) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        for (int i = 0; i < AuxStream::RING; ++i)
            if (cudaEventCreateWithFlags(&a.far_done[i], cudaEventDisableTiming) != cudaSuccess) return GPTQ_ERR_CUDA;
        for (int i = 0; i < 2; ++i)
            if (cudaEventCreateWithFlags(&a.zfar_done[i], cudaEventDisableTiming) != cudaSuccess) return GPTQ_ERR_CUDA;
    }
    *out = &a;
    return GPTQ_OK;
}

// U[r][c] = Z[d-1-c][d-1-r] for r <= c (U = P L'^-1 P = P Z^T P), 0 below the
// diagonal; NaN everywhere if the factorization failed.  A block writes a
// 64 x 64 tile of U: the matching tile of Z (rows d-c0-64 .., columns
// d-r0-64 ..) comes in as float4 rows into shared memory (row stride 65, so
// that the reversed, transposed reads below hit at most two ways of a bank),
// and goes out as float4 rows of U.  Tiles wholly below the diagonal read
// nothing.
constexpr int UT = 64;
__global__ void __launch_bounds__(256)
    write_u_kernel(const float* __restrict__ Z, int d, const int* __restrict__ info, float* __restrict__ U) {
    __shared__ float tile[UT][UT + 1];
    const int r0 = blockIdx.y * UT, c0 = blockIdx.x * UT, t = threadIdx.x;
    const bool bad = *info != 0;
    const bool below = c0 + UT - 1 < r0;
    if (!below && !bad) {
        const float* zt = Z + size_t(d - c0 - UT) * d + (d - r0 - UT);
        for (int idx = t; idx < UT * UT / 4; idx += 256) {
            const int zr = idx / (UT / 4), zc = (idx % (UT / 4)) * 4;
            const float4 v = *reinterpret_cast<const float4*>(zt + size_t(zr) * d + zc);
            tile[zr][zc] = v.x; tile[zr][zc + 1] = v.y; tile[zr][zc + 2] = v.z; tile[zr][zc + 3] = v.w;
        }
    }
    __syncthreads();
    for (int idx = t; idx < UT * UT / 4; idx += 256) {
        const int rl = idx / (UT / 4), cl = (idx % (UT / 4)) * 4;
        const int r = r0 + rl;
        float o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int c = c0 + cl + q;
            // U[r][c] = Z[d-1-c][d-1-r] = tile[(d-1-c) - (d-c0-UT)][(d-1-r) - (d-r0-UT)]
            o[q] = bad ? __int_as_float(0x7fc00000) : (!below && c >= r) ? tile[UT - 1 - (cl + q)][UT - 1 - rl] : 0.0f;
        }
        *reinterpret_cast<float4*>(U + size_t(r) * d + c0 + cl) = make_float4(o[0], o[1], o[2], o[3]);
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

    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(potrf_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(DIAG_SMEM)) !=
            cudaSuccess)
            return GPTQ_ERR_CUDA;
        attr_set[dev] = true;
    }

    // The internal streams and events of this caller stream's set; calls that
    // share a set enqueue one at a time.
    AuxStream* aux = nullptr;
    if (aux_stream(stream, &aux)) return GPTQ_ERR_CUDA;
    std::lock_guard<std::mutex> enqueue_lock(aux->enqueue);
    const cudaStream_t as = aux->s;
    const cudaStream_t caller = stream;
    stream = aux->main;
    if (cudaEventRecord(aux->fork, caller) != cudaSuccess || cudaStreamWaitEvent(stream, aux->fork, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;

    damp_lambda_kernel<<<1, 1024, 0, stream>>>(H, d, percdamp, lam, info, st); count_launch();
    reverse_damp_kernel<<<d, 256, 0, stream>>>(H, d, lam, A); count_launch();
    // fork: the inverse (stream `as`) starts from a zeroed Z; `ss` takes the
    // updates of the columns beyond the next super-panel
    const cudaStream_t ss = aux->side;
    if (cudaEventRecord(aux->fork, stream) != cudaSuccess || cudaStreamWaitEvent(as, aux->fork, 0) != cudaSuccess ||
        cudaStreamWaitEvent(ss, aux->fork, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    {
        const int rc = launch_fill(Z, int64_t(d) * d, 0.0f, as);
        if (rc) return rc;
    }
    // the diagonal kernels write Z's diagonal blocks: after the fill
    if (cudaEventRecord(aux->filled, as) != cudaSuccess || cudaStreamWaitEvent(stream, aux->filled, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;

    // Cholesky of A (lower), blocked right-looking, products on the tensor
    // cores, in super-panels of SUPER block columns [p0, p1):
    //  - step k of the super-panel, on `stream`: factor the diagonal block,
    //    solve the panel below it, then update the super-panel's later block
    //    columns (all rows below);
    //  - after the super-panel: the next super-panel's columns [p1, h1) get
    //    the whole super-panel's update, one product (p1 - p0) deep, on
    //    `stream`; the columns from h1 on get theirs on `ss`, beside the next
    //    super-panel's steps.
    // Every element of A thus receives its updates in a fixed order (by
    // super-panel, then by step): `ss` runs in order, and `stream` waits for
    // the previous super-panel's far update before it first touches the
    // columns that update covered.  So U does not depend on how the streams
    // interleave.
    // Z = L^-T (upper) on `as`: block step i needs only L's block column i and
    // Dinv_i, so it runs as soon as the factorization has them:
    //   Z[i][i] = Dinv_i^T;  Z[0:i0, i] <- Z[0:i0, i] Dinv_i^T;
    //   Z[0:i0+NB, i0+NB:p1] -= Z[0:i0+NB, i] L[i0+NB:p1, i]^T,
    // and after each super-panel Z[0:p1, p1:] -= Z[0:p1, p0:p1] L[p1:, p0:p1]^T
    // (the transpose of the block forward substitution Y = L^-1, deferred the
    // same way; Z's entries below the diagonal are zero, so the full row range
    // adds nothing; working on Z keeps every tensor-core operand K-major).
    int rc;
    for (int pb0 = 0, sp = 0; pb0 < nblk; pb0 += SUPER, ++sp) {
        const int pb1 = std::min(nblk, pb0 + SUPER);
        const int p0 = pb0 * NB, p1 = pb1 * NB;
        for (int k = pb0; k < pb1; ++k) {
            const int k0 = k * NB;
            float* dk = Dinv + size_t(k) * NB * NB;
            if (launch_pdl(potrf_diag_kernel, dim3(1), dim3(DIAG_THREADS), DIAG_SMEM, stream, static_cast<const float*>(A),
                           d, k0, dk, Z, info, st) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            count_launch();
            const int rest = d - k0 - NB;
            float* panel = A + size_t(k0 + NB) * d + k0;
            if (rest > 0) {
                // panel <- panel * Dinv_k^T.  In place is safe: N = NB is one output
                // tile column, so each CTA reads only the rows it writes, all before
                // its epilogue.
                rc = launch_tgemm(rest, NB, NB, 1.0f, panel, nullptr, d, dk, nullptr, NB, false, panel, d, false, stream, st);
                if (rc) return rc;
            }
            if (cudaEventRecord(aux->step, stream) != cudaSuccess || cudaStreamWaitEvent(as, aux->step, 0) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            const int ncols = p1 - k0 - NB;   // the super-panel's later columns
            if (ncols > 0) {
                rc = launch_tgemm(rest, ncols, NB, -1.0f, panel, nullptr, d, panel, nullptr, d, true,
                                  A + size_t(k0 + NB) * d + k0 + NB, d, true, stream, st);
                if (rc) return rc;
            }
            // inverse block step k on the auxiliary stream (Z's diagonal block k
            // was written by the diagonal kernel)
            if (k > 0) {
                float* zi = Z + k0;   // in place is safe for the same reason as the panel
                rc = launch_tgemm(k0, NB, NB, 1.0f, zi, nullptr, d, dk, nullptr, NB, false, zi, d, false, as, st);
                if (rc) return rc;
            }
            if (ncols > 0) {
                rc = launch_tgemm(k0 + NB, ncols, NB, -1.0f, Z + k0, nullptr, d, panel, nullptr, d, true, Z + k0 + NB, d,
                                  false, as, st);
                if (rc) return rc;
            }
        }
        if (p1 >= d) break;
        // the super-panel's update of the columns after it, from its operands
        // pre-split into tf32 parts and remainders (the products' fast form):
        // L'[p1:, p0:p1] into buffer sp % 2 (on `stream`, once the super-panel
        // two back no longer reads that buffer), Z[0:p1, p0:p1] (on `as`)
        const int h1 = std::min(d, p1 + SUPER * NB);   // end of the next super-panel
        const int kd = p1 - p0;
        const int lrows = d - p1;
        float* ls_hi = reinterpret_cast<float*>(base + L.ls_off) + size_t(sp % 2) * 2 * L.sp_elems;
        float* ls_lo = ls_hi + L.sp_elems;
        float* zs_hi = reinterpret_cast<float*>(base + L.zs_off);
        float* zs_lo = zs_hi + L.sp_elems;
        const unsigned split_blocks = 148 * 8;
        if (sp >= 2 && cudaStreamWaitEvent(stream, aux->zfar_done[sp % 2], 0) != cudaSuccess) return GPTQ_ERR_CUDA;
        split_cols_kernel<<<split_blocks, 256, 0, stream>>>(A + size_t(p1) * d + p0, d, lrows, kd, ls_hi, ls_lo);
        count_launch();
        split_cols_kernel<<<split_blocks, 256, 0, as>>>(Z + p0, d, p1, kd, zs_hi, zs_lo);
        count_launch();
        if (cudaEventRecord(aux->step, stream) != cudaSuccess || cudaStreamWaitEvent(ss, aux->step, 0) != cudaSuccess ||
            cudaStreamWaitEvent(as, aux->step, 0) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        if (h1 < d) {
            // columns [h1, d) on `ss`
            const float* hh = ls_hi + size_t(h1 - p1) * kd;
            const float* hl = ls_lo + size_t(h1 - p1) * kd;
            rc = launch_tgemm(d - h1, d - h1, kd, -1.0f, hh, hl, kd, hh, hl, kd, true, A + size_t(h1) * d + h1, d,
                              true, ss, st);
            if (rc) return rc;
        }
        if (cudaEventRecord(aux->far_done[sp % AuxStream::RING], ss) != cudaSuccess) return GPTQ_ERR_CUDA;
        // columns [p1, h1) on `stream`, after the previous super-panel's far
        // update (which covered them)
        if (sp > 0 && cudaStreamWaitEvent(stream, aux->far_done[(sp - 1) % AuxStream::RING], 0) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        rc = launch_tgemm(lrows, h1 - p1, kd, -1.0f, ls_hi, ls_lo, kd, ls_hi, ls_lo, kd, true, A + size_t(p1) * d + p1,
                          d, true, stream, st);
        if (rc) return rc;
        // Z's columns after the super-panel
        rc = launch_tgemm(p1, lrows, kd, -1.0f, zs_hi, zs_lo, kd, ls_hi, ls_lo, kd, true, Z + p1, d, false, as, st);
        if (rc) return rc;
        if (cudaEventRecord(aux->zfar_done[sp % 2], as) != cudaSuccess) return GPTQ_ERR_CUDA;
    }
    // join both auxiliary streams
    if (cudaEventRecord(aux->join, as) != cudaSuccess || cudaStreamWaitEvent(stream, aux->join, 0) != cudaSuccess ||
        cudaEventRecord(aux->join_side, ss) != cudaSuccess ||
        cudaStreamWaitEvent(stream, aux->join_side, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    write_u_kernel<<<dim3(d / UT, d / UT), 256, 0, stream>>>(Z, d, info, U); count_launch();
    // back to the caller's stream
    if (cudaEventRecord(aux->join, stream) != cudaSuccess || cudaStreamWaitEvent(caller, aux->join, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
