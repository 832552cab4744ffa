// Stages 3-5: the blocked column sweep, the lazy trailing update and the
// packed codes; plus the round-to-nearest baseline.
//
// Source: itwiki "GPTQ", "알고리즘" (Algorithm 1), "GPTQ의 세 가지 변경"
// rows 1-2 (shared column order; updates inside a block of B = 128 columns,
// one matrix product for the columns after it), "최소 구현" (per-row
// asymmetric min/max grid, q = clamp(round(w/s) + z, 0, maxq)), "실무 변형"
// (groups share a grid set from the latest updated weights); "문제 설정" (RTN).
//
// Sweep kernel design: rows are independent given U (the same U serves every
// row).  A CTA takes 32 rows (lane = row) and four warps, one per 32-column
// window of the 128-column block.  Warp q holds its window of every row in
// registers; it applies the E of every column of the windows p < q as soon
// as that column is done (each E goes through shared memory, followed by a
// per-window progress count), so that the windows' sequential chains
// overlap, then quantizes its own window column by column.  The 128 x 128 diagonal block of U
// arrives by one TMA copy; every lane of a warp reads the same U element at
// the same time (broadcast).  The block's E is written for the lazy trailing
// product on the tensor cores.  The codes are packed in registers
// (compile-time bit positions) and stored as vectors.
#include <atomic>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace sweep {

constexpr int B = 128;

// Per-row grid over columns [c0, c0 + len) of the ORIGINAL W: one warp per
// (row, group).  Writes fp16 scale/zero bit patterns.
__global__ void grid_kernel(const float* __restrict__ W, int d_out, int d_in, int group, int n_groups, float maxq,
                            uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros, DevStatus* st) {
    const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int r = warp_global / n_groups, g = warp_global % n_groups;
    if (r >= d_out) return;
    const float* row = W + size_t(r) * d_in + size_t(g) * group;
    float mn = INFINITY, mx = -INFINITY;
    for (int c = lane * 4; c < group; c += 128) {
        const float4 v = *reinterpret_cast<const float4*>(row + c);
        mn = fminf(fminf(mn, v.x), fminf(v.y, fminf(v.z, v.w)));
        mx = fmaxf(fmaxf(mx, v.x), fmaxf(v.y, fmaxf(v.z, v.w)));
    }
    for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) {
        float s, z;
        __half s16, z16;
        if (!grid_params(mn, mx, maxq, s, z, s16, z16)) record_error(st, GPTQ_ERR_NONFINITE, r);
        scales[size_t(r) * n_groups + g] = __half_as_ushort(s16);
        zeros[size_t(r) * n_groups + g] = __half_as_ushort(z16);
    }
}

constexpr int SUB = 32;          // window width = rows per CTA
constexpr int NWIN = B / SUB;    // windows per block = warps per CTA
constexpr int ELD = SUB + 1;     // E hand-over rows (conflict-free)

// Packer for one window: code j of the window goes to stream bits
// [j*BITS, (j+1)*BITS) of the window's BITS words.
template <int BITS>
struct Packer {
    uint32_t w[BITS];
    __device__ __forceinline__ Packer() {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = 0u;
    }
    template <int K>
    __device__ __forceinline__ void put(uint32_t c) {
        constexpr int pos = K * BITS, word = pos / 32, off = pos % 32;
        w[word] |= c << off;
        if constexpr (off + BITS > 32) w[word + 1] |= c >> (32 - off);
    }
    __device__ __forceinline__ void store(uint32_t* dst) const {
        if constexpr (BITS % 4 == 0) {
#pragma unroll
            for (int i = 0; i < BITS; i += 4)
                *reinterpret_cast<uint4*>(dst + i) = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
        } else if constexpr (BITS == 2) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
        } else {
#pragma unroll
            for (int i = 0; i < BITS; ++i) dst[i] = w[i];
        }
    }
};

struct Grid {
    float s, z, maxq, inv_s;   // inv_s = RN(1 / s)
};

// Column J of the window: quantize, pack, E = (w - q) / U_jj, the rank-1
// correction of the window's later columns and -- every PUB columns --
// publishing the E so far to the later windows (eh, then the window's
// progress count).  Row J of the U block (float4 broadcasts from shared
// memory) and 1 / U_jj arrive in ucur / icur: each column loads the next
// column's while it computes, so no load latency sits on the serial chain.
constexpr int PUB = 8;
constexpr int SUB4 = SUB / 4;
template <int BITS, int J>
struct WindowCol {
    __device__ __forceinline__ static void run(float (&w)[SUB], const float* __restrict__ Us, int wc,
                                               const float* __restrict__ invd, const Grid& gr, Packer<BITS>& pk,
                                               float* Qw, bool& finite, float* eh, volatile int* prog, int lane,
                                               const float4 (&ucur)[SUB4], float icur) {
        float4 unext[SUB4];
        float inext = 0.0f;
        if constexpr (J + 1 < SUB) {
            const float* nrow = Us + (wc + J + 1) * B + wc;
#pragma unroll
            for (int k4 = ((J + 2) / 4) * 4; k4 < SUB; k4 += 4) unext[k4 / 4] = *reinterpret_cast<const float4*>(nrow + k4);
            inext = invd[J + 1];
        }
        const float wj = w[J];
        const float c = quant_code(wj, gr.s, gr.inv_s, gr.z, gr.maxq);
        const float q = gr.s * (c - gr.z);
        const float e = (wj - q) * icur;
#pragma unroll
        for (int k4 = ((J + 1) / 4) * 4; k4 < SUB; k4 += 4) {
            const float4 u = ucur[k4 / 4];
            if (k4 + 0 > J) w[k4 + 0] = fmaf(-e, u.x, w[k4 + 0]);
            if (k4 + 1 > J) w[k4 + 1] = fmaf(-e, u.y, w[k4 + 1]);
            if (k4 + 2 > J) w[k4 + 2] = fmaf(-e, u.z, w[k4 + 2]);
            if (k4 + 3 > J) w[k4 + 3] = fmaf(-e, u.w, w[k4 + 3]);
        }
        w[J] = e;
        if (eh != nullptr && (J % PUB == PUB - 1)) {   // (the same in every lane of the warp)
#pragma unroll
            for (int j = J + 1 - PUB; j <= J; ++j) eh[j] = w[j];
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                *prog = J + 1;
            }
        }
        finite &= isfinite(e);
        if (Qw) Qw[J] = q;
        pk.template put<J>(static_cast<uint32_t>(c));
        if constexpr (J + 1 < SUB)
            WindowCol<BITS, J + 1>::run(w, Us, wc, invd, gr, pk, Qw, finite, eh, prog, lane, unext, inext);
    }
};

struct SweepArgs {
    float* W;
    const float* U;
    const float* Ut;     // [d_in, d_in] tf32-rounded hi parts of U^T (lazy trailing update)
    const float* Ut_lo;  // and their remainders
    int d_out, d_in, groupsize, n_groups;
    float maxq;
    uint32_t* codes;
    uint16_t* scales;
    uint16_t* zeros;
    float* Q;
    float* E;     // [d_out, e_ld] hi parts of the super-block's E (tf32-rounded)
    float* E_lo;  // [d_out, e_ld] remainders
    int e_ld;     // super-block width: block i0's E goes to columns i0 % e_ld ..
    DevStatus* st;
};

// Four warps per window.  Before a window's serial chain starts, its columns
// must receive the E of every earlier column (a rank-1 update per column); the
// four warps of the window share that work (8 columns each), then three of
// them hand their columns to the window's owner warp (h = 0), which runs the
// chain.
constexpr int HELP = 4;                       // warps per window
constexpr int HC = SUB / HELP;                // columns per warp while updating
constexpr int SWEEP_THREADS = 32 * NWIN * HELP;
constexpr int HLD = SUB + 1;                  // hand-over rows (conflict-free)

// shared memory: U block, E hand-over (one [32][ELD] per window), column
// hand-over to the owners ([NWIN][32][HLD]), 1/U_jj, min / max per warp and
// the grid, the U mbarrier and the progress counts
constexpr size_t SMEM = 1024 /*align slack*/ +
                        (size_t(B) * B + size_t(NWIN) * SUB * ELD + size_t(NWIN) * SUB * HLD + B +
                         2 * size_t(NWIN) * HELP * SUB + 2 * SUB) * sizeof(float) + 64;

template <int BITS>
__global__ void __launch_bounds__(SWEEP_THREADS) sweep_block_kernel(const __grid_constant__ CUtensorMap tmU,
                                                                    const SweepArgs a, int i0) {
    extern __shared__ uint8_t smem_raw[];
    float* sm = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* Us = sm;                            // Us[j][k] = U[i0+j][i0+k]  (TMA destination: 1024-aligned)
    float* Eh = Us + B * B;                    // Eh[p][row][j]: E of window p
    float* Hv = Eh + NWIN * SUB * ELD;         // Hv[q][row][k]: window q's columns after the update
    float* invd = Hv + NWIN * SUB * HLD;       // 1 / U[i0+j][i0+j]
    float* red = invd + B;                     // [2][NWIN * HELP][SUB] min / max per warp
    float* gsh = red + 2 * NWIN * HELP * SUB;  // [2][SUB] grid of each row
    uint64_t* bars = reinterpret_cast<uint64_t*>(gsh + 2 * SUB);   // [0] U landed
    int* prog = reinterpret_cast<int*>(bars + 1 + NWIN);   // [p]: columns of window p whose E is in Eh
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // window q's four warps are q, q + 4, q + 8, q + 12: one scheduler per
    // window, so a window's serial chain never shares issue slots with the
    // updates the later windows run meanwhile
    const int q = warp % NWIN, h = warp / NWIN;   // window, and this warp's share of it
    const int wc = q * SUB;                       // window's first column in the block
    const int hc = wc + h * HC;                   // this warp's columns while updating
    const int r = blockIdx.x * SUB + lane;
    const bool active = r < a.d_out;

    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        for (int p = 0; p < NWIN; ++p) prog[p] = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {   // U is not written by the kernel before this one: copy it before waiting
        mbar_arrive_expect_tx(&bars[0], B * B * sizeof(float));
        tma_load_2d(Us, &tmU, i0, i0, &bars[0]);   // one 128 x 128 fp32 box, no swizzle
    }
    pdl_wait();       // W as the previous trailing product left it
    pdl_trigger();

    // this warp's 8 columns of this lane's row, and their min / max
    float v[HC];
    {
        const float* wsrc = a.W + size_t(active ? r : 0) * a.d_in + i0 + hc;
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < HC; k += 4) {
            const float4 x = active ? *reinterpret_cast<const float4*>(wsrc + k) : make_float4(0.f, 0.f, 0.f, 0.f);
            v[k] = x.x; v[k + 1] = x.y; v[k + 2] = x.z; v[k + 3] = x.w;
            mn = fminf(fminf(mn, x.x), fminf(x.y, fminf(x.z, x.w)));
            mx = fmaxf(fmaxf(mx, x.x), fmaxf(x.y, fmaxf(x.z, x.w)));
        }
        red[warp * SUB + lane] = mn;
        red[(NWIN * HELP + warp) * SUB + lane] = mx;
    }
    __syncthreads();

    // grid of each row (warp 0), handed to the others through shared memory
    bool finite = true;
    if (warp == 0 && active) {
        float s, z;
        if (a.groupsize < 0) {
            s = __half2float(__ushort_as_half(a.scales[r]));
            z = __half2float(__ushort_as_half(a.zeros[r]));
        } else {
            const size_t gi = size_t(r) * a.n_groups + i0 / a.groupsize;
            if (i0 % a.groupsize == 0) {
                // grid from the current weights of the group: this block as loaded,
                // later columns of the group from W (already lazily updated)
                float gmn = red[lane], gmx = red[NWIN * HELP * SUB + lane];
#pragma unroll
                for (int p = 1; p < NWIN * HELP; ++p) {
                    gmn = fminf(gmn, red[p * SUB + lane]);
                    gmx = fmaxf(gmx, red[(NWIN * HELP + p) * SUB + lane]);
                }
                const float* rowp = a.W + size_t(r) * a.d_in + i0;
                for (int c = B; c < a.groupsize; c += 4) {
                    const float4 x = *reinterpret_cast<const float4*>(rowp + c);
                    gmn = fminf(fminf(gmn, x.x), fminf(x.y, fminf(x.z, x.w)));
                    gmx = fmaxf(fmaxf(gmx, x.x), fmaxf(x.y, fmaxf(x.z, x.w)));
                }
                __half s16, z16;
                finite &= grid_params(gmn, gmx, a.maxq, s, z, s16, z16);
                a.scales[gi] = __half_as_ushort(s16);
                a.zeros[gi] = __half_as_ushort(z16);
            } else {
                s = __half2float(__ushort_as_half(a.scales[gi]));
                z = __half2float(__ushort_as_half(a.zeros[gi]));
            }
        }
        gsh[lane] = s;
        gsh[SUB + lane] = z;
    }
    const bool loaded = mbar_wait(&bars[0], 0, a.st, 201);
    if (threadIdx.x < B) invd[threadIdx.x] = loaded ? 1.0f / Us[threadIdx.x * B + threadIdx.x] : 0.0f;
    __syncthreads();

    // E of the earlier windows' columns, applied to this warp's 8 columns as
    // each batch is published (in column order; the updates commute)
    {
        const int total = wc;
        int c = 0;
        uint32_t spins = 0;
        unsigned long long t0 = 0;
        while (c < total) {
            const int p = c / SUB;
            const int avail = p * SUB + __shfl_sync(0xffffffffu, static_cast<volatile int*>(prog)[p], 0);
            if (avail <= c) {
                if ((++spins & 255u) == 0u) {   // bounded wait for the earlier window
                    const unsigned long long now = globaltimer_ns();
                    if (t0 == 0) t0 = now;
                    else if (now - t0 > kWaitLimitNs) { record_error(a.st, GPTQ_ERR_TIMEOUT, 202); break; }
                }
                continue;
            }
            __threadfence_block();
            for (; c < avail; c += PUB) {   // windows publish PUB columns at a time
                float e[PUB];
#pragma unroll
                for (int t = 0; t < PUB; ++t) e[t] = Eh[(p * SUB + lane) * ELD + (c - p * SUB) + t];
#pragma unroll
                for (int t = 0; t < PUB; ++t) {
                    const float4* u4 = reinterpret_cast<const float4*>(Us + (c + t) * B + hc);
#pragma unroll
                    for (int k4 = 0; k4 < HC / 4; ++k4) {
                        const float4 u = u4[k4];
                        v[4 * k4 + 0] = fmaf(-e[t], u.x, v[4 * k4 + 0]);
                        v[4 * k4 + 1] = fmaf(-e[t], u.y, v[4 * k4 + 1]);
                        v[4 * k4 + 2] = fmaf(-e[t], u.z, v[4 * k4 + 2]);
                        v[4 * k4 + 3] = fmaf(-e[t], u.w, v[4 * k4 + 3]);
                    }
                }
            }
        }
    }

    // hand the updated columns to the window's owner
    if (h != 0) {
#pragma unroll
        for (int k = 0; k < HC; ++k) Hv[(q * SUB + lane) * HLD + h * HC + k] = v[k];
    }
    named_barrier_sync(1 + q, 32 * HELP);
    if (h != 0) return;

    // the owner: this window, column by column (each E published to the later windows)
    float w[SUB];
#pragma unroll
    for (int k = 0; k < HC; ++k) w[k] = v[k];
#pragma unroll
    for (int k = HC; k < SUB; ++k) w[k] = Hv[(q * SUB + lane) * HLD + k];
    const Grid gr{gsh[lane], gsh[SUB + lane], a.maxq, __frcp_rn(gsh[lane])};
    Packer<BITS> pk;
    float* qrow = (a.Q && active) ? a.Q + size_t(r) * a.d_in + i0 + wc : nullptr;
    float* eh = q + 1 < NWIN ? Eh + (q * SUB + lane) * ELD : nullptr;
    float4 u0[SUB4];
#pragma unroll
    for (int k4 = 0; k4 < SUB4; ++k4) u0[k4] = *reinterpret_cast<const float4*>(Us + wc * B + wc + 4 * k4);
    WindowCol<BITS, 0>::run(w, Us, wc, invd + wc, gr, pk, qrow, finite, eh, prog + q, lane, u0, invd[wc]);

    if (active) {
        // E leaves pre-split for the trailing product's tensor cores
        float* erow = a.E + size_t(r) * a.e_ld + i0 % a.e_ld + wc;
        float* elo = a.E_lo + size_t(r) * a.e_ld + i0 % a.e_ld + wc;
#pragma unroll
        for (int j = 0; j < SUB; j += 4) {
            float4 hi, lo;
            split_tf32(w[j], hi.x, lo.x); split_tf32(w[j + 1], hi.y, lo.y);
            split_tf32(w[j + 2], hi.z, lo.z); split_tf32(w[j + 3], hi.w, lo.w);
            *reinterpret_cast<float4*>(erow + j) = hi;
            *reinterpret_cast<float4*>(elo + j) = lo;
        }
        pk.store(a.codes + size_t(r) * (size_t(a.d_in) * BITS / 32) + size_t(i0 + wc) * BITS / 32);
        if (!finite) record_error(a.st, GPTQ_ERR_NONFINITE, r);
    }
}

// RTN: one thread per 32 consecutive codes of a row (one packing unit for
// every supported width); grid from the original W (grid_kernel).
template <int BITS>
__global__ void rtn_kernel(const float* __restrict__ W, int d_out, int d_in, int group, int n_groups, float maxq,
                           const uint16_t* __restrict__ scales, const uint16_t* __restrict__ zeros,
                           uint32_t* __restrict__ codes, float* __restrict__ Q) {
    const int units = d_in / 32;
    const size_t t = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= size_t(d_out) * units) return;
    const int r = int(t / units), u = int(t % units);
    const int c0 = u * 32;
    const size_t gi = size_t(r) * n_groups + c0 / group;
    const float s = __half2float(__ushort_as_half(scales[gi]));
    const float inv_s = __frcp_rn(s);
    const float z = __half2float(__ushort_as_half(zeros[gi]));
    const float* src = W + size_t(r) * d_in + c0;
    uint32_t words[BITS] = {};
#pragma unroll
    for (int k = 0; k < 32; k += 4) {
        const float4 v = *reinterpret_cast<const float4*>(src + k);
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t c = static_cast<uint32_t>(quant_code(vv[i], s, inv_s, z, maxq));
            const int pos = (k + i) * BITS, word = pos / 32, off = pos % 32;
            words[word] |= c << off;
            if (off + BITS > 32) words[word + 1] |= c >> (32 - off);
            if (Q) Q[size_t(r) * d_in + c0 + k + i] = s * (float(c) - z);
        }
    }
    uint32_t* dst = codes + size_t(r) * (size_t(d_in) * BITS / 32) + size_t(u) * BITS;
#pragma unroll
    for (int i = 0; i < BITS; ++i) dst[i] = words[i];
}

__global__ void widen_bf16_kernel(const uint16_t* __restrict__ src, float* __restrict__ dst, size_t n) {
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += size_t(gridDim.x) * blockDim.x)
        dst[i] = __uint_as_float(uint32_t(src[i]) << 16);
}

__global__ void fill_kernel(float* __restrict__ p, size_t n, float v) {
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += size_t(gridDim.x) * blockDim.x)
        p[i] = v;
}

// Ut[c][r] + Ut_lo[c][r] = U[r][c] (hi / lo split) for the tiles of U that
// reach the upper triangle (the trailing products read U's rows as K-major
// operands through Ut).
__global__ void transpose_upper_kernel(const float* __restrict__ U, int d, float* __restrict__ Ut,
                                       float* __restrict__ Ut_lo) {
    __shared__ float tile[32][33];
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    if (c0 + 31 < r0) return;
    for (int rr = threadIdx.y; rr < 32; rr += blockDim.y)
        tile[rr][threadIdx.x] = U[size_t(r0 + rr) * d + c0 + threadIdx.x];
    __syncthreads();
    for (int cc = threadIdx.y; cc < 32; cc += blockDim.y) {
        float h, l;
        split_tf32(tile[threadIdx.x][cc], h, l);
        Ut[size_t(c0 + cc) * d + r0 + threadIdx.x] = h;
        Ut_lo[size_t(c0 + cc) * d + r0 + threadIdx.x] = l;
    }
}

// The blocks in order, each followed by its share of the trailing update.
// Deferred super-block form (exact reformulation of the pages' lazy update:
// the trailing update is linear, so each column still holds, when the sweep
// reaches it, every earlier block's correction): the blocks are taken in
// super-blocks of a.e_ld columns.  After block i0, its E updates only the
// rest of its super-block, W[:, i0+B:s2] -= E_i0 U[i0:i0+B, i0+B:s2]; after
// the super-block's last block, the columns beyond it get one product with
// the super-block's whole E, W[:, s2:] -= E_sb U[s1:s2, s2:] (K = e_ld).  The
// far tail of W is then read and written once per super-block instead of
// once per block, and each product is e_ld deep instead of B.  With e_ld = B
// this is exactly the per-block form.  A group grid is set from the columns
// of its group, which therefore must lie inside one super-block (e_ld is a
// multiple of the group size).  Everything runs on one stream, in a fixed
// order, so the result does not depend on timing.
template <int BITS>
int run_sweep(const SweepArgs& a, cudaStream_t stream) {
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(sweep_block_kernel<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM)) !=
            cudaSuccess)
            return GPTQ_ERR_CUDA;
        attr_set[dev] = true;
    }
    CUtensorMap tmU;
    if (make_map_2d_f32(&tmU, a.U, uint64_t(a.d_in), uint64_t(a.d_in), uint64_t(a.d_in), B, B, false))
        return GPTQ_ERR_CUDA;
    const int blocks = (a.d_out + SUB - 1) / SUB;
    const int sbw = a.e_ld;
    for (int s1 = 0; s1 < a.d_in; s1 += sbw) {
        const int s2 = std::min(s1 + sbw, a.d_in);
        for (int i0 = s1; i0 < s2; i0 += B) {
            if (launch_pdl(sweep_block_kernel<BITS>, dim3(blocks), dim3(SWEEP_THREADS), SMEM, stream, tmU, a, i0) !=
                cudaSuccess)
                return GPTQ_ERR_CUDA;
            count_launch();
            const int near = s2 - i0 - B;
            if (near > 0) {
                // W[:, i0+B:s2] -= E_i0 U[i0:i0+B, i0+B:s2]   (U[i0+k][i0+B+n] = Ut[i0+B+n][i0+k])
                const size_t ut = size_t(i0 + B) * a.d_in + i0;
                const int rc = launch_tgemm(a.d_out, near, B, -1.0f, a.E + (i0 - s1), a.E_lo + (i0 - s1), sbw,
                                            a.Ut + ut, a.Ut_lo + ut, a.d_in, true, a.W + i0 + B, a.d_in, false,
                                            stream, a.st);
                if (rc) return rc;
            }
        }
        const int far = a.d_in - s2;
        if (far > 0) {
            // W[:, s2:] -= E_sb U[s1:s2, s2:]
            const size_t ut = size_t(s2) * a.d_in + s1;
            const int rc = launch_tgemm(a.d_out, far, s2 - s1, -1.0f, a.E, a.E_lo, sbw, a.Ut + ut, a.Ut_lo + ut,
                                        a.d_in, true, a.W + s2, a.d_in, false, stream, a.st);
            if (rc) return rc;
        }
    }
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace sweep

// Width of the super-blocks of the deferred trailing update: up to
// kSuperBlockCols columns, a multiple of the block and of the group size; the
// whole layer when it is narrower; the per-block form (B) for groups wider
// than kSuperBlockCols.
#ifndef GPTQ_SUPERBLOCK_COLS
#define GPTQ_SUPERBLOCK_COLS 1024
#endif
constexpr int kSuperBlockCols = GPTQ_SUPERBLOCK_COLS;   // a build-time tuning knob (128: per-block form)
static_assert(kSuperBlockCols % 128 == 0 && kSuperBlockCols >= 128 && kSuperBlockCols <= 8192, "super-block width");
int superblock_cols(int64_t d_in, int groupsize) {
    if (d_in <= kSuperBlockCols) return int(d_in);
    if (groupsize <= 0) return kSuperBlockCols;
    if (groupsize > kSuperBlockCols) return sweep::B;
    return (kSuperBlockCols / groupsize) * groupsize;
}

// E hi, E lo [d_out, min(d_in, kSuperBlockCols)] fp32, then U^T hi, U^T lo
// [d_in, d_in] fp32 (each 256-byte aligned)
namespace {
size_t e_bytes(int64_t d_out, int64_t d_in) {
    return (size_t(d_out) * size_t(std::min<int64_t>(d_in, kSuperBlockCols)) * sizeof(float) + 255) & ~size_t(255);
}
}  // namespace

size_t sweep_workspace_bytes(int64_t d_out, int64_t d_in) {
    return 2 * e_bytes(d_out, d_in) + 2 * size_t(d_in) * size_t(d_in) * sizeof(float);
}

int launch_quantize(float* W, int64_t d_out, int64_t d_in, const float* U, int bits, int groupsize,
                    uint32_t* codes, uint16_t* scales, uint16_t* zeros, float* Q, void* ws, cudaStream_t stream,
                    DevStatus* st) {
    using namespace sweep;
    SweepArgs a;
    a.W = W;
    a.U = U;
    a.d_out = int(d_out);
    a.d_in = int(d_in);
    a.groupsize = groupsize;
    a.n_groups = groupsize > 0 ? int(d_in / groupsize) : 1;
    a.maxq = float((1 << bits) - 1);
    a.codes = codes;
    a.scales = scales;
    a.zeros = zeros;
    a.Q = Q;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    a.E = reinterpret_cast<float*>(wsb);
    a.E_lo = reinterpret_cast<float*>(wsb + e_bytes(d_out, d_in));
    a.e_ld = superblock_cols(d_in, groupsize);
    float* Ut = reinterpret_cast<float*>(wsb + 2 * e_bytes(d_out, d_in));
    float* Ut_lo = Ut + size_t(d_in) * size_t(d_in);
    a.Ut = Ut;
    a.Ut_lo = Ut_lo;
    a.st = st;
    if (groupsize < 0) {
        const int warps = a.d_out;
        grid_kernel<<<(warps * 32 + 255) / 256, 256, 0, stream>>>(W, a.d_out, a.d_in, a.d_in, 1, a.maxq, scales,
                                                                  zeros, st); count_launch();
    }
    transpose_upper_kernel<<<dim3(unsigned(d_in / 32), unsigned(d_in / 32)), dim3(32, 8), 0, stream>>>(U, int(d_in), Ut, Ut_lo);
    count_launch();
    switch (bits) {
        case 2: return run_sweep<2>(a, stream);
        case 3: return run_sweep<3>(a, stream);
        case 4: return run_sweep<4>(a, stream);
        case 8: return run_sweep<8>(a, stream);
        default: return GPTQ_ERR_UNSUPPORTED;
    }
}

int launch_rtn(const float* W, int64_t d_out, int64_t d_in, int bits, int groupsize, uint32_t* codes,
               uint16_t* scales, uint16_t* zeros, float* Q, cudaStream_t stream, DevStatus* st) {
    using namespace sweep;
    const int group = groupsize > 0 ? groupsize : int(d_in);
    const int n_groups = int(d_in / group);
    const float maxq = float((1 << bits) - 1);
    const int64_t warps = d_out * n_groups;
    grid_kernel<<<unsigned((warps * 32 + 255) / 256), 256, 0, stream>>>(W, int(d_out), int(d_in), group, n_groups,
                                                                         maxq, scales, zeros, st); count_launch();
    const int64_t units = d_out * (d_in / 32);
    const unsigned blocks = unsigned((units + 255) / 256);
    switch (bits) {
        case 2: rtn_kernel<2><<<blocks, 256, 0, stream>>>(W, int(d_out), int(d_in), group, n_groups, maxq, scales, zeros, codes, Q); count_launch(); break;
        case 3: rtn_kernel<3><<<blocks, 256, 0, stream>>>(W, int(d_out), int(d_in), group, n_groups, maxq, scales, zeros, codes, Q); count_launch(); break;
        case 4: rtn_kernel<4><<<blocks, 256, 0, stream>>>(W, int(d_out), int(d_in), group, n_groups, maxq, scales, zeros, codes, Q); count_launch(); break;
        case 8: rtn_kernel<8><<<blocks, 256, 0, stream>>>(W, int(d_out), int(d_in), group, n_groups, maxq, scales, zeros, codes, Q); count_launch(); break;
        default: return GPTQ_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

int launch_widen_bf16(const uint16_t* src, float* dst, int64_t count, cudaStream_t stream) {
    if (count <= 0) return GPTQ_OK;
    const unsigned blocks = unsigned(std::min<int64_t>((count + 255) / 256, 148 * 32));
    sweep::widen_bf16_kernel<<<blocks, 256, 0, stream>>>(src, dst, size_t(count)); count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

int launch_fill(float* p, int64_t count, float value, cudaStream_t stream) {
    if (count <= 0) return GPTQ_OK;
    const unsigned blocks = unsigned(std::min<int64_t>((count + 255) / 256, 148 * 32));
    sweep::fill_kernel<<<blocks, 256, 0, stream>>>(p, size_t(count), value); count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
