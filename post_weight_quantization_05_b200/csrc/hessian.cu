// Stage 1: H += 2 X^T X on the tcgen05 tensor cores.
//
// Source: blog "GPTQ를 밑바닥부터 구현하며 배운 것들", section 3 (H = 2 X^T X);
// itwiki "GPTQ", "최소 구현" (X laid out [n, d_in]) and its closing paragraph
// (accumulated per layer over the calibration batches).
//
// Design (B200):
//  - H is symmetric, so only output tiles that reach the upper triangle are
//    computed.  Tile = 128 (a) x 256 (b) of H; the contraction runs over the
//    calibration rows r.  X is row-major [n, d], i.e. both operands of the
//    product X[:, a-tile]^T X[:, b-tile] are MN-major (the a / b index is the
//    contiguous one), which tcgen05 reads directly from 128-byte-swizzled
//    shared memory -- no transpose pass over X.
//  - Per stage a TMA load brings 64 calibration rows of the a-columns
//    (16 KB) and of the b-columns (32 KB); 4 stages in flight.  One thread
//    issues TMA, one thread issues tcgen05.mma (M=128, N=256, K=16, fp32
//    accumulator in 256 TMEM columns), and all four warps drain TMEM in the
//    epilogue and add 2*acc into H.
//  - fp32 inputs are split into three bf16 terms by `split3_kernel`; the
//    contraction then runs over the six leading cross products
//    (hh, hm, mh, mm, hl, lh), which the K loop walks one after another.
//  - No TMA multicast anywhere.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace hess {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int CHUNK_BYTES = 64 * BK * 2;  // one TMA box: 64 columns x 64 rows
constexpr int TMEM_COLS = 256;
constexpr int THREADS = 128;
constexpr size_t SMEM_BYTES = 1024 /*align slack*/ + size_t(STAGES) * STAGE_BYTES + 256 /*barriers*/;

struct Params {
    int d;          // d_in
    int n;          // calibration rows in this call
    int npairs;     // number of (A part, B part) products
    int pa[6];
    int pb[6];
    float alpha;    // 2.0
    int tiles_b;    // ceil(d / BN)
    int tiles_a;    // d / BM
};

// Map a linear tile index to (ti, tj): tiles (ti, tj) with ti*BM <= tj*BN + BN - 1.
__device__ __forceinline__ void tile_coords(int t, const Params& p, int& ti, int& tj) {
    int acc = 0;
    for (tj = 0; tj < p.tiles_b; ++tj) {
        int cnt = min(p.tiles_a, (tj * BN + BN - 1) / BM + 1);
        if (t < acc + cnt) {
            ti = t - acc;
            return;
        }
        acc += cnt;
    }
    ti = -1;
}

__global__ void __launch_bounds__(THREADS, 1)
    syrk_kernel(const __grid_constant__ CUtensorMap tmX, const Params p, float* __restrict__ H,
                DevStatus* st) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(STAGES) * STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* accum = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);

    int ti, tj;
    tile_coords(blockIdx.x, p, ti, tj);
    if (ti < 0) return;
    const int a0 = ti * BM;
    const int b0 = tj * BN;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tmX);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accum, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int kper = (p.n + BK - 1) / BK;
    const int ksteps = kper * p.npairs;
    bool ok = true;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer
        int last_round[STAGES];
#pragma unroll
        for (int s = 0; s < STAGES; ++s) last_round[s] = -1;
        for (int ks = 0; ks < ksteps; ++ks) {
            const int s = ks % STAGES;
            const uint32_t round = ks / STAGES;
            if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, st, 101)) { ok = false; break; }
            const int pair = ks / kper;
            const int r0 = (ks - pair * kper) * BK;
            uint8_t* sa = smem + size_t(s) * STAGE_BYTES;
            uint8_t* sb = sa + A_BYTES;
            mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
#pragma unroll
            for (int h = 0; h < BM / 64; ++h) tma_load_3d(sa + h * CHUNK_BYTES, &tmX, a0 + 64 * h, r0, p.pa[pair], &full[s]);
#pragma unroll
            for (int h = 0; h < BN / 64; ++h) tma_load_3d(sb + h * CHUNK_BYTES, &tmX, b0 + 64 * h, r0, p.pb[pair], &full[s]);
            last_round[s] = int(round);
        }
        if (!ok) {
            // let the copies already in flight land before the CTA can exit
#pragma unroll
            for (int s = 0; s < STAGES; ++s)
                if (last_round[s] >= 0) (void)mbar_wait(&full[s], uint32_t(last_round[s]) & 1u, st, 104);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        constexpr uint32_t idesc = idesc_bf16_mn_mn(BM, BN);
        for (int ks = 0; ks < ksteps; ++ks) {
            const int s = ks % STAGES;
            const uint32_t round = ks / STAGES;
            if (!mbar_wait(&full[s], round & 1u, st, 102)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + size_t(s) * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
                // 16 K rows = two 8-row groups of 128 bytes each
                const uint64_t da = sdesc_sw128(sa + kk * 2048, CHUNK_BYTES, 1024);
                const uint64_t db = sdesc_sw128(sb + kk * 2048, CHUNK_BYTES, 1024);
                umma_f16(tmem_base, da, db, idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&empty[s]);  // frees the stage once these MMAs are done
        }
        umma_commit(accum);          // accumulator complete (also on the error path)
    }

    // ---------------- epilogue: TMEM -> registers -> H += alpha * acc
    __syncwarp();
    const bool acc_ready = mbar_wait(accum, 0, st, 103);
    tc_fence_after();
    if (acc_ready && ksteps > 0) {
        const int m = warp * 32 + lane;  // TMEM lane == row of the tile
        const int a = a0 + m;
        float* hrow = H + size_t(a) * p.d;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
            float v[32];
            tmem_ld_32x32b_x32(tmem_base + (uint32_t(warp * 32) << 16) + uint32_t(c * 32), v);
            const int b = b0 + c * 32;
            if (b + 32 <= p.d) {
                float4* dst = reinterpret_cast<float4*>(hrow + b);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float4 h = dst[q];
                    h.x = fmaf(p.alpha, v[4 * q + 0], h.x);
                    h.y = fmaf(p.alpha, v[4 * q + 1], h.y);
                    h.z = fmaf(p.alpha, v[4 * q + 2], h.z);
                    h.w = fmaf(p.alpha, v[4 * q + 3], h.w);
                    dst[q] = h;
                }
            } else {
#pragma unroll
                for (int q = 0; q < 32; ++q)
                    if (b + q < p.d) hrow[b + q] = fmaf(p.alpha, v[q], hrow[b + q]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base, TMEM_COLS);
}

// x = h + m + l with h, m, l bf16 (each the bf16 rounding of what remains).
__global__ void split3_kernel(const float* __restrict__ X, __nv_bfloat16* __restrict__ out, size_t count) {
    const size_t stride = size_t(gridDim.x) * blockDim.x;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride) {
        const float x = X[i];
        const __nv_bfloat16 h = __float2bfloat16_rn(x);
        const float r1 = x - __bfloat162float(h);
        const __nv_bfloat16 m = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(m);
        out[i] = h;
        out[count + i] = m;
        out[2 * count + i] = __float2bfloat16_rn(r2);
    }
}

}  // namespace hess
}  // namespace gptq

namespace gptq {

int launch_hessian(const void* X, int dtype, int64_t n, int64_t d, float* H, void* ws, cudaStream_t stream,
                   DevStatus* st, PFN_encodeTiled encode) {
    using namespace hess;
    if (n == 0) return GPTQ_OK;
    const void* base = X;
    int parts = 1;
    Params p{};
    p.d = int(d);
    p.n = int(n);
    p.alpha = 2.0f;
    if (dtype == GPTQ_F32) {
        const size_t count = size_t(n) * size_t(d);
        int blocks = int(std::min<size_t>((count + 255) / 256, size_t(148) * 16));
        split3_kernel<<<blocks, 256, 0, stream>>>(static_cast<const float*>(X),
                                                  static_cast<__nv_bfloat16*>(ws), count); count_launch();
        base = ws;
        parts = 3;
        const int pa[6] = {0, 0, 1, 1, 0, 2};
        const int pb[6] = {0, 1, 0, 1, 2, 0};
        p.npairs = 6;
        for (int i = 0; i < 6; ++i) { p.pa[i] = pa[i]; p.pb[i] = pb[i]; }
    } else {
        p.npairs = 1;
        p.pa[0] = p.pb[0] = 0;
    }
    CUtensorMap tm;
    const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(n), cuuint64_t(parts)};
    const cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(d) * 2 * cuuint64_t(n)};
    const cuuint32_t box[3] = {64, BK, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return GPTQ_ERR_CUDA;
    p.tiles_a = int(d / BM);
    p.tiles_b = int((d + BN - 1) / BN);
    int tiles = 0;
    for (int tj = 0; tj < p.tiles_b; ++tj) tiles += std::min(p.tiles_a, (tj * BN + BN - 1) / BM + 1);
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(syrk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES)) !=
            cudaSuccess)
            return GPTQ_ERR_CUDA;
        attr_set[dev] = true;
    }
    syrk_kernel<<<tiles, THREADS, SMEM_BYTES, stream>>>(tm, p, H, st); count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
