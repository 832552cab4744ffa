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
//    accumulator in TMEM).
//  - Promotion: the tensor core's fp32 accumulation loses about half an ulp
//    per accumulation step (measured: relative error ~4e-5 over a chain of
//    16384 rows).  So the K loop is cut into chunks of 512 rows, each summed
//    into one of two TMEM buffers (2 x 256 columns) while eight epilogue warps
//    drain the other buffer and add it into fp32 registers (round to
//    nearest); at the end they add 2 * sum into H.
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
constexpr int CHUNK = 8;          // k-steps (of BK rows) summed in TMEM before promotion
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int CHUNK_BYTES = 64 * BK * 2;  // one TMA box: 64 columns x 64 rows
constexpr int TMEM_COLS = 2 * BN;         // two accumulator buffers
constexpr int EPI_WARPS = 8;              // 4 TMEM lane quadrants x 2 column halves
constexpr int THREADS = 32 * (2 + EPI_WARPS);
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
    uint64_t* tfull = empty + STAGES;   // [2] MMA -> epilogue: chunk summed in buffer b
    uint64_t* tempty = tfull + 2;       // [2] epilogue -> MMA: buffer b drained
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

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
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], EPI_WARPS);
        }
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
    const int nchunks = (ksteps + CHUNK - 1) / CHUNK;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            bool ok = true;
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
                for (int h = 0; h < BM / 64; ++h)
                    tma_load_3d(sa + h * CHUNK_BYTES, &tmX, a0 + 64 * h, r0, p.pa[pair], &full[s]);
#pragma unroll
                for (int h = 0; h < BN / 64; ++h)
                    tma_load_3d(sb + h * CHUNK_BYTES, &tmX, b0 + 64 * h, r0, p.pb[pair], &full[s]);
                last_round[s] = int(round);
            }
            if (!ok) {
                // let the copies already in flight land before the CTA can exit
#pragma unroll
                for (int s = 0; s < STAGES; ++s)
                    if (last_round[s] >= 0) (void)mbar_wait(&full[s], uint32_t(last_round[s]) & 1u, st, 104);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            constexpr uint32_t idesc = idesc_bf16_mn_mn(BM, BN);
            bool ok = true;
            for (int c = 0; c < nchunks && ok; ++c) {
                const int buf = c & 1;
                const int use = c >> 1;
                if (use > 0 && !mbar_wait(&tempty[buf], uint32_t(use - 1) & 1u, st, 105)) { ok = false; break; }
                tc_fence_after();
                const uint32_t dt = tmem_base + uint32_t(buf * BN);
                const int k_end = min(ksteps, (c + 1) * CHUNK);
                for (int ks = c * CHUNK; ks < k_end; ++ks) {
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
                        umma_f16(dt, da, db, idesc, (ks > c * CHUNK || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);  // frees the stage once these MMAs are done
                }
                umma_commit(&tfull[buf]);    // this chunk's sum is complete (also on the error path)
            }
        }
    } else {
        // ---------------- epilogue warps: promote each chunk into fp32 registers
        const int e = warp - 2;
        const int quad = warp & 3;           // TMEM lanes this warp may access
        const int half = e >> 2;             // which 128 of the 256 columns
        const uint32_t lane_addr = uint32_t(quad * 32) << 16;
        float acc[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int buf = c & 1;
            const int use = c >> 1;
            if (!mbar_wait(&tfull[buf], uint32_t(use) & 1u, st, 103)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float v[32];
                tmem_ld_32x32b_x32(tmem_base + lane_addr + uint32_t(buf * BN + half * 128 + cc * 32), v);
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[cc * 32 + i] += v[i];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
        }
        if (ok && nchunks > 0) {
            const int a = a0 + quad * 32 + lane;   // TMEM lane == row of the tile
            float* hrow = H + size_t(a) * p.d;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int b = b0 + half * 128 + cc * 32;
                if (b + 32 <= p.d) {
                    float4* dst = reinterpret_cast<float4*>(hrow + b);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 h = dst[q];
                        h.x = fmaf(p.alpha, acc[cc * 32 + 4 * q + 0], h.x);
                        h.y = fmaf(p.alpha, acc[cc * 32 + 4 * q + 1], h.y);
                        h.z = fmaf(p.alpha, acc[cc * 32 + 4 * q + 2], h.z);
                        h.w = fmaf(p.alpha, acc[cc * 32 + 4 * q + 3], h.w);
                        dst[q] = h;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        if (b + q < p.d) hrow[b + q] = fmaf(p.alpha, acc[cc * 32 + q], hrow[b + q]);
                }
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
