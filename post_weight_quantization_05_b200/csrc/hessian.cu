// Stage 1: H += 2 X^T X on the tcgen05 tensor cores.
//
// Source: blog "GPTQ를 밑바닥부터 구현하며 배운 것들", section 3 (H = 2 X^T X);
// itwiki "GPTQ", "최소 구현" (X laid out [n, d_in]) and its closing paragraph
// (accumulated per layer over the calibration batches).
//
// Design (B200):
//  - H is symmetric, so only the 256 x 256 output tiles (ta <= tb) that reach
//    the upper triangle are computed; the contraction runs over the
//    calibration rows r.  X is row-major [n, d], i.e. both operands of the
//    product X[:, a-tile]^T X[:, b-tile] are MN-major (the a / b index is the
//    contiguous one), which tcgen05 reads directly from 128-byte-swizzled
//    shared memory -- no transpose pass over X.
//  - A cluster of two CTAs (two SMs) owns a tile and runs it as cta_group::2
//    MMAs (M = 256, N = 256, K = 16, fp32 accumulators in TMEM): CTA r loads
//    128 calibration rows of its 128 a-columns and of its 128 of the 256
//    b-columns per stage (64 KB, three stages in flight; measured: 64-row
//    stages with six in flight ran 9% slower, 32-row stages 64% slower, so
//    the per-stage handshakes cost more than the shallower ring), and the pair's MMA
//    reads both CTAs' halves.  Per SM that is two thirds of the bytes a
//    single-CTA 128 x 256 tile would stream for the same MMA work, which is
//    what lets the loads stay ahead of the tensor cores.  One thread per CTA
//    issues TMA, one thread of CTA 0 issues the MMAs.
//  - Promotion: the tensor core's fp32 accumulation loses about half an ulp
//    per accumulation step (measured: relative error ~4e-5 over a chain of
//    16384 rows).  So the K loop is cut into chunks of 1024 rows, each summed
//    into one of two TMEM buffers (2 x 256 columns) while eight epilogue warps
//    per CTA drain the other buffer and add it into fp32 registers (round to
//    nearest); at the end they add 2 * sum into H.  Measured relative error
//    of H over 65536 bench rows: 6.5e-7 with 512-row chunks, 1.4e-6 with
//    1024, 3.3e-6 with 2048; 1024 rows take 2.4% less time than 512.
//  - fp32 inputs are split into three bf16 terms by `split3_kernel`; the
//    contraction then runs over the six leading cross products
//    (hh, hm, mh, mm, hl, lh), which the K loop walks one after another.
//  - No TMA load uses multicast (each CTA loads its own halves).
#include <atomic>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace hess {

// Build-time tuning knobs: calibration rows per stage, rows summed in TMEM
// before each promotion to fp32 registers, stages in the ring (default: a
// 192 KB ring).
#ifndef GPTQ_HESS_BK
#define GPTQ_HESS_BK 128
#endif
#ifndef GPTQ_HESS_PROMOTE_ROWS
#define GPTQ_HESS_PROMOTE_ROWS 1024
#endif
constexpr int BK = GPTQ_HESS_BK;            // calibration rows per stage
constexpr int CHUNK = GPTQ_HESS_PROMOTE_ROWS / BK;   // k-steps (of BK rows) summed in TMEM before promotion
static_assert(BK % 16 == 0 && BK <= 256 && CHUNK >= 1 && CHUNK * BK == GPTQ_HESS_PROMOTE_ROWS, "Hessian k-steps");
constexpr int CHUNK_BYTES = 64 * BK * 2;  // one TMA box: 64 columns x BK rows of bf16
constexpr int EPI_WARPS = 8;              // 4 TMEM lane quadrants x 2 column halves
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr int BMH = 128;                   // H rows per CTA (the pair covers 256)
constexpr int BNP = 256;                   // H columns per pair (128 loaded by each CTA)
constexpr int A_BYTES = BMH * BK * 2;      // 32 KB at BK = 128
constexpr int B_BYTES = (BNP / 2) * BK * 2;  // 32 KB at BK = 128
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
#ifndef GPTQ_HESS_STAGES
#define GPTQ_HESS_STAGES (196608 / STAGE_BYTES)
#endif
constexpr int STAGES = GPTQ_HESS_STAGES;
constexpr int TMEM_COLS = 2 * BNP;         // two accumulator buffers
constexpr int FLUSH_COLS = 32;                       // columns of H per reduce-add
constexpr int FLUSH_BYTES = BMH * FLUSH_COLS * 4;    // one staged slab: 128 rows x 32 fp32 (16 KB)
constexpr size_t SMEM_BYTES = 1024 /*align slack*/ + size_t(STAGES) * STAGE_BYTES +
                              2 * size_t(FLUSH_BYTES) /*one staging slab per column half*/ + 256 /*barriers*/;
static_assert(SMEM_BYTES <= 232448, "shared memory per block");
static_assert((2 * STAGES + 4) * 8 + 4 + 8 <= 256, "barrier area");

// Pair protocol: CTA r (r = 0, 1) loads a-columns a0 + 128 r .. + 127 and
// b-columns b0 + 128 r .. + 127 of each slab; both CTAs' TMA loads complete on
// CTA 0's `full` barrier; CTA 0's MMA commits arrive on both CTAs' `empty` and
// `tfull`; the epilogue warps of both CTAs arrive on CTA 0's `tempty`.  Each
// CTA's TMEM holds its 128 rows x 256 columns.

struct Params {
    int d, n, npairs;
    int pa[6], pb[6];
    float alpha;
    int tiles;      // T (T + 1) / 2 tiles (ta <= tb) of 256 x 256, T = ceil(d / 256)
    int T;
    int late_wait;  // the previous kernel in the stream is this kernel on another batch
    int wave;       // SM pairs of the device: the launch's clusters (one per pair)
};

// Launch order of the tiles (ta, tb), ta <= tb.  Pairs that run at the same
// time should read few distinct column slabs of X, so that a slab comes from
// HBM once and from L2 for the other tiles that use it (a slab is n_b x 256
// bf16: 4 MB at 8192 rows, so X of a 28672-wide layer is 112 slabs, far more
// than L2 holds).  Tiles are therefore taken in super-tiles of SUPER x SUPER
// tiles (about one wave of 74 pairs at SUPER = 8, reading at most 16 slabs),
// super-tiles by column J and then row I <= J, and inside a super-tile
// column-major with ta <= tb.  The order does not change any tile's
// arithmetic.
constexpr int SUPER = 8;
__device__ __forceinline__ void tile_of(int t, int T, int& ta, int& tb) {
    const int ns = (T + SUPER - 1) / SUPER;
    for (int J = 0; J < ns; ++J) {
        const int b0 = J * SUPER, b1 = min(T, b0 + SUPER);
        for (int I = 0; I <= J; ++I) {
            const int a0 = I * SUPER, a1 = min(T, a0 + SUPER);
            int cnt = 0;   // tiles of this super-tile with ta <= tb
            for (int b = b0; b < b1; ++b) cnt += max(0, min(a1, b + 1) - a0);
            if (t >= cnt) {
                t -= cnt;
                continue;
            }
            for (int b = b0; b < b1; ++b) {
                const int na = max(0, min(a1, b + 1) - a0);
                if (t < na) {
                    ta = a0 + t;
                    tb = b;
                    return;
                }
                t -= na;
            }
        }
    }
    ta = tb = 0;   // not reached for t < T (T + 1) / 2
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    syrk_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmH, const Params p,
                     DevStatus* st) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* flush_buf = smem + size_t(STAGES) * STAGE_BYTES;                            // [2][FLUSH_BYTES]
    uint64_t* full = reinterpret_cast<uint64_t*>(flush_buf + 2 * size_t(FLUSH_BYTES));    // CTA 0: both halves landed
    uint64_t* empty = full + STAGES;    // both CTAs: the pair's MMAs are done with the stage
    uint64_t* tfull = empty + STAGES;   // [2] both CTAs: chunk summed in buffer b
    uint64_t* tempty = tfull + 2;       // [2] CTA 0: buffer b drained by both CTAs
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    int* half_abort = reinterpret_cast<int*>(tmem_slot + 1);   // [2] an epilogue half gave up on a wait

    const uint32_t rank = cluster_ctarank();
    // Persistent: cluster cl takes tiles cl, cl + ncl, ... (round lt of its
    // tiles is wave lt of the launch).  The stage ring and the two TMEM
    // accumulators run on across tiles, so a tile's loads and MMAs start while
    // the previous tile's last chunk is promoted and added into H.
    const int cl = int(blockIdx.x >> 1), ncl = int(gridDim.x >> 1);
    const int my_tiles = p.tiles > cl ? (p.tiles - cl + ncl - 1) / ncl : 0;
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
            mbar_init(&tempty[b], 2 * EPI_WARPS);
            half_abort[b] = 0;
        }
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();          // barriers of both CTAs initialized, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Wait for the previous kernel in the stream before any global access --
    // unless it is this kernel on another batch (late_wait): that one never
    // writes X, so only the updates of H have to wait for it, and the main
    // loop overlaps its last tiles.
    if (!p.late_wait) pdl_wait();
    pdl_trigger();

    const int kper = (p.n + BK - 1) / BK;
    const int ksteps = kper * p.npairs;
    const int nchunks = (ksteps + CHUNK - 1) / CHUNK;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs).  Tiles of odd waves walk
            // the calibration rows backwards: they start on the rows the previous
            // wave read last, which are still in L2 (X of a 16384-row batch is
            // about the size of L2), instead of on the rows it evicted first.
            // Measured at 4096 x 16384: DRAM traffic per launch 308 -> 266 MB
            // (201 MB algorithmic), time unchanged (the kernel is not bound by
            // DRAM).  An L2 prefetch of X three steps ahead of the ring was
            // slower (3.62 against 3.41 ms per 16 batches).
            int gs = 0;   // stages issued so far, over all tiles
            bool ok = true;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                int ta = 0, tb = 0;
                tile_of(cl + lt * ncl, p.T, ta, tb);
                const int a0 = ta * BNP + int(rank) * BMH;   // this CTA's H rows
                const int b0 = tb * BNP;                     // the pair's H columns
                const bool rev = (lt & 1) != 0;
                for (int ks = 0; ks < ksteps; ++ks, ++gs) {
                    const int s = gs % STAGES;
                    const uint32_t round = uint32_t(gs / STAGES);
                    if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, st, 111)) { ok = false; break; }
                    const int kk = rev ? ksteps - 1 - ks : ks;
                    const int pair = kk / kper;
                    const int r0 = (kk - pair * kper) * BK;
                    uint8_t* sa = smem + size_t(s) * STAGE_BYTES;
                    uint8_t* sb = sa + A_BYTES;
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * STAGE_BYTES);
                    const uint32_t fb = mapa_shared(&full[s], 0);
#pragma unroll
                    for (int h = 0; h < BMH / 64; ++h)
                        tma_load_3d_pair(sa + h * CHUNK_BYTES, &tmX, a0 + 64 * h, r0, p.pa[pair], fb);
#pragma unroll
                    for (int h = 0; h < BNP / 128; ++h)
                        tma_load_3d_pair(sb + h * CHUNK_BYTES, &tmX, b0 + int(rank) * 128 + 64 * h, r0, p.pb[pair],
                                         fb);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer (CTA 0 only)
            constexpr uint32_t idesc = idesc_bf16_mn_mn(2 * BMH, BNP);
            int gs = 0, gc = 0;   // stages and chunks consumed so far, over all tiles
            bool ok = true;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                for (int c = 0; c < nchunks && ok; ++c, ++gc) {
                    const int buf = gc & 1;
                    const int use = gc >> 1;
                    if (use > 0 && !mbar_wait_cluster(&tempty[buf], uint32_t(use - 1) & 1u, st, 115)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t dt = tmem_base + uint32_t(buf * BNP);
                    const int k_end = min(ksteps, (c + 1) * CHUNK);
                    for (int ks = c * CHUNK; ks < k_end; ++ks, ++gs) {
                        const int s = gs % STAGES;
                        const uint32_t round = uint32_t(gs / STAGES);
                        if (!mbar_wait(&full[s], round & 1u, st, 112)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t sa = smem_u32(smem + size_t(s) * STAGE_BYTES);
                        const uint32_t sb = sa + A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint64_t da = sdesc_sw128(sa + kk * 2048, CHUNK_BYTES, 1024);
                            const uint64_t db = sdesc_sw128(sb + kk * 2048, CHUNK_BYTES, 1024);
                            umma_f16_pair(dt, da, db, idesc, (ks > c * CHUNK || kk > 0) ? 1u : 0u);
                        }
                        umma_commit_pair_both(&empty[s]);   // frees the stage in both CTAs
                    }
                    umma_commit_pair_both(&tfull[buf]);     // chunk complete (also on the error path)
                }
            }
        }
    } else {
        // ---------------- epilogue warps (both CTAs)
        const int e = warp - 2;
        const int quad = warp & 3;
        const int half = e >> 2;
        const uint32_t lane_addr = uint32_t(quad * 32) << 16;
        const uint32_t te = mapa_shared(&tempty[0], 0);   // CTA 0's tempty[0]; [1] is 8 bytes on
        int gc = 0;
        bool ok = true;
        volatile int* abort_flag = half_abort + half;
        for (int lt = 0; lt < my_tiles; ++lt) {
            int ta = 0, tb = 0;
            tile_of(cl + lt * ncl, p.T, ta, tb);
            const int a0 = ta * BNP + int(rank) * BMH;
            const int b0 = tb * BNP;
            float acc[128];
#pragma unroll
            for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            for (int c = 0; c < nchunks; ++c, ++gc) {
                const int buf = gc & 1;
                const int use = gc >> 1;
                if (!mbar_wait(&tfull[buf], uint32_t(use) & 1u, st, 113)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float v[32];
                    tmem_ld_32x32b_x32(tmem_base + lane_addr + uint32_t(buf * BNP + half * 128 + cc * 32), v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[cc * 32 + i] += v[i];
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(te + uint32_t(buf) * 8u);
            }
            // 2 * sum into H: the half's four warps stage 32 columns of their 128
            // rows at a time in shared memory (128-byte swizzle) and one thread
            // adds them into H with a TMA reduce-add, which the L2 applies as one
            // rounded fp32 addition per element (the same result as h + 2 sum
            // in the SM), without the SM waiting for H's old values.
            // the half's four warps decide together (a named barrier has no time
            // limit, so none may skip the ones below alone)
            if (!ok) *abort_flag = 1;
            named_barrier_sync(1 + half, 32 * EPI_WARPS / 2);
            if (*abort_flag) break;
            if (p.late_wait) pdl_wait();           // the previous batch's H is complete
            if (nchunks > 0) {
                const int row = quad * 32 + lane;  // TMEM lane == row of this CTA's 128
                uint8_t* buf = flush_buf + size_t(half) * FLUSH_BYTES;
                const bool issuer = (quad == 0 && lane == 0);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    if (issuer) bulk_wait_group_read<0>();   // the last reduce from this slab has read it
                    named_barrier_sync(1 + half, 32 * EPI_WARPS / 2);
                    uint8_t* rowp = buf + size_t(row) * (FLUSH_COLS * 4);
#pragma unroll
                    for (int q = 0; q < FLUSH_COLS / 4; ++q)
                        *reinterpret_cast<float4*>(rowp + ((q ^ (row & 7)) << 4)) =
                            make_float4(p.alpha * acc[cc * 32 + 4 * q], p.alpha * acc[cc * 32 + 4 * q + 1],
                                        p.alpha * acc[cc * 32 + 4 * q + 2], p.alpha * acc[cc * 32 + 4 * q + 3]);
                    fence_proxy_async_smem();
                    named_barrier_sync(1 + half, 32 * EPI_WARPS / 2);
                    if (issuer) {
                        tma_reduce_add_2d(&tmH, buf, b0 + half * 128 + cc * FLUSH_COLS, a0);
                        bulk_commit_group();
                    }
                }
            }
        }
        if (quad == 0 && lane == 0) bulk_wait_group<0>();   // every reduce has reached H
    }
    tc_fence_before();
    cluster_sync();          // no remote arrival or pair MMA is still pending
    if (warp == 0) tmem_dealloc_pair(tmem_base, TMEM_COLS);
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
                   DevStatus* st, PFN_encodeTiled encode, bool after_own_launch) {
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
    p.late_wait = (after_own_launch && dtype != GPTQ_F32) ? 1 : 0;
    {
        static std::atomic<int> sms[64];
        int dv = 0;
        if (cudaGetDevice(&dv) != cudaSuccess) return GPTQ_ERR_CUDA;
        if (dv < 64 && sms[dv].load() == 0) {
            int n = 0;
            if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dv) != cudaSuccess) return GPTQ_ERR_CUDA;
            sms[dv] = n;
        }
        p.wave = std::max(1, (dv < 64 ? sms[dv].load() : 148) / 2);
    }
    p.T = int((d + BNP - 1) / BNP);
    p.tiles = p.T * (p.T + 1) / 2;
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(syrk_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES)) !=
            cudaSuccess)
            return GPTQ_ERR_CUDA;
        attr_set[dev] = true;
    }
    const int clusters = std::max(1, std::min(p.tiles, p.wave));
    CUtensorMap tmH;   // H as fp32 [d, d], boxes of 32 columns x 128 rows, 128-byte swizzle
    {
        const cuuint64_t hd[2] = {cuuint64_t(d), cuuint64_t(d)};
        const cuuint64_t hs[1] = {cuuint64_t(d) * 4};
        const cuuint32_t hb[2] = {FLUSH_COLS, BMH};
        const cuuint32_t he[2] = {1, 1};
        if (encode(&tmH, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, H, hd, hs, hb, he, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GPTQ_ERR_CUDA;
    }
    if (launch_pdl(syrk_pair_kernel, dim3(2 * clusters), dim3(THREADS), SMEM_BYTES, stream, tm, tmH, p, st) !=
        cudaSuccess)
        return GPTQ_ERR_CUDA;
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
