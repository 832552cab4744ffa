// fp32-accurate GEMM on the tcgen05 tensor cores (kind::tf32, three passes).
//
// C[M,N] = beta * C_in + alpha * A[M,K] * op(B)[K,N]   (row-major, fp32)
//
// Every product in the factorization and in the sweep's lazy trailing update
// ([wiki] "알고리즘": W[:, i+B:] -= E U[i:i+B, i+B:]) needs about fp32
// accuracy: a single bf16 or tf32 product changes GPTQ codes.  Each operand x
// is split in shared memory into hi = x rounded to tf32 and lo = x - hi
// (exact in fp32; the MMA reads its leading 19 bits), and the product is
// accumulated as  A_hi B_hi + A_hi B_lo + A_lo B_hi  in fp32 TMEM, which is
// accurate to about 2^-21 relative (the dropped A_lo B_lo term and the tf32
// reading of the lo parts), comparable to an fp32 FMA chain of length K.
//
// Persistent kernel: one CTA per SM walks its share of the 128 x 128 output
// tiles; K <= 128 in chunks of 32 (one 128-byte swizzle row of fp32) flows
// through a 4-stage ring, and two TMEM accumulators let tile i+1's loads, split
// and MMAs run while tile i's epilogue drains.  Both operands are K-major: A[m * lda + k] and B(k, n) = Bt[n * ldb + k]
// (an MN-major tf32 operand would need a different shared-memory layout, so
// the callers arrange their data to avoid it).  Warp roles: one TMA producer
// (no multicast), six warps that split each chunk into hi (in place) / lo
// (two rotating buffers), one MMA issuer, four epilogue warps.  K must be a
// multiple of 32 and at most 128.
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace tg {

constexpr int BM = 128, BN = 128, BKC = 32;       // tile, K chunk (fp32 elements)
constexpr int MAX_K = 128;                         // K <= 128 (every caller uses 128)
constexpr int STAGES = 4;                          // ring of fp32 chunks (each becomes its hi part in place)
constexpr int LO_BUFS = 2;                         // lo parts, rotating
constexpr int A_BYTES = BM * BKC * 4;              // 16 KB
constexpr int B_BYTES = BN * BKC * 4;              // 16 KB
constexpr int CHUNK_BYTES = A_BYTES + B_BYTES;
constexpr int CONV_WARPS = 6;                      // warps 0-5 split chunks into hi / lo
constexpr int MMA_WARP = CONV_WARPS;               // warp 6 issues the MMAs
constexpr int PRODUCER_WARP = CONV_WARPS + 1;      // warp 7 issues TMA
constexpr int EPI_WARP0 = 8;                       // warps 8-15 drain TMEM: lane quadrant warp % 4,
constexpr int EPI_WARPS = 8;                       // column half (warp - 8) / 4
constexpr int THREADS = 32 * (EPI_WARP0 + EPI_WARPS);
constexpr int TMEM_COLS = 2 * BN;                  // two accumulators: tile i+1 runs while tile i drains
constexpr size_t SMEM_BYTES = 1024 + size_t(STAGES + LO_BUFS) * CHUNK_BYTES + 512;

// instruction descriptor: tf32 x tf32 -> f32, A and B K-major, M = BM, N = BN
__host__ __device__ constexpr uint32_t idesc_tf32() {
    return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
           (static_cast<uint32_t>(BM >> 4) << 24);
}

__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// x -> (hi, lo): hi = x rounded to the nearest tf32 value (ties away), lo = x - hi.
__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
    const uint32_t u = __float_as_uint(x);
    const uint32_t h = (u + 0x1000u) & 0xFFFFE000u;
    hi = isfinite(x) ? __uint_as_float(h) : x;
    lo = isfinite(x) ? x - hi : 0.0f;
}

struct Args {
    int M, N, K;
    float alpha, beta;
    const float* C_in;
    float* C_out;
    int ldc;
    int lower_only;
    int tiles_m, tiles_n, tiles;
    DevStatus* st;
};

// Tile t (row-major over (tm, tn); with lower_only only tn <= tm).
__device__ __forceinline__ void tile_coords(int t, const Args& g, int& tm, int& tn) {
    if (!g.lower_only) {
        tm = t / g.tiles_n;
        tn = t % g.tiles_n;
        return;
    }
    int acc = 0;
    for (tm = 0; tm < g.tiles_m; ++tm) {
        const int cnt = min(g.tiles_n, tm + 1);
        if (t < acc + cnt) {
            tn = t - acc;
            return;
        }
        acc += cnt;
    }
    tn = 0;
}

__global__ void __launch_bounds__(THREADS, 1)
    tgemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const Args g) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* lo_base = smem + size_t(STAGES) * CHUNK_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(lo_base + size_t(LO_BUFS) * CHUNK_BYTES);  // [STAGES] TMA landed
    uint64_t* conv = full + STAGES;          // [STAGES] one arrival per split warp: chunk split into hi / lo
    uint64_t* empty = conv + STAGES;         // [STAGES] MMA commit: stage may be reloaded
    uint64_t* lo_free = empty + STAGES;      // [LO_BUFS] MMA commit: lo buffer may be rewritten
    uint64_t* tfull = lo_free + LO_BUFS;     // [2] MMA commit: accumulator complete
    uint64_t* tempty = tfull + 2;            // [2] epilogue arrivals: accumulator drained
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = g.K / BKC;
    const int my_tiles = g.tiles > int(blockIdx.x) ? (g.tiles - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x) : 0;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], CONV_WARPS);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < LO_BUFS; ++b) mbar_init(&lo_free[b], 1);
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

    if (warp == PRODUCER_WARP) {
        if (lane == 0) {
            int gc = 0;
            bool ok = true;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                int tm, tn;
                tile_coords(int(blockIdx.x) + lt * int(gridDim.x), g, tm, tn);
                for (int c = 0; c < nk; ++c, ++gc) {
                    const int s = gc % STAGES;
                    const uint32_t round = uint32_t(gc / STAGES);
                    if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, g.st, 301)) { ok = false; break; }
                    uint8_t* base = smem + size_t(s) * CHUNK_BYTES;
                    mbar_arrive_expect_tx(&full[s], CHUNK_BYTES);
                    tma_load_2d(base, &tmA, c * BKC, tm * BM, &full[s]);             // A:   {32 k, 128 rows}
                    tma_load_2d(base + A_BYTES, &tmB, c * BKC, tn * BN, &full[s]);   // B^T: {32 k, 128 rows}
                }
            }
        }
    } else if (warp < CONV_WARPS) {
        // ---------------- split chunks into hi (in place) / lo
        const int ct = threadIdx.x;   // 0 .. 32*CONV_WARPS-1
        const int total = my_tiles * nk;
        for (int gc = 0; gc < total; ++gc) {
            const int s = gc % STAGES, l = gc % LO_BUFS;
            const uint32_t round = uint32_t(gc / STAGES), lround = uint32_t(gc / LO_BUFS);
            if (!mbar_wait(&full[s], round & 1u, g.st, 303)) break;
            if (!mbar_wait(&lo_free[l], (lround & 1u) ^ 1u, g.st, 306)) break;
            float4* x = reinterpret_cast<float4*>(smem + size_t(s) * CHUNK_BYTES);
            float4* lo = reinterpret_cast<float4*>(lo_base + size_t(l) * CHUNK_BYTES);
#pragma unroll 4
            for (int i = ct; i < CHUNK_BYTES / 16; i += 32 * CONV_WARPS) {
                float4 v = x[i], h, q;
                split_tf32(v.x, h.x, q.x); split_tf32(v.y, h.y, q.y);
                split_tf32(v.z, h.z, q.z); split_tf32(v.w, h.w, q.w);
                x[i] = h; lo[i] = q;
            }
            fence_proxy_async_smem();      // generic-proxy writes -> visible to tcgen05 reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&conv[s]);
        }
    } else if (warp == MMA_WARP) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_tf32();
            int gc = 0;
            bool ok = true;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                const int acc = lt & 1;
                const uint32_t use = uint32_t(lt >> 1);
                if (!mbar_wait(&tempty[acc], (use & 1u) ^ 1u, g.st, 307)) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + uint32_t(acc * BN);
                for (int c = 0; c < nk; ++c, ++gc) {
                    const int s = gc % STAGES, l = gc % LO_BUFS;
                    const uint32_t round = uint32_t(gc / STAGES);
                    if (!mbar_wait(&conv[s], round & 1u, g.st, 304)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_hi = smem_u32(smem + size_t(s) * CHUNK_BYTES), b_hi = a_hi + A_BYTES;
                    const uint32_t a_lo = smem_u32(lo_base + size_t(l) * CHUNK_BYTES), b_lo = a_lo + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BKC / 8; ++kk) {
                        // K-major: 8 k (32 bytes) per MMA inside the 128-byte swizzled
                        // rows; groups of 8 rows 1024 bytes apart
                        const uint64_t dah = sdesc_sw128(a_hi + kk * 32, 16, 1024);
                        const uint64_t dal = sdesc_sw128(a_lo + kk * 32, 16, 1024);
                        const uint64_t dbh = sdesc_sw128(b_hi + kk * 32, 16, 1024);
                        const uint64_t dbl = sdesc_sw128(b_lo + kk * 32, 16, 1024);
                        umma_tf32(dt, dah, dbl, idesc, (c > 0 || kk > 0) ? 1u : 0u);   // small terms first
                        umma_tf32(dt, dal, dbh, idesc, 1u);
                        umma_tf32(dt, dah, dbh, idesc, 1u);
                    }
                    umma_commit(&empty[s]);      // stage may be reloaded once these MMAs finish
                    umma_commit(&lo_free[l]);    // and its lo buffer rewritten
                }
                umma_commit(&tfull[acc]);        // tile complete (also on the error path)
            }
        }
    } else {
        // ---------------- epilogue warps: TMEM lanes (warp % 4) * 32 .. + 31 = tile rows,
        // columns half * 64 .. + 63
        const int quad = warp & 3;
        const int half = (warp - EPI_WARP0) >> 2;
        constexpr int HC = BN / 2;   // columns per epilogue thread
        for (int lt = 0; lt < my_tiles; ++lt) {
            const int acc = lt & 1;
            const uint32_t use = uint32_t(lt >> 1);
            int tm, tn;
            tile_coords(int(blockIdx.x) + lt * int(gridDim.x), g, tm, tn);
            const int m = tm * BM + quad * 32 + lane;
            const int n0 = tn * BN + half * HC;
            const bool in_range = m < g.M;
            const bool full_row = in_range && n0 + HC <= g.N;
            // C_in for this tile now, so that the loads overlap the tile's MMAs
            float4 ci[HC / 4];
            if (full_row && g.beta != 0.0f) {
                const float4* src = reinterpret_cast<const float4*>(g.C_in + size_t(m) * g.ldc + n0);
#pragma unroll
                for (int q = 0; q < HC / 4; ++q) ci[q] = src[q];
            } else {
#pragma unroll
                for (int q = 0; q < HC / 4; ++q) ci[q] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            }
            __syncwarp();
            if (!mbar_wait(&tfull[acc], use & 1u, g.st, 305)) break;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < HC / 32; ++cc) {
                const int n = n0 + cc * 32;
                float v[32];
                tmem_ld_32x32b_x32(tmem_base + (uint32_t(quad * 32) << 16) + uint32_t(acc * BN + half * HC + cc * 32), v);
                if (!in_range) continue;
                float* cout = g.C_out + size_t(m) * g.ldc + n;
                if (full_row) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 c4 = ci[cc * 8 + q];
                        *reinterpret_cast<float4*>(cout + 4 * q) =
                            make_float4(fmaf(g.alpha, v[4 * q], g.beta * c4.x), fmaf(g.alpha, v[4 * q + 1], g.beta * c4.y),
                                        fmaf(g.alpha, v[4 * q + 2], g.beta * c4.z), fmaf(g.alpha, v[4 * q + 3], g.beta * c4.w));
                    }
                } else {
                    const float* cin = g.C_in + size_t(m) * g.ldc + n;
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        if (n + q < g.N) cout[q] = fmaf(g.alpha, v[q], g.beta != 0.0f ? g.beta * cin[q] : 0.0f);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace tg

namespace {
PFN_encodeTiled g_enc = nullptr;
}

void set_tensor_map_encoder(PFN_encodeTiled f) { g_enc = f; }

int make_map_2d_f32(CUtensorMap* tm, const float* base, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                    uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
    if (g_enc == nullptr) return GPTQ_ERR_CUDA;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {ld_elems * 4};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box,
                             estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                             swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GPTQ_OK : GPTQ_ERR_CUDA;
}

int launch_tgemm(int M, int N, int K, float alpha, const float* A, int lda, const float* B, int ldb, bool trans_b,
                 float beta, const float* C_in, float* C_out, int ldc, bool lower_only, cudaStream_t stream,
                 DevStatus* st) {
    using namespace tg;
    if (M <= 0 || N <= 0) return GPTQ_OK;
    if (!trans_b || K <= 0 || K % BKC != 0 || K > MAX_K || g_enc == nullptr) return GPTQ_ERR_UNSUPPORTED;
    CUtensorMap ta, tb;
    int rc = make_map_2d_f32(&ta, A, uint64_t(K), uint64_t(M), uint64_t(lda), BKC, BM, true);
    if (rc) return rc;
    rc = make_map_2d_f32(&tb, B, uint64_t(K), uint64_t(N), uint64_t(ldb), BKC, BN, true);
    if (rc) return rc;
    Args g{};
    g.M = M; g.N = N; g.K = K; g.alpha = alpha; g.beta = beta; g.C_in = C_in; g.C_out = C_out; g.ldc = ldc;
    g.lower_only = lower_only ? 1 : 0;
    g.tiles_m = (M + BM - 1) / BM;
    g.tiles_n = (N + BN - 1) / BN;
    if (lower_only) {
        g.tiles = 0;
        for (int tm = 0; tm < g.tiles_m; ++tm) g.tiles += std::min(g.tiles_n, tm + 1);
    } else {
        g.tiles = g.tiles_m * g.tiles_n;
    }
    g.st = st;
    static bool attr_set[64] = {};
    static int sms[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(tgemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES)) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        attr_set[dev] = true;
    }
    const int grid = std::max(1, std::min(g.tiles, dev < 64 && sms[dev] > 0 ? sms[dev] : 148));
    tgemm_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(ta, tb, g);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
