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
// Tile 128 x 128 per CTA, K <= 128 in chunks of 32 (one 128-byte swizzle row
// of fp32), all chunks loaded at once so that the tile's latency is one load,
// not four.  Both operands are K-major: A[m * lda + k] and B(k, n) = Bt[n * ldb + k]
// (an MN-major tf32 operand would need a different shared-memory layout, so
// the callers arrange their data to avoid it).  Chunks travel by TMA (no
// multicast), eight warps split each into hi (in place) / lo (two rotating
// buffers), one thread issues the MMAs, and four warps drain TMEM into C.
// K must be a multiple of 32 and at most 128.
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace tg {

constexpr int BM = 128, BN = 128, BKC = 32;       // tile, K chunk (fp32 elements)
constexpr int MAX_CHUNKS = 4;                      // K <= 128: every chunk resident at once
constexpr int LO_BUFS = 2;                         // lo parts, double-buffered
constexpr int A_BYTES = BM * BKC * 4;              // 16 KB
constexpr int B_BYTES = BN * BKC * 4;              // 16 KB
constexpr int CHUNK_BYTES = A_BYTES + B_BYTES;     // fp32 chunk (becomes the hi part in place)
constexpr int CONV_WARPS = 8;                      // split hi/lo; warp 0 lane 0 issues MMAs; warps 0-3 drain TMEM
constexpr int PRODUCER_WARP = CONV_WARPS;          // TMA only
constexpr int THREADS = 32 * (CONV_WARPS + 1);
constexpr int TMEM_COLS = 128;
constexpr size_t SMEM_BYTES = 1024 + size_t(MAX_CHUNKS + LO_BUFS) * CHUNK_BYTES + 256;

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
    DevStatus* st;
};

__global__ void __launch_bounds__(THREADS, 1)
    tgemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const Args g) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* lo_base = smem + size_t(MAX_CHUNKS) * CHUNK_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(lo_base + size_t(LO_BUFS) * CHUNK_BYTES);  // [MAX_CHUNKS]
    uint64_t* conv = full + MAX_CHUNKS;      // [MAX_CHUNKS] 8 warp arrivals: chunk split into hi / lo
    uint64_t* lo_free = conv + MAX_CHUNKS;   // [LO_BUFS] MMA commit: lo buffer may be reused
    uint64_t* accum = lo_free + LO_BUFS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);

    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    if (g.lower_only && n0 > m0 + BM - 1) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        for (int c = 0; c < MAX_CHUNKS; ++c) {
            mbar_init(&full[c], 1);
            mbar_init(&conv[c], CONV_WARPS);
        }
        for (int b = 0; b < LO_BUFS; ++b) mbar_init(&lo_free[b], 1);
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
    const int nk = g.K / BKC;

    if (warp == PRODUCER_WARP) {
        if (lane == 0) {
            for (int c = 0; c < nk; ++c) {
                uint8_t* base = smem + size_t(c) * CHUNK_BYTES;
                mbar_arrive_expect_tx(&full[c], CHUNK_BYTES);
                tma_load_2d(base, &tmA, c * BKC, m0, &full[c]);              // A:   {32 k, 128 rows}
                tma_load_2d(base + A_BYTES, &tmB, c * BKC, n0, &full[c]);    // B^T: {32 k, 128 rows}
            }
            // every wait below is bounded; the copies are all waited for by the
            // converters before the CTA can reach its end
        }
    } else {
        // epilogue warps: fetch this thread's row of C_in now, so that its
        // latency overlaps the loads, the split and the MMAs
        const int m = m0 + (warp & 3) * 32 + lane;
        const bool pre = warp < 4 && g.beta != 0.0f && m < g.M && n0 + BN <= g.N;
        float4 cpre[BN / 4];
        if (pre) {
            const float4* src = reinterpret_cast<const float4*>(g.C_in + size_t(m) * g.ldc + n0);
#pragma unroll
            for (int q = 0; q < BN / 4; ++q) cpre[q] = src[q];
        }
        // ---------------- split each chunk into hi / lo; warp 0 lane 0 issues the MMAs
        constexpr uint32_t idesc = idesc_tf32();
        const int ct = threadIdx.x;   // 0 .. 32*CONV_WARPS-1
        bool ok = true;
        for (int c = 0; c < nk; ++c) {
            uint8_t* base = smem + size_t(c) * CHUNK_BYTES;
            uint8_t* lo = lo_base + size_t(c % LO_BUFS) * CHUNK_BYTES;
            const bool landed = mbar_wait(&full[c], 0, g.st, 303);
            ok = ok && landed;
            if (c >= LO_BUFS) ok = ok && mbar_wait(&lo_free[c % LO_BUFS], uint32_t(c / LO_BUFS - 1) & 1u, g.st, 306);
            if (ok) {
                float4* x = reinterpret_cast<float4*>(base);
                float4* l = reinterpret_cast<float4*>(lo);
                for (int i = ct; i < CHUNK_BYTES / 16; i += 32 * CONV_WARPS) {
                    float4 v = x[i], h, q;
                    split_tf32(v.x, h.x, q.x); split_tf32(v.y, h.y, q.y);
                    split_tf32(v.z, h.z, q.z); split_tf32(v.w, h.w, q.w);
                    x[i] = h; l[i] = q;
                }
            }
            fence_proxy_async_smem();      // generic-proxy writes -> visible to tcgen05 reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&conv[c]);
            if (warp == 0 && lane == 0) {
                const bool ready = ok && mbar_wait(&conv[c], 0, g.st, 304);
                if (ready) {
                    tc_fence_after();
                    const uint32_t a_hi = smem_u32(base), b_hi = a_hi + A_BYTES;
                    const uint32_t a_lo = smem_u32(lo), b_lo = a_lo + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BKC / 8; ++kk) {
                        // K-major: 8 k (32 bytes) per MMA inside the 128-byte swizzled
                        // rows; groups of 8 rows 1024 bytes apart
                        const uint64_t dah = sdesc_sw128(a_hi + kk * 32, 16, 1024);
                        const uint64_t dal = sdesc_sw128(a_lo + kk * 32, 16, 1024);
                        const uint64_t dbh = sdesc_sw128(b_hi + kk * 32, 16, 1024);
                        const uint64_t dbl = sdesc_sw128(b_lo + kk * 32, 16, 1024);
                        umma_tf32(tmem_base, dah, dbl, idesc, (c > 0 || kk > 0) ? 1u : 0u);   // small terms first
                        umma_tf32(tmem_base, dal, dbh, idesc, 1u);
                        umma_tf32(tmem_base, dah, dbh, idesc, 1u);
                    }
                }
                ok = ready;
                umma_commit(&lo_free[c % LO_BUFS]);   // this chunk's lo buffer is free once these MMAs finish
            }
            __syncwarp();
        }
        if (warp == 0 && lane == 0) umma_commit(accum);

        // ---------------- epilogue: warps 0..3 own TMEM lanes 32w..32w+31 (= tile rows)
        if (warp < 4) {
            __syncwarp();
            const bool ready = mbar_wait(accum, 0, g.st, 305);
            tc_fence_after();
            if (ready && nk > 0) {
#pragma unroll
                for (int cc = 0; cc < BN / 32; ++cc) {
                    float v[32];
                    tmem_ld_32x32b_x32(tmem_base + (uint32_t(warp * 32) << 16) + uint32_t(cc * 32), v);
                    const int n = n0 + cc * 32;
                    if (m >= g.M) continue;
                    float* cout = g.C_out + size_t(m) * g.ldc + n;
                    if (pre) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 ci = cpre[cc * 8 + q];
                            *reinterpret_cast<float4*>(cout + 4 * q) =
                                make_float4(fmaf(g.alpha, v[4 * q], g.beta * ci.x), fmaf(g.alpha, v[4 * q + 1], g.beta * ci.y),
                                            fmaf(g.alpha, v[4 * q + 2], g.beta * ci.z), fmaf(g.alpha, v[4 * q + 3], g.beta * ci.w));
                        }
                    } else if (n + 32 <= g.N) {
                        const float* cin = g.C_in + size_t(m) * g.ldc + n;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float4 r;
                            if (g.beta != 0.0f) {
                                const float4 ci = *reinterpret_cast<const float4*>(cin + 4 * q);
                                r = make_float4(fmaf(g.alpha, v[4 * q], g.beta * ci.x),
                                                fmaf(g.alpha, v[4 * q + 1], g.beta * ci.y),
                                                fmaf(g.alpha, v[4 * q + 2], g.beta * ci.z),
                                                fmaf(g.alpha, v[4 * q + 3], g.beta * ci.w));
                            } else {
                                r = make_float4(g.alpha * v[4 * q], g.alpha * v[4 * q + 1], g.alpha * v[4 * q + 2],
                                                g.alpha * v[4 * q + 3]);
                            }
                            *reinterpret_cast<float4*>(cout + 4 * q) = r;
                        }
                    } else {
                        const float* cin = g.C_in + size_t(m) * g.ldc + n;
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            if (n + q < g.N) cout[q] = fmaf(g.alpha, v[q], g.beta != 0.0f ? g.beta * cin[q] : 0.0f);
                    }
                }
            }
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
    if (!trans_b || K <= 0 || K % BKC != 0 || K > BKC * MAX_CHUNKS || g_enc == nullptr) return GPTQ_ERR_UNSUPPORTED;
    CUtensorMap ta, tb;
    int rc = make_map_2d_f32(&ta, A, uint64_t(K), uint64_t(M), uint64_t(lda), BKC, BM, true);
    if (rc) return rc;
    rc = make_map_2d_f32(&tb, B, uint64_t(K), uint64_t(N), uint64_t(ldb), BKC, BN, true);
    if (rc) return rc;
    Args g{M, N, K, alpha, beta, C_in, C_out, ldc, lower_only ? 1 : 0, st};
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(tgemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_BYTES)) !=
            cudaSuccess)
            return GPTQ_ERR_CUDA;
        attr_set[dev] = true;
    }
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
    tgemm_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(ta, tb, g);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
