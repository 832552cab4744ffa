// fp32-accurate GEMM on the tcgen05 tensor cores (kind::tf32, three passes).
//
// C[M,N] = alpha * A[M,K] * op(B)[K,N]        (accumulate = false)
// C[M,N] += alpha * A[M,K] * op(B)[K,N]       (accumulate = true)
// row-major fp32, op(B)(k, n) = Bt[n * ldb + k].
//
// Every product in the factorization and in the sweep's lazy trailing update
// ([wiki] "알고리즘": W[:, i+B:] -= E U[i:i+B, i+B:]) needs about fp32
// accuracy: a single bf16 or tf32 product changes GPTQ codes.  Each operand x
// is split into hi = x rounded to tf32 and lo = x - hi (exact in fp32; the MMA
// reads its leading 19 bits), and the product is accumulated as
// A_hi B_hi + A_hi B_lo + A_lo B_hi  in fp32 TMEM, which is accurate to about
// 2^-21 relative (the dropped A_lo B_lo term and the tf32 reading of the lo
// parts), comparable to an fp32 FMA chain of length K.
//
// Two ways to get the split:
//  - pre-split: the caller stores hi and lo in global memory (the sweep writes
//    E that way and transposes U that way); TMA brings all four operand parts
//    and no thread touches them, which keeps shared memory free for the MMAs
//    (at M = N = 128 the tf32 MMAs alone need most of its bandwidth);
//  - in-kernel: six warps split each TMA-loaded chunk into hi (in place) and lo
//    (two rotating buffers), for operands that other kernels produce as plain
//    fp32 (the factorization).
//
// Persistent kernel: one CTA per SM walks its share of the 128 x 128 output
// tiles; K in chunks of 32 (one 128-byte swizzle row of fp32) flows through a
// ring of stages, and two TMEM accumulators let tile i+1's loads and MMAs run
// while tile i's epilogue drains.  Both operands are K-major (an MN-major tf32
// operand would need a different shared-memory layout, so the callers arrange
// their data to avoid it).  The epilogue moves the accumulator to shared memory
// 32 columns at a time (128-byte swizzle, conflict-free) and writes it with one
// TMA store, or one TMA reduce-add when accumulating, so C leaves the SM as
// whole lines and is never read by the SM.  No TMA load uses multicast.
#include <atomic>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace tg {

constexpr int BM = 128, BN = 128, BKC = 32;        // tile, K chunk (fp32 elements)
constexpr int MAX_K = 8192;
constexpr int PART_BYTES = BM * BKC * 4;           // one 128 x 32 fp32 operand part: 16 KB
constexpr int EPI_WARPS = 4;                       // one per TMEM lane quadrant
constexpr int SLAB = 32;                           // epilogue columns per TMA store
constexpr int SLAB_BYTES = BM * SLAB * 4;          // 16 KB
constexpr int SLAB_BUFS = 2;
constexpr int TMEM_COLS = 2 * BN;                  // two accumulators: tile i+1 runs while tile i drains
constexpr int EPI_BARRIER = 1;                     // named barrier of the epilogue warps

// Shared-memory and warp layout of the two variants.
template <bool PRESPLIT>
struct Cfg {
    // pre-split: a stage holds A_hi, B_hi, A_lo, B_lo of one chunk.
    // in-kernel: a stage holds A, B (split to hi in place); lo goes to LO_BUFS buffers.
    static constexpr int STAGE_BYTES = PRESPLIT ? 4 * PART_BYTES : 2 * PART_BYTES;
    static constexpr int STAGES = PRESPLIT ? 3 : 4;
    static constexpr int LO_BUFS = PRESPLIT ? 0 : 2;
    static constexpr int CONV_WARPS = PRESPLIT ? 0 : 6;
    static constexpr int MMA_WARP = CONV_WARPS;
    static constexpr int PRODUCER_WARP = CONV_WARPS + 1;
    static constexpr int EPI_WARP0 = PRESPLIT ? 4 : 8;   // multiple of 4: warp % 4 = TMEM lane quadrant
    static constexpr int THREADS = 32 * (EPI_WARP0 + EPI_WARPS);
    static constexpr size_t SMEM_BYTES =
        1024 + size_t(STAGES) * STAGE_BYTES + size_t(LO_BUFS) * 2 * PART_BYTES + size_t(SLAB_BUFS) * SLAB_BYTES + 256;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

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

struct Args {
    int M, N, K;
    float alpha;
    int accumulate;
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

// The operand tensor maps: A_hi, B_hi, A_lo, B_lo (pre-split) or A, B.
struct Maps {
    CUtensorMap a, b, a_lo, b_lo, c;
};

template <bool PRESPLIT>
__global__ void __launch_bounds__(Cfg<PRESPLIT>::THREADS, 1)
    tgemm_kernel(const __grid_constant__ Maps maps, const Args g) {
    using C = Cfg<PRESPLIT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* lo_base = smem + size_t(C::STAGES) * C::STAGE_BYTES;
    uint8_t* cbuf = lo_base + size_t(C::LO_BUFS) * 2 * PART_BYTES;                 // [SLAB_BUFS][128 rows][128 B]
    uint64_t* full = reinterpret_cast<uint64_t*>(cbuf + size_t(SLAB_BUFS) * SLAB_BYTES);  // [STAGES] TMA landed
    uint64_t* conv = full + C::STAGES;       // [STAGES] one arrival per split warp (in-kernel split)
    uint64_t* empty = conv + C::STAGES;      // [STAGES] MMA commit: stage may be reloaded
    uint64_t* lo_free = empty + C::STAGES;   // [2] MMA commit: lo buffer may be rewritten (in-kernel split)
    uint64_t* tfull = lo_free + 2;           // [2] MMA commit: accumulator complete
    uint64_t* tempty = tfull + 2;            // [2] epilogue arrivals: accumulator drained
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    int* epi_abort = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = g.K / BKC;
    const int my_tiles = g.tiles > int(blockIdx.x) ? (g.tiles - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x) : 0;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&maps.a);
        tma_prefetch_desc(&maps.b);
        tma_prefetch_desc(&maps.c);
        if (PRESPLIT) {
            tma_prefetch_desc(&maps.a_lo);
            tma_prefetch_desc(&maps.b_lo);
        }
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], C::CONV_WARPS > 0 ? C::CONV_WARPS : 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&lo_free[b], 1);
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], EPI_WARPS);
        }
        *epi_abort = 0;
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
    pdl_wait();       // the previous kernel's output (our operands, C) is complete
    pdl_trigger();

    if (warp == C::PRODUCER_WARP) {
        if (lane == 0) {
            int gc = 0;
            bool ok = true;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                int tm, tn;
                tile_coords(int(blockIdx.x) + lt * int(gridDim.x), g, tm, tn);
                for (int c = 0; c < nk; ++c, ++gc) {
                    const int s = gc % C::STAGES;
                    const uint32_t round = uint32_t(gc / C::STAGES);
                    if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, g.st, 301)) { ok = false; break; }
                    uint8_t* base = smem + size_t(s) * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
                    tma_load_2d(base, &maps.a, c * BKC, tm * BM, &full[s]);                  // {32 k, 128 rows}
                    tma_load_2d(base + PART_BYTES, &maps.b, c * BKC, tn * BN, &full[s]);
                    if (PRESPLIT) {
                        tma_load_2d(base + 2 * PART_BYTES, &maps.a_lo, c * BKC, tm * BM, &full[s]);
                        tma_load_2d(base + 3 * PART_BYTES, &maps.b_lo, c * BKC, tn * BN, &full[s]);
                    }
                }
            }
        }
    } else if (warp < C::CONV_WARPS) {
        // ---------------- in-kernel split: chunk -> hi (in place) / lo
        const int ct = threadIdx.x;   // 0 .. 32*CONV_WARPS-1
        const int total = my_tiles * nk;
        for (int gc = 0; gc < total; ++gc) {
            constexpr int LB = C::LO_BUFS > 0 ? C::LO_BUFS : 1;   // (this branch runs only when LO_BUFS > 0)
            const int s = gc % C::STAGES, l = gc % LB;
            const uint32_t round = uint32_t(gc / C::STAGES), lround = uint32_t(gc / LB);
            if (!mbar_wait(&full[s], round & 1u, g.st, 303)) break;
            if (!mbar_wait(&lo_free[l], (lround & 1u) ^ 1u, g.st, 306)) break;
            float4* x = reinterpret_cast<float4*>(smem + size_t(s) * C::STAGE_BYTES);
            float4* lo = reinterpret_cast<float4*>(lo_base + size_t(l) * 2 * PART_BYTES);
#pragma unroll 4
            for (int i = ct; i < 2 * PART_BYTES / 16; i += 32 * C::CONV_WARPS) {
                float4 v = x[i], h, q;
                split_tf32(v.x, h.x, q.x); split_tf32(v.y, h.y, q.y);
                split_tf32(v.z, h.z, q.z); split_tf32(v.w, h.w, q.w);
                x[i] = h; lo[i] = q;
            }
            fence_proxy_async_smem();      // generic-proxy writes -> visible to tcgen05 reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&conv[s]);
        }
    } else if (warp == C::MMA_WARP) {
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
                    const int s = gc % C::STAGES;
                    const int l = PRESPLIT ? 0 : gc % 2;
                    const uint32_t round = uint32_t(gc / C::STAGES);
                    if (!mbar_wait(PRESPLIT ? &full[s] : &conv[s], round & 1u, g.st, 304)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_hi = smem_u32(smem + size_t(s) * C::STAGE_BYTES), b_hi = a_hi + PART_BYTES;
                    const uint32_t a_lo = PRESPLIT ? a_hi + 2 * PART_BYTES
                                                   : smem_u32(lo_base + size_t(l) * 2 * PART_BYTES);
                    const uint32_t b_lo = a_lo + PART_BYTES;
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
                    umma_commit(&empty[s]);                  // stage may be reloaded once these MMAs finish
                    if (!PRESPLIT) umma_commit(&lo_free[l]); // and its lo buffer rewritten
                }
                umma_commit(&tfull[acc]);        // tile complete (also on the error path)
            }
        }
    } else if (warp >= C::EPI_WARP0) {
        // ---------------- epilogue: thread et owns tile row et (TMEM lane et)
        const int quad = warp - C::EPI_WARP0;
        const int et = threadIdx.x - 32 * C::EPI_WARP0;
        volatile int* abort_flag = epi_abort;
        int gs = 0;   // slabs issued so far (selects the staging buffer)
        for (int lt = 0; lt < my_tiles; ++lt) {
            const int acc = lt & 1;
            const uint32_t use = uint32_t(lt >> 1);
            int tm, tn;
            tile_coords(int(blockIdx.x) + lt * int(gridDim.x), g, tm, tn);
            if (!mbar_wait(&tfull[acc], use & 1u, g.st, 305)) *abort_flag = 1;
            named_barrier_sync(EPI_BARRIER, 32 * EPI_WARPS);   // all four warps leave together on a timeout
            if (*abort_flag) break;
            tc_fence_after();
#pragma unroll 1
            for (int j = 0; j < BN / SLAB; ++j, ++gs) {
                float v[32];
                tmem_ld_32x32b_x32(tmem_base + (uint32_t(quad * 32) << 16) + uint32_t(acc * BN + j * SLAB), v);
                if (j == BN / SLAB - 1) {   // accumulator drained: the MMAs of tile lt + 2 may start
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[acc]);
                }
                uint8_t* buf = cbuf + size_t(gs & 1) * SLAB_BYTES;
                if (et == 0) bulk_wait_group_read<1>();   // the store that last used this buffer has read it
                named_barrier_sync(EPI_BARRIER, 32 * EPI_WARPS);
                // row et, 16-byte chunk q at position q ^ (et % 8): TMA's 128-byte swizzle,
                // and eight consecutive rows cover all 32 banks
                uint8_t* row = buf + size_t(et) * (SLAB * 4);
#pragma unroll
                for (int q = 0; q < SLAB / 4; ++q)
                    *reinterpret_cast<float4*>(row + ((q ^ (et & 7)) << 4)) =
                        make_float4(g.alpha * v[4 * q], g.alpha * v[4 * q + 1], g.alpha * v[4 * q + 2],
                                    g.alpha * v[4 * q + 3]);
                fence_proxy_async_smem();
                named_barrier_sync(EPI_BARRIER, 32 * EPI_WARPS);
                if (et == 0) {
                    const int x = tn * BN + j * SLAB;
                    if (x < g.N) {
                        if (g.accumulate)
                            tma_reduce_add_2d(&maps.c, buf, x, tm * BM);
                        else
                            tma_store_2d(&maps.c, buf, x, tm * BM);
                    }
                    bulk_commit_group();
                }
            }
        }
        if (et == 0) bulk_wait_group<0>();   // every store has reached global memory
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base, TMEM_COLS);
}

// ---------------------------------------------------------------------------
// The same pre-split three-pass product on SM pairs, for long contractions
// (the far updates, K = 256 .. 8192).  A cluster of two CTAs owns a 256 x 256
// output tile and runs it as cta_group::2 MMAs (M = 256, N = 256, K = 8):
// CTA r loads rows 128 r .. 128 r + 127 of the tile's A rows and of its Bt
// rows (its half of N), all four operand parts per 32-wide K chunk (64 KB per
// stage, three stages); both CTAs' loads complete on CTA 0's barrier; CTA 0
// issues the MMAs, whose commits arrive on both CTAs' barriers; each CTA's
// TMEM holds its 128 rows x 256 columns (two accumulators, 512 columns).
// Per SM this streams half the operand bytes of a 128 x 128 tile for the
// same MMA work, which keeps shared memory below its bandwidth: the single-CTA
// kernel's three passes over 128 x 128 tiles read and write about 200 bytes
// of shared memory per clock at full tensor rate, against about 106 here.
// Persistent: cluster c walks tiles c, c + clusters, ...; no TMA load uses
// multicast.
constexpr int PBM = 256, PBN = 256;              // pair tile
constexpr int P_ROWS = 128;                      // A rows and Bt rows each CTA loads per chunk
constexpr int P_PART = P_ROWS * BKC * 4;         // 16 KB
constexpr int P_STAGE = 4 * P_PART;              // A_hi, B_hi, A_lo, B_lo
constexpr int P_STAGES = 3;
constexpr int P_EPI_WARP0 = 4;                   // warp % 4 = TMEM lane quadrant
constexpr int P_THREADS = 32 * (P_EPI_WARP0 + EPI_WARPS);
constexpr int P_TMEM_COLS = 2 * PBN;
constexpr size_t P_SMEM_BYTES = 1024 + size_t(P_STAGES) * P_STAGE + size_t(SLAB_BUFS) * SLAB_BYTES + 256;
static_assert(P_SMEM_BYTES <= 232448, "shared memory");

__host__ __device__ constexpr uint32_t idesc_tf32_pair() {
    return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(PBN >> 3) << 17) |
           (static_cast<uint32_t>(PBM >> 4) << 24);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_THREADS, 1)
    tgemm_pair_kernel(const __grid_constant__ Maps maps, const Args g) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* cbuf = smem + size_t(P_STAGES) * P_STAGE;                                   // [SLAB_BUFS][128 rows][128 B]
    uint64_t* full = reinterpret_cast<uint64_t*>(cbuf + size_t(SLAB_BUFS) * SLAB_BYTES);  // CTA 0: both halves landed
    uint64_t* empty = full + P_STAGES;   // both CTAs: the pair's MMAs are done with the stage
    uint64_t* tfull = empty + P_STAGES;  // [2] both CTAs: accumulator complete
    uint64_t* tempty = tfull + 2;        // [2] CTA 0: accumulator drained by both CTAs
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    int* epi_abort = reinterpret_cast<int*>(tmem_slot + 1);

    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cl = int(blockIdx.x >> 1), ncl = int(gridDim.x >> 1);
    const int nk = g.K / BKC;
    const int my_tiles = g.tiles > cl ? (g.tiles - cl + ncl - 1) / ncl : 0;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&maps.a);
        tma_prefetch_desc(&maps.b);
        tma_prefetch_desc(&maps.a_lo);
        tma_prefetch_desc(&maps.b_lo);
        tma_prefetch_desc(&maps.c);
        for (int s = 0; s < P_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * EPI_WARPS);
        }
        *epi_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(tmem_slot, P_TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();          // barriers of both CTAs initialized, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs)
            const uint32_t fb0 = mapa_shared(&full[0], 0);
            int gc = 0;
            bool ok = true;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                int tm, tn;
                tile_coords(cl + lt * ncl, g, tm, tn);
                const int ar = tm * PBM + int(rank) * P_ROWS, br = tn * PBN + int(rank) * P_ROWS;
                for (int c = 0; c < nk; ++c, ++gc) {
                    const int s = gc % P_STAGES;
                    const uint32_t round = uint32_t(gc / P_STAGES);
                    if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, g.st, 311)) { ok = false; break; }
                    uint8_t* base = smem + size_t(s) * P_STAGE;
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * P_STAGE);
                    const uint32_t fb = fb0 + uint32_t(s) * 8u;
                    tma_load_2d_pair(base, &maps.a, c * BKC, ar, fb);
                    tma_load_2d_pair(base + P_PART, &maps.b, c * BKC, br, fb);
                    tma_load_2d_pair(base + 2 * P_PART, &maps.a_lo, c * BKC, ar, fb);
                    tma_load_2d_pair(base + 3 * P_PART, &maps.b_lo, c * BKC, br, fb);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer (CTA 0)
            constexpr uint32_t idesc = idesc_tf32_pair();
            int gc = 0;
            bool ok = true;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                const int acc = lt & 1;
                const uint32_t use = uint32_t(lt >> 1);
                if (use > 0 && !mbar_wait_cluster(&tempty[acc], (use - 1) & 1u, g.st, 317)) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + uint32_t(acc * PBN);
                for (int c = 0; c < nk; ++c, ++gc) {
                    const int s = gc % P_STAGES;
                    const uint32_t round = uint32_t(gc / P_STAGES);
                    if (!mbar_wait(&full[s], round & 1u, g.st, 314)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_hi = smem_u32(smem + size_t(s) * P_STAGE), b_hi = a_hi + P_PART;
                    const uint32_t a_lo = a_hi + 2 * P_PART, b_lo = a_hi + 3 * P_PART;
#pragma unroll
                    for (int kk = 0; kk < BKC / 8; ++kk) {
                        const uint64_t dah = sdesc_sw128(a_hi + kk * 32, 16, 1024);
                        const uint64_t dal = sdesc_sw128(a_lo + kk * 32, 16, 1024);
                        const uint64_t dbh = sdesc_sw128(b_hi + kk * 32, 16, 1024);
                        const uint64_t dbl = sdesc_sw128(b_lo + kk * 32, 16, 1024);
                        umma_tf32_pair(dt, dah, dbl, idesc, (c > 0 || kk > 0) ? 1u : 0u);   // small terms first
                        umma_tf32_pair(dt, dal, dbh, idesc, 1u);
                        umma_tf32_pair(dt, dah, dbh, idesc, 1u);
                    }
                    umma_commit_pair_both(&empty[s]);      // the stage may be reloaded in both CTAs
                }
                umma_commit_pair_both(&tfull[acc]);        // tile complete (also on the error path)
            }
        }
    } else if (warp >= P_EPI_WARP0) {
        // ---------------- epilogue (both CTAs): thread et owns row et of this CTA's 128
        const int quad = warp - P_EPI_WARP0;
        const int et = threadIdx.x - 32 * P_EPI_WARP0;
        const uint32_t te = mapa_shared(&tempty[0], 0);
        volatile int* abort_flag = epi_abort;
        int gs = 0;
        for (int lt = 0; lt < my_tiles; ++lt) {
            const int acc = lt & 1;
            const uint32_t use = uint32_t(lt >> 1);
            int tm, tn;
            tile_coords(cl + lt * ncl, g, tm, tn);
            if (!mbar_wait(&tfull[acc], use & 1u, g.st, 315)) *abort_flag = 1;
            named_barrier_sync(EPI_BARRIER, 32 * EPI_WARPS);   // all four warps leave together on a timeout
            if (*abort_flag) break;
            tc_fence_after();
            const int y = tm * PBM + int(rank) * P_ROWS;
#pragma unroll 1
            for (int j = 0; j < PBN / SLAB; ++j, ++gs) {
                float v[32];
                tmem_ld_32x32b_x32(tmem_base + (uint32_t(quad * 32) << 16) + uint32_t(acc * PBN + j * SLAB), v);
                if (j == PBN / SLAB - 1) {   // accumulator drained in this CTA
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(te + uint32_t(acc) * 8u);
                }
                uint8_t* buf = cbuf + size_t(gs & 1) * SLAB_BYTES;
                if (et == 0) bulk_wait_group_read<1>();   // the store that last used this buffer has read it
                named_barrier_sync(EPI_BARRIER, 32 * EPI_WARPS);
                uint8_t* row = buf + size_t(et) * (SLAB * 4);
#pragma unroll
                for (int q = 0; q < SLAB / 4; ++q)
                    *reinterpret_cast<float4*>(row + ((q ^ (et & 7)) << 4)) =
                        make_float4(g.alpha * v[4 * q], g.alpha * v[4 * q + 1], g.alpha * v[4 * q + 2],
                                    g.alpha * v[4 * q + 3]);
                fence_proxy_async_smem();
                named_barrier_sync(EPI_BARRIER, 32 * EPI_WARPS);
                if (et == 0) {
                    const int x = tn * PBN + j * SLAB;
                    if (x < g.N && y < g.M) {
                        if (g.accumulate)
                            tma_reduce_add_2d(&maps.c, buf, x, y);
                        else
                            tma_store_2d(&maps.c, buf, x, y);
                    }
                    bulk_commit_group();
                }
            }
        }
        if (et == 0) bulk_wait_group<0>();   // every store has reached global memory
    }
    tc_fence_before();
    cluster_sync();          // no remote arrival or pair MMA is still pending
    if (warp == 0) tmem_dealloc_pair(tmem_base, P_TMEM_COLS);
}

}  // namespace tg

namespace {
PFN_encodeTiled g_enc = nullptr;

template <bool PRESPLIT>
int launch_variant(const tg::Maps& maps, const tg::Args& g, cudaStream_t stream) {
    using C = tg::Cfg<PRESPLIT>;
    static std::atomic<bool> attr_set[64];
    static std::atomic<int> sms[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (dev < 64 && !attr_set[dev]) {
        int n = 0;
        if (cudaFuncSetAttribute(tg::tgemm_kernel<PRESPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(C::SMEM_BYTES)) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        sms[dev] = n;
        attr_set[dev] = true;
    }
    const int n_sms = dev < 64 ? sms[dev].load() : 0;
    const int grid = std::max(1, std::min(g.tiles, n_sms > 0 ? n_sms : 148));
    if (launch_pdl(tg::tgemm_kernel<PRESPLIT>, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, stream, maps, g) !=
        cudaSuccess)
        return GPTQ_ERR_CUDA;
    count_launch();
    return GPTQ_OK;
}
// Pre-split products at least this deep (and wider than one 128-row tile in
// both M and N) run on SM pairs.  A build-time tuning knob.
#ifndef GPTQ_TGEMM_PAIR_MIN_K
#define GPTQ_TGEMM_PAIR_MIN_K 256
#endif

int launch_pair(const tg::Maps& maps, tg::Args g, cudaStream_t stream) {
    using namespace tg;
    static std::atomic<bool> attr_set[64];
    static std::atomic<int> sms[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (dev < 64 && !attr_set[dev]) {
        int n = 0;
        if (cudaFuncSetAttribute(tgemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(P_SMEM_BYTES)) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        sms[dev] = n;
        attr_set[dev] = true;
    }
    g.tiles_m = (g.M + PBM - 1) / PBM;
    g.tiles_n = (g.N + PBN - 1) / PBN;
    if (g.lower_only) {
        g.tiles = 0;
        for (int tm = 0; tm < g.tiles_m; ++tm) g.tiles += std::min(g.tiles_n, tm + 1);
    } else {
        g.tiles = g.tiles_m * g.tiles_n;
    }
    const int n_sms = dev < 64 ? sms[dev].load() : 0;
    const int clusters = std::max(1, std::min(g.tiles, (n_sms > 0 ? n_sms : 148) / 2));
    if (launch_pdl(tgemm_pair_kernel, dim3(2 * clusters), dim3(P_THREADS), P_SMEM_BYTES, stream, maps, g) !=
        cudaSuccess)
        return GPTQ_ERR_CUDA;
    count_launch();
    return GPTQ_OK;
}
}  // namespace

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

int launch_tgemm(int M, int N, int K, float alpha, const float* A, const float* A_lo, int lda, const float* Bt,
                 const float* Bt_lo, int ldb, bool accumulate, float* C, int ldc, bool lower_only,
                 cudaStream_t stream, DevStatus* st) {
    using namespace tg;
    if (M <= 0 || N <= 0) return GPTQ_OK;
    const bool presplit = A_lo != nullptr;
    if (K <= 0 || K % BKC != 0 || K > MAX_K || (Bt_lo != nullptr) != presplit || g_enc == nullptr)
        return GPTQ_ERR_UNSUPPORTED;
    Maps maps;
    std::memset(&maps, 0, sizeof(maps));
    int rc = make_map_2d_f32(&maps.a, A, uint64_t(K), uint64_t(M), uint64_t(lda), BKC, BM, true);
    if (!rc) rc = make_map_2d_f32(&maps.b, Bt, uint64_t(K), uint64_t(N), uint64_t(ldb), BKC, BN, true);
    if (!rc && presplit) rc = make_map_2d_f32(&maps.a_lo, A_lo, uint64_t(K), uint64_t(M), uint64_t(lda), BKC, BM, true);
    if (!rc && presplit) rc = make_map_2d_f32(&maps.b_lo, Bt_lo, uint64_t(K), uint64_t(N), uint64_t(ldb), BKC, BN, true);
    if (!rc) rc = make_map_2d_f32(&maps.c, C, uint64_t(N), uint64_t(M), uint64_t(ldc), SLAB, BM, true);
    if (rc) return rc;
    Args g{};
    g.M = M; g.N = N; g.K = K; g.alpha = alpha;
    g.accumulate = accumulate ? 1 : 0;
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
    if (presplit && K >= GPTQ_TGEMM_PAIR_MIN_K && M > BM && N > BN) return launch_pair(maps, g, stream);
    return presplit ? launch_variant<true>(maps, g, stream) : launch_variant<false>(maps, g, stream);
}

}  // namespace gptq
