// The layer output computed from the stored form (itwiki "GPTQ", section
// "결과": a dedicated inference kernel unpacks the weights as it needs them;
// blog "GPTQ를 밑바닥부터 구현하며 배운 것들", section 5: INT4 codes are
// stored and dequantized during inference):
//
//   y[t][r] = sum_k s[r][g(k)] (c[r][k] - z[r][g(k)]) x[t][perm[k]]
//
// for a handful of tokens t (decode).  The work streams the packed codes from
// HBM (half a byte per weight); the design keeps that stream long and
// contiguous and spends as few instructions per weight as possible.
//
// prep_x_kernel (one warp per token and 128-column block): x in processing
//   order (through perm), scaled by a power of two 2^-e so that the block's
//   max |x| lies in [2^14, 2^15), as fp16 -- exact for every bf16 value down
//   to 2^-28 of that maximum (the 8-bit bf16 significand fits fp16's 11
//   bits) -- stored in the k order of the MMA fragments below, plus the
//   block's sum of those fp16 values and 2^e, in fp32.
//
// w4_kernel (one block per 32 rows, two blocks per SM): the rows' codes
//   stream by TMA through a ring of shared-memory stages, 512 contiguous bytes
//   of each row per stage, with x for the same 1024 columns; warp w takes
//   column block w of each stage, and the last warp to finish reading a stage
//   refills it.  A lane turns one 32-bit word (8 codes) into four
//   fp16 pairs with one shift, four LOPs and four packed FMAs (the nibble is
//   ORed into the mantissa of 1024.0 -- or 1024 + 16 c for the upper nibble of
//   a byte -- and the bias removed exactly), which go straight from registers
//   into warp-level fp16 MMAs (m16n8k16: 16 rows x 8 tokens, exact products,
//   fp32 accumulation).  Each column block is then scaled in fp32 as
//   2^e s (sum c x - z sum x); a shared-memory reduction over the 8 warps
//   finishes y in a fixed order.  The block's scale / zero pairs (one padded
//   word per row and group) and the tokens' block sums are staged in shared
//   memory once, so the loop reads nothing else from global memory.
// A word's nibbles are taken in pairs (p, p + 4) -- the two halves of a packed
// fp16 register -- and x is stored in the same pairing, with the four lanes'
// 16-byte chunks interleaved, so no permute is left in the inner loop and the
// x reads are free of bank conflicts.
#include <atomic>
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace gemv {

constexpr int WARPS = 8;                  // consumer warps: column block w of each stage
constexpr int ROWS = 32;                  // rows per block (two 16-row MMA tiles per warp)
constexpr int KB = 128;                   // codes per column block (4 lanes x 32)
constexpr int KPS = 8;                    // column blocks per stage (one per consumer warp)
constexpr int THREADS = 32 * WARPS;
constexpr int MAX_TOKENS = 8;
constexpr int MAX_STAGES = 4;
constexpr int CODE_BYTES = ROWS * KPS * KB / 2;      // 32 rows x 512 contiguous bytes: 16 KB
constexpr int XBLK_BYTES = KPS * KB * 2;             // one token's x for a stage: 2 KB
constexpr int PREP_THREADS = 256;

struct Args {
    const uint16_t* scales;   // fp16 bits [d_out, n_groups]
    const uint16_t* zeros;
    const float2* xaux;       // [m][d_in / 128]: {sum of the block's fp16 x, 2^e}
    float* y;                 // [m, d_out]
    int d_out, d_in, m, group, n_groups;
    // fp16x2 constants of the code conversion (1024, -1024, 1/16, -64), passed
    // as launch arguments: an instruction can take one of them straight from
    // the constant bank next to an immediate mask, where two immediates would
    // cost an extra move per use
    uint32_t k_mag, k_sub, k_s16, k_sub64;
    uint32_t kpg_magic;       // ceil(2^32 / (group / 128)), 0 when group = 128: the group of column block kb
    int side_off;             // byte offset of the staged scales / zeros / block data in shared memory
};

struct Maps {
    CUtensorMap codes;   // u32 [d_out][d_in / 8], box 128 words x 32 rows
    CUtensorMap x;       // fp16 [m][d_in / 128][128] (fragment order), box 128 x 8 x m
};

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// Codes to fp16 (in compute_tile): the low nibble of each byte of a word is
// ORed into the mantissa of 1024.0 and 1024 subtracted; the high nibble gives
// 1024 + 16 c, times 1/16, minus 64.  Both exact; one LOP and one packed FMA
// per two codes, the pairs (p, p + 4) of a word sharing a register.
__device__ __forceinline__ uint32_t hadd2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One warp's share of a column block, in registers: 16 bytes of codes of each
// of the lane's 4 rows (g + 8 i) and 64 bytes of its token's x.
struct Tile {
    uint4 c[4];
    uint4 x[4];
};

// MMA (j, h) of the block covers word j of every row and x words 4 j + 2 h,
// 4 j + 2 h + 1: k slots 2q, 2q+1 <-> nibbles (2h, 2h+4), slots 8+2q, 9+2q
// <-> nibbles (2h+1, 2h+5) of word j.  Then y += 2^e s (acc - z sum x).
__device__ __forceinline__ void compute_tile(const Tile& t, const float (&sv)[4], const float (&zv)[4], float2 xa0,
                                             float2 xa1, float (&yacc)[2][4], const Args& A) {
    const uint32_t X[16] = {t.x[0].x, t.x[0].y, t.x[0].z, t.x[0].w, t.x[1].x, t.x[1].y, t.x[1].z, t.x[1].w,
                            t.x[2].x, t.x[2].y, t.x[2].z, t.x[2].w, t.x[3].x, t.x[3].y, t.x[3].z, t.x[3].w};
    const uint32_t C[4][4] = {{t.c[0].x, t.c[0].y, t.c[0].z, t.c[0].w}, {t.c[1].x, t.c[1].y, t.c[1].z, t.c[1].w},
                              {t.c[2].x, t.c[2].y, t.c[2].z, t.c[2].w}, {t.c[3].x, t.c[3].y, t.c[3].z, t.c[3].w}};
    float acc[2][4] = {};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t b0 = X[4 * j + 2 * h], b1 = X[4 * j + 2 * h + 1];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                // rows g + 16 r (A rows 0..7) and g + 16 r + 8 (A rows 8..15)
                const uint32_t wl = h ? (C[2 * r][j] >> 8) : C[2 * r][j];
                const uint32_t wh = h ? (C[2 * r + 1][j] >> 8) : C[2 * r + 1][j];
                const uint32_t a0 = hadd2((wl & 0x000F000Fu) | A.k_mag, A.k_sub);
                const uint32_t a1 = hadd2((wh & 0x000F000Fu) | A.k_mag, A.k_sub);
                const uint32_t a2 = hfma2((wl & 0x00F000F0u) | A.k_mag, A.k_s16, A.k_sub64);
                const uint32_t a3 = hfma2((wh & 0x00F000F0u) | A.k_mag, A.k_s16, A.k_sub64);
                mma_f16(acc[r], a0, a1, a2, a3, b0, b1);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int i = 2 * r + hf;
            yacc[r][2 * hf] = fmaf(sv[i] * xa0.y, fmaf(-zv[i], xa0.x, acc[r][2 * hf]), yacc[r][2 * hf]);
            yacc[r][2 * hf + 1] = fmaf(sv[i] * xa1.y, fmaf(-zv[i], xa1.x, acc[r][2 * hf + 1]), yacc[r][2 * hf + 1]);
        }
    }
}

// One block: rows [r0, r0 + 32).  Lane (g = lane / 4, q = lane % 4) of
// warp w: rows g + 8 i of the block, codes 32 q .. 32 q + 31 of column block
// w of each stage, token g (lanes past m read no x: their MMA columns stay 0
// and nothing of them is stored).  Rows past d_out and columns past d_in
// arrive from TMA as zeros.
__global__ void __launch_bounds__(THREADS, 2) w4_kernel(const __grid_constant__ Maps maps, Args a, int stages,
                                                     DevStatus* st) {
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ uint64_t full[MAX_STAGES];
    __shared__ int released[MAX_STAGES];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int r0 = blockIdx.x * ROWS;
    const int nkb = a.d_in / KB;
    const int nst = (nkb + KPS - 1) / KPS;
    const uint32_t stage_bytes = CODE_BYTES + uint32_t(a.m) * XBLK_BYTES;
    // a stage holds 512 contiguous bytes of each of the 32 rows (column blocks
    // it*8 .. it*8+7), row-major: long row runs keep the HBM stream efficient
    auto issue_codes = [&](int it, int sidx) {
        mbar_arrive_expect_tx(&full[sidx], stage_bytes);
        tma_load_2d(ring + size_t(sidx) * stage_bytes, &maps.codes, it * (KPS * KB / 8), r0, &full[sidx]);
    };
    auto issue_x = [&](int it, int sidx) {
        tma_load_3d(ring + size_t(sidx) * stage_bytes + CODE_BYTES, &maps.x, 0, it * KPS, 0, &full[sidx]);
    };

    const int first = min(stages, nst);
    if (threadIdx.x == 0) {
        for (int i = 0; i < stages; ++i) {
            mbar_init(&full[i], 1);
            released[i] = 0;
        }
        fence_mbar_init();
        // the codes of the first stages do not depend on the x preparation
        // that runs just before this kernel: start them first
        for (int it = 0; it < first; ++it) issue_codes(it, it);
    }
    // scales and zeros of the block's rows (all groups) and the tokens' block
    // data, staged once: the loop then reads only shared memory.  The scales
    // and zeros do not depend on the x preparation: stage them before waiting.
    const int rows_here = min(ROWS, a.d_out - r0);
    const int ng = a.n_groups, sstride = ng + 1;        // words per row: the 8 rows of a warp on distinct banks
    uint32_t* sSZ = reinterpret_cast<uint32_t*>(ring + a.side_off);   // (s | z << 16) per row and group
    float2* sXA = reinterpret_cast<float2*>(ring + a.side_off + ((size_t(ROWS) * sstride * 4 + 15) & ~size_t(15)));
    {
        uint16_t* h = reinterpret_cast<uint16_t*>(sSZ);
        const int n_el = rows_here * ng;
        const float inv_ng = 1.0f / float(ng);
        auto put = [&](int idx, uint16_t v, int half) {
            const int row = int((float(idx) + 0.5f) * inv_ng);
            h[2 * (row * sstride + (idx - row * ng)) + half] = v;
        };
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint16_t* src = (half ? a.zeros : a.scales) + size_t(r0) * ng;
            int done = 0;
            if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {   // 16-byte loads, all in flight
                const int n16 = n_el / 8;
                uint4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int c = threadIdx.x + u * THREADS;
                    if (c < n16) v[u] = __ldg(reinterpret_cast<const uint4*>(src) + c);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int c = threadIdx.x + u * THREADS;
                    if (c < n16) {
                        const uint32_t wv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                        for (int e = 0; e < 8; ++e) put(8 * c + e, uint16_t(wv[e >> 1] >> (16 * (e & 1))), half);
                    }
                }
                done = 8 * min(n16, 4 * THREADS);
            }
            for (int idx = done + threadIdx.x; idx < n_el; idx += THREADS) put(idx, src[idx], half);
            // rows past d_out: scale 0, zero 0
            for (int idx = n_el + threadIdx.x; idx < ROWS * ng; idx += THREADS) put(idx, uint16_t(0), half);
        }
    }
    pdl_wait();                 // x and its block data come from the x preparation
    if (threadIdx.x == 0)
        for (int it = 0; it < first; ++it) issue_x(it, it);
    for (int e = threadIdx.x; e < a.m * nkb; e += THREADS) sXA[e] = a.xaux[e];
    __syncthreads();

    const int g = lane >> 2, q = lane & 3;
    const bool xvalid = g < a.m;
    // this lane's two token columns of the block data (tokens past m read
    // token 0: their outputs are not stored)
    const float2* xa0p = sXA + (2 * q < a.m ? 2 * q : 0) * nkb;
    const float2* xa1p = sXA + (2 * q + 1 < a.m ? 2 * q + 1 : 0) * nkb;

    float yacc[2][4] = {};
    Tile t;
#pragma unroll
    for (int i = 0; i < 4; ++i) t.x[i] = make_uint4(0, 0, 0, 0);
    int sidx = 0;
    uint32_t par = 0;
    for (int it = 0; it < nst; ++it) {
        const int kb = it * KPS + w;
        const bool active = kb < nkb;
        if (!mbar_wait(&full[sidx], par, st, 40)) break;
        const uint8_t* src = ring + size_t(sidx) * stage_bytes;
        if (active) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                t.c[i] = *reinterpret_cast<const uint4*>(src + (g + 8 * i) * (KPS * KB / 2) + w * (KB / 2) + q * 16);
            if (xvalid) {
                const uint8_t* xsrc = src + CODE_BYTES + g * XBLK_BYTES + w * (KB * 2) + q * 16;
#pragma unroll
                for (int i = 0; i < 4; ++i) t.x[i] = *reinterpret_cast<const uint4*>(xsrc + i * 64);
            }
        }
        // this warp's reads of the stage are ordered before the TMA that
        // refills it (generic-proxy reads, then an async-proxy write); the
        // last warp to release the stage issues the refill
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            if (atomicAdd(&released[sidx], 1) == WARPS - 1) {
                __threadfence_block();
                released[sidx] = 0;
                if (it + stages < nst) {
                    fence_proxy_async_smem();
                    issue_codes(it + stages, sidx);
                    issue_x(it + stages, sidx);
                }
            }
        }
        if (active) {
            const int gi = a.kpg_magic ? int(__umulhi(uint32_t(kb), a.kpg_magic)) : kb;
            float sv[4], zv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t v = sSZ[(g + 8 * i) * sstride + gi];
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&v));
                sv[i] = f.x;
                zv[i] = f.y;
            }
            compute_tile(t, sv, zv, xa0p[kb], xa1p[kb], yacc, a);
        }
        if (++sidx == stages) { sidx = 0; par ^= 1u; }
    }
    // lane holds rows g + 16 r + 8 hf, tokens 2q, 2q + 1; the reduction reuses
    // the ring (every stage has been consumed)
    __syncthreads();
    float (*red)[ROWS][MAX_TOKENS + 1] = reinterpret_cast<float (*)[ROWS][MAX_TOKENS + 1]>(ring);
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            red[w][g + 16 * r + 8 * hf][2 * q] = yacc[r][2 * hf];
            red[w][g + 16 * r + 8 * hf][2 * q + 1] = yacc[r][2 * hf + 1];
        }
    __syncthreads();
    for (int e = threadIdx.x; e < ROWS * a.m; e += THREADS) {
        const int row = e % ROWS, tok = e / ROWS;
        float v = 0.0f;
#pragma unroll
        for (int ww = 0; ww < WARPS; ++ww) v += red[ww][row][tok];
        if (r0 + row < a.d_out) a.y[size_t(tok) * a.d_out + r0 + row] = v;
    }
}

// Warp (t, b) -- token t = blockIdx.y, column block b = blockIdx.x * 8 +
// warp: amax = max |x[t][perm[k]]| over the block, e with amax 2^-e in
// [2^14, 2^15) (e = 0 for amax 0 or not finite), xh[t][slot] =
// fp16(x[t][perm[k]] 2^-e) with the slot of k in the order the product's
// lanes read (pairs (p, p + 4) of each group of 8 adjacent, the four lanes'
// 16-byte chunks interleaved), and xaux[t][b] = {sum of the block's fp16
// values in fp32 (fixed order), 2^e}.  An index outside [0, d_in) is reported
// and read as NaN.
__global__ void __launch_bounds__(PREP_THREADS)
    prep_x_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int d_in,
                  uint16_t* __restrict__ xh, float2* __restrict__ xaux, DevStatus* st) {
    pdl_trigger();              // the product kernel may set up meanwhile
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.y, b = blockIdx.x * (PREP_THREADS / 32) + (threadIdx.x >> 5);
    const int nkb = d_in / KB;
    if (b >= nkb) return;
    const uint16_t* xt = x + size_t(t) * d_in;
    float v[4];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // physical slot 4 lane + i of the block holds 16-byte chunk c = slot / 8:
        // lane q = c % 4 of the product reads chunk j = c / 4 as its j-th 16
        // bytes, i.e. fragment position f = 32 q + 8 j + (slot % 8), which is
        // k = 8u + {0,4,1,5,2,6,3,7}[f % 8] with u = f / 8
        const int slot = 4 * lane + i, c = slot >> 3;
        const int f = (c & 3) * 32 + (c >> 2) * 8 + (slot & 7);
        const int p = f & 7;
        const int k = b * KB + (f & ~7) + (p >> 1) + ((p & 1) ? 4 : 0);
        int src = k;
        bool ok = true;
        if (perm) {
            src = perm[k];
            ok = src >= 0 && src < d_in;
            if (!ok) record_error(st, GPTQ_ERR_INVALID_ARG, k);
        }
        v[i] = ok ? __uint_as_float(uint32_t(xt[src]) << 16) : __int_as_float(0x7fc00000);
        amax = fmaxf(amax, fabsf(v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int e = 0;
    if (amax > 0.0f && amax <= 3.4028235e38f) {
        int E;
        frexpf(amax, &E);           // amax in [2^(E-1), 2^E)
        e = E - 15;
    }
    float part = 0.0f;
    uint16_t hv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half h = __float2half_rn(ldexpf(v[i], -e));
        hv[i] = __half_as_ushort(h);
        part += __half2float(h);
    }
    *reinterpret_cast<uint2*>(xh + size_t(t) * d_in + b * KB + 4 * lane) =
        make_uint2(uint32_t(hv[0]) | (uint32_t(hv[1]) << 16), uint32_t(hv[2]) | (uint32_t(hv[3]) << 16));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) xaux[size_t(t) * nkb + b] = make_float2(part, ldexpf(1.0f, e));
}

}  // namespace gemv

namespace {
size_t r256(size_t b) { return (b + 255) & ~size_t(255); }
}  // namespace

// x in fragment order (fp16), then {block sum, block scale} per token and block.
size_t gemv_workspace_bytes(int64_t m, int64_t d_in, bool) {
    return r256(size_t(m) * size_t(d_in) * 2) + r256(size_t(m) * size_t(d_in / gemv::KB) * 8);
}

int launch_dequant_gemv(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                        int64_t d_in, int groupsize, const int32_t* perm, const uint16_t* x, int64_t m, float* y,
                        void* ws, cudaStream_t stream, DevStatus* st, PFN_encodeTiled encode) {
    using namespace gemv;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    uint16_t* xh = reinterpret_cast<uint16_t*>(wsb);
    float2* xaux = reinterpret_cast<float2*>(wsb + r256(size_t(m) * size_t(d_in) * 2));

    Maps maps;
    {
        const cuuint64_t dims[2] = {cuuint64_t(d_in / 8), cuuint64_t(d_out)};
        const cuuint64_t strides[1] = {cuuint64_t(d_in / 2)};
        const cuuint32_t box[2] = {KPS * KB / 8, ROWS};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&maps.codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GPTQ_ERR_CUDA;
    }
    {
        const cuuint64_t dims[3] = {cuuint64_t(KB), cuuint64_t(d_in / KB), cuuint64_t(m)};
        const cuuint64_t strides[2] = {cuuint64_t(KB * 2), cuuint64_t(d_in * 2)};
        const cuuint32_t box[3] = {KB, KPS, cuuint32_t(m)};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (encode(&maps.x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, xh, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GPTQ_ERR_CUDA;
    }
    Args a;
    a.scales = scales;
    a.zeros = zeros;
    a.xaux = xaux;
    a.y = y;
    a.d_out = int(d_out);
    a.d_in = int(d_in);
    a.m = int(m);
    a.group = groupsize > 0 ? groupsize : int(d_in);
    a.n_groups = groupsize > 0 ? int(d_in / groupsize) : 1;
    // kb / kpg as umulhi(kb, ceil(2^32 / kpg)) -- exact for kb, kpg <= 256; 0 marks kpg = 1
    a.k_mag = 0x64006400u;
    a.k_sub = 0xE400E400u;
    a.k_s16 = 0x2C002C00u;
    a.k_sub64 = 0xD400D400u;
    const uint64_t kpg = uint64_t(a.group / KB);
    a.kpg_magic = kpg == 1 ? 0u : uint32_t(((uint64_t(1) << 32) + kpg - 1) / kpg);
    // shared memory: the ring, then the staged scale / zero pairs (u32, 32 rows
    // x (n_groups + 1)) and block data (float2, m x d_in / 128); as many stages
    // (4, 3, 2) as keep two blocks on an SM
    const size_t stage_bytes = CODE_BYTES + size_t(m) * XBLK_BYTES;
    const size_t side = ((size_t(ROWS) * (a.n_groups + 1) * 4 + 15) & ~size_t(15)) + size_t(m) * (d_in / KB) * 8;
    int stages = 4;
    while (stages > 2 && size_t(stages) * stage_bytes + side > size_t(110) * 1024) --stages;
    const size_t ring_bytes = std::max(size_t(stages) * stage_bytes, size_t(WARPS) * ROWS * (MAX_TOKENS + 1) * 4);
    a.side_off = int(ring_bytes);
    const size_t smem = ring_bytes + side;
    constexpr size_t SMEM_CAP = size_t(160) * 1024;   // largest case (m = 8, d_in = 32768): about 112 KB
    if (smem > SMEM_CAP) return GPTQ_ERR_UNSUPPORTED;
    static std::atomic<bool> attr_done[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        // two blocks per SM need the whole shared-memory carveout (the
        // driver would otherwise size it for one)
        if (cudaFuncSetAttribute(w4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(SMEM_CAP)) != cudaSuccess ||
            cudaFuncSetAttribute(w4_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 int(cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    const dim3 pgrid(unsigned((d_in / KB + PREP_THREADS / 32 - 1) / (PREP_THREADS / 32)), unsigned(m));
    prep_x_kernel<<<pgrid, PREP_THREADS, 0, stream>>>(x, perm, int(d_in), xh, xaux, st);
    count_launch();
    if (launch_pdl(w4_kernel, dim3(unsigned((d_out + ROWS - 1) / ROWS)), dim3(THREADS), smem, stream, maps, a,
                   stages, st) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
