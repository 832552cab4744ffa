// The layer output computed from the stored form (itwiki "GPTQ", section
// "결과": a dedicated inference kernel unpacks the weights as it needs them;
// blog "GPTQ를 밑바닥부터 구현하며 배운 것들", section 5: INT4 codes are
// stored and dequantized during inference):
//
//   y[t][r] = sum_k s[r][g(k)] (c[r][k] - z[r][g(k)]) x[t][perm[k]]
//
// for a handful of tokens t (decode).  The work is bound by reading the
// packed codes from HBM (half a byte per weight), so the design goal is a
// full-bandwidth stream of coalesced 16-byte loads with as few instructions
// per weight as possible:
//  - each block owns 32 rows; its 8 warps split d_in, and a shared-memory
//    reduction combines them (deterministic order);
//  - per 128-column block a lane loads 16 bytes (32 codes) of each of its 4
//    rows and 64 bytes of its token's x;
//  - codes become exact bf16 integers with one OR into a bf16 with exponent
//    2^7 (value 128 + c) and one packed FMA that subtracts 128, two codes per
//    instruction, and go straight from registers into warp-level bf16 MMAs
//    (m16n8k16: 16 rows x 8 tokens, fp32 accumulation, exact products); the
//    tensor core is only the dot-product engine here, far from its limit;
//  - the zero point is applied per 128-column block as s (sum c x - z sum x),
//    with sum x from one more MMA against an all-ones operand.
// The k order inside an MMA does not matter for a dot product: the codes are
// taken as nibble pairs (p, p+4) of a word, and x is paired the same way with
// byte permutes.
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace gemv {

constexpr int WARPS = 8;                  // K split of a block's rows
constexpr int ROWS = 32;                  // two 16-row MMA tiles per warp
constexpr int KB = 128;                   // codes per column block (4 lanes x 32)
constexpr int THREADS = 32 * WARPS;
constexpr int MAX_TOKENS = 8;

struct Args {
    const uint32_t* codes;    // [d_out, d_in / 8]
    const uint16_t* scales;   // fp16 bits [d_out, n_groups]
    const uint16_t* zeros;
    const uint16_t* x;        // bf16 bits [m, d_in], processing order
    float* y;                 // [m, d_out]
    int d_out, d_in, m, group, n_groups;
};

// bf16x2 (128 + c_lo, 128 + c_hi) from the nibbles at bits sh and sh + 16,
// then minus (128, 128): both codes as exact bf16 values.
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, int sh) {
    const uint32_t t = ((w >> sh) & 0x000F000Fu) | 0x43004300u;
    uint32_t r;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(t), "r"(0x3F803F80u), "r"(0xC300C300u));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// One block: rows [r0, r0 + 32); warp w: column blocks [kb0, kb1).
// Lane (g = lane / 4, q = lane % 4): rows r0 + g + 8 i (i = 0..3), codes
// 32 q .. 32 q + 31 of each column block, token g of x.
__global__ void __launch_bounds__(THREADS) w4_kernel(Args a) {
    __shared__ float red[WARPS][ROWS][MAX_TOKENS + 1];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int g = lane >> 2, q = lane & 3;
    const int r0 = blockIdx.x * ROWS;
    const int nkb = a.d_in / KB;
    const int kb0 = int((int64_t(nkb) * w) / WARPS), kb1 = int((int64_t(nkb) * (w + 1)) / WARPS);
    const int words_per_row = a.d_in / 8;

    const uint32_t* crow[4];
    bool rvalid[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + g + 8 * i;
        rvalid[i] = r < a.d_out;
        crow[i] = a.codes + size_t(rvalid[i] ? r : 0) * words_per_row + q * 4;
    }
    const bool xvalid = g < a.m;
    const uint16_t* xrow = a.x + size_t(xvalid ? g : 0) * a.d_in + q * 32;

    float yacc[2][4] = {};
    uint4 cw[4], xw[4];
    auto load = [&](int kb, uint4 (&c)[4], uint4 (&xv)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) c[i] = rvalid[i] ? ldg_stream(crow[i] + size_t(kb) * 16) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            xv[i] = xvalid ? __ldg(reinterpret_cast<const uint4*>(xrow + size_t(kb) * KB) + i) : make_uint4(0, 0, 0, 0);
    };
    if (kb0 < kb1) load(kb0, cw, xw);
    for (int kb = kb0; kb < kb1; ++kb) {
        uint4 cn[4], xn[4];
        if (kb + 1 < kb1) load(kb + 1, cn, xn);
        const uint32_t X[16] = {xw[0].x, xw[0].y, xw[0].z, xw[0].w, xw[1].x, xw[1].y, xw[1].z, xw[1].w,
                                xw[2].x, xw[2].y, xw[2].z, xw[2].w, xw[3].x, xw[3].y, xw[3].z, xw[3].w};
        const uint32_t C[4][4] = {{cw[0].x, cw[0].y, cw[0].z, cw[0].w}, {cw[1].x, cw[1].y, cw[1].z, cw[1].w},
                                  {cw[2].x, cw[2].y, cw[2].z, cw[2].w}, {cw[3].x, cw[3].y, cw[3].z, cw[3].w}};
        float acc[2][4] = {}, xs[4] = {};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t b0 = prmt(X[4 * j + h], X[4 * j + h + 2], 0x5410u);
                const uint32_t b1 = prmt(X[4 * j + h], X[4 * j + h + 2], 0x7632u);
                mma_bf16(xs, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u, b0, b1);
#pragma unroll
                for (int t = 0; t < 2; ++t)
                    mma_bf16(acc[t], nib_pair(C[2 * t][j], 8 * h), nib_pair(C[2 * t + 1][j], 8 * h),
                             nib_pair(C[2 * t][j], 8 * h + 4), nib_pair(C[2 * t + 1][j], 8 * h + 4), b0, b1);
            }
        }
        // scale this column block: y += s (acc - z sum x)
        const int gi = (kb * KB) / a.group;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int i = 2 * t + hf;
                float s = 0.0f, z = 0.0f;
                if (rvalid[i]) {
                    const size_t o = size_t(r0 + g + 8 * i) * a.n_groups + gi;
                    s = h2f(__ldg(a.scales + o));
                    z = h2f(__ldg(a.zeros + o));
                }
                yacc[t][2 * hf] = fmaf(s, fmaf(-z, xs[0], acc[t][2 * hf]), yacc[t][2 * hf]);
                yacc[t][2 * hf + 1] = fmaf(s, fmaf(-z, xs[1], acc[t][2 * hf + 1]), yacc[t][2 * hf + 1]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) { cw[i] = cn[i]; xw[i] = xn[i]; }
    }
    // lane holds rows g + 16 t + 8 hf, tokens 2q, 2q + 1
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            red[w][g + 16 * t + 8 * hf][2 * q] = yacc[t][2 * hf];
            red[w][g + 16 * t + 8 * hf][2 * q + 1] = yacc[t][2 * hf + 1];
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

// xp[t][k] = x[t][perm[k]]; an index outside [0, d_in) is reported and gives NaN.
__global__ void gather_x_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int d_in, int m,
                                uint16_t* __restrict__ xp, DevStatus* st) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= d_in) return;
    const int p = perm[k];
    const bool ok = p >= 0 && p < d_in;
    if (!ok) record_error(st, GPTQ_ERR_INVALID_ARG, k);
    for (int t = 0; t < m; ++t) xp[size_t(t) * d_in + k] = ok ? x[size_t(t) * d_in + p] : uint16_t(0x7FC0);
}

}  // namespace gemv

size_t gemv_workspace_bytes(int64_t m, int64_t d_in, bool with_perm) {
    return with_perm ? ((size_t(m) * size_t(d_in) * 2 + 255) & ~size_t(255)) : 0;
}

int launch_dequant_gemv(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                        int64_t d_in, int groupsize, const int32_t* perm, const uint16_t* x, int64_t m, float* y,
                        void* ws, cudaStream_t stream, DevStatus* st) {
    using namespace gemv;
    const uint16_t* xin = x;
    if (perm) {
        uint16_t* xp = static_cast<uint16_t*>(ws);
        gather_x_kernel<<<unsigned((d_in + 255) / 256), 256, 0, stream>>>(x, perm, int(d_in), int(m), xp, st);
        count_launch();
        xin = xp;
    }
    Args a;
    a.codes = codes;
    a.scales = scales;
    a.zeros = zeros;
    a.x = xin;
    a.y = y;
    a.d_out = int(d_out);
    a.d_in = int(d_in);
    a.m = int(m);
    a.group = groupsize > 0 ? groupsize : int(d_in);
    a.n_groups = groupsize > 0 ? int(d_in / groupsize) : 1;
    w4_kernel<<<unsigned((d_out + ROWS - 1) / ROWS), THREADS, 0, stream>>>(a);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
