// The weights rebuilt from the stored form (note "Model Quantization",
// section "주요 양자화 기법", the GPTQ entry: at inference the INT4 weights are
// restored to FP16 for the computation; blog "GPTQ를 밑바닥부터 구현하며 배운
// 것들", section 5: codes stored, dequantized for use):
//
//   Wq[r][perm[k]] = s[r][g(k)] (c[r][k] - z[r][g(k)])
//
// for codes of 2, 3, 4 or 8 bits in the packed little-endian stream, groups in
// processing order, and the act-order permutation undone (perm = NULL: the
// natural order).  Each value is one fused multiply-add, s c + (-s z): s z is
// exact in fp32 (two 11-bit significands), so the result is s (c - z)
// rounded once -- exact in fp32 whenever it fits 24 bits (an integer zero
// point always does); fp16 / bf16 outputs round that to nearest even.
//
// Both kernels write 16-byte output vectors (4 fp32 or 8 fp16 / bf16 values),
// consecutive lanes to consecutive vectors, so every warp store covers 512
// contiguous bytes.  Without a permutation a flat grid-stride loop walks all
// vectors of the matrix and each vector reads its own codes.  With one, a
// block keeps the inverse permutation in shared memory, decodes one or two
// rows in processing order into shared memory, and gathers each output
// column from there.  Bound by HBM: bits / 8 bytes per weight in, 2 or 4 out.
#include <atomic>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace dq {

constexpr int VEC_THREADS = 256;
constexpr int GATHER_THREADS = 1024;
constexpr int UNROLL = 2;            // direct kernel: vectors per lane and row
constexpr int ROWS = 4;              // direct kernel: rows per block
constexpr int CHUNK = VEC_THREADS * UNROLL;   // direct kernel: vectors per block and row

struct Shape {
    int64_t d_out;
    int d_in, wpr, vpr;              // code words and output vectors per row
    int n_groups;
    uint32_t g_inv;                  // ceil(2^16 / (group / 128))
};

// Group of column k: floor((k / 128) / (group / 128)) by a reciprocal
// multiply, exact for k / 128 < 256 and group / 128 <= 256 (d_in <= 32768).
__device__ __forceinline__ int group_of(int k, uint32_t g_inv) { return int((uint32_t(k >> 7) * g_inv) >> 16); }

// An exact float of a code c < 2^23 without the conversion unit.
__device__ __forceinline__ float code_f(uint32_t c) { return __int_as_float(0x4B000000 | c) - 8388608.0f; }

template <int OUT>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    if constexpr (OUT == 1) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<const uint32_t*>(&h);
    } else {
        const __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
}

template <int OUT, int E>
__device__ __forceinline__ uint4 to_vec(const float (&v)[E]) {
    if constexpr (OUT == 0) {
        return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
    } else {
        return make_uint4(pack2<OUT>(v[0], v[1]), pack2<OUT>(v[2], v[3]), pack2<OUT>(v[4], v[5]), pack2<OUT>(v[6], v[7]));
    }
}

// Without a permutation.  Output vector v of a row holds columns E v ..
// E v + E - 1, whose codes are VB = E * BITS consecutive bits of the row's
// stream starting at bit VB v: one word for 2, 4 and 8 bits (two for 8-bit
// codes into fp16 / bf16); 3-bit vectors may straddle two words.  A block
// takes ROWS rows x CHUNK vectors; warp w of it the vectors 64 w + lane and
// 64 w + 32 + lane of the chunk, so that its stores are two adjacent 512-byte
// runs per row.  A lane's column offsets and groups are the same in every row:
// they are computed once, and the rows only advance the pointers.
template <int BITS, int OUT>
__global__ void __launch_bounds__(VEC_THREADS)
    dequant_vec_kernel(const uint32_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                       const uint16_t* __restrict__ zeros, Shape sh, uint4* __restrict__ out) {
    constexpr int E = OUT == 0 ? 4 : 8;
    constexpr int VB = E * BITS;
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    constexpr bool TWO_WORDS = VB == 64 || BITS == 3;
    const int n_chunks = (sh.vpr + CHUNK - 1) / CHUNK;
    const int64_t r0 = int64_t(blockIdx.x / n_chunks) * ROWS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int vv[UNROLL], wi[UNROLL], off[UNROLL], gi[UNROLL];
    bool ok[UNROLL], hi[UNROLL];
#pragma unroll
    for (int i = 0; i < UNROLL; ++i) {
        vv[i] = int(blockIdx.x % n_chunks) * CHUNK + warp * (32 * UNROLL) + 32 * i + lane;
        ok[i] = vv[i] < sh.vpr;
        const int bit = vv[i] * VB;
        wi[i] = bit >> 5;
        off[i] = bit & 31;
        hi[i] = VB == 64 || off[i] + VB > 32;     // the vector's last bits are in the next word of the row
        gi[i] = ok[i] ? group_of(vv[i] * E, sh.g_inv) : 0;
    }
    const int nrows = int(min(int64_t(ROWS), sh.d_out - r0));
    const uint32_t* crow = codes + size_t(r0) * sh.wpr;
    const uint16_t* srow = scales + size_t(r0) * sh.n_groups;
    const uint16_t* zrow = zeros + size_t(r0) * sh.n_groups;
    uint4* orow = out + size_t(r0) * sh.vpr;
    // every load of the block's rows first, then the arithmetic and the stores
    uint32_t lo[ROWS][UNROLL], up[ROWS][UNROLL];
    uint16_t sc[ROWS][UNROLL], zp[ROWS][UNROLL];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
#pragma unroll
        for (int i = 0; i < UNROLL; ++i) {
            if (r < nrows && ok[i]) {
                lo[r][i] = crow[size_t(r) * sh.wpr + wi[i]];
                if constexpr (TWO_WORDS) up[r][i] = hi[i] ? crow[size_t(r) * sh.wpr + wi[i] + 1] : 0u;
                sc[r][i] = srow[size_t(r) * sh.n_groups + gi[i]];
                zp[r][i] = zrow[size_t(r) * sh.n_groups + gi[i]];
            }
        }
    }
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
#pragma unroll
        for (int i = 0; i < UNROLL; ++i) {
            if (r < nrows && ok[i]) {
                uint32_t w;
                if constexpr (TWO_WORDS) w = uint32_t(((uint64_t(up[r][i]) << 32) | lo[r][i]) >> off[i]);
                else w = lo[r][i] >> off[i];
                const float s = __half2float(__ushort_as_half(sc[r][i]));
                const float nsz = -(s * __half2float(__ushort_as_half(zp[r][i])));   // exact
                float val[E];
                if constexpr (VB == 64) {   // 8-bit codes into 16-bit values: the upper four from the next word
#pragma unroll
                    for (int j = 0; j < 4; ++j) val[j] = fmaf(s, code_f((lo[r][i] >> (8 * j)) & MASK), nsz);
#pragma unroll
                    for (int j = 0; j < 4; ++j) val[4 + j] = fmaf(s, code_f((up[r][i] >> (8 * j)) & MASK), nsz);
                } else {
#pragma unroll
                    for (int j = 0; j < E; ++j) val[j] = fmaf(s, code_f((w >> (j * BITS)) & MASK), nsz);
                }
                orow[size_t(r) * sh.vpr + vv[i]] = to_vec<OUT, E>(val);
            }
        }
    }
}

// With a permutation.  Shared memory holds the inverse permutation
// ip[j] = k with perm[k] = j (16-bit) and one 32-bit slot per code column k,
// plus slot d_in, which holds NaN: ip points there where no entry lands.  A block takes RPB rows at a time:
//   A: decode them in processing order (contiguous codes and groups,
//      conflict-free 16-byte stores) into the slots: the fp32 value of one
//      row, or for 16-bit outputs the rounded values of two rows side by side;
//   B: output column j reads slot ip[j] -- one random shared-memory read per
//      value for fp32, one per two values for fp16 / bf16 -- and each row's
//      16-byte vectors are stored coalesced.
// A column that no entry reaches is NaN.
template <int BITS, int OUT>
__global__ void __launch_bounds__(GATHER_THREADS, 1)
    dequant_gather_kernel(const uint32_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                          const uint16_t* __restrict__ zeros, const int32_t* __restrict__ perm, Shape sh,
                          uint4* __restrict__ out, DevStatus* st) {
    constexpr int E = OUT == 0 ? 4 : 8;       // values per output vector
    constexpr int RPB = OUT == 0 ? 1 : 2;     // rows per slot
    constexpr int DB = 8;                     // columns decoded per step of A
    constexpr int VB = DB * BITS;
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    constexpr uint32_t NAN_SLOT = OUT == 0 ? 0x7fc00000u : OUT == 1 ? 0x7fc07fc0u : 0x7e007e00u;
    extern __shared__ __align__(16) uint8_t smem[];
    uint16_t* ip = reinterpret_cast<uint16_t*>(smem);                                              // [d_in]
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + ((size_t(sh.d_in) * 2 + 15) & ~size_t(15)));   // [d_in]
    const int t = threadIdx.x;
    for (int j = t; j < sh.d_in; j += GATHER_THREADS) ip[j] = uint16_t(sh.d_in);   // d_in <= 32768
    if (t == 0) slot[sh.d_in] = NAN_SLOT;
    __syncthreads();
    for (int k = t; k < sh.d_in; k += GATHER_THREADS) {
        const int j = perm[k];
        if (j >= 0 && j < sh.d_in) ip[j] = uint16_t(k);
        else if (blockIdx.x == 0) record_error(st, GPTQ_ERR_INVALID_ARG, k);
    }
    // A's global reads for the next rows are issued before B of the current
    // ones and land in registers untouched (no instruction uses them until the
    // next A), so their latency hides behind B.
    const int steps = sh.d_in / DB;
    constexpr int QMAX = 32768 / DB / GATHER_THREADS;      // steps per thread at the largest d_in
    constexpr bool HI = VB == 64 || BITS == 3;             // a step's codes may need a second word
    uint32_t lo[QMAX][RPB], hi[QMAX][RPB];
    uint16_t sc[QMAX][RPB], zp[QMAX][RPB];
    auto fetch = [&](int64_t r0) {
        const bool two = RPB == 2 && r0 + 1 < sh.d_out;
#pragma unroll
        for (int i = 0; i < QMAX; ++i) {
            const int q = t + i * GATHER_THREADS;
            if (q >= steps) break;
            const int bit = q * VB, wi = bit >> 5, off = bit & 31;
            const int gi = group_of(q * DB, sh.g_inv);
#pragma unroll
            for (int rr = 0; rr < RPB; ++rr) {
                const int64_t r = (rr == 1 && !two) ? r0 : r0 + rr;    // a missing second row repeats the first
                const uint32_t* crow = codes + size_t(r) * sh.wpr;
                lo[i][rr] = crow[wi];
                if constexpr (HI) hi[i][rr] = (VB == 64 || off + VB > 32) ? crow[wi + 1] : 0u;   // still inside the row
                sc[i][rr] = scales[size_t(r) * sh.n_groups + gi];
                zp[i][rr] = zeros[size_t(r) * sh.n_groups + gi];
            }
        }
    };
    const int64_t stride = int64_t(gridDim.x) * RPB;
    if (int64_t(blockIdx.x) * RPB < sh.d_out) fetch(int64_t(blockIdx.x) * RPB);
    for (int64_t r0 = int64_t(blockIdx.x) * RPB; r0 < sh.d_out; r0 += stride) {
        const bool two = RPB == 2 && r0 + 1 < sh.d_out;
        __syncthreads();   // B of the previous rows is done with the slots (and ip is complete)
        // ---- A
#pragma unroll
        for (int i = 0; i < QMAX; ++i) {
            const int q = t + i * GATHER_THREADS;
            if (q >= steps) break;
            const int off = (q * VB) & 31;
            float val[RPB][DB];
#pragma unroll
            for (int rr = 0; rr < RPB; ++rr) {
                uint64_t w = lo[i][rr];
                if constexpr (HI) w |= uint64_t(hi[i][rr]) << 32;
                w >>= off;
                const float s = __half2float(__ushort_as_half(sc[i][rr]));
                const float nsz = -(s * __half2float(__ushort_as_half(zp[i][rr])));
#pragma unroll
                for (int j = 0; j < DB; ++j) val[rr][j] = fmaf(s, code_f(uint32_t(w >> (j * BITS)) & MASK), nsz);
            }
            uint32_t o[DB];
#pragma unroll
            for (int j = 0; j < DB; ++j) {
                if constexpr (OUT == 0) o[j] = __float_as_uint(val[0][j]);
                else o[j] = pack2<OUT>(val[0][j], val[RPB - 1][j]);
            }
            uint4* dst = reinterpret_cast<uint4*>(slot + q * DB);
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
        if (r0 + stride < sh.d_out) fetch(r0 + stride);
        __syncthreads();
        // ---- B
        uint4* orow = out + size_t(r0) * sh.vpr;
        for (int vec = t; vec < sh.vpr; vec += GATHER_THREADS) {
            uint32_t g[E];
            if constexpr (E == 8) {
                const uint4 q = *reinterpret_cast<const uint4*>(ip + vec * 8);
                const uint32_t qa[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    g[2 * i] = slot[qa[i] & 0xFFFFu];
                    g[2 * i + 1] = slot[qa[i] >> 16];
                }
            } else {
                const uint2 q = *reinterpret_cast<const uint2*>(ip + vec * 4);
                const uint32_t qa[2] = {q.x, q.y};
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    g[2 * i] = slot[qa[i] & 0xFFFFu];
                    g[2 * i + 1] = slot[qa[i] >> 16];
                }
            }
            if constexpr (OUT == 0) {
                orow[vec] = make_uint4(g[0], g[1], g[2], g[3]);
            } else {
                // row r0: the low halves; row r0 + 1: the high halves
                orow[vec] = make_uint4(__byte_perm(g[0], g[1], 0x5410), __byte_perm(g[2], g[3], 0x5410),
                                       __byte_perm(g[4], g[5], 0x5410), __byte_perm(g[6], g[7], 0x5410));
                if (two)
                    orow[sh.vpr + vec] = make_uint4(__byte_perm(g[0], g[1], 0x7632), __byte_perm(g[2], g[3], 0x7632),
                                                    __byte_perm(g[4], g[5], 0x7632), __byte_perm(g[6], g[7], 0x7632));
            }
        }
    }
}

// The gather kernel's shared memory: ip (16-bit, padded to 16 bytes) and
// d_in + 1 slots; 196,612 bytes at the largest d_in (32768).
inline size_t gather_smem(int d_in) { return ((size_t(d_in) * 2 + 15) & ~size_t(15)) + size_t(d_in + 1) * 4; }

template <int BITS, int OUT>
int launch_typed(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, const int32_t* perm,
                 Shape sh, void* out, cudaStream_t stream, DevStatus* st) {
    uint4* o = static_cast<uint4*>(out);
    if (!perm) {
        const int64_t n_chunks = (sh.vpr + CHUNK - 1) / CHUNK;
        const int64_t blocks = (sh.d_out + ROWS - 1) / ROWS * n_chunks;      // <= 2^22 * 16
        dequant_vec_kernel<BITS, OUT><<<unsigned(blocks), VEC_THREADS, 0, stream>>>(codes, scales, zeros, sh, o);
    } else {
        // once per device: the shared-memory limit for the largest d_in, and the SM count
        static std::atomic<bool> ready[64];   // zero-initialized (static storage)
        static std::atomic<int> sms[64];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
        if (!ready[dev]) {
            int n = 0;
            if (cudaFuncSetAttribute(dequant_gather_kernel<BITS, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(gather_smem(32768))) != cudaSuccess ||
                cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            sms[dev] = n;
            ready[dev] = true;
        }
        const size_t smem = gather_smem(sh.d_in);
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dequant_gather_kernel<BITS, OUT>, GATHER_THREADS,
                                                          smem) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        const int64_t units = OUT == 0 ? sh.d_out : (sh.d_out + 1) / 2;     // rows per block step: 1 or 2
        const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(units, int64_t(sms[dev].load()) * std::max(per_sm, 1)));
        dequant_gather_kernel<BITS, OUT><<<unsigned(blocks), GATHER_THREADS, smem, stream>>>(codes, scales, zeros,
                                                                                             perm, sh, o, st);
    }
    count_launch();
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

template <int BITS>
int launch_bits(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, const int32_t* perm,
                const Shape& sh, int out_dtype, void* out, cudaStream_t stream, DevStatus* st) {
    switch (out_dtype) {
        case 0: return launch_typed<BITS, 0>(codes, scales, zeros, perm, sh, out, stream, st);
        case 1: return launch_typed<BITS, 1>(codes, scales, zeros, perm, sh, out, stream, st);
        case 2: return launch_typed<BITS, 2>(codes, scales, zeros, perm, sh, out, stream, st);
        default: return GPTQ_ERR_INVALID_ARG;
    }
}

}  // namespace dq

int launch_dequantize(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                      int64_t d_in, int bits, int groupsize, const int32_t* perm, int out_dtype, void* out,
                      cudaStream_t stream, DevStatus* st) {
    using namespace dq;
    const int group = groupsize > 0 ? groupsize : int(d_in);
    Shape sh{};
    sh.d_out = d_out;
    sh.d_in = int(d_in);
    sh.wpr = int(d_in * bits / 32);
    sh.vpr = int(d_in / (out_dtype == 0 ? 4 : 8));
    sh.n_groups = int(d_in / group);
    sh.g_inv = (65536u + uint32_t(group / 128) - 1u) / uint32_t(group / 128);
    switch (bits) {
        case 2: return launch_bits<2>(codes, scales, zeros, perm, sh, out_dtype, out, stream, st);
        case 3: return launch_bits<3>(codes, scales, zeros, perm, sh, out_dtype, out, stream, st);
        case 4: return launch_bits<4>(codes, scales, zeros, perm, sh, out_dtype, out, stream, st);
        case 8: return launch_bits<8>(codes, scales, zeros, perm, sh, out_dtype, out, stream, st);
        default: return GPTQ_ERR_UNSUPPORTED;
    }
}

}  // namespace gptq
