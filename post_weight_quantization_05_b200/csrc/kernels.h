// Host-side launchers shared between the translation units of libgptq.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

namespace gptq {

struct DevStatus;

// Host-side count of kernels enqueued by this library (gptq_launch_count).
void count_launch();


typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// api.cu: this device's status word, the driver's tensor-map encoder, and
// the host-side checks of gptq_quantize_layer's arguments (all but ws).
int status_ptr(DevStatus** out);
int encode_fn(PFN_encodeTiled* out);
int validate_quantize_args(const float* W, int64_t d_out, int64_t d_in, const float* U, int bits, int blocksize,
                           int groupsize, const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros,
                           const float* Q);

// hessian.cu.  after_own_launch: the previous kernel in `stream` is this
// library's H accumulation of another batch (bf16 only: the kernel then waits
// for it only before updating H).
int launch_hessian(const void* X, int dtype, int64_t n, int64_t d, float* H, void* ws, cudaStream_t stream,
                   DevStatus* st, PFN_encodeTiled encode, bool after_own_launch = false);

// tgemm.cu: C[M,N] = alpha * A[M,K] * B (accumulate = false) or
// C[M,N] += alpha * A[M,K] * B (accumulate = true), B(k, n) = Bt[n * ldb + k],
// fp32 row-major, on the tensor cores (kind::tf32, hi/lo split, three passes;
// fp32-class accuracy).  A_lo / Bt_lo null: the kernel splits A and Bt itself;
// both non-null: A and Bt hold the tf32-rounded hi parts and A_lo / Bt_lo the
// remainders (split_tf32).  K must be a multiple of 32; pointers and leading
// dimensions must satisfy TMA's 16-byte rules.  lower_only skips 128 x 128
// output tiles entirely above the diagonal.  C may be one of the operands when
// N <= 128 (each CTA then reads only the rows it writes, before writing them).
void set_tensor_map_encoder(PFN_encodeTiled f);
// 2-D fp32 tensor map (row stride ld_elems), 128-byte swizzle or none.
int make_map_2d_f32(CUtensorMap* tm, const float* base, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                    uint32_t box_inner, uint32_t box_outer, bool swizzle128);
int launch_tgemm(int M, int N, int K, float alpha, const float* A, const float* A_lo, int lda, const float* Bt,
                 const float* Bt_lo, int ldb, bool accumulate, float* C, int ldc, bool lower_only,
                 cudaStream_t stream, DevStatus* st);

// factor.cu
size_t factor_workspace_bytes(int64_t d);
int launch_prepare_hinv(const float* H, int64_t d, float percdamp, float* U, int* info, void* ws,
                        cudaStream_t stream, DevStatus* st);

// sweep.cu
size_t sweep_workspace_bytes(int64_t d_out, int64_t d_in);
int launch_quantize(float* W, int64_t d_out, int64_t d_in, const float* U, int bits, int groupsize,
                    uint32_t* codes, uint16_t* scales, uint16_t* zeros, float* Q, void* ws, cudaStream_t stream,
                    DevStatus* st);
int launch_rtn(const float* W, int64_t d_out, int64_t d_in, int bits, int groupsize, uint32_t* codes,
               uint16_t* scales, uint16_t* zeros, float* Q, cudaStream_t stream, DevStatus* st);
int launch_widen_bf16(const uint16_t* src, float* dst, int64_t count, cudaStream_t stream);

// gemv.cu: y = x W^T from the stored form (4-bit codes), m <= 8 tokens; with
// perm, x is first gathered into ws (gemv_workspace_bytes).
size_t gemv_workspace_bytes(int64_t m, int64_t d_in, bool with_perm);
int launch_dequant_gemv(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                        int64_t d_in, int groupsize, const int32_t* perm, const uint16_t* x, int64_t m, float* y,
                        void* ws, cudaStream_t stream, DevStatus* st, PFN_encodeTiled encode);

// dequant.cu: the weights rebuilt from the stored form (2/3/4/8-bit codes,
// act-order undone), out_dtype 0 fp32, 1 bf16, 2 fp16.
int launch_dequantize(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                      int64_t d_in, int bits, int groupsize, const int32_t* perm, int out_dtype, void* out,
                      cudaStream_t stream, DevStatus* st);

// permute.cu (act-order): the processing order from diag(H), the permuted
// Hessian, and the column permutation of a row-major matrix (in place allowed).
int launch_act_order_perm(const float* H, int64_t d, int32_t* perm, cudaStream_t stream);
int launch_permute_hessian(const float* H, int64_t d, const int32_t* perm, float* Hp, cudaStream_t stream,
                           DevStatus* st);
int launch_permute_columns(const float* src, int64_t rows, int64_t cols, const int32_t* perm, bool inverse,
                           float* dst, cudaStream_t stream, DevStatus* st);
int launch_fill(float* p, int64_t count, float value, cudaStream_t stream);

}  // namespace gptq
