// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "dbf.h"

namespace dbf {

constexpr int kMaxEll = 8;

// Every workspace starts with this many bytes of header that only the
// single-launch decode kernel uses (its grid barrier counter); they must be
// zero before the workspace's first use and every call leaves them valid.
constexpr size_t kWsHeaderBytes = 256;
// Header layout: bytes 0..7 the decode kernel's grid-barrier word (arrival
// count in the low 32 bits, epoch in the high 32 bits; zero at first use),
// bytes 8..11 a sticky int32 status that kernels whose bounded wait expired
// set to DBF_ERR_TIMEOUT (never cleared by the library).
constexpr size_t kWsStatusOffset = 8;

// ---- packed layout helpers (see "Packed sign layout" in dbf.h) -----------
__host__ __device__ inline int64_t pitch_words(int64_t k) { return (k + 31) / 32; }

// ---- per-device launch state (dbf_device.cu) -------------------------------
// SM count of the current device (148 if it cannot be read).
int device_sms();
// Allow 'kernel' at least 'bytes' of dynamic shared memory on the current
// device (cudaFuncSetAttribute once per device and size; optionally the
// largest shared-memory carve-out too).
cudaError_t allow_smem(const void *kernel, int bytes, bool max_shared_carveout = false);

// ---- launchers (each returns the first CUDA error it meets) --------------
cudaError_t launch_pack(const void *src, dbf_dtype dt, int64_t rows, int64_t k, uint32_t *dst,
                        int32_t *status, cudaStream_t s);
// the same with a destination row stride of dst_ld >= pitch_words(k) words
cudaError_t launch_pack_ld(const void *src, dbf_dtype dt, int64_t rows, int64_t k, uint32_t *dst,
                           int64_t dst_ld, int32_t *status, cudaStream_t s);
cudaError_t launch_unpack(const uint32_t *src, int64_t rows, int64_t k, int8_t *dst,
                          cudaStream_t s);
cudaError_t launch_transpose(const uint32_t *src, int64_t rows, int64_t k, uint32_t *dst,
                             cudaStream_t s);
cudaError_t launch_ste(const float *db, const void *h, dbf_dtype hd, int64_t n, float tau, float *dh,
                       int accumulate, cudaStream_t s);

// single-launch decode kernels (integer tensor-core products): dbf_decode.cu
// for one layer with at most eight (token, envelope) columns, and
// dbf_decode_multi.cu for more columns and for segmented adapters (M <= 8192,
// at most 512 segments); *_fits says whether a call takes that kernel
bool decode_fits(const dbf_layer &L, int64_t T);
size_t decode_workspace_bytes(const dbf_layer &L, int64_t T);
cudaError_t decode_forward(const dbf_layer &L, const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                           int flags, void *ws, cudaStream_t s);
bool multi_fits(const dbf_layer &L, int64_t T);
size_t multi_workspace_bytes(const dbf_layer &L, int64_t T);
cudaError_t multi_forward(const dbf_layer &L, const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                          int flags, void *ws, cudaStream_t s);
bool multi_segmented_fits(int32_t S, int32_t max_R, int32_t max_ell, int32_t M, int32_t N, int64_t T);
size_t multi_segmented_workspace_bytes(int32_t max_R, int32_t max_ell, int64_t T);
cudaError_t multi_forward_segmented(const dbf_layer *adapters, int32_t num_adapters, const int32_t *seg_off,
                                    const int32_t *seg_adp, int32_t S, int32_t max_R, int32_t max_ell, int32_t M,
                                    int32_t N, const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                                    int flags, void *ws, int32_t *status, cudaStream_t s);
// limit of the decode kernels' grid-barrier wait (dbf_device.cu): the value
// for launches, and the setting for later calls (0: the default, 2 s)
unsigned long long decode_wait_ns();
void set_decode_wait_ns(unsigned long long ns);

// decode path
size_t gemv_workspace_bytes(int64_t R, int64_t ell, int64_t T);   // two-launch and segmented kernels
size_t gemv_layer_workspace_bytes(const dbf_layer &L, int64_t T);  // dbf_forward on the GEMV path
int gemv_launches(const dbf_layer &L, int64_t T);   // 1 (single launch) or 2
cudaError_t gemv_forward(const dbf_layer &L, const void *x, dbf_dtype xd, void *y, dbf_dtype yd,
                         int64_t T, int flags, void *ws, cudaStream_t s);
cudaError_t gemv_forward_segmented(const dbf_layer *adapters, int32_t num_adapters,
                                   const int32_t *seg_off, const int32_t *seg_adp, int32_t S,
                                   int32_t max_R, int32_t max_ell, int32_t M, int32_t N,
                                   const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                                   int flags, void *ws, int32_t *status, cudaStream_t s);

// grouped prefill of adapters of one shape (segmented serving)
constexpr int kMaxGroupsPerLaunch = 48;
cudaError_t gemm_forward_grouped(const dbf_layer *const *layers, const int *off, const int *n, int count,
                                 const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T, int flags,
                                 void *ws, cudaStream_t s);

// multi-boolean-kernel layer (tcgen05 GEMM for any T)
bool mbok_shape_ok(int64_t M, int64_t N, int64_t K);
size_t mbok_workspace_bytes(int64_t M, int64_t K, int64_t T);
cudaError_t mbok_forward(int M, int N, int K, const uint32_t *w_packed, const uint16_t *s_in,
                         const uint16_t *s_out, const void *x, dbf_dtype xd, void *y, dbf_dtype yd,
                         int64_t T, int flags, void *ws, cudaStream_t s);

// SVID (sign times the best rank-1 fit of the magnitudes), by power iteration
size_t svid_scratch_bytes(int64_t n, int64_t m, int iters);
int *svid_count_slot(void *scratch, int64_t n, int64_t m, int iters);   // power iterations the last call ran
// the power iteration alone: fp16 and/or fp32 scale outputs (null ones skipped)
cudaError_t svid_power(const float *X, int64_t n, int64_t m, int iters, uint16_t *s_out, uint16_t *s_in,
                       float *s_out32, float *s_in32, void *scratch, cudaStream_t s);
cudaError_t svid_run(float *X, int64_t n, int64_t m, int iters, int subtract, uint32_t *signs,
                     int64_t signs_ld, uint16_t *s_out, uint16_t *s_in, void *scratch, cudaStream_t s);

// dense fp32 GEMM on the tensor cores (three TF32 products): Cout = alpha A B^T
// + beta Cin, A [M x K] and B [N x K] K-major; tf32x3_ok says whether the
// operands qualify (16-byte aligned, pitches a multiple of 4 floats); the lo
// planes of A and B go to lo_scratch (tf32x3_scratch_floats(M, N, K) floats,
// 16-byte aligned). lower (M == N, no sumsq): only the tiles that reach the
// lower triangle are computed; Cout entries above the diagonal outside them
// are left as they were. max_ctas > 0: at most that many CTAs (one per SM),
// leaving the other SMs to work on another stream. A_lo / B_lo: the lo
// planes of A / B already formed (pitch ceil4(K); then not split again);
// Cout_lo: also write the lo plane of the result (pitch ceil4(N)).
// lo(x) = x - (x with its low 13 mantissa bits cleared), exact.
__device__ __forceinline__ float tf32_lo(float x) { return x - __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }
bool tf32x3_ok(int64_t M, int64_t N, int64_t K, const float *A, int64_t lda, const float *B, int64_t ldb);
size_t tf32x3_scratch_floats(int64_t M, int64_t N, int64_t K);
cudaError_t tf32x3_gemm(int64_t M, int64_t N, int64_t K, float alpha, const float *A, int64_t lda, const float *B,
                        int64_t ldb, float beta, const float *Cin, int64_t ldci, float *Cout, int64_t ldco,
                        double *sumsq, int32_t *status, float *lo_scratch, size_t lo_scratch_floats, cudaStream_t s,
                        bool lower = false, int max_ctas = 0, const float *A_lo = nullptr,
                        const float *B_lo = nullptr, float *Cout_lo = nullptr);

// DBF factorisation (alternating ADMM with the SVID projection, fp32)
size_t factorize_workspace_bytes(int64_t n, int64_t m, int64_t k, int outer, int svid_iters);
cudaError_t factorize_run(const float *W, int64_t n, int64_t m, int64_t k, const float *U0, const float *V0,
                          int outer, int admm_iters, int svid_iters, float rho_rel, uint32_t *A_packed,
                          uint32_t *B_packed, uint16_t *alpha, uint16_t *beta, uint16_t *gamma, float *objective,
                          void *ws, cudaStream_t s);

// prefill path (tcgen05)
bool gemm_shape_ok(const dbf_layer &L);
// launches of one prefill forward: the pre-pass and both stages in one
// launch when both stages are at least 32 K steps deep, else three
int gemm_forward_launches(const dbf_layer &L);
size_t gemm_workspace_bytes(const dbf_layer &L, int64_t T);
cudaError_t gemm_forward(const dbf_layer &L, const void *x, dbf_dtype xd, void *y, dbf_dtype yd,
                         int64_t T, int flags, void *ws, cudaStream_t s);
bool gemm_backward_shape_ok(const dbf_layer &L);
size_t gemm_backward_workspace_bytes(const dbf_layer &L, int64_t T, bool signs);
cudaError_t gemm_backward(const dbf_layer &L, const uint32_t *b1t, const uint32_t *b2t, const void *x,
                          dbf_dtype xd, const void *dy, dbf_dtype dyd, int64_t T, float *dx,
                          float *dalpha, float *dbeta, float *dgamma, float *db1, float *db2,
                          int flags, void *ws, cudaStream_t s);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace dbf

// ---- small device helpers -------------------------------------------------
namespace dbf {

__device__ __forceinline__ float load_act(const void *p, dbf_dtype dt, int64_t i)
{
    if (dt == DBF_F32) return static_cast<const float *>(p)[i];
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

__device__ __forceinline__ void store_act(void *p, dbf_dtype dt, int64_t i, float v)
{
    if (dt == DBF_F32)
        static_cast<float *>(p)[i] = v;
    else
        static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float h2f(uint16_t h)
{
    return __half2float(__ushort_as_half(h));
}

}  // namespace dbf
