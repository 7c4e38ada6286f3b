// Sign-value-independent decomposition (SVID) of a dense fp32 matrix.
//
// DBF page, section 2: the SVID projection (from OneBit) keeps the binary
// structure inside the factorisation's alternating minimisation;
// Multi-Boolean Architectures page, section 2: W ~ W_bool . (s_out s_in^T)
// with W_bool = sign(W), and successive extraction of further kernels from
// the residuals. Here: X ~ sign(X) . (s_out s_in^T) where s_out s_in^T is
// the best rank-1 approximation of |X|, found by power iteration from the
// all-positive start (the top singular vectors of a nonnegative matrix are
// nonnegative), split evenly between the two scale vectors.
//
// One iteration reads X twice (u = |X| v row by row, one warp per row; then
// v = |X|^T u, a thread per column over a band of rows, atomics across
// bands). Norms are accumulated by atomics into a per-iteration slot, so
// consecutive kernels need no other synchronisation. HBM-bound.
#include "dbf_internal.cuh"

namespace dbf {
namespace {

constexpr int kSvidThreads = 256;
constexpr int kBandRows = 128;   // rows per band of the column pass

// u[i] = sum_j |X[i, j]| v[j] * vs, vs = rsqrt(norm2_in) (1 when norm2_in is null);
// norm2_out += |u|^2
__global__ void __launch_bounds__(kSvidThreads) svid_rows_kernel(const float *__restrict__ X, int64_t n, int64_t m,
                                                                 const float *__restrict__ v, const float *norm2_in,
                                                                 float *__restrict__ u, float *norm2_out)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const float vs = norm2_in ? rsqrtf(*norm2_in) : 1.f;
    float sq = 0.f;
    for (int64_t i = warp; i < n; i += nwarps) {
        const float *row = X + i * m;
        float acc = 0.f;
        for (int64_t j = lane; j < m; j += 32) acc += fabsf(row[j]) * v[j];
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        acc *= vs;
        if (lane == 0) {
            u[i] = acc;
            sq += acc * acc;
        }
    }
    if (lane == 0 && sq != 0.f) atomicAdd(norm2_out, sq);
}

// v[j] += sum_{i in band} |X[i, j]| u[i] * us (v zeroed before), us = rsqrt(norm2_in)
__global__ void __launch_bounds__(kSvidThreads) svid_cols_kernel(const float *__restrict__ X, int64_t n, int64_t m,
                                                                 const float *__restrict__ u, const float *norm2_in,
                                                                 float *__restrict__ v)
{
    const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t i0 = static_cast<int64_t>(blockIdx.y) * kBandRows;
    if (j >= m) return;
    const float us = rsqrtf(*norm2_in);
    const int64_t i1 = i0 + kBandRows < n ? i0 + kBandRows : n;
    float acc = 0.f;
    for (int64_t i = i0; i < i1; ++i) acc += fabsf(X[i * m + j]) * u[i];
    atomicAdd(v + j, acc * us);
}

__global__ void __launch_bounds__(kSvidThreads) svid_norm_kernel(const float *__restrict__ v, int64_t m, float *norm2)
{
    float sq = 0.f;
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < m;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x)
        sq += v[j] * v[j];
    for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if ((threadIdx.x & 31) == 0 && sq != 0.f) atomicAdd(norm2, sq);
}

// u is A v / |.| of the last row pass (norm2_u), v is A^T u_hat unnormalised
// with |v|^2 = norm2_v = sigma^2: s_out = sqrt(sigma) u_hat, s_in = v / sqrt(sigma)
__global__ void __launch_bounds__(kSvidThreads) svid_scales_kernel(const float *__restrict__ u, int64_t n,
                                                                   const float *norm2_u, const float *__restrict__ v,
                                                                   int64_t m, const float *norm2_v, uint16_t *s_out,
                                                                   uint16_t *s_in)
{
    const float sigma = sqrtf(*norm2_v);
    const float r = sqrtf(sigma);
    const float cu = r * rsqrtf(*norm2_u), cv = 1.f / r;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n + m;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (i < n) s_out[i] = __half_as_ushort(__float2half_rn(cu * u[i]));
        else s_in[i - n] = __half_as_ushort(__float2half_rn(cv * v[i - n]));
    }
}

// X[i, j] -= sign(X[i, j]) s_out[i] s_in[j] with the stored fp16 scales
__global__ void __launch_bounds__(kSvidThreads) svid_subtract_kernel(float *__restrict__ X, int64_t n, int64_t m,
                                                                     const uint16_t *s_out, const uint16_t *s_in)
{
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n * m;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = idx / m, j = idx - i * m;
        const float x = X[idx];
        const float r = h2f(s_out[i]) * h2f(s_in[j]);
        X[idx] = x < 0.f ? x + r : x - r;
    }
}

__global__ void svid_fill_kernel(float *__restrict__ p, int64_t count, float value)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[i] = value;
}

int sms_count()
{
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    return (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) ? v : 148;
}

}  // namespace

// Scratch: u [n], v [m], packed signs [n][ceil(m/32)], 2 iters + 2 norm slots.
size_t svid_scratch_bytes(int64_t n, int64_t m, int iters)
{
    return align_up(static_cast<size_t>(n) * 4, 256) + align_up(static_cast<size_t>(m) * 4, 256) +
           align_up(static_cast<size_t>(n) * pitch_words(m) * 4, 256) +
           align_up(static_cast<size_t>(2 * iters + 2) * 4, 256);
}

cudaError_t svid_run(float *X, int64_t n, int64_t m, int iters, int subtract, uint32_t *signs, int64_t signs_ld,
                     uint16_t *s_out, uint16_t *s_in, void *scratch, cudaStream_t s)
{
    char *p = static_cast<char *>(scratch);
    float *u = reinterpret_cast<float *>(p);
    p += align_up(static_cast<size_t>(n) * 4, 256);
    float *v = reinterpret_cast<float *>(p);
    p += align_up(static_cast<size_t>(m) * 4, 256);
    uint32_t *packed = reinterpret_cast<uint32_t *>(p);
    p += align_up(static_cast<size_t>(n) * pitch_words(m) * 4, 256);
    float *norms = reinterpret_cast<float *>(p);
    const int sms = sms_count();
    cudaError_t e;
    // signs first: the subtraction below changes X
    if ((e = launch_pack(X, DBF_F32, n, m, packed, nullptr, s)) != cudaSuccess) return e;
    const size_t pw = static_cast<size_t>(pitch_words(m)) * 4;
    if ((e = cudaMemcpy2DAsync(signs, static_cast<size_t>(signs_ld) * 4, packed, pw, pw, static_cast<size_t>(n),
                               cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
        return e;
    if ((e = cudaMemsetAsync(norms, 0, static_cast<size_t>(2 * iters + 2) * 4, s)) != cudaSuccess) return e;
    svid_fill_kernel<<<(m + 255) / 256 < sms * 4 ? static_cast<int>((m + 255) / 256) : sms * 4, 256, 0, s>>>(
        v, m, 1.0f / sqrtf(static_cast<float>(m)));
    const int rows_grid = static_cast<int>((n * 32 + kSvidThreads - 1) / kSvidThreads < sms * 16
                                               ? (n * 32 + kSvidThreads - 1) / kSvidThreads
                                               : sms * 16);
    const dim3 cols_grid(static_cast<unsigned>((m + kSvidThreads - 1) / kSvidThreads),
                         static_cast<unsigned>((n + kBandRows - 1) / kBandRows));
    const float *vnorm = nullptr;   // the start vector is unit length
    for (int it = 0; it < iters; ++it) {
        float *nu = norms + 2 * it, *nv = norms + 2 * it + 1;
        svid_rows_kernel<<<rows_grid, kSvidThreads, 0, s>>>(X, n, m, v, vnorm, u, nu);
        if ((e = cudaMemsetAsync(v, 0, static_cast<size_t>(m) * 4, s)) != cudaSuccess) return e;
        svid_cols_kernel<<<cols_grid, kSvidThreads, 0, s>>>(X, n, m, u, nu, v);
        svid_norm_kernel<<<sms, kSvidThreads, 0, s>>>(v, m, nv);
        vnorm = nv;
    }
    svid_scales_kernel<<<sms, kSvidThreads, 0, s>>>(u, n, norms + 2 * (iters - 1), v, m, norms + 2 * (iters - 1) + 1,
                                                   s_out, s_in);
    if (subtract) svid_subtract_kernel<<<sms * 8, kSvidThreads, 0, s>>>(X, n, m, s_out, s_in);
    return cudaGetLastError();
}

}  // namespace dbf
