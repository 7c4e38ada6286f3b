// Sign packing into the one-bit-per-weight layout of dbf.h.
//
// LoRDBA page, section 2 ("Arquitetura Central": sign carriers at 1 bit per
// weight; training pipeline step 2: B = sign(H)); DBF page, section 2 (the
// factors are {-1, +1} sign matrices).
//
// One warp builds one 32-bit word per step with a single ballot: lane L reads
// the column that bit L of the word holds (bit p < 16 -> column 2p, bit
// 16 + p -> column 2p + 1), so the ballot result is the packed word itself.
// The 32 lanes read one 32-column span of the row, which is contiguous.
#include "dbf_internal.cuh"

namespace dbf {
namespace {

template <typename T>
__device__ __forceinline__ bool is_negative(T v, bool &nan);

template <>
__device__ __forceinline__ bool is_negative<int8_t>(int8_t v, bool &nan)
{
    nan = false;
    return v < 0;
}
template <>
__device__ __forceinline__ bool is_negative<float>(float v, bool &nan)
{
    nan = isnan(v);
    return v < 0.0f;   // -0.0 and NaN compare false -> +1
}
template <>
__device__ __forceinline__ bool is_negative<__half>(__half v, bool &nan)
{
    float f = __half2float(v);
    nan = isnan(f);
    return f < 0.0f;
}
template <>
__device__ __forceinline__ bool is_negative<__nv_bfloat16>(__nv_bfloat16 v, bool &nan)
{
    float f = __bfloat162float(v);
    nan = isnan(f);
    return f < 0.0f;
}

// A work item is a run of up to kPackSeg words of one row (one division per
// item, not per word); the warp issues the loads of U words before their
// ballots so U row segments are in flight at once. Lane u < U stores word u.
constexpr int kPackSeg = 64;

template <typename T>
__global__ void __launch_bounds__(256) pack_kernel(const T *__restrict__ src, int64_t rows,
                                                   int64_t k, uint32_t *__restrict__ dst,
                                                   int64_t dst_ld, int32_t *status)
{
    constexpr int U = sizeof(T) == 1 ? 8 : 4;
    const int lane = threadIdx.x & 31;
    const int64_t pitch = pitch_words(k);
    const int64_t segs = (pitch + kPackSeg - 1) / kPackSeg;
    const int64_t total = rows * segs;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    // column of this lane inside a 32-column word
    const int col = lane < 16 ? 2 * lane : 2 * (lane - 16) + 1;
    bool saw_nan = false;
    for (int64_t item = warp; item < total; item += nwarps) {
        const int64_t row = item / segs;
        const int64_t w0 = (item - row * segs) * kPackSeg;
        const int64_t w1 = w0 + kPackSeg < pitch ? w0 + kPackSeg : pitch;
        const T *rp = src + row * k;
        uint32_t *dp = dst + row * dst_ld;
        for (int64_t w = w0; w < w1; w += U) {
            T v[U];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t c = (w + u) * 32 + col;
                ok[u] = w + u < w1 && c < k;
                v[u] = ok[u] ? rp[c] : T();
            }
            uint32_t mine = 0u;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                bool nan = false, neg = false;
                if (ok[u]) neg = is_negative<T>(v[u], nan);
                saw_nan |= nan;
                const uint32_t word = __ballot_sync(0xffffffffu, neg);
                if (lane == u) mine = word;
            }
            if (lane < U && w + lane < w1) dp[w + lane] = mine;
        }
    }
    if (saw_nan && status) atomicExch(status, static_cast<int32_t>(DBF_ERR_INVALID_ARG));
}

__global__ void __launch_bounds__(256) unpack_kernel(const uint32_t *__restrict__ src, int64_t rows,
                                                     int64_t k, int8_t *__restrict__ dst)
{
    const int64_t pitch = pitch_words(k);
    const int64_t n = rows * k;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = i / k;
        const int64_t c = i - row * k;
        const int j = static_cast<int>(c & 31);
        const int bit = (j & 1) ? 16 + (j >> 1) : (j >> 1);
        const uint32_t word = src[row * pitch + (c >> 5)];
        dst[i] = ((word >> bit) & 1u) ? int8_t(-1) : int8_t(1);
    }
}

// Transpose of a packed sign matrix: src is rows x k (packed along k), dst is
// k x rows (packed along rows). A warp takes one 32 x 32 block: lane L loads
// the src word of row r0 + col(L), where col(L) is the in-word column that
// bit L of a packed word holds; then for each of the block's 32 columns c one
// ballot of "bit of column c is set" is already the dst word of row 32w + c
// (its bit L is old row r0 + col(L)). Rows past 'rows' load as zero, which
// keeps the dst padding bits zero.
__global__ void __launch_bounds__(256) transpose_kernel(const uint32_t *__restrict__ src, int64_t rows,
                                                        int64_t k, uint32_t *__restrict__ dst)
{
    const int lane = threadIdx.x & 31;
    const int64_t sp = pitch_words(k), dp = pitch_words(rows);
    const int64_t nblk = dp * sp;   // (row block, word column) pairs
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int col = lane < 16 ? 2 * lane : 2 * (lane - 16) + 1;
    for (int64_t b = warp; b < nblk; b += nwarps) {
        const int64_t rb = b / sp, w = b - rb * sp;
        const int64_t row = rb * 32 + col;
        const uint32_t word = row < rows ? src[row * sp + w] : 0u;
        uint32_t mine = 0u;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            const int bit = (c & 1) ? 16 + (c >> 1) : (c >> 1);
            const uint32_t t = __ballot_sync(0xffffffffu, (word >> bit) & 1u);
            if (lane == c) mine = t;
        }
        const int64_t nrow = w * 32 + lane;   // dst row = src column
        if (nrow < k) dst[nrow * dp + rb] = mine;
    }
}

// Straight-through estimator on the latents: dH = dB * s'(H) with the
// surrogate s = tanh(H / tau) (tau > 0) or the identity clipped to |H| <= 1.
template <typename T>
__device__ __forceinline__ float latent_value(const T *h, int64_t i);
template <>
__device__ __forceinline__ float latent_value<float>(const float *h, int64_t i) { return h[i]; }
template <>
__device__ __forceinline__ float latent_value<__half>(const __half *h, int64_t i) { return __half2float(h[i]); }
template <>
__device__ __forceinline__ float latent_value<__nv_bfloat16>(const __nv_bfloat16 *h, int64_t i)
{
    return __bfloat162float(h[i]);
}

template <typename T>
__global__ void __launch_bounds__(256) ste_kernel(const float *__restrict__ db, const T *__restrict__ h, int64_t n,
                                                  float tau, float *__restrict__ dh, int accumulate)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float v = latent_value<T>(h, i);
        float d;
        if (tau > 0.f) {
            const float th = tanhf(v / tau);
            d = (1.f - th * th) / tau;
        } else {
            d = fabsf(v) <= 1.f ? 1.f : 0.f;
        }
        const float g = db[i] * d;
        dh[i] = accumulate ? dh[i] + g : g;
    }
}

int grid_for(int64_t work, int per_block)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t g = (work + per_block - 1) / per_block;
    const int64_t cap = static_cast<int64_t>(sms) * 16;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return static_cast<int>(g);
}

}  // namespace

cudaError_t launch_pack(const void *src, dbf_dtype dt, int64_t rows, int64_t k, uint32_t *dst,
                        int32_t *status, cudaStream_t s)
{
    return launch_pack_ld(src, dt, rows, k, dst, pitch_words(k), status, s);
}

cudaError_t launch_pack_ld(const void *src, dbf_dtype dt, int64_t rows, int64_t k, uint32_t *dst,
                           int64_t dst_ld, int32_t *status, cudaStream_t s)
{
    const int64_t items = rows * ((pitch_words(k) + kPackSeg - 1) / kPackSeg);
    const int grid = grid_for(items, 8);   // 8 warps per block, one item each per step
    switch (dt) {
    case DBF_I8:
        pack_kernel<int8_t><<<grid, 256, 0, s>>>(static_cast<const int8_t *>(src), rows, k, dst, dst_ld, status);
        break;
    case DBF_F32:
        pack_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float *>(src), rows, k, dst, dst_ld, status);
        break;
    case DBF_F16:
        pack_kernel<__half><<<grid, 256, 0, s>>>(static_cast<const __half *>(src), rows, k, dst, dst_ld, status);
        break;
    case DBF_BF16:
        pack_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(src), rows, k,
                                                        dst, dst_ld, status);
        break;
    default:
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_ste(const float *db, const void *h, dbf_dtype hd, int64_t n, float tau, float *dh,
                       int accumulate, cudaStream_t s)
{
    const int grid = grid_for(n, 256);
    switch (hd) {
    case DBF_F32: ste_kernel<float><<<grid, 256, 0, s>>>(db, static_cast<const float *>(h), n, tau, dh, accumulate); break;
    case DBF_F16: ste_kernel<__half><<<grid, 256, 0, s>>>(db, static_cast<const __half *>(h), n, tau, dh, accumulate); break;
    case DBF_BF16:
        ste_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(db, static_cast<const __nv_bfloat16 *>(h), n, tau, dh, accumulate);
        break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_transpose(const uint32_t *src, int64_t rows, int64_t k, uint32_t *dst, cudaStream_t s)
{
    const int grid = grid_for(pitch_words(rows) * pitch_words(k), 8);
    transpose_kernel<<<grid, 256, 0, s>>>(src, rows, k, dst);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const uint32_t *src, int64_t rows, int64_t k, int8_t *dst, cudaStream_t s)
{
    const int grid = grid_for(rows * k, 256);
    unpack_kernel<<<grid, 256, 0, s>>>(src, rows, k, dst);
    return cudaGetLastError();
}

}  // namespace dbf
