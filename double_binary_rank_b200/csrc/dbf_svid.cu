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
// One power iteration is u = |X| v_hat, then v = |X|^T u. When a row of X is
// at most 12288 floats (a multiple of 4, 16-byte aligned) one persistent
// kernel does both from a single read of X: each CTA streams bands of whole
// rows into shared memory with bulk copies (a ring of two buffers, mbarrier
// completion), forms u for the band's rows by a block reduction, then adds
// |X_band|^T u_band into per-thread registers (a thread owns fixed columns),
// and flushes them with vector atomics at the end. Otherwise two kernels
// read X once each (rows: a warp per row; columns: a thread per column over
// a band of rows, atomics across bands). HBM-bound either way.
#include "dbf_internal.cuh"

namespace dbf {
namespace {

constexpr int kSvidThreads = 256;
constexpr int kBandRows = 128;   // rows per band of the two-pass column kernel

// ---- two-pass iteration -----------------------------------------------------

// u[i] = sum_j |X[i, j]| v[j] * vs, vs = rsqrt(norm2_in) (1 when norm2_in is null);
// norm2_out += |u|^2. Four loads of the row in flight per lane.
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
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        int64_t j = lane;
        for (; j + 96 < m; j += 128) {
            const float x0 = row[j], x1 = row[j + 32], x2 = row[j + 64], x3 = row[j + 96];
            a0 += fabsf(x0) * v[j];
            a1 += fabsf(x1) * v[j + 32];
            a2 += fabsf(x2) * v[j + 64];
            a3 += fabsf(x3) * v[j + 96];
        }
        for (; j < m; j += 32) a0 += fabsf(row[j]) * v[j];
        float acc = (a0 + a1) + (a2 + a3);
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

// ---- single-read iteration --------------------------------------------------

constexpr int kFuseThreads = 256;
constexpr int kFuseWarps = kFuseThreads / 32;
constexpr int64_t kFuseMaxCols = 12288;         // 12 float4 columns per thread
constexpr int kFuseMaxBand = 16;                // rows per band
constexpr int kFuseStages = 2;                  // band buffers in the ring
// Converged power iteration (single-read path): the unit vectors v_in / |v_in|
// and v_prev / |v_prev| of two successive iterations agree to within this in
// every element; the remaining iterations then pass v on unchanged.
constexpr float kSvidTol = 1e-6f;
constexpr size_t kFuseBufBudget = 200 * 1024;   // bytes of all band buffers
constexpr unsigned long long kWaitNs = 2000000000ull;   // bounded waits: 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void bar_init(uint64_t *bar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Expect 'bytes' on the barrier, then bulk-copy them (16-byte aligned ends,
// a multiple of 16 bytes) in pieces of at most 32 KB. One thread.
__device__ __forceinline__ void band_copy(float *dst, const float *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
    for (uint32_t off = 0; off < bytes; off += 32768u)
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                smem_u32(reinterpret_cast<char *>(dst) + off)),
            "l"(reinterpret_cast<const char *>(src) + off), "r"(min(32768u, bytes - off)), "r"(smem_u32(bar))
            : "memory");
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase 'parity' of the barrier; false if kWaitNs passed first.
__device__ __forceinline__ bool bar_wait(uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_u32(bar);
    const unsigned long long t0 = global_ns();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
        if (global_ns() - t0 > kWaitNs) return false;
    }
}

__device__ __forceinline__ float dot_abs(float4 x, float4 v)
{
    return fabsf(x.x) * v.x + fabsf(x.y) * v.y + fabsf(x.z) * v.z + fabsf(x.w) * v.w;
}

__device__ __forceinline__ void fma_abs(float4 &a, float4 x, float s)
{
    a.x += fabsf(x.x) * s;
    a.y += fabsf(x.y) * s;
    a.z += fabsf(x.z) * s;
    a.w += fabsf(x.w) * s;
}

// One power iteration from one read of X: v_hat = v_in / |v_in| (each CTA
// sums |v_in|^2 itself, in the same order), u = |X| v_hat (stored, |u|^2
// added to *norm2_u), v_out += |X|^T u (v_out zero before). v_clear (the
// accumulator of the iteration after next) is zeroed on the way. Thread t
// owns columns 4t + 1024c, c < NCH. CTA b takes bands b, b + grid, ... of
// 'band' rows through a ring of kFuseStages buffers, so kFuseStages - 1
// bands are in flight while one is reduced. Launched as a programmatic
// dependent of the previous iteration: the bands of X (read only) are
// requested before the wait for the previous iteration's v. A band wait that
// times out makes every thread of the CTA stop (decided together), wait
// (bounded) for the copies still in flight, and add NaN to *norm2_u and
// v_out[0], so the scales come out NaN: the result is visibly void.
template <int NCH>
__global__ void __launch_bounds__(kFuseThreads, 1)
    svid_iter_kernel(const float *__restrict__ X, int64_t n, int m, int band, const float *__restrict__ v_in,
                     float *__restrict__ v_out, float *__restrict__ v_clear, float *__restrict__ u, float *norm2_u,
                     const float *__restrict__ v_prev, int *count, int *conv, int prefetch_early)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const size_t buf_floats = static_cast<size_t>(band) * m;
    float *bufs = reinterpret_cast<float *>(smem);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kFuseStages * buf_floats * sizeof(float));
    float *red = reinterpret_cast<float *>(bar + kFuseStages);   // [kFuseWarps][kFuseMaxBand]
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t nb = (n + band - 1) / band;
    const int64_t grid = gridDim.x;

    // band j of this CTA (b = blockIdx.x + j grid) goes to buffer j % S as
    // that buffer's (j / S)-th fill: its wait parity is (j / S) & 1
    auto issue = [&](int64_t j) {
        const int64_t b = blockIdx.x + j * grid;
        if (b >= nb) return;
        const int64_t r0 = b * band;
        const int64_t rows = n - r0 < band ? n - r0 : band;
        band_copy(bufs + (j % kFuseStages) * buf_floats, X + r0 * m, static_cast<uint32_t>(rows * m * 4),
                  &bar[j % kFuseStages]);
    };

    // the first iterations fetch their first bands while the previous kernel
    // still runs; later ones first look whether an earlier iteration found
    // the iterate converged (then they read no band at all)
    if (tid == 0) {
        for (int st = 0; st < kFuseStages; ++st) bar_init(&bar[st], 1);
        if (prefetch_early)
            for (int st = 0; st < kFuseStages; ++st) issue(st);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");   // v_in complete, v_clear no longer read
    __syncthreads();

    for (int64_t j = static_cast<int64_t>(blockIdx.x) * kFuseThreads + tid; j < m; j += grid * kFuseThreads)
        v_clear[j] = 0.f;
    if (!prefetch_early) {
        int f = 0;
        if (tid == 0) f = *reinterpret_cast<volatile int *>(conv);
        if (__syncthreads_or(f)) {
            for (int64_t j = static_cast<int64_t>(blockIdx.x) * kFuseThreads + tid; j < m; j += grid * kFuseThreads)
                v_out[j] = v_in[j];
            if (blockIdx.x == 0 && tid == 0) *norm2_u = *(norm2_u - 2);
            asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
            return;
        }
        if (tid == 0)
            for (int st = 0; st < kFuseStages; ++st) issue(st);
    }

    float4 vh[NCH], acc[NCH];
    float sq = 0.f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int col = 4 * tid + 1024 * c;
        vh[c] = col < m ? *reinterpret_cast<const float4 *>(v_in + col) : make_float4(0.f, 0.f, 0.f, 0.f);
        acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        sq += vh[c].x * vh[c].x + vh[c].y * vh[c].y + vh[c].z * vh[c].z + vh[c].w * vh[c].w;
    }
    for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) red[wid] = sq;
    __syncthreads();
    float n2 = 0.f;
#pragma unroll
    for (int w = 0; w < kFuseWarps; ++w) n2 += red[w];
    const float vs = rsqrtf(n2);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        vh[c].x *= vs;
        vh[c].y *= vs;
        vh[c].z *= vs;
        vh[c].w *= vs;
    }
    __syncthreads();   // red is reused below

    if (v_prev) {
        // converged? v_prev is the previous iteration's input: every CTA
        // reads the same vectors and reduces them in the same order, so all
        // of them take the same decision
        float4 vp[NCH];
        float psq = 0.f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int col = 4 * tid + 1024 * c;
            vp[c] = col < m ? *reinterpret_cast<const float4 *>(v_prev + col) : make_float4(0.f, 0.f, 0.f, 0.f);
            psq += vp[c].x * vp[c].x + vp[c].y * vp[c].y + vp[c].z * vp[c].z + vp[c].w * vp[c].w;
        }
        for (int o = 16; o; o >>= 1) psq += __shfl_xor_sync(0xffffffffu, psq, o);
        if (lane == 0) red[wid] = psq;
        __syncthreads();
        float p2 = 0.f;
#pragma unroll
        for (int w = 0; w < kFuseWarps; ++w) p2 += red[w];
        const float ps = rsqrtf(p2);
        float d = 0.f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            d = fmaxf(d, fabsf(vh[c].x - vp[c].x * ps));
            d = fmaxf(d, fabsf(vh[c].y - vp[c].y * ps));
            d = fmaxf(d, fabsf(vh[c].z - vp[c].z * ps));
            d = fmaxf(d, fabsf(vh[c].w - vp[c].w * ps));
        }
        for (int o = 16; o; o >>= 1) d = fmaxf(d, __shfl_xor_sync(0xffffffffu, d, o));
        __syncthreads();   // every warp has read its p2 terms
        if (lane == 0) red[wid] = d;
        __syncthreads();
        float dmax = 0.f;
#pragma unroll
        for (int w = 0; w < kFuseWarps; ++w) dmax = fmaxf(dmax, red[w]);
        if (dmax <= kSvidTol) {
            // pass the iterate on: v_out = v_in, |u|^2 as before (u itself is
            // unchanged), and tell the later iterations; the band copies
            // issued above land before the exit
            if (blockIdx.x == 0 && tid == 0) *conv = 1;
            if (tid == 0)
                for (int64_t j = 0; j < kFuseStages; ++j)
                    if (blockIdx.x + j * grid < nb) bar_wait(&bar[j], 0u);
            for (int64_t j = static_cast<int64_t>(blockIdx.x) * kFuseThreads + tid; j < m; j += grid * kFuseThreads)
                v_out[j] = v_in[j];
            if (blockIdx.x == 0 && tid == 0) *norm2_u = *(norm2_u - 2);
            asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
            return;
        }
        __syncthreads();   // red is reused below
    }
    if (blockIdx.x == 0 && tid == 0) atomicAdd(count, 1);   // iterations that ran

    float usq = 0.f;
    bool ok = true;
    int64_t k = 0;
    int64_t b = blockIdx.x;
    for (; b < nb; b += grid, ++k) {
        const int st = static_cast<int>(k % kFuseStages);
        const bool done = bar_wait(&bar[st], static_cast<uint32_t>((k / kFuseStages) & 1));
        if (__syncthreads_or(!done)) {
            ok = false;
            break;
        }
        const int64_t r0 = b * band;
        const int rows = static_cast<int>(n - r0 < band ? n - r0 : band);
        const float *xb = bufs + st * buf_floats;
        for (int r = 0; r < rows; ++r) {
            const float *xr = xb + static_cast<size_t>(r) * m;
            float p = 0.f;
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const int col = 4 * tid + 1024 * c;
                if (col < m) p += dot_abs(*reinterpret_cast<const float4 *>(xr + col), vh[c]);
            }
            for (int o = 16; o; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            if (lane == 0) red[wid * kFuseMaxBand + r] = p;
        }
        __syncthreads();
        for (int r = 0; r < rows; ++r) {
            float ur = 0.f;
#pragma unroll
            for (int w = 0; w < kFuseWarps; ++w) ur += red[w * kFuseMaxBand + r];
            if (tid == 0) {
                u[r0 + r] = ur;
                usq += ur * ur;
            }
            const float *xr = xb + static_cast<size_t>(r) * m;
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const int col = 4 * tid + 1024 * c;
                if (col < m) fma_abs(acc[c], *reinterpret_cast<const float4 *>(xr + col), ur);
            }
        }
        __syncthreads();   // buffer st and red are free again
        if (tid == 0) issue(k + kFuseStages);
    }
    if (!ok) {
        // in flight: the copies of bands k .. k + S - 1 that exist (band k is
        // the failed wait)
        if (tid == 0) {
            for (int64_t j = k; j < k + kFuseStages; ++j)
                if (blockIdx.x + j * grid < nb)
                    bar_wait(&bar[j % kFuseStages], static_cast<uint32_t>((j / kFuseStages) & 1));
            const float nan = __int_as_float(0x7fffffff);
            atomicAdd(norm2_u, nan);
            atomicAdd(v_out, nan);   // poisons every later iteration and the scales
        }
        return;
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int col = 4 * tid + 1024 * c;
        if (col < m) atomicAdd(reinterpret_cast<float4 *>(v_out + col), acc[c]);
    }
    if (tid == 0 && usq != 0.f) atomicAdd(norm2_u, usq);
}

// Final scales from the last iteration's u (|u|^2 = *norm2_u) and v
// (|v|^2 = *norm2_v). Two-pass path: v = |X|^T u_hat, so sigma = |v|.
// Single-read path (v_times_u): v = |X|^T u = |u| |X|^T u_hat, so
// sigma = |v| / |u|. s_out = sqrt(sigma) u_hat, s_in = (|X|^T u_hat) /
// sqrt(sigma). fp16 and/or fp32 outputs (null ones are skipped).
__global__ void __launch_bounds__(kSvidThreads) svid_scales_kernel(const float *__restrict__ u, int64_t n,
                                                                   const float *norm2_u, const float *__restrict__ v,
                                                                   int64_t m, const float *norm2_v, int v_times_u,
                                                                   uint16_t *s_out, uint16_t *s_in, float *s_out32,
                                                                   float *s_in32)
{
    const float nu = sqrtf(*norm2_u), nv = sqrtf(*norm2_v);
    const float sigma = v_times_u ? nv / nu : nv;
    const float r = sqrtf(sigma);
    const float cu = r / nu, cv = v_times_u ? 1.f / (r * nu) : 1.f / r;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n + m;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (i < n) {
            const float a = cu * u[i];
            if (s_out) s_out[i] = __half_as_ushort(__float2half_rn(a));
            if (s_out32) s_out32[i] = a;
        } else {
            const float b = cv * v[i - n];
            if (s_in) s_in[i - n] = __half_as_ushort(__float2half_rn(b));
            if (s_in32) s_in32[i - n] = b;
        }
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

// rows per band of the single-read kernel, 0 when it does not apply
int fuse_band(const float *X, int64_t m)
{
    if (m % 4 != 0 || m > kFuseMaxCols || (reinterpret_cast<uintptr_t>(X) & 15) != 0) return 0;
    const int64_t b = static_cast<int64_t>(kFuseBufBudget) / (kFuseStages * 4 * m);
    return static_cast<int>(b < kFuseMaxBand ? b : kFuseMaxBand);
}

// v_prev: the previous iteration's input (its norm slot is two floats
// before norm2_u), or null for the first iteration; count: iterations that
// ran; conv: set once the iterate converged; prefetch_early: fetch the first
// bands before the previous kernel's results are visible (no look at conv)
template <int NCH>
cudaError_t launch_iter(const float *X, int64_t n, int m, int band, const float *v_in, float *v_out, float *v_clear,
                        float *u, float *norm2_u, const float *v_prev, int *count, int *conv, int prefetch_early,
                        int sms, cudaStream_t s)
{
    const size_t smem = kFuseStages * (static_cast<size_t>(band) * m * sizeof(float) + sizeof(uint64_t)) +
                        sizeof(float) * kFuseWarps * kFuseMaxBand;
    cudaError_t e = cudaFuncSetAttribute(svid_iter_kernel<NCH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t nb = (n + band - 1) / band;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(nb < sms ? nb : sms));
    cfg.blockDim = dim3(kFuseThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, svid_iter_kernel<NCH>, X, n, m, band, v_in, v_out, v_clear, u, norm2_u, v_prev,
                              count, conv, prefetch_early);
}

}  // namespace

// Scratch: u [n], four v buffers [m] each, 2 iters + 2 norm slots, the count
// of iterations that ran, the converged flag.
size_t svid_scratch_bytes(int64_t n, int64_t m, int iters)
{
    return align_up(static_cast<size_t>(n) * 4, 256) + 4 * align_up(static_cast<size_t>(m) * 4, 256) +
           align_up(static_cast<size_t>(2 * iters + 4) * 4, 256);
}

// the count slot of a scratch laid out for (n, m, iters)
int *svid_count_slot(void *scratch, int64_t n, int64_t m, int iters)
{
    return reinterpret_cast<int *>(static_cast<char *>(scratch) + align_up(static_cast<size_t>(n) * 4, 256) +
                                   4 * align_up(static_cast<size_t>(m) * 4, 256)) +
           2 * iters + 2;
}

namespace {
__global__ void svid_set_count_kernel(int *count, int v) { *count = v; }
}  // namespace

cudaError_t svid_power(const float *X, int64_t n, int64_t m, int iters, uint16_t *s_out, uint16_t *s_in,
                       float *s_out32, float *s_in32, void *scratch, cudaStream_t s)
{
    char *p = static_cast<char *>(scratch);
    float *u = reinterpret_cast<float *>(p);
    p += align_up(static_cast<size_t>(n) * 4, 256);
    float *vb[4];
    for (int i = 0; i < 4; ++i) {
        vb[i] = reinterpret_cast<float *>(p);
        p += align_up(static_cast<size_t>(m) * 4, 256);
    }
    float *norms = reinterpret_cast<float *>(p);
    const int sms = sms_count();
    cudaError_t e;
    int *count = reinterpret_cast<int *>(norms) + 2 * iters + 2, *conv = count + 1;
    if ((e = cudaMemsetAsync(norms, 0, static_cast<size_t>(2 * iters + 4) * 4, s)) != cudaSuccess) return e;
    const int fill_grid = (m + 255) / 256 < sms * 4 ? static_cast<int>((m + 255) / 256) : sms * 4;
    svid_fill_kernel<<<fill_grid, 256, 0, s>>>(vb[0], m, 1.0f / sqrtf(static_cast<float>(m)));
    const int band = fuse_band(X, m);
    if (band > 0) {
        // iteration it reads vb[it % 4] (and, for the convergence test, its
        // own predecessor's input vb[(it + 3) % 4]), accumulates into
        // vb[(it + 1) % 4] and clears vb[(it + 2) % 4]
        if ((e = cudaMemsetAsync(vb[1], 0, static_cast<size_t>(m) * 4, s)) != cudaSuccess) return e;
        const int mi = static_cast<int>(m);
        for (int it = 0; it < iters; ++it) {
            const float *vin = vb[it % 4], *vprev = it > 0 ? vb[(it + 3) % 4] : nullptr;
            float *vout = vb[(it + 1) % 4], *vclr = vb[(it + 2) % 4];
            float *nu = norms + 2 * it;
            if (m <= 4096) e = launch_iter<4>(X, n, mi, band, vin, vout, vclr, u, nu, vprev, count, conv, it < 2, sms, s);
            else if (m <= 8192) e = launch_iter<8>(X, n, mi, band, vin, vout, vclr, u, nu, vprev, count, conv, it < 2, sms, s);
            else e = launch_iter<12>(X, n, mi, band, vin, vout, vclr, u, nu, vprev, count, conv, it < 2, sms, s);
            if (e != cudaSuccess) return e;
        }
        float *vlast = vb[iters % 4], *nv = norms + 2 * (iters - 1) + 1;
        svid_norm_kernel<<<sms, kSvidThreads, 0, s>>>(vlast, m, nv);
        svid_scales_kernel<<<sms, kSvidThreads, 0, s>>>(u, n, norms + 2 * (iters - 1), vlast, m, nv, 1, s_out, s_in,
                                                       s_out32, s_in32);
        return cudaGetLastError();
    }
    float *v = vb[0];
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
                                                   0, s_out, s_in, s_out32, s_in32);
    svid_set_count_kernel<<<1, 1, 0, s>>>(count, iters);   // the two-pass path runs them all
    return cudaGetLastError();
}

cudaError_t svid_run(float *X, int64_t n, int64_t m, int iters, int subtract, uint32_t *signs, int64_t signs_ld,
                     uint16_t *s_out, uint16_t *s_in, void *scratch, cudaStream_t s)
{
    cudaError_t e;
    // signs first: the subtraction below changes X
    if ((e = launch_pack_ld(X, DBF_F32, n, m, signs, signs_ld, nullptr, s)) != cudaSuccess) return e;
    if ((e = svid_power(X, n, m, iters, s_out, s_in, nullptr, nullptr, scratch, s)) != cudaSuccess) return e;
    if (subtract) svid_subtract_kernel<<<sms_count() * 8, kSvidThreads, 0, s>>>(X, n, m, s_out, s_in);
    return cudaGetLastError();
}

}  // namespace dbf
