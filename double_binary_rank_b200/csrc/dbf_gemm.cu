// Prefill-regime forward on the 5th-generation tensor cores (tcgen05).
//
// LoRDBA page, section 2 ("Kernel de Inferencia"): two sign-accumulation
// products with per-channel scaling between them; with many tokens each
// product is a dense contraction, so it runs as a GEMM:
//   stage 1:  h[r, (i,t)] = sum_m B2[r, m] u_i[t, m],  u_i = fp16(gamma_i . x_t)
//             v[t, i R + r] = fp16(beta_i[r] h[r, (i,t)])
//   stage 2:  y[t, n] = [acc] y[t, n] + sum_{i,r} (alpha_i[n] B1[n, r]) v[t, i R + r]
// In stage 2 the envelope sum is one longer contraction (K = ell R) whose A
// operand is the exact fp16 product alpha_i[n] * (+-1).
//
// One CTA computes a 128 x 256 tile of D = A B^T (A: 128 sign rows, B: 256
// token rows) with the accumulator in tensor memory:
//   warp 0      TMA producer: fp16 activation tiles (64 K x 256 rows, 128-byte
//               swizzle) into a 4-stage ring;
//   warp 1      allocates 256 TMEM columns; one thread issues tcgen05.mma
//               (M = 128, N = 256, K = 16) and commits each stage back;
//   warps 2..5  one sign row per thread: the packed words are streamed with
//               cp.async into a private ring 7 pairs of K steps ahead and
//               expanded to exact fp16 +-1 (or +-alpha) pairs -- a shift and
//               one LOP3 per two signs, the packed layout keeping columns 2p and
//               2p+1 in bits p and 16+p -- written in the same 128-byte swizzled
//               K-major layout; after the K loop the same warps read the
//               accumulator back (tcgen05.ld) and run the epilogue.
// Every wait is bounded; on expiry the CTA records DBF_ERR_TIMEOUT, stops
// issuing work, and still frees its tensor memory.
#include "dbf_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace dbf {
namespace {

constexpr int BM = 128;             // sign rows per tile (MMA M)
constexpr int BN = 256;             // token rows per tile (MMA N)
constexpr int BK = 64;              // K per stage: one 128-byte swizzle row of fp16
constexpr int STAGES = 4;
constexpr int kThreads = 192;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int B_BYTES = BN * BK * 2;   // 32 KB
constexpr int RING = 8;                // cp.async ring slots per expansion thread (16 B each)
constexpr int TMEM_COLS = 256;
constexpr unsigned long long kWaitNs = 1000000000ull;   // bounded waits: 1 s

struct GemmArgs {
    // A operand: packed sign rows
    const uint32_t *signs;
    int pitch;          // words per packed row
    int P;              // sign rows (R for stage 1, N for stage 2)
    int Kp;             // columns per envelope block of K (M for stage 1, R for stage 2)
    int Ktot;           // total K (M, or ell R)
    const uint16_t *arow_scale;   // stage 2: alpha [ell][N]; stage 1: null (+-1)
    int C;              // token rows of B
    int stage;
    // stage 1 epilogue: v
    __half *V;          // [T][ell R]
    const uint16_t *beta;   // [ell][R]
    int T, ell, R;
    // stage 2 epilogue: y
    void *y;
    dbf_dtype yd;
    int N;
    int accumulate;
    int32_t *status;
};

// ---- small PTX helpers --------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void bar_init(uint64_t *bar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void bar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void bar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool bar_try(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait; false (and the abort flag raised) when the limit passes or
// another role already aborted.
__device__ __forceinline__ bool bar_wait(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    if (bar_try(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (bar_try(bar, parity)) return true;
        if (*abort) return false;
        if (global_ns() - t0 > kWaitNs) {
            *abort = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), version 1 (sm_100).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);           // start address
    d |= static_cast<uint64_t>(1u) << 16;                           // leading byte offset (unused here)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;                   // stride byte offset
    d |= static_cast<uint64_t>(1u) << 46;                           // descriptor version
    d |= static_cast<uint64_t>(2u) << 61;                           // swizzle: 128 bytes
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, fp16 A and B, both
// K-major, N = BN, M = BM.
constexpr uint32_t kIdesc = (1u << 4) | (static_cast<uint32_t>(BN >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// fp16 pair of in-word columns (2p, 2p+1) from bits p and 16+p: the sign bits
// land on bits 15 and 31 and are xored into the pair's magnitude pattern.
__device__ __forceinline__ uint32_t sign_pair(uint32_t w, int p, uint32_t mag2)
{
    return ((w << (15 - p)) & 0x80008000u) ^ mag2;
}

struct GemmSmem {
    uint64_t full_a[STAGES], full_b[STAGES], empty[STAGES], acc_full;
    uint32_t tmem_base;
    int abort;
};

__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ CUtensorMap tmB, const GemmArgs g)
{
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *smA = smem;
    uint8_t *smB = smA + STAGES * A_BYTES;
    uint4 *ring = reinterpret_cast<uint4 *>(smB + STAGES * B_BYTES);   // [RING][128]
    GemmSmem *sh = reinterpret_cast<GemmSmem *>(ring + RING * BM);
    volatile int *abort = &sh->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int p0 = blockIdx.x * BM;    // first sign row
    const int c0 = blockIdx.y * BN;    // first token row
    const int nk = g.Ktot / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            bar_init(&sh->full_a[s], 128);
            bar_init(&sh->full_b[s], 1);
            bar_init(&sh->empty[s], 1);
        }
        bar_init(&sh->acc_full, 1);
        sh->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh->tmem_base)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            for (int s = 0; s < nk; ++s) {
                const int st = s % STAGES;
                if (!bar_wait(&sh->empty[st], ((s / STAGES) & 1) ^ 1, abort)) break;
                bar_expect_tx(&sh->full_b[st], B_BYTES);
                tma_load_2d(smB + st * B_BYTES, &tmB, s * BK, c0, &sh->full_b[st]);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool ok = true;
            for (int s = 0; s < nk && ok; ++s) {
                const int st = s % STAGES;
                const uint32_t ph = (s / STAGES) & 1;
                ok = bar_wait(&sh->full_a[st], ph, abort) && bar_wait(&sh->full_b[st], ph, abort);
                if (!ok) break;
                tc_fence_after();
                const uint64_t da = sw128_desc(smem_u32(smA + st * A_BYTES));
                const uint64_t db = sw128_desc(smem_u32(smB + st * B_BYTES));
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)   // 32 bytes of K per MMA: +2 in 16-byte units
                    mma_f16(tmem, da + 2 * kk, db + 2 * kk, (s | kk) != 0);
                mma_commit(&sh->empty[st]);
            }
            mma_commit(&sh->acc_full);   // also after an abort: completes once issued MMAs are done
        }
    } else {
        // ---------------- sign expansion, then epilogue ----------------
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int prow = q * 32 + lane;         // tile row of this thread
        const int grow = p0 + prow;             // sign row
        const bool valid = grow < g.P;
        const uint32_t *srow = g.signs + static_cast<int64_t>(valid ? grow : 0) * g.pitch;
        // cp.async ring: slot j holds the 4 words (2 K steps) of pair j mod RING
        const int npairs = (nk + 1) / 2;
        auto issue = [&](int pr) {
            if (pr < npairs) {
                const int k = pr * 2 * BK;      // first column of the pair
                const int env = k / g.Kp, kk = k - env * g.Kp;
                cp_async16(&ring[(pr % RING) * BM + prow], srow + kk / 32);
            }
            cp_async_commit();
        };
#pragma unroll
        for (int pr = 0; pr < RING - 1; ++pr) issue(pr);
        uint32_t mag_env = 0x3C003C00u;   // +-1
        int cur_env = -1;
        for (int s = 0; s < nk; ++s) {
            const int st = s % STAGES;
            if ((s & 1) == 0) cp_async_wait<RING - 2>();   // pair s/2 has landed
            const uint4 w4 = ring[((s >> 1) % RING) * BM + prow];
            if (s & 1) issue((s >> 1) + RING - 1);        // refill the slot consumed last
            const int env = (s * BK) / g.Kp;
            if (env != cur_env) {
                cur_env = env;
                if (g.arow_scale) {
                    const uint32_t a = valid ? __ldg(g.arow_scale + static_cast<int64_t>(env) * g.N + grow) : 0u;
                    mag_env = a | (a << 16);
                }
            }
            const uint32_t w0 = valid ? ((s & 1) ? w4.z : w4.x) : 0u;
            const uint32_t w1 = valid ? ((s & 1) ? w4.w : w4.y) : 0u;
            const uint32_t mag = valid ? mag_env : 0u;
            if (!bar_wait(&sh->empty[st], ((s / STAGES) & 1) ^ 1, abort)) break;
            uint8_t *arow = smA + st * A_BYTES + prow * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j) {   // 16-byte chunk j: columns 8j..8j+7
                const uint32_t w = j < 4 ? w0 : w1;
                const int pb = 4 * (j & 3);
                uint4 v;
                v.x = valid ? sign_pair(w, pb + 0, mag) : 0u;
                v.y = valid ? sign_pair(w, pb + 1, mag) : 0u;
                v.z = valid ? sign_pair(w, pb + 2, mag) : 0u;
                v.w = valid ? sign_pair(w, pb + 3, mag) : 0u;
                *reinterpret_cast<uint4 *>(arow + ((j ^ (prow & 7)) << 4)) = v;
            }
            fence_proxy_async();   // generic-proxy writes -> visible to the tensor core
            bar_arrive(&sh->full_a[st]);
        }
        cp_async_wait<0>();

        // ---------------- epilogue ----------------
        if (bar_wait(&sh->acc_full, 0, abort)) {
            tc_fence_after();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
            if (g.stage == 1) {
                // column c = i T + t; v[t, i R + r] = fp16(beta_i[r] h)
                const int r = grow;
                for (int cc = 0; cc < BN; cc += 16) {
                    uint32_t v[16];
                    tmem_ld16(taddr + cc, v);
                    if (r < g.R) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int c = c0 + cc + e;
                            if (c < g.C) {
                                const int i = c / g.T, t = c - i * g.T;
                                const float b = h2f(g.beta[static_cast<int64_t>(i) * g.R + r]);
                                g.V[static_cast<int64_t>(t) * g.ell * g.R + static_cast<int64_t>(i) * g.R + r] =
                                    __float2half_rn(b * __uint_as_float(v[e]));
                            }
                        }
                    }
                }
            } else {
                const int n = grow;
                for (int cc = 0; cc < BN; cc += 16) {
                    uint32_t v[16];
                    tmem_ld16(taddr + cc, v);
                    if (n < g.N) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int t = c0 + cc + e;
                            if (t < g.C) {
                                const int64_t idx = static_cast<int64_t>(t) * g.N + n;
                                float yv = __uint_as_float(v[e]);
                                if (g.accumulate) yv += load_act(g.y, g.yd, idx);
                                store_act(g.y, g.yd, idx, yv);
                            }
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (sh->abort && threadIdx.x == 0 && g.status) atomicExch(g.status, static_cast<int32_t>(DBF_ERR_TIMEOUT));
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}

// u[(i T + t), m] = fp16(gamma_i[m] x[t, m])
__global__ void __launch_bounds__(256) scale_cast_kernel(const void *x, dbf_dtype xd, const uint16_t *gamma, int M,
                                                         int T, int ell, __half *U)
{
    const int64_t total = static_cast<int64_t>(ell) * T * M;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = idx / M;
        const int m = static_cast<int>(idx - row * M);
        const int i = static_cast<int>(row / T);
        const int64_t t = row - static_cast<int64_t>(i) * T;
        U[idx] = __float2half_rn(h2f(gamma[static_cast<int64_t>(i) * M + m]) * load_act(x, xd, t * M + m));
    }
}

// ---- host side ----------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D fp16 map of a [rows x K] row-major matrix, boxes of 64 K x 256 rows.
bool make_map(CUtensorMap *map, const void *base, int64_t K, int64_t rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {BK, BN};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kGemmSmem = 1024 + STAGES * (A_BYTES + B_BYTES) + RING * BM * 16 + sizeof(GemmSmem) + 64;

cudaError_t launch_gemm(const CUtensorMap &map, const GemmArgs &a, cudaStream_t s)
{
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kGemmSmem));
        if (e != cudaSuccess) return e;
        configured = true;
    }
    dim3 grid((a.P + BM - 1) / BM, (a.C + BN - 1) / BN);
    gemm_kernel<<<grid, kThreads, kGemmSmem, s>>>(map, a);
    return cudaGetLastError();
}

size_t u_bytes(const dbf_layer &L, int64_t T) { return align_up(static_cast<size_t>(L.ell) * T * L.M * 2, 256); }
size_t v_bytes(const dbf_layer &L, int64_t T) { return align_up(static_cast<size_t>(T) * L.ell * L.R * 2, 256); }

}  // namespace

bool gemm_shape_ok(const dbf_layer &L)
{
    return L.M % 128 == 0 && L.R % 128 == 0 && L.M > 0 && L.R > 0 && L.N > 0;
}

size_t gemm_workspace_bytes(const dbf_layer &L, int64_t T) { return u_bytes(L, T) + v_bytes(L, T); }

cudaError_t gemm_forward(const dbf_layer &L, const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                         int flags, void *ws, cudaStream_t s)
{
    if (T > (1 << 30) / L.ell) return cudaErrorInvalidValue;
    __half *U = static_cast<__half *>(ws);
    __half *V = reinterpret_cast<__half *>(static_cast<char *>(ws) + u_bytes(L, T));
    const int Ti = static_cast<int>(T);
    {
        const int64_t total = static_cast<int64_t>(L.ell) * T * L.M;
        int64_t blocks = (total + 255) / 256;
        if (blocks > 148 * 32) blocks = 148 * 32;
        scale_cast_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(x, xd, L.gamma, L.M, Ti, L.ell, U);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mu, mv;
    if (!make_map(&mu, U, L.M, static_cast<int64_t>(L.ell) * T)) return cudaErrorInvalidValue;
    if (!make_map(&mv, V, static_cast<int64_t>(L.ell) * L.R, T)) return cudaErrorInvalidValue;
    GemmArgs a1 = {};
    a1.signs = L.b2_packed;
    a1.pitch = static_cast<int>(pitch_words(L.M));
    a1.P = L.R;
    a1.Kp = L.M;
    a1.Ktot = L.M;
    a1.arow_scale = nullptr;
    a1.C = L.ell * Ti;
    a1.stage = 1;
    a1.V = V;
    a1.beta = L.beta;
    a1.T = Ti;
    a1.ell = L.ell;
    a1.R = L.R;
    a1.N = L.N;
    cudaError_t e = launch_gemm(mu, a1, s);
    if (e != cudaSuccess) return e;
    GemmArgs a2 = {};
    a2.signs = L.b1_packed;
    a2.pitch = static_cast<int>(pitch_words(L.R));
    a2.P = L.N;
    a2.Kp = L.R;
    a2.Ktot = L.ell * L.R;
    a2.arow_scale = L.alpha;
    a2.C = Ti;
    a2.stage = 2;
    a2.T = Ti;
    a2.ell = L.ell;
    a2.R = L.R;
    a2.y = y;
    a2.yd = yd;
    a2.N = L.N;
    a2.accumulate = (flags & DBF_ACCUMULATE) ? 1 : 0;
    return launch_gemm(mv, a2, s);
}

}  // namespace dbf
