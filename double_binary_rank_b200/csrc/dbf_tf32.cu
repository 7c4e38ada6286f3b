// Dense fp32 GEMM on the fifth-generation tensor cores, fp32-accurate by
// splitting each operand into a TF32 head and an exact remainder:
// x = hi + lo with hi = x with its low 13 mantissa bits cleared (exactly a
// TF32 value) and lo = x - hi (exact in fp32), and
//     A B^T ~ hi(A) hi(B)^T + hi(A) lo(B)^T + lo(A) hi(B)^T
// accumulated in fp32 in tensor memory (the dropped lo lo term and the TF32
// rounding of lo are below 2^-20 of |a||b| per product; the accumulator's
// round-toward-zero adds a bias of about 3K/8 units of 2^-24).
//
// Cout[M x N] = alpha A B^T + beta Cin, A [M x K] and B [N x K] fp32
// row-major (K contiguous: both operands K-major). The tensor cores read an
// fp32 word as its top 19 bits, so A and B themselves are their hi parts;
// a split pass writes the lo planes of A and B once per call. The three
// products are then one GEMM over K' = 3K: the first third of K' pairs
// (A, B), the second (A, lo B), the third (lo A, B). Persistent kernel, one
// CTA per SM, 128 x BN output tiles in groups of 16 row tiles (so the tiles
// running together share their A and B blocks in L2), 32 fp32 of K per
// pipeline stage (one 128-byte swizzle row):
//   warp 0     TMA: the A and B tiles of a stage from the plane the K'
//              segment names (no multicast);
//   warp 1     allocates 2 BN TMEM columns (two accumulators) and issues four
//              tcgen05.mma.kind::tf32 (M 128, N BN, K 8) per stage;
//   warps 2-5  epilogue: tcgen05.ld 32 columns at a time, alpha acc + beta
//              Cin, stored (or squared and summed for a residual norm).
// Every wait is bounded (1 s); on expiry the CTA stops issuing work, raises
// *status (if given), waits (bounded) for its loads and MMAs in flight and
// still frees its tensor memory.
#include "dbf_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace dbf {
namespace {

constexpr int XM = 128, XK = 32;               // tile rows; 32 fp32 of K = one 128-byte swizzle row
constexpr int kEpiWarps = 4;
constexpr int X_THREADS = 32 * (2 + kEpiWarps);
constexpr int X_A_TILE = XM * XK * 4;          // 16 KB
constexpr int kRasterRows = 16;                // row tiles per raster group
constexpr unsigned long long kWaitNs = 1000000000ull;

// Tile width BN (128 or 256) and pipeline stages S.
template <int BN_, int S_>
struct XCfg {
    static constexpr int BN = BN_, S = S_;
    static constexpr int B_TILE = BN * XK * 4;
    static constexpr int STAGE = X_A_TILE + B_TILE;
    static constexpr int TMEM_COLS = 2 * BN;   // two accumulators
    // Instruction descriptor, kind::tf32: fp32 accumulator (bits 4-5 = 1), A
    // and B TF32 (bits 7-9 and 10-12 = 2), both K-major, N >> 3 at bit 17,
    // M >> 4 at bit 24.
    static constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                       (static_cast<uint32_t>(XM >> 4) << 24);
    static_assert(BN == 128 || BN == 256, "tile width");
    static_assert(1024 + S * STAGE + 256 <= 227 * 1024, "shared memory");
};
using XDefault = XCfg<256, 4>;

struct XArgs {
    int64_t M, N, K;
    float alpha, beta;
    const float *Cin;
    int64_t ldci;
    float *Cout;
    int64_t ldco;
    double *sumsq;     // non-null: add the squares of the results, store nothing
    int vec_c;         // Cin / Cout rows allow float4 access
    int32_t *status;   // optional: DBF_ERR_TIMEOUT on a wait that expired
    int lower;         // M == N: only the tiles that reach the lower triangle (row >= column somewhere)
    float *Cout_lo;    // optional: the lo plane of the result, pitch ldlo
    int64_t ldlo;
};

template <int S>
struct XSmem {
    uint64_t full[S], empty[S], acc_full[2], acc_empty[2], drain;
    uint32_t tmem_base;
    int abort;
};

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

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = bar_wait(bar, parity, abort);
    return __shfl_sync(0xffffffffu, ok, 0);
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart, version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Tiles of a lower-triangle product (M == N, BN = r XM): column tile nt
// holds row tiles r nt .. n_m - 1, the ones whose rows reach its columns
__host__ __device__ __forceinline__ int lower_tiles(int n_m, int n_n, int r)
{
    int t = 0;
    for (int nt = 0; nt < n_n && r * nt < n_m; ++nt) t += n_m - r * nt;
    return t;
}

// Row tile and column tile of tile t: groups of kRasterRows row tiles, row
// tile fastest inside a group; lower-triangle products column by column
// (their operands are a few MB: L2 holds them in any order).
__device__ __forceinline__ void tile_pos(int t, int n_m, int n_n, int &mt, int &nt, int lower = 0, int r = 1)
{
    if (lower) {
        nt = 0;
        for (int c = n_m; t >= c && nt + 1 < n_n; c = n_m - r * nt) {
            t -= c;
            ++nt;
        }
        mt = r * nt + t;
        return;
    }
    const int per_group = kRasterRows * n_n;
    const int grp = t / per_group;
    const int local = t - grp * per_group;
    const int rows = n_m - grp * kRasterRows < kRasterRows ? n_m - grp * kRasterRows : kRasterRows;
    mt = grp * kRasterRows + local % rows;
    nt = local / rows;
}

// 32 result columns c0 .. c0 + 31 of one row: alpha acc + beta Cin, stored or
// squared into sq
__device__ __forceinline__ void epi_chunk(const XArgs &g, int64_t row, int64_t c0, const uint32_t (&v)[32], float &sq)
{
    const int64_t n_ok = g.N - c0;
    if (n_ok <= 0) return;
    const bool full = g.vec_c && n_ok >= 32;
    float out[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) out[e] = g.alpha * __uint_as_float(v[e]);
    if (g.beta != 0.f) {
        const float *cin = g.Cin + row * g.ldci + c0;
        if (full) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 c = *reinterpret_cast<const float4 *>(cin + e);
                out[e] += g.beta * c.x;
                out[e + 1] += g.beta * c.y;
                out[e + 2] += g.beta * c.z;
                out[e + 3] += g.beta * c.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
                if (e < n_ok) out[e] += g.beta * cin[e];
        }
    }
    if (g.sumsq) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (e < n_ok) sq += out[e] * out[e];
        return;
    }
    float *cout = g.Cout + row * g.ldco + c0;
    if (full) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4 *>(cout + e) = make_float4(out[e], out[e + 1], out[e + 2], out[e + 3]);
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (e < n_ok) cout[e] = out[e];
    }
    if (g.Cout_lo) {
        float *clo = g.Cout_lo + row * g.ldlo + c0;
        if (full) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4 *>(clo + e) =
                    make_float4(tf32_lo(out[e]), tf32_lo(out[e + 1]), tf32_lo(out[e + 2]), tf32_lo(out[e + 3]));
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
                if (e < n_ok) clo[e] = tf32_lo(out[e]);
        }
    }
}

// lo = x - (x with its low 13 mantissa bits cleared), rows x cols of a
// row-major matrix with pitch ld into a plane with pitch ldl (both multiples
// of 4; columns up to the next multiple of 4 are processed, which stays
// inside both pitches)
__global__ void split_lo_kernel(const float *__restrict__ x, int64_t rows, int64_t cols4, int64_t ld,
                                float *__restrict__ lo, int64_t ldl)
{
    const int64_t total = rows * cols4;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / cols4, c = (i - r * cols4) * 4;
        const float4 v = *reinterpret_cast<const float4 *>(x + r * ld + c);
        float4 l;
        l.x = tf32_lo(v.x);
        l.y = tf32_lo(v.y);
        l.z = tf32_lo(v.z);
        l.w = tf32_lo(v.w);
        *reinterpret_cast<float4 *>(lo + r * ldl + c) = l;
    }
}

template <class Cfg>
__global__ void __launch_bounds__(X_THREADS, 1)
    tf32x3_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAl,
                  const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmBl,
                  const __grid_constant__ XArgs g)
{
    constexpr int S = Cfg::S, BN = Cfg::BN, B_TILE = Cfg::B_TILE, STAGE = Cfg::STAGE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    XSmem<S> *sh = reinterpret_cast<XSmem<S> *>(smem + S * STAGE);
    volatile int *abort = &sh->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_m = static_cast<int>((g.M + XM - 1) / XM);
    const int n_n = static_cast<int>((g.N + BN - 1) / BN);
    const int ntiles = g.lower ? lower_tiles(n_m, n_n, BN / XM) : n_m * n_n;
    const int my_tiles = static_cast<int>(blockIdx.x) < ntiles ? (ntiles - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;
    const int nk = static_cast<int>((g.K + XK - 1) / XK);
    const int nk3 = 3 * nk;   // stages per tile: K' = 3K

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            bar_init(&sh->full[i], 1);
            bar_init(&sh->empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            bar_init(&sh->acc_full[i], 1);
            bar_init(&sh->acc_empty[i], kEpiWarps);
        }
        bar_init(&sh->drain, 1);
        sh->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmAl) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmBl) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh->tmem_base)),
                     "r"(Cfg::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int s = 0;
            for (int j = 0; j < my_tiles && !*abort; ++j) {
                int mt, nt;
                tile_pos(static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x), n_m, n_n, mt, nt, g.lower,
                         BN / XM);
                for (int kq = 0; kq < nk3; ++kq, ++s) {
                    const int seg = kq / nk, k = kq - seg * nk;   // segment 0: (A, B), 1: (A, lo B), 2: (lo A, B)
                    const int st = s % S;
                    if (!bar_wait(&sh->empty[st], ((s / S) & 1) ^ 1, abort)) break;
                    uint8_t *base = smem + st * STAGE;
                    bar_expect_tx(&sh->full[st], X_A_TILE + B_TILE);
                    tma_load_2d(base, seg == 2 ? &tmAl : &tmA, k * XK, mt * XM, &sh->full[st]);
                    tma_load_2d(base + X_A_TILE, seg == 1 ? &tmBl : &tmB, k * XK, nt * BN, &sh->full[st]);
                }
            }
            // after an abort: the loads already issued land before the CTA
            // ends (bounded: the last S stages)
            if (*abort)
                for (int b = s - 1; b >= 0 && b >= s - S; --b) {
                    const unsigned long long t0 = global_ns();
                    while (!bar_try(&sh->full[b % S], (b / S) & 1) && global_ns() - t0 < kWaitNs) {
                    }
                }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int s = 0;
            bool ok = true;
            for (int j = 0; j < my_tiles && ok; ++j) {
                const int ab = j & 1;
                ok = bar_wait(&sh->acc_empty[ab], ((j >> 1) & 1) ^ 1, abort);
                if (!ok) break;
                tc_fence_after();
                const uint32_t dt = tmem + static_cast<uint32_t>(ab * BN);
                for (int kq = 0; kq < nk3; ++kq, ++s) {
                    const int st = s % S;
                    ok = bar_wait(&sh->full[st], (s / S) & 1, abort);
                    if (!ok) break;
                    tc_fence_after();
                    uint8_t *base = smem + st * STAGE;
                    const uint64_t da = sw128_desc(smem_u32(base));
                    const uint64_t db = sw128_desc(smem_u32(base + X_A_TILE));
#pragma unroll
                    for (int kk = 0; kk < XK / 8; ++kk)   // 8 fp32 = 32 bytes of K per MMA: +2 in 16-byte units
                        mma_tf32(dt, da + 2 * kk, db + 2 * kk, Cfg::kIdesc, (kq | kk) != 0);
                    mma_commit(&sh->empty[st]);   // arrives once these MMAs are done
                }
                if (ok) mma_commit(&sh->acc_full[ab]);
            }
            // every MMA issued has completed before tensor memory is freed
            mma_commit(&sh->drain);
            const unsigned long long t0 = global_ns();
            while (!bar_try(&sh->drain, 0) && global_ns() - t0 < kWaitNs) {
            }
        }
    } else {
        // ---------------- epilogue: one TMEM lane quarter per warp ----------------
        const int q = warp & 3;   // a warp reads TMEM lanes 32 (warp % 4) .. + 31
        for (int j = 0; j < my_tiles; ++j) {
            const int ab = j & 1;
            if (!warp_wait(&sh->acc_full[ab], (j >> 1) & 1, abort)) break;
            tc_fence_after();
            int mt, nt;
            tile_pos(static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x), n_m, n_n, mt, nt, g.lower, BN / XM);
            const int64_t row = static_cast<int64_t>(mt) * XM + q * 32 + lane;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(ab * BN);
            float sq = 0.f;
            for (int cc = 0; cc < BN; cc += 32) {
                uint32_t v[32];
                tmem_ld32(taddr + cc, v);   // every lane takes part (.sync.aligned)
                if (row < g.M) epi_chunk(g, row, static_cast<int64_t>(nt) * BN + cc, v, sq);
            }
            if (g.sumsq) {
                for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
                if (lane == 0 && sq != 0.f) atomicAdd(g.sumsq, static_cast<double>(sq));
            }
            tc_fence_before();   // the accumulator reads are done before it is handed back
            __syncwarp();
            if (lane == 0) bar_arrive(&sh->acc_empty[ab]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (sh->abort && threadIdx.x == 0 && g.status) atomicExch(g.status, static_cast<int32_t>(DBF_ERR_TIMEOUT));
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cfg::TMEM_COLS));
    }
}

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

// K-major fp32 operand [rows x K], row pitch ld: 32 x box_rows boxes, 128-byte swizzle
bool make_map_f32(CUtensorMap *map, const float *base, int64_t K, int64_t rows, int64_t ld, int box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4};
    const cuuint32_t box[2] = {XK, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

template <class Cfg>
constexpr size_t x_smem() { return 1024 + Cfg::S * Cfg::STAGE + sizeof(XSmem<Cfg::S>) + 64; }

int64_t ceil4(int64_t v) { return (v + 3) / 4 * 4; }

template <class Cfg>
cudaError_t launch_tf32x3(int64_t M, int64_t N, int64_t K, float alpha, const float *A, int64_t lda, const float *B,
                          int64_t ldb, float beta, const float *Cin, int64_t ldci, float *Cout, int64_t ldco,
                          double *sumsq, int32_t *status, float *lo, bool lower, int max_ctas, const float *A_lo,
                          const float *B_lo, float *Cout_lo, cudaStream_t s)
{
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
    // lo planes of A and B (B's is A's when B is A)
    const int64_t ldl = ceil4(K);
    float *Alo = lo, *Blo = lo + M * ldl;
    auto split = [&](const float *x, int64_t rows, int64_t ld, float *out) {
        const int64_t total = rows * (ldl / 4);
        const int64_t grid = (total + 255) / 256 < sms * 8 ? (total + 255) / 256 : sms * 8;
        split_lo_kernel<<<static_cast<unsigned>(grid > 0 ? grid : 1), 256, 0, s>>>(x, rows, ldl / 4, ld, out, ldl);
    };
    if (A_lo) Alo = const_cast<float *>(A_lo);
    else split(A, M, lda, Alo);
    if (B_lo) Blo = const_cast<float *>(B_lo);
    else if (B == A && ldb == lda && N == M) Blo = Alo;   // the same operand: the same plane
    else split(B, N, ldb, Blo);
    CUtensorMap ma, mal, mb, mbl;
    if (!make_map_f32(&ma, A, K, M, lda, XM) || !make_map_f32(&mal, Alo, K, M, ldl, XM) ||
        !make_map_f32(&mb, B, K, N, ldb, Cfg::BN) || !make_map_f32(&mbl, Blo, K, N, ldl, Cfg::BN))
        return cudaErrorInvalidValue;
    XArgs g;
    g.M = M;
    g.N = N;
    g.K = K;
    g.alpha = alpha;
    g.beta = beta;
    g.Cin = Cin;
    g.ldci = ldci;
    g.Cout = Cout;
    g.ldco = ldco;
    g.sumsq = sumsq;
    g.vec_c = (sumsq || (aligned16(Cout) && ldco % 4 == 0)) && (beta == 0.f || (aligned16(Cin) && ldci % 4 == 0));
    g.status = status;
    g.lower = lower && M == N && !sumsq;
    g.Cout_lo = sumsq ? nullptr : Cout_lo;
    g.ldlo = ceil4(N);
    if (g.Cout_lo && !aligned16(g.Cout_lo)) g.vec_c = 0;
    {
        cudaError_t e = allow_smem(reinterpret_cast<const void *>(tf32x3_kernel<Cfg>), static_cast<int>(x_smem<Cfg>()));
        if (e != cudaSuccess) return e;
    }
    const int64_t n_m = (M + XM - 1) / XM, n_n = (N + Cfg::BN - 1) / Cfg::BN;
    if (n_m * n_n >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
    const int64_t tiles = g.lower ? lower_tiles(static_cast<int>(n_m), static_cast<int>(n_n), Cfg::BN / XM) : n_m * n_n;
    if (max_ctas > 0 && max_ctas < sms) sms = max_ctas;   // SMs left to other work on the device
    tf32x3_kernel<Cfg><<<static_cast<unsigned>(tiles < sms ? tiles : sms), X_THREADS, x_smem<Cfg>(), s>>>(ma, mal, mb,
                                                                                                         mbl, g);
    return cudaGetLastError();
}

}  // namespace

bool tf32x3_ok(int64_t M, int64_t N, int64_t K, const float *A, int64_t lda, const float *B, int64_t ldb)
{
    return M > 0 && N > 0 && K > 0 && M < (int64_t(1) << 31) && N < (int64_t(1) << 31) && K < (int64_t(1) << 31) &&
           aligned16(A) && aligned16(B) && lda % 4 == 0 && ldb % 4 == 0 && lda >= K && ldb >= K;
}

size_t tf32x3_scratch_floats(int64_t M, int64_t N, int64_t K)
{
    return static_cast<size_t>(M + N) * static_cast<size_t>(ceil4(K));
}

cudaError_t tf32x3_gemm(int64_t M, int64_t N, int64_t K, float alpha, const float *A, int64_t lda, const float *B,
                        int64_t ldb, float beta, const float *Cin, int64_t ldci, float *Cout, int64_t ldco,
                        double *sumsq, int32_t *status, float *lo_scratch, size_t lo_scratch_floats, cudaStream_t s,
                        bool lower, int max_ctas, const float *A_lo, const float *B_lo, float *Cout_lo)
{
    if (!tf32x3_ok(M, N, K, A, lda, B, ldb) || !lo_scratch || !aligned16(lo_scratch) ||
        lo_scratch_floats < tf32x3_scratch_floats(M, N, K))
        return cudaErrorInvalidValue;
    return launch_tf32x3<XDefault>(M, N, K, alpha, A, lda, B, ldb, beta, Cin, ldci, Cout, ldco, sumsq, status,
                                   lo_scratch, lower, max_ctas, A_lo, B_lo, Cout_lo, s);
}

}  // namespace dbf
