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
// Persistent kernel, one CTA per SM; each CTA walks 128 x 256 tiles of
// D = A B^T (A: 128 sign rows, B: 256 token rows) with two 256-column
// accumulators in tensor memory, so the epilogue of one tile overlaps the
// K loop of the next. Warp roles (FwdCfg below, the single-CTA instance used
// by the grouped, MBOK and dense products):
//   warp 0       TMA producer: fp16 activation tiles (64 K x 256 rows,
//                128-byte swizzle) into a ring of SB stages;
//   warp 1       allocates 512 TMEM columns; one thread issues tcgen05.mma
//                (M = 128, N = 256, K = 16) into the free accumulator and
//                commits each stage back;
//   warps 2..9   sign expansion in two groups of four warps that take turns
//                by pairs of K steps, one tile row per thread: the row's
//                packed words are read 16 bytes (two K steps) at a time into
//                a register queue four loads deep, by a cursor that walks the
//                CTA's tiles without divisions, and expanded to exact fp16
//                +-1 (or +-alpha) pairs -- a shift and one LOP3 per two
//                signs, the packed layout keeping columns 2p and 2p+1 in bits
//                p and 16+p -- written in the same 128-byte swizzled K-major
//                layout into a ring of SA stages;
//   warps 10..13 epilogue, one per TMEM lane quarter: tcgen05.ld of a
//                finished accumulator, scaling, stores, then the accumulator
//                is handed back to the MMA warp.
// The forward stages (FwdPairCfg) and the backward sign GEMMs (BwdPairCfg:
// one expansion group, eight epilogue warps) run on CTA pairs: clusters of
// two CTAs, tcgen05 cta_group::2 with M = 256 over the pair, each CTA
// expanding its 128 sign rows and loading half of the token tile (2-SM TMA
// loads without multicast, counted by the leader CTA's barrier); the leader
// issues the MMAs and commits to both CTAs' barriers, and each CTA's tensor
// memory holds its 128 rows of the 256 x 256 accumulator. The one-launch
// forward (FusedCfg, also the MBOK layer) takes 256 x 512 pair tiles: each
// expanded sign stage feeds two MMAs, one per 256-token half, and the two
// accumulators hold the two halves of one tile.
// Every wait is bounded; on expiry the CTA records DBF_ERR_TIMEOUT and stops
// issuing work; before it frees its tensor memory and ends, the TMA loads
// and MMAs it already issued are waited for (bounded as well).
#include "dbf_internal.cuh"

#include <cuda.h>
#include <algorithm>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>
#include <cudaTypedefs.h>

namespace dbf {
namespace {

constexpr int BM = 128;             // sign rows per tile (MMA M)
constexpr int BN = 256;             // token rows per tile (MMA N)
constexpr int BK = 64;              // K per stage: one 128-byte swizzle row of fp16
// Pipeline shapes, per kernel instance. The forward keeps two expansion
// groups (alternating pairs of K steps) and four epilogue warps; the
// one-launch forward, whose 512-column tiles leave no accumulator free for
// the next tile during an epilogue, and the backward, whose epilogues read
// and write an operand per element, take eight epilogue warps (two per TMEM
// lane quarter, each with half of the columns) and one expansion group (a
// 512-column tile needs half the expanded signs per flop).
template <int kGroups, int kSA, int kSB, int kEpi, bool kBackward, bool kPairMode = false, bool kFusedMode = false,
          bool kWideMode = false>
struct GemmCfg {
    static constexpr bool kBwd = kBackward;      // epilogues of stages 3..6 compiled in
    static constexpr bool kFused = kFusedMode;   // both forward stages in one launch (gemm_fused_kernel)
    // 512-token pair tiles: every expanded sign stage feeds two MMAs, one
    // per 256-token half, into two accumulators that fill the 512 tensor
    // memory columns (so one tile's epilogue is not overlapped with the next
    // tile's MMAs); halves the sign expansion per flop
    static constexpr bool kWide = kWideMode;
    static constexpr int kTBN = kWideMode ? 2 * BN : BN;   // token rows per tile
    // CTA pairs (a cluster of two): tcgen05 cta_group::2 with M = 256 over the
    // two SMs; each CTA holds its 128 sign rows of A and half of the 256 token
    // rows of B, and its TMEM the accumulator of its 128 rows
    static constexpr bool kPair = kPairMode;
    static constexpr int kBRows = kPairMode ? 128 : 256;   // B rows a CTA loads per stage
    static constexpr int kBBytes = kBRows * 64 * 2 * (kWideMode ? 2 : 1);   // B bytes a CTA holds per stage
    static constexpr int SA = kSA;               // stages of expanded sign tiles (produced on chip)
    static constexpr int SB = kSB;               // stages of TMA activation tiles
    static constexpr int kExpandGroups = kGroups;
    static constexpr int kExpandWarps = 4 * kGroups;
    static constexpr int kEpiWarps = kEpi;       // multiple of 4: kEpi / 4 warps per TMEM lane quarter
    static constexpr int kThreads = 32 * (2 + kExpandWarps + kEpiWarps);
};
using FwdCfg = GemmCfg<2, 6, 4, 4, false>;
using GrpCfg = GemmCfg<2, 6, 4, 8, false>;   // grouped (segmented) launches: short K loops, epilogue-heavy
using FwdPairCfg = GemmCfg<2, 6, 6, 4, false, true>;
using FusedCfg = GemmCfg<1, 6, 4, 8, false, true, true, true>;
using BwdPairCfg = GemmCfg<1, 6, 6, 8, true, true>;
using BwdFusedCfg = GemmCfg<1, 6, 6, 8, true, true, true>;   // two sign GEMMs of the backward in one launch
constexpr int kMaxStages = 8;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int TMEM_COLS = 512;          // two 256-column accumulators
constexpr unsigned long long kWaitNs = 1000000000ull;   // bounded waits: 1 s

// One adapter's share of a grouped launch (segmented serving): its sign rows,
// scales and token rows; tiles tile0 .. of the launch belong to it.
constexpr int kMaxGroups = 48;
struct GroupRef {
    const uint32_t *signs;      // stage 1: B2, stage 2: B1 of this adapter
    const uint16_t *arow;       // stage 2: alpha [ell][N]
    const uint16_t *beta;       // stage 1: beta [ell][R]
    int off, n;                 // token rows off .. off + n - 1
    int tile0;                  // first tile of the group
    int ncpe;                   // token tiles per envelope: ceil(n / BN)
};

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
    // backward epilogues (stages 3..6); columns c = i T + t (envelope-major)
    float *H32;               // stage 3 writes h [C][P]; stage 4 reads it
    __half *Vout;             // stages 3, 4: fp16(cscale_i[p] acc) [C][P]
    const uint16_t *cscale;   // stages 3, 4: beta [ell][P]; stage 6: gamma [ell][P]
    float *red;               // stages 4, 5, 6 (optional): [ell][P] += sum_t acc * W (stage 4: * H32)
    const void *W;            // stage 5: dy [T][P]; stage 6: x [T][P]
    dbf_dtype wd;
    float *dx;                // stage 6 (optional): [T][P] receives sum_i gamma_i[p] acc
    int dx_mode;              // 0 store, 1 add, 2 atomic add
    int dense_a;              // A is a dense fp16 [P][Ktot] matrix loaded by TMA (tmA), not packed signs
    int env_advance;          // K blocks of Kp columns read successive blocks of the sign row (one sign
                              // matrix per block, multi-kernel layers) instead of the same row again
    // grouped launch (stages 1 and 2): ngroups adapters of one shape, tiles_total tiles
    int ngroups, tiles_total;
    GroupRef grp[kMaxGroups];
};

// Where tile 'tile' of the launch reads and writes: its sign-row block p0,
// its first B row, its token range [t0, t1) and envelope (grouped stage 1
// tiles stay inside one envelope), and its group (null when not grouped).
struct TileRef {
    int p0, brow, t0, t1, env;
    const GroupRef *gr;
};

__device__ __forceinline__ TileRef tile_ref(const GemmArgs &g, int tile, int n_p, int pair_rank = -1, int bn = BN)
{
    TileRef r;
    if (pair_rank >= 0) {
        // a pair tile: 256 sign rows, this CTA's 128 of them
        r.p0 = (tile % n_p) * 2 * BM + pair_rank * BM;
        r.brow = (tile / n_p) * bn;
        r.t0 = r.brow;
        r.t1 = g.C;
        r.env = 0;
        r.gr = nullptr;
        return r;
    }
    if (g.ngroups == 0) {
        r.p0 = (tile % n_p) * BM;
        r.brow = (tile / n_p) * BN;
        r.t0 = r.brow;
        r.t1 = g.C;
        r.env = 0;
        r.gr = nullptr;
        return r;
    }
    int gi = 0;
    while (gi + 1 < g.ngroups && tile >= g.grp[gi + 1].tile0) ++gi;
    const GroupRef &G = g.grp[gi];
    const int local = tile - G.tile0;
    const int c = local / n_p;
    r.p0 = (local - c * n_p) * BM;
    r.env = g.stage == 1 ? c / G.ncpe : 0;
    r.t0 = G.off + (c - r.env * G.ncpe) * BN;
    r.t1 = G.off + G.n;
    r.brow = g.stage == 1 ? r.env * g.T + r.t0 : r.t0;
    r.gr = &G;
    return r;
}

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

// Wait for phase 'parity' of a barrier whatever the abort flag says, bounded
// by the same limit: used on the way out so that no asynchronous copy or MMA
// of this CTA is still in flight when its shared and tensor memory are freed.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity)
{
    const unsigned long long t0 = global_ns();
    while (!bar_try(bar, parity) && global_ns() - t0 < kWaitNs) {
    }
}

// ---- CTA-pair helpers ------------------------------------------------------
// Shared-memory address of the same object in CTA 0 of the pair: bit 24 of
// a shared::cluster address selects the CTA of the pair.
__device__ __forceinline__ uint32_t pair_leader_addr(const void *p) { return smem_u32(p) & 0xFEFFFFFFu; }

// Arrive on a barrier of the pair's CTA 0 (its MMA reads the tiles this CTA
// wrote: the writer fences its generic stores to the async proxy first).
__device__ __forceinline__ void bar_arrive_leader(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(pair_leader_addr(bar)) : "memory");
}

// Arrive on the same barrier in CTA 'rank' of the cluster.
__device__ __forceinline__ void bar_arrive_rank(uint64_t *bar, uint32_t rank)
{
    asm volatile(
        "{\n\t.reg .b32 ra;\n\t"
        "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
        "mbarrier.arrive.shared::cluster.b64 _, [ra];\n\t}" ::"r"(smem_u32(bar)),
        "r"(rank)
        : "memory");
}

// Tile load of one CTA of a pair: the bytes are counted on CTA 0's barrier.
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(pair_leader_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}


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

// The pair's MMA (issued by CTA 0): M = 256 (128 rows from each CTA's A
// tile), N = 256 (128 columns from each CTA's B tile); each CTA's TMEM gets
// the accumulator of its rows.
constexpr uint32_t kIdescPair = (1u << 4) | (static_cast<uint32_t>(BN >> 3) << 17) | (static_cast<uint32_t>((2 * BM) >> 4) << 24);

__device__ __forceinline__ void mma_f16_pair(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(kIdescPair), "r"(accumulate)
        : "memory");
}

// Commit of the pair's MMAs to the same barrier in both CTAs.
__device__ __forceinline__ void mma_commit_pair_both(uint64_t *bar)
{
    asm volatile(
        "{\n\t.reg .b16 msk;\n\t"
        "mov.b16 msk, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], msk;\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mma_commit_pair_own(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
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

// fp16 pair of in-word columns (2p, 2p+1) from bits p and 16+p: the sign bits
// land on bits 15 and 31 and are xored into the pair's magnitude pattern.
__device__ __forceinline__ uint32_t sign_pair(uint32_t w, int p, uint32_t mag2)
{
    return ((w << (15 - p)) & 0x80008000u) ^ mag2;
}

constexpr int kRing = 4;   // tile ring of the fused forward: entries in flight

struct GemmSmem {
    uint64_t full_a[kMaxStages], empty_a[kMaxStages], full_b[kMaxStages], empty_b[kMaxStages], acc_full[2], acc_empty[2];
    uint64_t tfull[kRing], tempty[kRing];   // fused forward: tile ring entries posted / given back
    int ring[kRing];
    uint64_t drain;   // the MMA thread's last commit: every MMA it issued has completed
    uint64_t exit_bar;   // CTA pairs: the peer is done with this CTA's shared memory
    uint32_t tmem_base;
    int abort;
};

// Epilogue of a grouped tile, 32 columns = tokens t0 .. t0 + 31 (those below
// the group's end): stage 1 writes v = fp16(beta h) of envelope tr.env,
// stage 2 writes y.
__device__ __forceinline__ void grouped_chunk(const GemmArgs &g, const TileRef &tr, const uint32_t (&v)[32], int t0,
                                              int p)
{
    const int n_ok = tr.t1 - t0;
    if (n_ok <= 0) return;   // a chunk past the group's end: nothing to read or write
    if (g.stage == 1) {
        const float b = h2f(tr.gr->beta[static_cast<int64_t>(tr.env) * g.R + p]);
        const int64_t ts = static_cast<int64_t>(g.ell) * g.R;
        __half *vp = g.V + static_cast<int64_t>(t0) * ts + static_cast<int64_t>(tr.env) * g.R + p;
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (e < n_ok) vp[e * ts] = __float2half_rn(b * __uint_as_float(v[e]));
    } else if (g.yd == DBF_BF16) {
        __nv_bfloat16 *yp = static_cast<__nv_bfloat16 *>(g.y) + static_cast<int64_t>(t0) * g.N + p;
#pragma unroll
        for (int e0 = 0; e0 < 32; e0 += 8) {
            float yin[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                yin[e] = g.accumulate ? __bfloat162float(yp[static_cast<int64_t>(e0 + e < n_ok ? e0 + e : 0) * g.N]) : 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (e0 + e < n_ok) yp[static_cast<int64_t>(e0 + e) * g.N] = __float2bfloat16_rn(__uint_as_float(v[e0 + e]) + yin[e]);
        }
    } else {
        float *yp = static_cast<float *>(g.y) + static_cast<int64_t>(t0) * g.N + p;
#pragma unroll
        for (int e0 = 0; e0 < 32; e0 += 8) {
            float yin[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                yin[e] = g.accumulate ? yp[static_cast<int64_t>(e0 + e < n_ok ? e0 + e : 0) * g.N] : 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (e0 + e < n_ok) yp[static_cast<int64_t>(e0 + e) * g.N] = __uint_as_float(v[e0 + e]) + yin[e];
        }
    }
}

__device__ __forceinline__ float load_w(const void *w, dbf_dtype wd, int64_t i)
{
    return wd == DBF_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(w)[i])
                          : static_cast<const float *>(w)[i];
}

// Backward epilogue of 32 accumulator columns c = cb .. cb + 31 of tile row
// p (see GemmArgs): c = i T + t, so (i, t) advance with c. Every operand the
// chunk reads (H32 or W) is loaded first, all 32 loads in flight together;
// then the per-(i, p) sums over tokens are formed and flushed with one
// atomic add when i changes and at the end of the chunk.
__device__ __forceinline__ void backward_chunk(const GemmArgs &g, const uint32_t (&v)[32], int cb, int p)
{
    const int i0 = cb / g.T, t0 = cb - i0 * g.T;
    // the operand of each of the 32 columns, all loads issued before any is
    // used (one straight block per operand type; dy and x through the
    // read-only path, h not: the same launch may have written it)
    float w[32];
    if (g.stage == 4) {
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = g.H32[cb + e < g.C ? static_cast<int64_t>(cb + e) * g.P + p : 0];
    } else if (g.stage >= 5 && g.red) {
        int64_t off[32];
        int t = t0;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            off[e] = cb + e < g.C ? static_cast<int64_t>(t) * g.P + p : 0;
            if (++t == g.T) t = 0;
        }
        if (g.wd == DBF_BF16) {
            const __nv_bfloat16 *wp = static_cast<const __nv_bfloat16 *>(g.W);
            __nv_bfloat16 wb[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) wb[e] = __ldg(wp + off[e]);
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = __bfloat162float(wb[e]);
        } else {
            const float *wp = static_cast<const float *>(g.W);
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = __ldg(wp + off[e]);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = 0.f;
    }
    int i = i0, t = t0;
    float cs = (g.cscale && i < g.ell) ? h2f(g.cscale[static_cast<int64_t>(i) * g.P + p]) : 0.f;
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int c = cb + e;
        if (c < g.C) {
            const float a = __uint_as_float(v[e]);
            const int64_t ic = static_cast<int64_t>(c) * g.P + p;
            if (g.stage == 3) {
                g.H32[ic] = a;
                g.Vout[ic] = __float2half_rn(cs * a);
            } else if (g.stage == 4) {
                part += a * w[e];
                g.Vout[ic] = __float2half_rn(cs * a);
            } else {
                part += a * w[e];
                if (g.stage == 6 && g.dx) {
                    const int64_t it = static_cast<int64_t>(t) * g.P + p;
                    const float d = cs * a;
                    if (g.dx_mode == 0) g.dx[it] = d;
                    else if (g.dx_mode == 1) g.dx[it] += d;
                    else atomicAdd(g.dx + it, d);
                }
            }
        }
        if (++t == g.T) {
            if (g.red && i < g.ell) atomicAdd(g.red + static_cast<int64_t>(i) * g.P + p, part);
            part = 0.f;
            t = 0;
            ++i;
            cs = (g.cscale && i < g.ell) ? h2f(g.cscale[static_cast<int64_t>(i) * g.P + p]) : 0.f;
        }
    }
    if (g.red && i < g.ell && part != 0.f) atomicAdd(g.red + static_cast<int64_t>(i) * g.P + p, part);
}

// ---- the forward's two stages in one launch ---------------------------------
// Stage-1 tiles (B2 rows x columns of u) come first, then the stage-2 tiles
// (B1 rows x tokens), the last nsk of them split in two halves of K, so that
// the last tiles to run are short: each half sums its share of K, the half
// that finishes first leaves its partial sums in the workspace and the other
// adds them (fp32 addition commutes, so the sum does not depend on which
// half finishes first) and writes y. A pair takes its first tile by its
// index and every later one from a claim counter, one tile ahead of the tile
// it starts, so that the pairs that finish first take the remaining tiles;
// CTA 0's producer posts each claimed tile in a ring of kRing entries in both
// CTAs' shared memory, from which every role reads it. A stage-2 tile loads
// rows of v that the stage-1 epilogues of other pairs write: each stage-1
// epilogue warp counts its finished tile on the flag of the tile's column
// block, and a producer loads v only once the flags of every block its tokens
// need are complete (bounded wait). Tiles are claimed in order and a pair
// only claims while it runs, so every stage-1 tile a stage-2 tile waits for
// is held by a running pair that does not wait itself.
struct FusedSched {
    int n1, n2f, nsk;        // stage-1 tiles; stage-2 tiles run whole; stage-2 tiles split in K
    // what stage-2 tiles read of stage-1 output (flags, counted by stage-1
    // epilogue warps): 1 their B operand, whole column blocks (the forward's
    // v; flag per column block); 2 in their epilogue, the stage-1 tile of the
    // same index (the backward's h; flag per tile); 0 nothing
    int dep;
    int ksplit;              // K steps of the first half of a split tile (even)
    int n_p1, n_p2;          // pair row tiles per column block in stages 1 and 2
    unsigned *ctr;           // claim counter (zeroed by the pre-pass)
    unsigned *flags;         // finished stage-1 epilogue warps per column block (dep 1) or tile (dep 2); zeroed by the pre-pass
    unsigned flag_target;    // arrivals that complete a block or tile
    // per split tile, CTA and TMEM lane quarter (zeroed by the pre-pass):
    unsigned *sk_count;      // halves that reached the epilogue
    unsigned *sk_ready;      // the first half's partial sums are written
    float *sk_part;          // per split tile and CTA: 128 rows x 256 columns of partial sums, column-major
};

struct FusedTile {
    int stage, t, part;      // part: -1 for a whole tile, else which half of K of tile t
};

__device__ __forceinline__ FusedTile fused_decode(const FusedSched &fs, int u)
{
    FusedTile f;
    if (u < fs.n1) {
        f.stage = 1;
        f.t = u;
        f.part = -1;
    } else if (u < fs.n1 + fs.n2f) {
        f.stage = 2;
        f.t = u - fs.n1;
        f.part = -1;
    } else {
        const int h = u - fs.n1 - fs.n2f;
        f.stage = 2;
        f.t = fs.n2f + (h >> 1);
        f.part = h & 1;
    }
    return f;
}

// K steps [kb, ke) of a claimed tile with nk K steps in all.
__device__ __forceinline__ void fused_krange(const FusedSched &fs, const FusedTile &f, int nk, int &kb, int &ke)
{
    kb = f.part == 1 ? fs.ksplit : 0;
    ke = f.part == 0 ? fs.ksplit : nk;
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Wait with acquire at cluster scope (the ring's entries are written by CTA 0).
__device__ __forceinline__ bool bar_try_cluster(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Release-arrive on the barrier at shared::cluster address 'addr'.
__device__ __forceinline__ void bar_arrive_cluster_addr(uint32_t addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

__device__ __forceinline__ uint32_t peer_addr(const void *p, uint32_t rank)
{
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    return a;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait with acquire at cluster scope; false (and the abort flag
// raised) when the limit passes or another role already aborted.
__device__ __forceinline__ bool bar_wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    if (bar_try_cluster(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (bar_try_cluster(bar, parity)) return true;
        if (*abort) return false;
        if (global_ns() - t0 > kWaitNs) {
            *abort = 1;
            return false;
        }
    }
}

// Entry j of the pair's tile ring (one thread): the claimed tile, -1 after
// the last one; false when the wait expired or another role aborted. The
// slot is handed back to CTA 0's producer once read.
__device__ __forceinline__ bool ring_get(GemmSmem *sh, int j, int &u)
{
    const int s = j % kRing;
    if (!bar_wait_cluster(&sh->tfull[s], (j / kRing) & 1, &sh->abort)) return false;
    u = *reinterpret_cast<volatile int *>(&sh->ring[s]);
    bar_arrive_cluster_addr(pair_leader_addr(&sh->tempty[s]));
    return true;
}

// The same for a whole warp: lane 0 reads, every lane gets the entry.
__device__ __forceinline__ bool ring_get_warp(GemmSmem *sh, int j, int &u)
{
    int v = -1;
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = ring_get(sh, j, v) ? 1 : 0;
    u = __shfl_sync(0xffffffffu, v, 0);
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Persistent: CTA b takes tiles b, b + gridDim.x, ... (token-tile major, so
// the CTAs running together share activation tiles in L2); in the fused
// forward (g2 and fs given) the pairs claim tiles instead (see above), tmB
// being the map of u and tmA the map of v.
template <class Cfg>
__device__ __forceinline__ void gemm_body(const CUtensorMap &tmB, const CUtensorMap &tmA, const GemmArgs &g,
                                          const GemmArgs *g2, const FusedSched *fs)
{
    constexpr int SA = Cfg::SA, SB = Cfg::SB, kExpandGroups = Cfg::kExpandGroups;
    constexpr int kExpandWarps = Cfg::kExpandWarps, kEpiWarps = Cfg::kEpiWarps;
    constexpr bool kFused = Cfg::kFused, kWide = Cfg::kWide;
    constexpr int TBN = Cfg::kTBN;   // token rows per tile
    static_assert(SA <= kMaxStages && SB <= kMaxStages && kEpiWarps % 4 == 0 && TBN % (32 * (kEpiWarps / 4)) == 0,
                  "pipeline shape");
    static_assert(!kWide || (kFused && Cfg::kPair), "512-token tiles: the one-launch forward on CTA pairs");
    static_assert(!kFused || Cfg::kPair, "tiles are claimed by CTA pairs");
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *smA = smem;
    constexpr bool kPair = Cfg::kPair;
    constexpr int kBBytes = Cfg::kBBytes;
    uint8_t *smB = smA + SA * A_BYTES;
    GemmSmem *sh = reinterpret_cast<GemmSmem *>(smB + SB * kBBytes);
    volatile int *abort = &sh->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // tiles are walked per CTA, or per CTA pair (rank 0 issues the pair's MMAs)
    uint32_t rank = 0;
    if (kPair) asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    const int unit = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int nunits = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    const int tile_rank = kPair ? static_cast<int>(rank) : -1;
    const int n_p = (g.P + (kPair ? 2 * BM : BM) - 1) / (kPair ? 2 * BM : BM);
    const int n_c = (g.C + TBN - 1) / TBN;
    const int ntiles = g.ngroups ? g.tiles_total : n_p * n_c;
    const int my_tiles = unit < ntiles ? (ntiles - 1 - unit) / nunits + 1 : 0;
    const int nk = g.Ktot / BK;
    auto wait = [&](uint64_t *bar, uint32_t parity) { return bar_wait(bar, parity, abort); };
    // the fused forward's view of a claimed tile: its stage's arguments, row
    // tiles per column block, tile index and half
    auto fused_args = [&](const FusedTile &f) -> const GemmArgs & { return f.stage == 1 ? g : *g2; };

    if (threadIdx.x == 0) {
        for (int i = 0; i < SA; ++i) {
            // the TMA producer, or the four warps of one expansion group (of both CTAs of a pair)
            bar_init(&sh->full_a[i], g.dense_a ? 1 : (kPair ? 8 : 4));
            bar_init(&sh->empty_a[i], 1);
        }
        for (int i = 0; i < SB; ++i) {
            bar_init(&sh->full_b[i], 1);
            bar_init(&sh->empty_b[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            bar_init(&sh->acc_full[i], 1);
            bar_init(&sh->acc_empty[i], kPair ? 2 * kEpiWarps : kEpiWarps);
        }
        if (kFused) {
            // every reader of the ring in both CTAs gives each entry back: the
            // MMA thread of CTA 0, the producer of CTA 1, and the expansion and
            // epilogue warps of both
            for (int i = 0; i < kRing; ++i) {
                bar_init(&sh->tfull[i], 1);
                bar_init(&sh->tempty[i], 2 + 2 * (kExpandWarps + kEpiWarps));
            }
        }
        bar_init(&sh->drain, 1);
        bar_init(&sh->exit_bar, 1);
        sh->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
        if (g.dense_a || kFused) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
    }
    if (warp == 1) {
        if (kPair) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh->tmem_base)),
                         "r"(TMEM_COLS));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh->tmem_base)),
                         "r"(TMEM_COLS));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
    }
    // A launch that follows with programmatic stream serialisation (the next
    // decode call) may be set up now: it cannot become resident before this
    // grid's CTAs leave their SMs, and it waits (griddepcontrol.wait) for
    // this grid to complete before it touches anything this grid writes.
    if (kFused) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    if (kPair) {
        // both CTAs' barriers are initialised before either reaches the other's
        asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
        asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    }
    tc_fence_after();
    const uint32_t tmem = sh->tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int s = 0;
            int nb_issued = 0, na_issued = 0;   // TMA loads issued on each ring
            if (kFused) {
                const int total = fs->n1 + fs->n2f + 2 * fs->nsk;
                // CTA 0 claims tile k of the pair and posts it in both rings
                // (-1: no tile left); -2 when the ring wait gave up
                auto claim = [&](int k) -> int {
                    const int sl = k % kRing;
                    if (!bar_wait_cluster(&sh->tempty[sl], ((k / kRing) & 1) ^ 1, abort)) return -2;
                    int u = k == 0 ? unit : nunits + static_cast<int>(atomicAdd(fs->ctr, 1u));
                    if (u >= total) u = -1;
                    *reinterpret_cast<volatile int *>(&sh->ring[sl]) = u;
                    const uint32_t peer_ring = peer_addr(&sh->ring[sl], 1u);
                    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_ring), "r"(u) : "memory");
                    bar_arrive_cluster_addr(smem_u32(&sh->tfull[sl]));
                    bar_arrive_cluster_addr(peer_addr(&sh->tfull[sl], 1u));
                    return u;
                };
                // the pair's first tile is its index: posted before the wait for
                // the pre-pass, so that the sign expansion starts meanwhile
                int u = -1;
                if (rank == 0) u = claim(0);
                griddep_wait();   // u and the claim state come from the pre-pass launched before
                if (rank != 0 && !ring_get(sh, 0, u)) u = -1;
                for (int j = 0; u >= 0 && !*abort; ++j) {
                    int un = -1;   // the pair's next tile, claimed (CTA 0) or read (CTA 1) one tile ahead
                    if (rank == 0) {
                        un = claim(j + 1);
                        if (un == -2) break;
                    }
                    const FusedTile f = fused_decode(*fs, u);
                    const GemmArgs &gs = fused_args(f);
                    const TileRef tr = tile_ref(gs, f.t, f.stage == 1 ? fs->n_p1 : fs->n_p2, tile_rank, TBN);
                    const int c0 = tr.brow;
                    const CUtensorMap *mp = f.stage == 1 ? &tmB : &tmA;
                    bool ok = true;
                    if (f.stage == 2 && fs->dep == 1 && c0 < g.T) {
                        // the v rows of tokens [c0, t_hi) of every envelope: stage-1
                        // column blocks (i T + t) / TBN
                        const int t_hi = min(c0 + TBN, g.T);
                        const unsigned long long t0 = global_ns();
                        for (int i = 0; i < g.ell && ok; ++i) {
                            const int b_lo = (i * g.T + c0) / TBN, b_hi = (i * g.T + t_hi - 1) / TBN;
                            for (int b = b_lo; b <= b_hi && ok; ++b) {
                                while (ld_acquire_u32(fs->flags + b) < fs->flag_target) {
                                    if (*abort) { ok = false; break; }
                                    if (global_ns() - t0 > kWaitNs) {
                                        *abort = 1;
                                        ok = false;
                                        break;
                                    }
                                }
                            }
                        }
                        // v was written through the generic proxy; the loads below use the async one
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                    }
                    if (!ok) break;
                    int kb, ke;
                    fused_krange(*fs, f, gs.Ktot / BK, kb, ke);
                    for (int k = kb; k < ke; ++k, ++s) {
                        const int st = s % SB;
                        if (!wait(&sh->empty_b[st], ((s / SB) & 1) ^ 1)) break;
                        if (rank == 0) bar_expect_tx(&sh->full_b[st], 2 * kBBytes);
                        tma_load_2d_pair(smB + st * kBBytes, mp, k * BK, c0 + static_cast<int>(rank) * Cfg::kBRows,
                                         &sh->full_b[st]);
                        if (kWide)   // the second 256-token half, 16 KB further on
                            tma_load_2d_pair(smB + st * kBBytes + kBBytes / 2, mp, k * BK,
                                             c0 + BN + static_cast<int>(rank) * Cfg::kBRows, &sh->full_b[st]);
                        nb_issued = s + 1;
                    }
                    if (rank == 0) {
                        u = un;
                    } else if (!ring_get(sh, j + 1, u)) {
                        break;
                    }
                }
            } else {
                for (int j = 0; j < my_tiles && !*abort; ++j) {
                    const TileRef tr = tile_ref(g, unit + j * nunits, n_p, tile_rank, TBN);
                    const int c0 = tr.brow;
                    const int p0 = tr.p0;
                    for (int k = 0; k < nk; ++k, ++s) {
                        const int st = s % SB;
                        if (!wait(&sh->empty_b[st], ((s / SB) & 1) ^ 1)) break;
                        if (kPair) {
                            // CTA 0's barrier counts the bytes of both halves of B
                            if (rank == 0) bar_expect_tx(&sh->full_b[st], 2 * kBBytes);
                            tma_load_2d_pair(smB + st * kBBytes, &tmB, k * BK, c0 + static_cast<int>(rank) * Cfg::kBRows,
                                             &sh->full_b[st]);
                        } else {
                            bar_expect_tx(&sh->full_b[st], kBBytes);
                            tma_load_2d(smB + st * kBBytes, &tmB, k * BK, c0, &sh->full_b[st]);
                        }
                        nb_issued = s + 1;
                        if (g.dense_a) {
                            // a dense fp16 A operand: its tile comes by TMA too, in the
                            // same swizzled K-major layout the expansion writes
                            const int sa = s % SA;
                            if (!bar_wait(&sh->empty_a[sa], ((s / SA) & 1) ^ 1, abort)) break;
                            bar_expect_tx(&sh->full_a[sa], A_BYTES);
                            tma_load_2d(smA + sa * A_BYTES, &tmA, k * BK, p0, &sh->full_a[sa]);
                            na_issued = s + 1;
                        }
                    }
                }
            }
            // After an abort, the loads already issued (at most the last SB,
            // resp. SA, of each ring: earlier ones were consumed) land before
            // the CTA ends and its shared memory is released. Bounded. (In a
            // pair, CTA 0's barriers count both CTAs' loads; CTA 1 is held by
            // the exit handshake until CTA 0 has waited for them.)
            if (*abort && (!kPair || rank == 0)) {
                for (int b = nb_issued - 1; b >= 0 && b >= nb_issued - SB; --b) drain_wait(&sh->full_b[b % SB], (b / SB) & 1);
                for (int b = na_issued - 1; b >= 0 && b >= na_issued - SA; --b) drain_wait(&sh->full_a[b % SA], (b / SA) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (CTA 0 of a pair issues for both) ----------------
        if (lane == 0 && (!kPair || rank == 0)) {
            int s = 0;
            bool ok = true;
            for (int j = 0; ok; ++j) {
                int kb = 0, ke = nk;
                if (kFused) {
                    int u = -1;
                    if (!ring_get(sh, j, u) || u < 0) break;
                    const FusedTile f = fused_decode(*fs, u);
                    fused_krange(*fs, f, fused_args(f).Ktot / BK, kb, ke);
                } else if (j >= my_tiles) {
                    break;
                }
                // two accumulators taking turns by tile, or (wide) one tile's
                // two halves in them
                const int ab = kWide ? 0 : (j & 1);
                ok = wait(&sh->acc_empty[ab], (kWide ? (j & 1) : ((j >> 1) & 1)) ^ 1);
                if (!ok) break;
                tc_fence_after();
                const uint32_t dt = tmem + static_cast<uint32_t>(ab * BN);
                for (int k = kb; k < ke; ++k, ++s) {
                    const int sa = s % SA, sb = s % SB;
                    ok = wait(&sh->full_a[sa], (s / SA) & 1) && wait(&sh->full_b[sb], (s / SB) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t da = sw128_desc(smem_u32(smA + sa * A_BYTES));
                    const uint64_t db = sw128_desc(smem_u32(smB + sb * kBBytes));
                    if (kWide) {
                        // the same sign stage for both token halves
                        const uint64_t db1 = sw128_desc(smem_u32(smB + sb * kBBytes + kBBytes / 2));
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            mma_f16_pair(dt, da + 2 * kk, db + 2 * kk, (k != kb || kk) != 0);
                            mma_f16_pair(dt + static_cast<uint32_t>(BN), da + 2 * kk, db1 + 2 * kk, (k != kb || kk) != 0);
                        }
                        mma_commit_pair_both(&sh->empty_a[sa]);
                        mma_commit_pair_both(&sh->empty_b[sb]);
                    } else if (kPair) {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            mma_f16_pair(dt, da + 2 * kk, db + 2 * kk, (k != kb || kk) != 0);
                        mma_commit_pair_both(&sh->empty_a[sa]);   // both CTAs' stages are free again
                        mma_commit_pair_both(&sh->empty_b[sb]);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)   // 32 bytes of K per MMA: +2 in 16-byte units
                            mma_f16(dt, da + 2 * kk, db + 2 * kk, (k != kb || kk) != 0);
                        mma_commit(&sh->empty_a[sa]);   // each commit arrives once these MMAs are done
                        mma_commit(&sh->empty_b[sb]);
                    }
                }
                if (ok) {
                    if (kPair) mma_commit_pair_both(&sh->acc_full[ab]);
                    else mma_commit(&sh->acc_full[ab]);
                }
            }
            // every MMA issued (also on an abort) has completed before tensor
            // memory is freed and the CTA ends
            if (kPair) mma_commit_pair_own(&sh->drain);
            else mma_commit(&sh->drain);
            drain_wait(&sh->drain, 0);
        }
    } else if (warp < 2 + kExpandWarps) {
        if (g.dense_a) goto teardown;   // A tiles come by TMA
        // ---------------- sign expansion: one tile row per thread ----------------
        // kExpandGroups groups of four warps take turns by pairs of K steps;
        // each thread of a group owns one tile row.
        const int grp = (warp - 2) >> 2;
        const int prow = ((warp - 2) & 3) * 32 + lane;
        const uint32_t swz = static_cast<uint32_t>(prow & 7) << 4;
        // cursor over this CTA's (tile, pair) sequence, advanced without
        // divisions; calive turns false past the last tile
        int cj = 0, cpair = 0, cword = 0, cenv = 0, cgrow = 0, cbase = 0;   // cbase: first word of the envelope block
        int cnpairs = nk / 2;                     // pairs of K steps of the tile (K is a multiple of 128)
        int cenv_words = g.Kp / 32;               // packed words of one envelope block of K
        const GemmArgs *cg = &g;                  // the tile's arguments (fused: its stage's)
        const uint32_t *crow = nullptr;
        bool cvalid = false, calive = true;
        uint32_t cmag = 0u;
        const uint16_t *carow = g.arow_scale;
        auto seat_mag = [&]() {
            if (carow) {
                const uint32_t a = cvalid ? __ldg(carow + static_cast<int64_t>(cenv) * cg->N + cgrow) : 0u;
                cmag = a | (a << 16);
            } else {
                cmag = cvalid ? 0x3C003C00u : 0u;   // +-1
            }
        };
        auto seat_tile = [&]() {
            int t = unit + cj * nunits, np = n_p;
            if (kFused) {
                int u = -1;
                if (!ring_get_warp(sh, cj, u) || u < 0) {
                    calive = false;
                    return;
                }
                const FusedTile f = fused_decode(*fs, u);
                cg = &fused_args(f);
                np = f.stage == 1 ? fs->n_p1 : fs->n_p2;
                t = f.t;
                int kb, ke;
                fused_krange(*fs, f, cg->Ktot / BK, kb, ke);
                cnpairs = (ke - kb) / 2;
                cenv_words = cg->Kp / 32;
                if (kb > 0) {
                    // the second half of K starts inside the row: its envelope
                    // block, and the word in it (a multiple of four: Kp % 128 == 0)
                    cenv = kb * BK / cg->Kp;
                    cword = (kb * BK - cenv * cg->Kp) / 32;
                    cbase = cg->env_advance ? cenv * cenv_words : 0;
                }
            } else if (cj >= my_tiles) {
                calive = false;
                return;
            }
            const TileRef tr = tile_ref(*cg, t, np, tile_rank, TBN);
            cgrow = tr.p0 + prow;
            cvalid = cgrow < cg->P;
            carow = tr.gr ? tr.gr->arow : cg->arow_scale;
            crow = (tr.gr ? tr.gr->signs : cg->signs) + static_cast<int64_t>(cvalid ? cgrow : 0) * cg->pitch;
            seat_mag();
        };
        auto advance = [&]() {
            if (!calive) return;
            if (++cpair == cnpairs) {
                cpair = 0;
                cword = 0;
                cenv = 0;
                cbase = 0;
                ++cj;
                seat_tile();
            } else {
                cword += 4;
                if (cword == cenv_words) {
                    cword = 0;
                    ++cenv;
                    cbase += cg->env_advance ? cenv_words : 0;   // a new block of the row, or the same row again
                    seat_mag();
                }
            }
        };
        // this row's four words of the cursor's pair (two K steps) and the
        // magnitude pattern of its envelope block; then move on to the group's
        // next pair. False when the cursor is past the last tile.
        auto fetch = [&](uint4 &w, uint32_t &mag) -> bool {
            if (!calive) return false;
            w = cvalid ? __ldg(reinterpret_cast<const uint4 *>(crow + cbase + cword)) : make_uint4(0u, 0u, 0u, 0u);
            mag = cmag;
#pragma unroll
            for (int e = 0; e < kExpandGroups; ++e) advance();
            return true;
        };
        seat_tile();
#pragma unroll
        for (int e = 0; e < kExpandGroups; ++e)
            if (e < grp) advance();
        constexpr int D = 4;   // pairs in flight per thread
        uint4 qw[D];
        uint32_t qm[D];
        bool qa[D];
#pragma unroll
        for (int d = 0; d < D; ++d) {
            qw[d] = make_uint4(0u, 0u, 0u, 0u);
            qm[d] = 0u;
            qa[d] = fetch(qw[d], qm[d]);
        }
        bool ok = true;
        auto write_stage = [&](int st, uint32_t w0, uint32_t w1, uint32_t mag) {
            uint8_t *arow = smA + st * A_BYTES + prow * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j) {   // 16-byte chunk j: columns 8j .. 8j + 7
                const uint32_t w = j < 4 ? w0 : w1;
                const int pb = 4 * (j & 3);
                uint4 v;
                v.x = sign_pair(w, pb + 0, mag);
                v.y = sign_pair(w, pb + 1, mag);
                v.z = sign_pair(w, pb + 2, mag);
                v.w = sign_pair(w, pb + 3, mag);
                *reinterpret_cast<uint4 *>(arow + ((static_cast<uint32_t>(j) << 4) ^ swz)) = v;
            }
        };
        // both K steps of pair p, one proxy fence for the two stages
        auto expand_pair = [&](int p, const uint4 &w, uint32_t mag) {
            const int s0 = 2 * p, s1 = 2 * p + 1;
            const int st0 = s0 % SA, st1 = s1 % SA;
            ok = wait(&sh->empty_a[st0], ((s0 / SA) & 1) ^ 1) && wait(&sh->empty_a[st1], ((s1 / SA) & 1) ^ 1);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) return;
            write_stage(st0, w.x, w.y, mag);
            write_stage(st1, w.z, w.w, mag);
            fence_proxy_async();   // generic-proxy writes -> visible to the tensor core
            __syncwarp();
            if (lane == 0) {
                if (kPair) {   // CTA 0 issues the MMAs that read both CTAs' tiles
                    bar_arrive_leader(&sh->full_a[st0]);
                    bar_arrive_leader(&sh->full_a[st1]);
                } else {
                    bar_arrive(&sh->full_a[st0]);
                    bar_arrive(&sh->full_a[st1]);
                }
            }
        };
        // slot d of the queue holds the group's pairs base + d * kExpandGroups
        for (int base = grp; ok && qa[0]; base += D * kExpandGroups) {
#pragma unroll
            for (int d = 0; d < D; ++d) {
                if (qa[d] && ok) {
                    const int p = base + d * kExpandGroups;
                    const uint4 w = qw[d];
                    const uint32_t mag = qm[d];
                    qa[d] = fetch(qw[d], qm[d]);
                    expand_pair(p, w, mag);
                } else {
                    qa[0] = false;   // the pairs after an empty slot are empty too
                }
            }
        }
    } else {
        // ---------------- epilogue: one warp per TMEM lane quarter ----------------
        const int q = warp & 3;   // a warp reads the TMEM lane quarter warp % 4
        const int ch = kEpiWarps == 4 ? 0 : (warp - 2 - kExpandWarps) >> 2;   // which share of the columns
        constexpr int kColShare = TBN / (kEpiWarps / 4);
        if (kFused) griddep_wait();   // the flags it counts on are zeroed by the pre-pass
        for (int j = 0;; ++j) {
            TileRef tr;
            const GemmArgs *ge = &g;
            int stage1 = g.stage == 1;
            int sk = -1;         // a tile split in K: its slot (tile, CTA, epilogue warp)
            int flag_out = -1;   // a stage-1 tile whose epilogue counts on a flag (dep 1: column block; 2: tile)
            int flag_in = -1;    // a stage-2 tile whose epilogue waits for the stage-1 tile of this index (dep 2)
            if (kFused) {
                int u = -1;
                if (!ring_get_warp(sh, j, u) || u < 0) break;
                const FusedTile f = fused_decode(*fs, u);
                ge = &fused_args(f);
                tr = tile_ref(*ge, f.t, f.stage == 1 ? fs->n_p1 : fs->n_p2, tile_rank, TBN);
                stage1 = ge->stage == 1;   // the forward's stage 1 (v); the backward's GEMMs have stages 3..6
                if (!Cfg::kBwd && f.part >= 0)   // only the forward splits tiles in K
                    sk = ((f.t - fs->n2f) * 2 + static_cast<int>(rank)) * kEpiWarps + (warp - 2 - kExpandWarps);
                if (f.stage == 1 && fs->dep == 1) flag_out = tr.brow / TBN;
                if (f.stage == 1 && fs->dep == 2) flag_out = f.t;
                if (f.stage == 2 && fs->dep == 2) flag_in = f.t;
            } else {
                if (j >= my_tiles) break;
                tr = tile_ref(g, unit + j * nunits, n_p, tile_rank, TBN);
            }
            const GemmArgs &ga = *ge;
            const int ab = kWide ? 0 : (j & 1);
            bool got = true;
            if (lane == 0) got = wait(&sh->acc_full[ab], kWide ? (j & 1) : ((j >> 1) & 1));
            if (!__shfl_sync(0xffffffffu, got, 0)) break;
            tc_fence_after();
            if (kFused && flag_in >= 0) {
                // the stage-1 tile this epilogue reads (its h) is complete
                if (lane == 0) {
                    const unsigned long long t0 = global_ns();
                    while (ld_acquire_u32(fs->flags + flag_in) < fs->flag_target) {
                        if (*abort) break;
                        if (global_ns() - t0 > kWaitNs) {
                            *abort = 1;
                            break;
                        }
                    }
                }
                __syncwarp();
            }
            const int p0 = tr.p0, c0 = tr.brow;
            const int grow = p0 + q * 32 + lane;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(ab * BN);
            const bool row_ok = grow < ga.P;
            // a split tile: the half that reaches its epilogue first stores its
            // partial sums (this CTA's 128 rows, column-major) and the other
            // waits for them, adds them to its own and writes y
            bool sk_first = false;
            float *sk_base = nullptr;
            if (kFused && sk >= 0) {
                unsigned old = 0;
                if (lane == 0) old = atomicAdd(fs->sk_count + sk, 1u);
                sk_first = __shfl_sync(0xffffffffu, old, 0) == 0;
                sk_base = fs->sk_part + static_cast<int64_t>(sk / kEpiWarps) * (BM * TBN) + q * 32 + lane;
                if (!sk_first && lane == 0) {
                    const unsigned long long t0 = global_ns();
                    while (ld_acquire_u32(fs->sk_ready + sk) == 0) {
                        if (*abort) break;
                        if (global_ns() - t0 > kWaitNs) {
                            *abort = 1;
                            break;
                        }
                    }
                }
                __syncwarp();
            }
            for (int cc = ch * kColShare; cc < (ch + 1) * kColShare; cc += 32) {
                uint32_t v[32];
                tmem_ld32(taddr + cc, v);   // every lane takes part (.sync.aligned)
                if (kFused && sk >= 0) {
                    float *pc = sk_base + static_cast<int64_t>(cc) * BM;
                    if (sk_first) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) pc[e * BM] = __uint_as_float(v[e]);
                        continue;
                    }
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) + pc[e * BM]);
                }
                if (!row_ok) continue;
                if (tr.gr) {
                    grouped_chunk(ga, tr, v, tr.t0 + cc, grow);
                    continue;
                }
                const int cb = c0 + cc;
                if (cb >= ga.C) continue;   // a chunk past the last token (a ragged tile): nothing to read or write
                if (stage1) {
                    // column c = i T + t; v[t, i R + r] = fp16(beta_i[r] h); (i, t)
                    // advance with c, beta reloaded only when i changes
                    int i = cb / ga.T, t = cb - i * ga.T;
                    const int64_t tstride = static_cast<int64_t>(ga.ell) * ga.R;
                    float b = i < ga.ell ? h2f(ga.beta[static_cast<int64_t>(i) * ga.R + grow]) : 0.f;
                    __half *vp = ga.V + static_cast<int64_t>(t) * tstride + static_cast<int64_t>(i) * ga.R + grow;
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        if (cb + e < ga.C) *vp = __float2half_rn(b * __uint_as_float(v[e]));
                        vp += tstride;
                        if (++t == ga.T) {
                            t = 0;
                            ++i;
                            b = i < ga.ell ? h2f(ga.beta[static_cast<int64_t>(i) * ga.R + grow]) : 0.f;
                            vp = ga.V + static_cast<int64_t>(i) * ga.R + grow;
                        }
                    }
                } else if (Cfg::kBwd) {
                    backward_chunk(ga, v, cb, grow);
                } else {
                    const int64_t base = static_cast<int64_t>(cb) * ga.N + grow;
                    const int n_ok = ga.C - cb;   // tokens of this chunk inside the batch
                    // with accumulation the y_in values are loaded eight at a time,
                    // all eight in flight together
                    if (ga.yd == DBF_BF16) {
                        __nv_bfloat16 *yp = static_cast<__nv_bfloat16 *>(ga.y) + base;
#pragma unroll
                        for (int e0 = 0; e0 < 32; e0 += 8) {
                            float yin[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                yin[e] = ga.accumulate ? __bfloat162float(yp[static_cast<int64_t>(e0 + e < n_ok ? e0 + e : 0) * ga.N]) : 0.f;
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                if (e0 + e < n_ok)
                                    yp[static_cast<int64_t>(e0 + e) * ga.N] = __float2bfloat16_rn(__uint_as_float(v[e0 + e]) + yin[e]);
                        }
                    } else {
                        float *yp = static_cast<float *>(ga.y) + base;
#pragma unroll
                        for (int e0 = 0; e0 < 32; e0 += 8) {
                            float yin[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                yin[e] = ga.accumulate ? yp[static_cast<int64_t>(e0 + e < n_ok ? e0 + e : 0) * ga.N] : 0.f;
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                if (e0 + e < n_ok) yp[static_cast<int64_t>(e0 + e) * ga.N] = __uint_as_float(v[e0 + e]) + yin[e];
                        }
                    }
                }
            }
            tc_fence_before();   // the accumulator reads are done before it is handed back
            __syncwarp();
            if (lane == 0) {
                if (kPair) bar_arrive_leader(&sh->acc_empty[ab]);
                else bar_arrive(&sh->acc_empty[ab]);
            }
            if (kFused && sk >= 0 && sk_first) {
                // the partial sums are written: the other half may read them
                __threadfence();
                __syncwarp();
                if (lane == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(fs->sk_ready + sk) : "memory");
            }
            if (kFused && flag_out >= 0) {
                // this warp's rows of the tile are written: count them on the
                // flag (every lane's stores ordered before it, for the generic
                // and the async proxy)
                asm volatile("fence.proxy.async.global;" ::: "memory");
                __threadfence();
                __syncwarp();
                if (lane == 0)
                    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(fs->flags + flag_out) : "memory");
            }
        }
    }

teardown:
    tc_fence_before();
    __syncthreads();
    if (kPair) {
        // neither CTA of a pair ends while the other may still reach its shared
        // memory (remote arrivals, the pair's MMAs and their commits, the
        // tile ring): each tells the other it is done and waits (bounded) for
        // the other
        if (threadIdx.x == 0) {
            bar_arrive_rank(&sh->exit_bar, rank ^ 1u);
            const unsigned long long t0 = global_ns();
            while (!bar_try(&sh->exit_bar, 0) && global_ns() - t0 < kWaitNs) {
            }
        }
        __syncthreads();
    }
    if (sh->abort && threadIdx.x == 0 && g.status) atomicExch(g.status, static_cast<int32_t>(DBF_ERR_TIMEOUT));
    if (warp == 1) {
        tc_fence_after();
        if (kPair) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
        else asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads, 1) gemm_kernel(const __grid_constant__ CUtensorMap tmB,
                                                                const __grid_constant__ CUtensorMap tmA, const __grid_constant__ GemmArgs g)
{
    gemm_body<Cfg>(tmB, tmA, g, nullptr, nullptr);
}

// The forward's two stages in one launch (see FusedSched): tmU and tmV are the
// maps of u and v, g1 and g2 the two stages' arguments.
template <class Cfg>
__global__ void __launch_bounds__(Cfg::kThreads, 1) gemm_fused_kernel(const __grid_constant__ CUtensorMap tmU,
                                                                      const __grid_constant__ CUtensorMap tmV,
                                                                      const __grid_constant__ GemmArgs g1,
                                                                      const __grid_constant__ GemmArgs g2,
                                                                      const __grid_constant__ FusedSched fs)
{
    gemm_body<Cfg>(tmU, tmV, g1, &g2, &fs);
}

// out[k][c] = in[c][k] for an fp16 matrix in[C][K]; columns C .. Cp-1 of out
// are zero (the row pitch of out is Cp). 32 x 32 tiles through shared memory.
__global__ void __launch_bounds__(256) transpose_f16_kernel(const uint16_t *__restrict__ in, int C, int K,
                                                            uint16_t *__restrict__ out, int Cp)
{
    __shared__ uint16_t tile[32][34];
    const int k0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads
    for (int r = ty; r < 32; r += 8) {
        const int c = c0 + r, k = k0 + tx;
        tile[r][tx] = (c < C && k < K) ? in[static_cast<int64_t>(c) * K + k] : uint16_t(0);
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int k = k0 + r, c = c0 + tx;
        if (k < K && c < Cp) out[static_cast<int64_t>(k) * Cp + c] = tile[tx][r];
    }
}

// Eight fp16 products of a row's 16-byte piece m8 (x in bf16 or fp32).
__device__ __forceinline__ uint4 scale8(const uint4 &gw, const uint4 &xa, const uint4 &xb, dbf_dtype xd)
{
    float xv[8];
    if (xd == DBF_BF16) {
        const __nv_bfloat16 *xh = reinterpret_cast<const __nv_bfloat16 *>(&xa);
#pragma unroll
        for (int e = 0; e < 8; ++e) xv[e] = __bfloat162float(xh[e]);
    } else {
        const float *f0 = reinterpret_cast<const float *>(&xa);
        const float *f1 = reinterpret_cast<const float *>(&xb);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            xv[e] = f0[e];
            xv[4 + e] = f1[e];
        }
    }
    const __half *gh = reinterpret_cast<const __half *>(&gw);
    uint4 out;
    __half *oh = reinterpret_cast<__half *>(&out);
#pragma unroll
    for (int e = 0; e < 8; ++e) oh[e] = __float2half_rn(__half2float(gh[e]) * xv[e]);
    return out;
}

// One row u[row] = fp16(gamma . x[t]) by one warp: four 16-byte pieces per
// lane in flight at a time (vectorised when M % 8 == 0 and gamma is 16-byte
// aligned), else one column per lane.
__device__ __forceinline__ void scale_row_warp(const void *x, dbf_dtype xd, const uint16_t *gp, int64_t xr, int M,
                                               __half *up, bool vec8, int lane)
{
    if (vec8) {
        const int M8 = M / 8;
        for (int base = lane; base < M8; base += 4 * 32) {
            uint4 gw[4], xa[4], xb[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int m8 = base + 32 * v;
                if (m8 >= M8) continue;
                gw[v] = __ldg(reinterpret_cast<const uint4 *>(gp) + m8);
                if (xd == DBF_BF16) {
                    xa[v] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(x) + xr) + m8);
                } else {
                    const uint4 *xf = reinterpret_cast<const uint4 *>(static_cast<const float *>(x) + xr) + 2 * m8;
                    xa[v] = __ldg(xf);
                    xb[v] = __ldg(xf + 1);
                }
            }
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int m8 = base + 32 * v;
                if (m8 < M8) reinterpret_cast<uint4 *>(up)[m8] = scale8(gw[v], xa[v], xb[v], xd);
            }
        }
    } else {
        for (int m = lane; m < M; m += 32) up[m] = __float2half_rn(h2f(gp[m]) * load_act(x, xd, xr + m));
    }
}

constexpr int kCastPiece = 1024;   // columns a warp of the pre-pass converts at a time (a multiple of 8)

// u[(i T + t), m] = fp16(gamma_i[m] x[t, m]); with M % 8 == 0 and gamma
// 16-byte aligned a warp takes whole rows with 16-byte loads and stores,
// else one column per thread.
// tok_major: output row t ell + i (U is [T][ell M], blocks of one token side
// by side) instead of i T + t.
// zero[0 .. nzero-1] are cleared too (the fused forward's claim state), and
// the launch that follows may start as soon as every block has begun.
__global__ void __launch_bounds__(256) scale_cast_kernel(const void *x, dbf_dtype xd, const uint16_t *gamma, int M,
                                                         int T, int ell, __half *U, int vec8, int tok_major,
                                                         unsigned *zero, int nzero)
{
    asm volatile("griddepcontrol.launch_dependents;");
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0u;
    const int64_t total = static_cast<int64_t>(ell) * T * M;
    if (vec8) {
        // one piece of kCastPiece columns of a row per warp step (see
        // scale_row_warp): enough warps to keep HBM busy at small T
        const int lane = threadIdx.x & 31;
        const int npieces = (M + kCastPiece - 1) / kCastPiece;
        const int64_t nitems = static_cast<int64_t>(ell) * T * npieces;
        const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
        for (int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; w < nitems; w += nw) {
            const int row = static_cast<int>(w / npieces);
            const int c0 = static_cast<int>(w - static_cast<int64_t>(row) * npieces) * kCastPiece;
            const int i = tok_major ? row % ell : row / T;
            const int t = tok_major ? row / ell : row - i * T;
            scale_row_warp(x, xd, gamma + static_cast<int64_t>(i) * M + c0, static_cast<int64_t>(t) * M + c0,
                           min(kCastPiece, M - c0), U + static_cast<int64_t>(row) * M + c0, true, lane);
        }
        return;
    }
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = idx / M;
        const int m = static_cast<int>(idx - row * M);
        const int i = tok_major ? static_cast<int>(row % ell) : static_cast<int>(row / T);
        const int64_t t = tok_major ? row / ell : row - static_cast<int64_t>(i) * T;
        U[idx] = __float2half_rn(h2f(gamma[static_cast<int64_t>(i) * M + m]) * load_act(x, xd, t * M + m));
    }
}

// Grouped pre-pass: u[(i T + t), m] = fp16(gamma_{a(t), i}[m] x[t, m]) where
// a(t) is the group holding token t; rows of tokens outside every group are
// not written (no tile reads them into a stored column).
struct GammaGroups {
    int ngroups;
    int off[kMaxGroups], n[kMaxGroups];
    const uint16_t *gamma[kMaxGroups];
};

__global__ void __launch_bounds__(256) scale_cast_grouped_kernel(const void *x, dbf_dtype xd,
                                                                 const __grid_constant__ GammaGroups gg, int M, int T,
                                                                 int ell, __half *U, int vec8)
{
    // one row (i T + t) per warp step; the row's group is found by the warp
    // together (lane k tests groups k, k + 32, ...)
    const int lane = threadIdx.x & 31;
    const int nrows = ell * T;   // <= 2^30
    const int nw = static_cast<int>((gridDim.x * blockDim.x) >> 5);
    for (int row = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5); row < nrows; row += nw) {
        const int i = row / T;
        const int t = row - i * T;
        int gi = -1;
        for (int k = lane; k < gg.ngroups; k += 32)
            if (t >= gg.off[k] && t < gg.off[k] + gg.n[k]) gi = k;
        const unsigned found = __ballot_sync(0xffffffffu, gi >= 0);
        if (!found) continue;
        gi = __shfl_sync(0xffffffffu, gi, __ffs(found) - 1);
        const uint16_t *gp = gg.gamma[gi] + static_cast<int64_t>(i) * M;
        scale_row_warp(x, xd, gp, static_cast<int64_t>(t) * M, M, U + static_cast<int64_t>(row) * M,
                       vec8 && (reinterpret_cast<uintptr_t>(gp) & 15u) == 0, lane);
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
// box_rows: BN for the B operand, BM for a dense A operand; ld: elements
// per row (>= K, a multiple of 8).
bool make_map(CUtensorMap *map, const void *base, int64_t K, int64_t rows, int box_rows = BN, int64_t ld = 0)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld > 0 ? ld : K) * 2};
    const cuuint32_t box[2] = {BK, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class Cfg>
constexpr size_t gemm_smem() { return 1024 + Cfg::SA * A_BYTES + Cfg::SB * Cfg::kBBytes + sizeof(GemmSmem) + 64; }

template <class Cfg>
cudaError_t launch_gemm(const CUtensorMap &map, const GemmArgs &args, cudaStream_t s, const CUtensorMap *map_a,
                        int32_t *status)
{
    GemmArgs a = args;
    a.status = status;   // a bounded wait that expires stores DBF_ERR_TIMEOUT here
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(gemm_kernel<Cfg>), static_cast<int>(gemm_smem<Cfg>()));
    if (e != cudaSuccess) return e;
    const int sms = device_sms();
    const int tiles = a.ngroups ? a.tiles_total : ((a.P + BM - 1) / BM) * ((a.C + BN - 1) / BN);
    gemm_kernel<Cfg><<<tiles < sms ? tiles : sms, Cfg::kThreads, gemm_smem<Cfg>(), s>>>(map, map_a ? *map_a : map, a);
    return cudaGetLastError();
}

// CTA pairs of 'kernel' (launched as in cfg) that can be resident at once:
// queried once per kernel and device (the query is slow next to a launch).
template <class K>
int resident_pairs(K kernel, cudaLaunchConfig_t cfg)
{
    static std::mutex lock;
    static std::map<std::pair<int, const void *>, int> resident;
    int dev = 0;
    cudaGetDevice(&dev);
    int pairs = device_sms() / 2;
    std::lock_guard<std::mutex> guard(lock);
    const auto key = std::make_pair(dev, reinterpret_cast<const void *>(kernel));
    auto it = resident.find(key);
    if (it == resident.end()) {
        cfg.gridDim = dim3(2 * pairs);
        int n = 0;
        const int r = (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) == cudaSuccess && n > 0) ? n : pairs;
        (void)cudaGetLastError();
        it = resident.emplace(key, r).first;
    }
    return it->second < pairs ? it->second : pairs;
}

// The forward's GEMMs on CTA pairs: clusters of two CTAs, each pair walking
// 256-row x 256-token tiles (as many pairs as can be resident at once).
template <class Cfg>
cudaError_t launch_gemm_pair(const CUtensorMap &map, const GemmArgs &args, cudaStream_t s, int32_t *status)
{
    GemmArgs a = args;
    a.status = status;
    const size_t smem = gemm_smem<Cfg>();
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(gemm_kernel<Cfg>), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int tiles = ((a.P + 2 * BM - 1) / (2 * BM)) * ((a.C + BN - 1) / BN);
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int pairs = resident_pairs(gemm_kernel<Cfg>, cfg);
    if (pairs > tiles) pairs = tiles;
    if (pairs < 1) pairs = 1;
    cfg.gridDim = dim3(2 * pairs);
    e = cudaLaunchKernelEx(&cfg, gemm_kernel<Cfg>, map, map, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// ---- the fused forward's schedule ----------------------------------------------
constexpr int kMaxSplit = 64;   // stage-2 tiles at most that run split in K
// a split tile's counters: one per (split tile, CTA of the pair, epilogue warp)
constexpr int kSkSlots = kMaxSplit * 2 * FusedCfg::kEpiWarps;

// Makespan of the claim order (each pair claims its next tile when it starts
// one) when the last nsk stage-2 tiles run as two halves of K, under a cost
// model: a tile costs its K steps plus two, a half its share plus three (the
// exchange of partial sums).
double fused_makespan(int pairs, int n1, int n2, int nsk, int nk1, int nk2)
{
    const int total = n1 + n2 + nsk;
    auto cost = [&](int u) {
        if (u < n1) return nk1 + 2.0;
        if (u < n1 + n2 - nsk) return nk2 + 2.0;
        return 0.5 * nk2 + 3.0;
    };
    std::vector<double> end(pairs, 0.0);
    // min-heap of (time of the pair's next claim, pair)
    std::priority_queue<std::pair<double, int>, std::vector<std::pair<double, int>>, std::greater<>> claims;
    int u = 0;
    for (int p = 0; p < pairs && u < total; ++p, ++u) {
        end[p] = cost(u);
        claims.push({0.0, p});
    }
    for (; u < total; ++u) {
        const auto c = claims.top();
        claims.pop();
        const int p = c.second;
        claims.push({end[p], p});   // it starts this tile when its current one ends, and claims again
        end[p] += cost(u);
    }
    double m = 0.0;
    for (double e : end) m = e > m ? e : m;
    return m;
}

// Stage-2 tiles to split in K (at most smax): the count with the smallest
// modelled makespan (the smallest such count), memoised per shape.
int fused_splits(int pairs, int n1, int n2, int nk1, int nk2, int smax)
{
    static std::mutex lock;
    static std::map<std::tuple<int, int, int, int, int, int>, int> memo;
    const auto key = std::make_tuple(pairs, n1, n2, nk1, nk2, smax);
    {
        std::lock_guard<std::mutex> guard(lock);
        const auto it = memo.find(key);
        if (it != memo.end()) return it->second;
    }
    const int hmax = std::min(n2, smax);
    const int step = std::max(1, pairs / 16);
    int best = 0;
    double best_t = fused_makespan(pairs, n1, n2, 0, nk1, nk2);
    for (int nsk = step; nsk <= hmax; nsk += step) {
        const double t = fused_makespan(pairs, n1, n2, nsk, nk1, nk2);
        if (t < best_t - 1e-9) {
            best_t = t;
            best = nsk;
        }
    }
    std::lock_guard<std::mutex> guard(lock);
    if (memo.size() > 256) memo.clear();
    memo[key] = best;
    return best;
}

constexpr int kFusedMinSteps = 32;   // K steps per stage below which the two-launch path runs

// Two GEMMs in one launch on CTA pairs (Cfg: FusedCfg for the forward's two
// stages, BwdFusedCfg for pairs of the backward's independent sign GEMMs):
// fs.n1 tiles of the first, n2 of the second. With pdl the launch allows
// programmatic stream serialisation, so that its prologue and first sign
// expansions overlap the pre-pass before it (which clears the claim state
// it waits for). The forward (fs.dep) splits its last stage-2 tiles in K.
template <class Cfg>
cudaError_t launch_fused(const CUtensorMap &mu, const CUtensorMap &mv, const GemmArgs &a1, const GemmArgs &a2,
                         FusedSched fs, int n2, int nk1, int nk2, bool pdl, cudaStream_t s, int32_t *status)
{
    GemmArgs g1 = a1, g2 = a2;
    g1.status = status;
    g2.status = status;
    const size_t smem = gemm_smem<Cfg>();
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(gemm_fused_kernel<Cfg>), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int pairs = resident_pairs(gemm_fused_kernel<Cfg>, cfg);
    cfg.numAttrs = pdl ? 2 : 1;
    // only the forward (dep 1) splits tiles in K: the backward's epilogues
    // have no exchange of partial sums
    fs.nsk = fs.dep == 1 ? fused_splits(pairs, fs.n1, n2, nk1, nk2, std::min(n2, kMaxSplit)) : 0;
    fs.ksplit = (nk2 / 2) & ~1;
    fs.n2f = n2 - fs.nsk;
    const int total = fs.n1 + fs.n2f + 2 * fs.nsk;
    if (total <= 0) return cudaSuccess;
    if (pairs > total) pairs = total;
    if (pairs < 1) pairs = 1;
    cfg.gridDim = dim3(2 * pairs);
    e = cudaLaunchKernelEx(&cfg, gemm_fused_kernel<Cfg>, mu, mv, g1, g2, fs);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// the sticky status word of a workspace header
int32_t *ws_status(void *ws) { return reinterpret_cast<int32_t *>(static_cast<char *>(ws) + kWsStatusOffset); }

size_t u_bytes(const dbf_layer &L, int64_t T) { return align_up(static_cast<size_t>(L.ell) * T * L.M * 2, 256); }
size_t v_bytes(const dbf_layer &L, int64_t T) { return align_up(static_cast<size_t>(T) * L.ell * L.R * 2, 256); }

}  // namespace

int gemm_forward_launches(const dbf_layer &L)
{
    return (L.M / BK >= kFusedMinSteps && L.ell * L.R / BK >= kFusedMinSteps) ? 2 : 3;
}

bool gemm_shape_ok(const dbf_layer &L)
{
    return L.M % 128 == 0 && L.R % 128 == 0 && L.M > 0 && L.R > 0 && L.N > 0;
}

// the fused forward's claim state: the claim counter, the stage-1
// column-block flags and the split tiles' counters (zeroed by the pre-pass)
int ctl_words(const dbf_layer &L, int64_t T)
{
    constexpr int TBN = FusedCfg::kTBN;
    return static_cast<int>(1 + (static_cast<int64_t>(L.ell) * T + TBN - 1) / TBN + 2 * kSkSlots);
}

// the split tiles' partial sums: 256 x TBN fp32 per split tile
size_t part_bytes(const dbf_layer &L, int64_t T)
{
    constexpr int TBN = FusedCfg::kTBN;
    if (gemm_forward_launches(L) != 2) return 0;
    const int64_t n2 = ((L.N + 2 * BM - 1) / (2 * BM)) * ((T + TBN - 1) / TBN);
    return static_cast<size_t>(std::min<int64_t>(n2, kMaxSplit)) * 2 * BM * TBN * 4;
}

size_t gemm_workspace_bytes(const dbf_layer &L, int64_t T)
{
    return kWsHeaderBytes + u_bytes(L, T) + v_bytes(L, T) + align_up(4 * static_cast<size_t>(ctl_words(L, T)), 256) +
           part_bytes(L, T);
}

cudaError_t gemm_forward(const dbf_layer &L, const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                         int flags, void *ws, cudaStream_t s)
{
    int32_t *st = ws_status(ws);
    if (T > (1 << 30) / L.ell) return cudaErrorInvalidValue;
    char *body = static_cast<char *>(ws) + kWsHeaderBytes;   // the header belongs to the decode path
    __half *U = reinterpret_cast<__half *>(body);
    __half *V = reinterpret_cast<__half *>(body + u_bytes(L, T));
    const int Ti = static_cast<int>(T);
    unsigned *ctl = reinterpret_cast<unsigned *>(body + u_bytes(L, T) + v_bytes(L, T));
    const int nk1 = L.M / BK, nk2 = L.ell * L.R / BK;
    constexpr int TBN = FusedCfg::kTBN;   // the one-launch forward's token rows per tile
    const int n_c1 = static_cast<int>((static_cast<int64_t>(L.ell) * T + TBN - 1) / TBN);
    const bool fused = gemm_forward_launches(L) == 2;
    {
        const int64_t total = static_cast<int64_t>(L.ell) * T * L.M;
        const int vec8 = (L.M % 8 == 0) && ((reinterpret_cast<uintptr_t>(L.gamma) & 15u) == 0);
        const int64_t pieces = (L.M + kCastPiece - 1) / kCastPiece;
        int64_t blocks = vec8 ? (static_cast<int64_t>(L.ell) * T * pieces + 7) / 8 : (total + 255) / 256;
        if (blocks > 8 * device_sms()) blocks = 8 * device_sms();
        scale_cast_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(x, xd, L.gamma, L.M, Ti, L.ell, U, vec8, 0,
                                                                   fused ? ctl : nullptr, fused ? ctl_words(L, T) : 0);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // CTA pairs: each CTA loads 128 of a tile's 256 token rows
    CUtensorMap mu, mv;
    if (!make_map(&mu, U, L.M, static_cast<int64_t>(L.ell) * T, FwdPairCfg::kBRows)) return cudaErrorInvalidValue;
    if (!make_map(&mv, V, static_cast<int64_t>(L.ell) * L.R, T, FwdPairCfg::kBRows)) return cudaErrorInvalidValue;
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
    if (fused) {
        FusedSched fs = {};
        fs.n_p1 = (L.R + 2 * BM - 1) / (2 * BM);
        fs.n_p2 = (L.N + 2 * BM - 1) / (2 * BM);
        fs.n1 = fs.n_p1 * n_c1;
        fs.ctr = ctl;
        fs.flags = ctl + 1;
        fs.flag_target = static_cast<unsigned>(fs.n_p1 * 2 * FusedCfg::kEpiWarps);
        fs.sk_count = ctl + 1 + n_c1;
        fs.sk_ready = fs.sk_count + kSkSlots;
        fs.sk_part = reinterpret_cast<float *>(reinterpret_cast<char *>(ctl) + align_up(4 * static_cast<size_t>(ctl_words(L, T)), 256));
        const int n2 = fs.n_p2 * ((Ti + TBN - 1) / TBN);
        fs.dep = 1;
        return launch_fused<FusedCfg>(mu, mv, a1, a2, fs, n2, nk1, nk2, true, s, st);
    }
    cudaError_t e = launch_gemm_pair<FwdPairCfg>(mu, a1, s, st);
    if (e != cudaSuccess) return e;
    return launch_gemm_pair<FwdPairCfg>(mv, a2, s, st);
}

}  // namespace dbf

// The one-launch forward's schedule as chosen for a layer and token count
// with 'pairs' resident CTA pairs (host-side model; see dbf.h).
extern "C" dbf_status dbf_debug_fused_schedule(const dbf_layer *L, int64_t T, int32_t pairs, int32_t *tiles,
                                               double *makespan)
{
    using namespace dbf;
    if (!L || !tiles || !makespan || T < 1 || pairs < 1 || L->M <= 0 || L->N <= 0 || L->R <= 0 || L->ell < 1)
        return DBF_ERR_INVALID_ARG;
    if (!gemm_shape_ok(*L) || gemm_forward_launches(*L) != 2) return DBF_ERR_UNSUPPORTED;
    const int nk1 = L->M / BK, nk2 = L->ell * L->R / BK;
    constexpr int TBN = FusedCfg::kTBN;
    const int n_c1 = static_cast<int>((static_cast<int64_t>(L->ell) * T + TBN - 1) / TBN);
    const int n1 = ((L->R + 2 * BM - 1) / (2 * BM)) * n_c1;
    const int n2 = ((L->N + 2 * BM - 1) / (2 * BM)) * static_cast<int>((T + TBN - 1) / TBN);
    const int nsk = fused_splits(pairs, n1, n2, nk1, nk2, std::min(n2, kMaxSplit));
    tiles[0] = n1;
    tiles[1] = n2;
    tiles[2] = nsk;
    makespan[0] = fused_makespan(pairs, n1, n2, 0, nk1, nk2);
    makespan[1] = fused_makespan(pairs, n1, n2, nsk, nk1, nk2);
    return DBF_OK;
}

// ---- backward (tcgen05, four sign GEMMs) ---------------------------------------
namespace dbf {
namespace {

cudaError_t scale_cast(const void *x, dbf_dtype xd, const uint16_t *scale, int K, int64_t T, int ell, __half *out,
                       cudaStream_t s, int tok_major = 0, unsigned *zero = nullptr, int nzero = 0)
{
    const int64_t total = static_cast<int64_t>(ell) * T * K;
    const int vec8 = (K % 8 == 0) && ((reinterpret_cast<uintptr_t>(scale) & 15u) == 0);
    const int64_t pieces = (K + kCastPiece - 1) / kCastPiece;
    int64_t blocks = vec8 ? (static_cast<int64_t>(ell) * T * pieces + 7) / 8 : (total + 255) / 256;
    if (blocks > 8 * device_sms()) blocks = 8 * device_sms();
    scale_cast_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(x, xd, scale, K, static_cast<int>(T), ell, out, vec8,
                                                               tok_major, zero, nzero);
    return cudaGetLastError();
}

struct BwdLayout {
    size_t ctl;                     // claim counters of the two fused launches (256 bytes)
    size_t u, a, h32, vh, vg;       // offsets after the header
    size_t ut, at, vht, vgt;        // transposed operands of the sign-matrix gradients
    size_t total;
    int64_t cp;                     // row pitch of the transposed operands (elements)
};

BwdLayout bwd_layout(const dbf_layer &L, int64_t T, bool signs)
{
    const int64_t C = static_cast<int64_t>(L.ell) * T;
    BwdLayout b;
    b.cp = (C + 7) / 8 * 8;
    b.ctl = 0;
    // claim counters of the two fused launches and one flag per G3 tile
    b.u = align_up(4 * static_cast<size_t>(2 + ((L.R + 255) / 256) * ((C + 255) / 256)), 256);
    b.a = b.u + align_up(static_cast<size_t>(C) * L.M * 2, 256);
    b.h32 = b.a + align_up(static_cast<size_t>(C) * L.N * 2, 256);
    b.vh = b.h32 + align_up(static_cast<size_t>(C) * L.R * 4, 256);
    b.vg = b.vh + align_up(static_cast<size_t>(C) * L.R * 2, 256);
    b.total = b.vg + align_up(static_cast<size_t>(C) * L.R * 2, 256);
    b.ut = b.at = b.vht = b.vgt = 0;
    if (signs) {
        b.ut = b.total;
        b.at = b.ut + align_up(static_cast<size_t>(b.cp) * L.M * 2, 256);
        b.vht = b.at + align_up(static_cast<size_t>(b.cp) * L.N * 2, 256);
        b.vgt = b.vht + align_up(static_cast<size_t>(b.cp) * L.R * 2, 256);
        b.total = b.vgt + align_up(static_cast<size_t>(b.cp) * L.R * 2, 256);
    }
    return b;
}

cudaError_t transpose_f16(const __half *in, int64_t C, int64_t K, __half *out, int64_t Cp, cudaStream_t s)
{
    const dim3 grid(static_cast<unsigned>((K + 31) / 32), static_cast<unsigned>((Cp + 31) / 32));
    transpose_f16_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint16_t *>(in), static_cast<int>(C),
                                              static_cast<int>(K), reinterpret_cast<uint16_t *>(out),
                                              static_cast<int>(Cp));
    return cudaGetLastError();
}

// out[q][p] (+)= sum_c A[p][c] Bm[q][c] over the Kpad contraction (fp16
// operands [P][cp] and [Q][cp], zero past the real length), fp32 out with row
// pitch P: the dense GEMM of the sign-matrix gradients.
cudaError_t dense_outer(const __half *A, int64_t P, const __half *Bm, int64_t Q, int64_t cp, float *out, bool acc,
                        int32_t *st, cudaStream_t s)
{
    CUtensorMap ma, mb;
    if (!make_map(&ma, A, cp, P, BM) || !make_map(&mb, Bm, cp, Q, BN)) return cudaErrorInvalidValue;
    GemmArgs g = {};
    g.dense_a = 1;
    g.P = static_cast<int>(P);
    g.Ktot = g.Kp = static_cast<int>((cp + 2 * BK - 1) / (2 * BK) * (2 * BK));
    g.pitch = 1;
    g.C = static_cast<int>(Q);
    g.T = static_cast<int>(Q);
    g.ell = 1;
    g.stage = 2;
    g.y = out;
    g.yd = DBF_F32;
    g.N = static_cast<int>(P);
    g.accumulate = acc ? 1 : 0;
    return launch_gemm<FwdCfg>(mb, g, s, &ma, st);
}

GemmArgs sign_gemm_args(const uint32_t *signs, int P, int K, int C, int T, int ell, int stage)
{
    GemmArgs a = {};
    a.signs = signs;
    a.pitch = static_cast<int>(pitch_words(K));
    a.P = P;
    a.Kp = K;
    a.Ktot = K;
    a.C = C;
    a.T = T;
    a.ell = ell;
    a.stage = stage;
    return a;
}

}  // namespace

bool gemm_backward_shape_ok(const dbf_layer &L)
{
    return L.M % 128 == 0 && L.N % 128 == 0 && L.R % 128 == 0 && L.M > 0 && L.N > 0 && L.R > 0;
}

size_t gemm_backward_workspace_bytes(const dbf_layer &L, int64_t T, bool signs)
{
    return kWsHeaderBytes + bwd_layout(L, T, signs).total;
}

// Gradients through the forward (see dbf.h, dbf_backward), as four sign
// GEMMs whose epilogues do the per-channel scalings and the reductions over
// tokens. Columns of every GEMM are c = i T + t (envelope-major).
//   G3: h_i = B2 u_i,      u_i = fp16(gamma_i . x)    -> H32 = h, Vh = fp16(beta_i . h)
//   G4: g_i = B1^T a_i,    a_i = fp16(alpha_i . dy)   -> dbeta_i += sum_t g h, Vg = fp16(beta_i . g)
//   G5: z_i = B1 Vh_i                                 -> dalpha_i += sum_t z dy
//   G6: e_i = B2^T Vg_i                               -> dgamma_i += sum_t e x, dx = sum_i gamma_i . e
cudaError_t gemm_backward(const dbf_layer &L, const uint32_t *b1t, const uint32_t *b2t, const void *x, dbf_dtype xd,
                          const void *dy, dbf_dtype dyd, int64_t T, float *dx, float *dalpha, float *dbeta,
                          float *dgamma, float *db1, float *db2, int flags, void *ws, cudaStream_t s)
{
    int32_t *st = ws_status(ws);
    if (T > (1 << 30) / L.ell) return cudaErrorInvalidValue;
    const bool acc = (flags & DBF_ACCUMULATE) != 0;
    const int ell = L.ell, Ti = static_cast<int>(T), C = ell * Ti;
    const bool signs = db1 || db2;
    const BwdLayout b = bwd_layout(L, T, signs);
    char *body = static_cast<char *>(ws) + kWsHeaderBytes;
    __half *U = reinterpret_cast<__half *>(body + b.u);
    __half *A = reinterpret_cast<__half *>(body + b.a);
    float *H32 = reinterpret_cast<float *>(body + b.h32);
    __half *Vh = reinterpret_cast<__half *>(body + b.vh);
    __half *Vg = reinterpret_cast<__half *>(body + b.vg);
    cudaError_t e;
    if (!acc) {
        if (dalpha && (e = cudaMemsetAsync(dalpha, 0, sizeof(float) * ell * L.N, s)) != cudaSuccess) return e;
        if (dbeta && (e = cudaMemsetAsync(dbeta, 0, sizeof(float) * ell * L.R, s)) != cudaSuccess) return e;
        if (dgamma && (e = cudaMemsetAsync(dgamma, 0, sizeof(float) * ell * L.M, s)) != cudaSuccess) return e;
        if (dx && ell > 1 && (e = cudaMemsetAsync(dx, 0, sizeof(float) * T * L.M, s)) != cudaSuccess) return e;
    }
    // G4 and G3, then G5 and G6, as two launches with tiles claimed at run time
    // when every contraction is at least 32 K steps deep (else one launch each)
    const bool fused = L.M / BK >= kFusedMinSteps && L.N / BK >= kFusedMinSteps && L.R / BK >= kFusedMinSteps;
    unsigned *ctl = reinterpret_cast<unsigned *>(body + b.ctl);
    constexpr int TBN = BwdFusedCfg::kTBN;   // token columns per tile of the fused launches
    const int n_g3 = ((L.R + 2 * BM - 1) / (2 * BM)) * ((C + TBN - 1) / TBN);   // G3 tiles (G4 the same)
    if ((e = scale_cast(x, xd, L.gamma, L.M, T, ell, U, s, 0, fused ? ctl : nullptr, fused ? 2 + n_g3 : 0)) !=
        cudaSuccess)
        return e;
    if ((e = scale_cast(dy, dyd, L.alpha, L.N, T, ell, A, s)) != cudaSuccess) return e;
    CUtensorMap mu, ma, mvh, mvg;
    // the four sign GEMMs run on CTA pairs (each CTA loads half of a token tile)
    constexpr int kb = BwdPairCfg::kBRows;
    if (!make_map(&mu, U, L.M, C, kb) || !make_map(&ma, A, L.N, C, kb) || !make_map(&mvh, Vh, L.R, C, kb) ||
        !make_map(&mvg, Vg, L.R, C, kb))
        return cudaErrorInvalidValue;
    GemmArgs g3 = sign_gemm_args(L.b2_packed, L.R, L.M, C, Ti, ell, 3);
    g3.H32 = H32;
    g3.Vout = Vh;
    g3.cscale = L.beta;
    GemmArgs g4 = sign_gemm_args(b1t, L.R, L.N, C, Ti, ell, 4);
    g4.H32 = H32;
    g4.Vout = Vg;
    g4.cscale = L.beta;
    g4.red = dbeta;
    GemmArgs g5 = {}, g6 = {};
    if (dalpha) {
        g5 = sign_gemm_args(L.b1_packed, L.N, L.R, C, Ti, ell, 5);
        g5.red = dalpha;
        g5.W = dy;
        g5.wd = dyd;
    }
    if (dx || dgamma) {
        g6 = sign_gemm_args(b2t, L.M, L.R, C, Ti, ell, 6);
        g6.red = dgamma;
        g6.W = x;
        g6.wd = xd;
        g6.cscale = L.gamma;
        g6.dx = dx;
        g6.dx_mode = ell > 1 ? 2 : (acc ? 1 : 0);
    }
    if (fused) {
        // pair row tiles of P rows, token tiles of the C columns
        auto rows = [](int P) { return (P + 2 * BM - 1) / (2 * BM); };
        const int n_c = (C + TBN - 1) / TBN;
        // G3 first, then G4, whose epilogue reads the h of the G3 tile of the
        // same index: it waits for that tile's flag (G3 tiles are claimed
        // first and never wait, so every flag is set)
        FusedSched f1 = {};
        f1.dep = 2;
        f1.n_p1 = rows(L.R);
        f1.n1 = f1.n_p1 * n_c;
        f1.n_p2 = rows(L.R);
        f1.ctr = ctl;
        f1.flags = ctl + 2;
        f1.flag_target = 2 * BwdFusedCfg::kEpiWarps;
        if ((e = launch_fused<BwdFusedCfg>(mu, ma, g3, g4, f1, f1.n_p2 * n_c, L.M / BK, L.N / BK, true, s, st)) !=
            cudaSuccess)
            return e;
        // G5 and G6 read what G3 and G4 wrote: a plain launch after them
        FusedSched f2 = {};
        f2.n_p1 = rows(L.N);
        f2.n1 = dalpha ? f2.n_p1 * n_c : 0;
        f2.n_p2 = rows(L.M);
        f2.ctr = ctl + 1;
        if ((e = launch_fused<BwdFusedCfg>(mvh, mvg, g5, g6, f2, (dx || dgamma) ? f2.n_p2 * n_c : 0, L.R / BK,
                                           L.R / BK, false, s, st)) != cudaSuccess)
            return e;
    } else {
        if ((e = launch_gemm_pair<BwdPairCfg>(mu, g3, s, st)) != cudaSuccess) return e;
        if ((e = launch_gemm_pair<BwdPairCfg>(ma, g4, s, st)) != cudaSuccess) return e;
        if (dalpha && (e = launch_gemm_pair<BwdPairCfg>(mvh, g5, s, st)) != cudaSuccess) return e;
        if ((dx || dgamma) && (e = launch_gemm_pair<BwdPairCfg>(mvg, g6, s, st)) != cudaSuccess) return e;
    }
    // sign-matrix gradients: dB1 = sum_c a_c v_c^T (N x R), dB2 = sum_c w_c u_c^T
    // (R x M), dense products contracting over the envelope-major token index
    if (signs) {
        __half *Ut = reinterpret_cast<__half *>(body + b.ut), *At = reinterpret_cast<__half *>(body + b.at);
        __half *Vht = reinterpret_cast<__half *>(body + b.vht), *Vgt = reinterpret_cast<__half *>(body + b.vgt);
        if (db1) {
            if ((e = transpose_f16(Vh, C, L.R, Vht, b.cp, s)) != cudaSuccess) return e;
            if ((e = transpose_f16(A, C, L.N, At, b.cp, s)) != cudaSuccess) return e;
            if ((e = dense_outer(Vht, L.R, At, L.N, b.cp, db1, acc, st, s)) != cudaSuccess) return e;
        }
        if (db2) {
            if ((e = transpose_f16(U, C, L.M, Ut, b.cp, s)) != cudaSuccess) return e;
            if ((e = transpose_f16(Vg, C, L.R, Vgt, b.cp, s)) != cudaSuccess) return e;
            if ((e = dense_outer(Ut, L.M, Vgt, L.R, b.cp, db2, acc, st, s)) != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

}  // namespace dbf

// ---- multi-boolean-kernel layer (MBOK) on the same GEMM -------------------------
// Multi-Boolean Architectures page, section 2: y = sum_k s_out_k . (W_k (s_in_k . x)).
// One GEMM with K blocks of M contraction columns: the A operand of block k
// is s_out_k[n] * W_k[n, :] (the packed row of W holds the K kernels' rows
// side by side, so the cursor moves on to the next block instead of reading
// the same row again), the B operand is u[t][k M + m] = fp16(s_in_k[m] x[t, m]).
namespace dbf {

bool mbok_shape_ok(int64_t M, int64_t N, int64_t K) { return M > 0 && N > 0 && K >= 1 && K <= 64 && M % 128 == 0; }

// header, the fp16 operand (T x K M), the claim counter of the GEMM's tiles
size_t mbok_workspace_bytes(int64_t M, int64_t K, int64_t T)
{
    return kWsHeaderBytes + align_up(static_cast<size_t>(T) * K * M * 2, 256) + 256;
}

cudaError_t mbok_forward(int M, int N, int K, const uint32_t *w_packed, const uint16_t *s_in, const uint16_t *s_out,
                         const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T, int flags, void *ws,
                         cudaStream_t s)
{
    int32_t *st = ws_status(ws);
    if (T > (1 << 30) / K) return cudaErrorInvalidValue;
    __half *U = reinterpret_cast<__half *>(static_cast<char *>(ws) + kWsHeaderBytes);
    unsigned *ctl = reinterpret_cast<unsigned *>(static_cast<char *>(ws) + kWsHeaderBytes +
                                                 align_up(static_cast<size_t>(T) * K * M * 2, 256));
    cudaError_t e = scale_cast(x, xd, s_in, M, T, K, U, s, 1, ctl, 1);   // also zeroes the claim counter
    if (e != cudaSuccess) return e;
    CUtensorMap mu;
    // CTA pairs: each CTA loads 128 of a tile's 256 token rows
    if (!make_map(&mu, U, static_cast<int64_t>(K) * M, T, FwdPairCfg::kBRows)) return cudaErrorInvalidValue;
    GemmArgs a = {};
    a.signs = w_packed;
    a.pitch = static_cast<int>(pitch_words(static_cast<int64_t>(K) * M));
    a.P = N;
    a.Kp = M;
    a.Ktot = K * M;
    a.arow_scale = s_out;
    a.env_advance = 1;
    a.C = static_cast<int>(T);
    a.T = static_cast<int>(T);
    a.ell = K;
    a.stage = 2;
    a.y = y;
    a.yd = yd;
    a.N = N;
    a.accumulate = (flags & DBF_ACCUMULATE) ? 1 : 0;
    // the one-launch kernel's 512-token pair tiles, all of them output tiles
    // (no first stage), claimed at run time
    constexpr int TBN = FusedCfg::kTBN;
    FusedSched fs = {};
    fs.n_p2 = (N + 2 * BM - 1) / (2 * BM);
    fs.ctr = ctl;
    const int n2 = fs.n_p2 * static_cast<int>((T + TBN - 1) / TBN);
    return launch_fused<FusedCfg>(mu, mu, a, a, fs, n2, 0, K * M / BK, true, s, st);
}

}  // namespace dbf

// ---- grouped forward (segmented serving of adapters of one shape) ----------------
namespace dbf {

// Adapters 'layers[k]' (same M, N, R, ell; GEMM-eligible) on token rows
// [off[k], off[k] + n[k]) of x / y, count <= kMaxGroups: one pre-pass and two
// grouped GEMM launches, tiles of all groups side by side in each launch.
cudaError_t gemm_forward_grouped(const dbf_layer *const *layers, const int *off, const int *n, int count,
                                 const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T, int flags, void *ws,
                                 cudaStream_t s)
{
    int32_t *st = ws_status(ws);
    if (count < 1 || count > kMaxGroups) return cudaErrorInvalidValue;
    const dbf_layer &L = *layers[0];
    if (T > (1 << 30) / L.ell) return cudaErrorInvalidValue;
    char *body = static_cast<char *>(ws) + kWsHeaderBytes;
    __half *U = reinterpret_cast<__half *>(body);
    __half *V = reinterpret_cast<__half *>(body + u_bytes(L, T));
    const int Ti = static_cast<int>(T);
    GammaGroups gg = {};
    gg.ngroups = count;
    for (int k = 0; k < count; ++k) {
        gg.off[k] = off[k];
        gg.n[k] = n[k];
        gg.gamma[k] = layers[k]->gamma;
    }
    {
        int64_t blocks = (static_cast<int64_t>(L.ell) * T + 7) / 8;   // a warp per row
        if (blocks > 8 * device_sms()) blocks = 8 * device_sms();
        scale_cast_grouped_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(x, xd, gg, L.M, Ti, L.ell, U, L.M % 8 == 0);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mu, mv;
    if (!make_map(&mu, U, L.M, static_cast<int64_t>(L.ell) * T)) return cudaErrorInvalidValue;
    if (!make_map(&mv, V, static_cast<int64_t>(L.ell) * L.R, T)) return cudaErrorInvalidValue;
    // stage 1: per group ell x ceil(n / BN) token tiles, each inside one envelope
    GemmArgs a1 = {};
    a1.pitch = static_cast<int>(pitch_words(L.M));
    a1.P = L.R;
    a1.Kp = L.M;
    a1.Ktot = L.M;
    a1.C = L.ell * Ti;
    a1.stage = 1;
    a1.V = V;
    a1.T = Ti;
    a1.ell = L.ell;
    a1.R = L.R;
    a1.N = L.N;
    GemmArgs a2 = {};
    a2.pitch = static_cast<int>(pitch_words(L.R));
    a2.P = L.N;
    a2.Kp = L.R;
    a2.Ktot = L.ell * L.R;
    a2.C = Ti;
    a2.stage = 2;
    a2.T = Ti;
    a2.ell = L.ell;
    a2.R = L.R;
    a2.y = y;
    a2.yd = yd;
    a2.N = L.N;
    a2.accumulate = (flags & DBF_ACCUMULATE) ? 1 : 0;
    const int np1 = (L.R + BM - 1) / BM, np2 = (L.N + BM - 1) / BM;
    int t1 = 0, t2 = 0;
    for (int k = 0; k < count; ++k) {
        const int ncpe = (n[k] + BN - 1) / BN;
        a1.grp[k] = GroupRef{layers[k]->b2_packed, nullptr, layers[k]->beta, off[k], n[k], t1, ncpe};
        a2.grp[k] = GroupRef{layers[k]->b1_packed, layers[k]->alpha, nullptr, off[k], n[k], t2, ncpe};
        t1 += np1 * L.ell * ncpe;
        t2 += np2 * ncpe;
    }
    a1.ngroups = a2.ngroups = count;
    a1.tiles_total = t1;
    a2.tiles_total = t2;
    cudaError_t e = launch_gemm<GrpCfg>(mu, a1, s, nullptr, st);
    if (e != cudaSuccess) return e;
    return launch_gemm<GrpCfg>(mv, a2, s, nullptr, st);
}

}  // namespace dbf
