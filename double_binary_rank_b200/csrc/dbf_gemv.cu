// Decode-regime forward in two launches: two sign-accumulation GEMVs with
// per-channel scaling, for the calls neither single-launch kernel
// (dbf_decode.cu, dbf_decode_multi.cu) takes: M above 8192, more than 512
// segments, or no plan that fits in shared memory.
//
// LoRDBA page, section 2 ("Kernel de Inferencia"): the forward is two
// sign-accumulation matrix products interleaved with per-channel scaling;
// DBF page, section 2 ("Inferencia"): the dense product becomes additions and
// scalar-vector products. Stage 1 computes v_i = beta_i . (B2 (gamma_i . x)),
// stage 2 computes y = [acc] y + sum_i alpha_i . (B1 v_i).
//
// Arithmetic. A sign is s = 1 - 2b with b in {0, 1} the packed bit, so
//   sum_k s_k a_k = sum_k a_k - 2 sum_k b_k a_k .
// Every activation column a (one token and envelope) becomes the integers
// q_k = round(a_k 2^sh), |q| <= 2^22, with one power-of-two scale per column
// (q is exact whenever a is a small dyadic value), written as three balanced
// base-256 int8 digits. mma.sync m16n8k32 u8 x s8 accumulates sum_k b_k d_k
// exactly in int32. The A operand needs no shifts: masking a packed word
// with 0x01010101 << j gives bytes in {0, 2^j}, so the eight masks j = 0..7
// of one word feed eight MMAs whose accumulators carry the weight 2^j and are
// folded with an exact right shift. The digit planes are recombined in int64
// and converted once: (sum q - 2 sum b q) 2^-sh. Integer accumulation makes
// the result independent of how K is split across warps.
//
// Stage 1 digitises gamma.x from max|gamma.x|. For v = beta.h it fixes the
// scale in advance from the bound |v_r| <= max|beta| sum_m |q_m| 2^-sh
// (integers and bit patterns only, so every CTA derives the same value), and
// its epilogue writes v straight into the digit image stage 2 consumes, plus
// its share of sum q. Stage 2's prologue is then one bulk copy.
//
// Data movement. A CTA owns a contiguous range of 16-row blocks; its slice of
// the packed sign matrix is copied to shared memory by one bulk async copy
// (cp.async.bulk with mbarrier completion) at kernel start. Both stages are
// programmatic dependent launches: each lets the next kernel launch at once,
// and with static weights starts its sign copy before the previous kernel
// has finished; every other read and every write waits for it.
#include "dbf_internal.cuh"

#include <algorithm>

namespace dbf {
namespace {

constexpr int kRows = 16;          // rows per MMA block
constexpr int kPlanes = 3;         // int8 digits per activation
constexpr int kMaxGroups = 3;      // MMA column groups per pass (24 digit columns)
constexpr int kMaxBcols = 8 * kMaxGroups;
constexpr int kMaxNcl = kMaxBcols / kPlanes;   // logical columns per pass (8)
constexpr int kGroupWords = 8;     // words per work unit (256 columns of K)
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxCtas = 160;      // per segment; sizes the per-CTA partial sums
constexpr int kSmemCap = 220 * 1024;
constexpr int kPrefetchCap = 128 * 1024;
constexpr unsigned long long kWaitNs = 2000000000ull;   // bounded wait: 2 s

struct GemvParams {
    dbf_layer layer;              // single-layer mode
    const dbf_layer *adapters;    // segmented mode
    int32_t num_adapters;
    const int32_t *seg_off;
    const int32_t *seg_adp;
    int32_t M, N, max_R, max_ell;
    const void *x;
    dbf_dtype xd;
    void *y;
    dbf_dtype yd;
    int flags;                    // DBF_ACCUMULATE | DBF_WEIGHTS_STATIC
    // workspace, per logical column c = t * ell_cap + i
    char *img;                    // digit image of v: [c][kPlanes][cb2]
    long long *qpart;             // per stage-1 CTA sum of q: [kMaxCtas][T * ell_cap]
    int *sh2;                     // scale exponent of v: [T * ell_cap]
    int32_t ell_cap, R_cap;
    int32_t cb2;                  // bytes per digit column of v
    int64_t T;
    int32_t *status;
    int32_t stage1_ctas;          // CTAs per segment of stage 1
    // shared-memory plan (host computed)
    int32_t ncl_pass;             // logical columns per pass (>= ell)
    int32_t pitch_max;            // words per row (largest over adapters)
    int32_t prefetch_rows;        // rows of the sign slice held in shared memory (0 = none)
    int32_t off_digits, off_colinfo, off_tiles, off_bar, off_ubuf, off_rscale;
    int32_t nb_max;               // row blocks per CTA batch (tiles)
    int32_t pdl_wait;             // launched as a programmatic dependent of the previous kernel
};

// Bytes per digit column: 32 per packed word (one byte per column of K),
// padded so that columns start 32 bytes apart modulo 128. The 8-byte
// B-fragment loads of a half warp (columns g..g+3, threads t = 0..3) then
// cover all 32 banks once.
__host__ __device__ inline int col_bytes(int pitch)
{
    const int words = (pitch + kGroupWords - 1) / kGroupWords * kGroupWords;
    return words * 32 + 32;
}

// Digit layout inside a 256-column group (8 packed words): for mask j and MMA
// thread t, 8 bytes at j*32 + t*8: b0 = digits of word 2t, bits j + 8i, and
// b1 = digits of word 2t+1, bits j + 8i (i = byte 0..3). Packed layout: in-word
// column 2p sits at bit p, column 2p+1 at bit 16+p.
__device__ __forceinline__ int digit_offset(int k)
{
    const int word = k >> 5, j = k & 31;
    const int bit = (j & 1) ? 16 + (j >> 1) : (j >> 1);
    const int grp = word >> 3, wi = word & 7;
    return grp * 256 + (bit & 7) * 32 + (wi >> 1) * 8 + (wi & 1) * 4 + (bit >> 3);
}

// A "quad" is the four columns whose digits form one aligned 32-bit word of
// the layout above: quad Q covers k0, k0+16, k0+1, k0+17 (in byte order) with
// k0 = 32 (Q >> 3) + 2 (Q & 7); its word sits at digit_offset(k0).
__device__ __forceinline__ int quad_k0(int Q) { return 32 * (Q >> 3) + 2 * (Q & 7); }

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---- mbarrier + bulk copy -------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void bar_init(uint64_t *bar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void bar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Copy 'bytes' (a multiple of 16, both ends 16-byte aligned) with completion
// on 'bar'. Called by one thread, after one bar_expect_tx for all the bytes
// of the barrier's phase.
__device__ __forceinline__ void bulk_copy(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    for (uint32_t off = 0; off < bytes; off += 32768u)
        bulk_g2s(static_cast<char *>(dst) + off, static_cast<const char *>(src) + off, min(32768u, bytes - off), bar);
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

__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void set_status(int32_t *status, dbf_status s)
{
    if (status) atomicExch(status, static_cast<int32_t>(s));
}

// exact 2^e as a float for |e| <= 126
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

__device__ __forceinline__ float scale_pow2(float v, int e)
{
    return (e >= -126 && e <= 126) ? v * exp2i(e) : ldexpf(v, e);
}

// |q| <= 2^22 for every value below 'bound': sh = 22 - e with bound < 2^e
__device__ __forceinline__ int scale_exponent(float bound) { return bound > 0.f ? 22 - (ilogbf(bound) + 1) : 0; }

__device__ __forceinline__ long long warp_sum64(long long v)
{
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ unsigned warp_max(unsigned v)
{
    for (int o = 16; o; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// ---- shared memory ----------------------------------------------------------
struct ColInfo {
    long long qsum;      // sum_k q_k of the column
    long long qabs;      // sum_k |q_k| (stage 1: bounds v)
    int sh;              // q = round(a 2^sh)
    int sh_next;         // stage 1: scale of v for stage 2
    unsigned amax;       // reduction scratch
};

struct Smem {
    char *digits;        // [kPlanes * ncl_pass + 1][cb]; the last column is zero
    char *zero_col;
    ColInfo *col;        // [kMaxNcl]
    unsigned *bmax;      // max |beta| over the rank and envelopes (bit pattern)
    float *rscale;       // [ell][rows of this CTA]: beta (stage 1) or alpha (stage 2)
    int *tiles;          // [nb_max][16][kMaxBcols] int32
    uint32_t *signs;     // [prefetch_rows][pitch]
    float4 *ubuf;        // staging of gamma.x quads when K needs several load rounds
    uint64_t *bar;       // [0] sign slice, [1] digit image
    int *flag;
};

constexpr int kQuadsPerRound = 4;     // gamma.x quads loaded per thread per round
constexpr int kBetaPerRound = 16;     // beta values loaded per thread in the first round
constexpr int kScalesPerThread = 8;   // row scales per thread (rows per CTA * ell <= 8 * 256)

__device__ __forceinline__ float ldg_h(const uint16_t *p) { return __half2float(__ushort_as_half(__ldg(p))); }

template <bool XBF16>
__device__ __forceinline__ float ldg_x(const void *x, int64_t i)
{
    if (XBF16) return __bfloat162float(__ldg(static_cast<const __nv_bfloat16 *>(x) + i));
    return __ldg(static_cast<const float *>(x) + i);
}

// q = round-to-nearest-even(u 2^sh) for |u 2^sh| < 2^22, through the fp32
// adder: 1.5 * 2^23 + v has an ulp of 1.
__device__ __forceinline__ int quantize(float u, float scale, int sh, bool plain)
{
    if (plain) return __float_as_int(fmaf(u, scale, 12582912.0f)) - 0x4B400000;
    return __float2int_rn(ldexpf(u, sh));
}

// The three balanced base-256 digits of q (|q| <= 2^22) as int8 bytes 0..2:
// the bytes of q + 0x808080 are d_i + 128, and xor 0x80 turns d_i + 128 into
// the int8 bit pattern of d_i.
__device__ __forceinline__ uint32_t digit_bytes(int q) { return static_cast<uint32_t>(q + 0x808080) ^ 0x808080u; }

// Write the digit words of one quad (four values in byte order) to the three planes.
__device__ __forceinline__ void store_quad(char *plane0, int cb, int woff, int q0, int q1, int q2, int q3)
{
    const uint32_t p0 = digit_bytes(q0), p1 = digit_bytes(q1), p2 = digit_bytes(q2), p3 = digit_bytes(q3);
    const uint32_t lo01 = __byte_perm(p0, p1, 0x5140), lo23 = __byte_perm(p2, p3, 0x5140);
    const uint32_t hi01 = __byte_perm(p0, p1, 0x0062), hi23 = __byte_perm(p2, p3, 0x0062);
    *reinterpret_cast<uint32_t *>(plane0 + woff) = __byte_perm(lo01, lo23, 0x5410);
    *reinterpret_cast<uint32_t *>(plane0 + cb + woff) = __byte_perm(lo01, lo23, 0x7632);
    *reinterpret_cast<uint32_t *>(plane0 + 2 * cb + woff) = __byte_perm(hi01, hi23, 0x5410);
}

// CTA row scales (beta rows for stage 1, alpha rows for stage 2) into shared
// memory; all loads issued before any store.
__device__ __forceinline__ void load_row_scales(const uint16_t *scale, int ld, int ell, int row_lo, int nrows,
                                                float *dst)
{
    const int n = nrows * ell;
    float v[kScalesPerThread];
#pragma unroll
    for (int e = 0; e < kScalesPerThread; ++e) {
        const int idx = threadIdx.x + e * kThreads;
        const int ok = idx < n;
        const int i = ok ? idx / nrows : 0, r = ok ? idx - (idx / nrows) * nrows : 0;
        v[e] = ldg_h(scale + static_cast<int64_t>(i) * ld + row_lo + r);
    }
#pragma unroll
    for (int e = 0; e < kScalesPerThread; ++e) {
        const int idx = threadIdx.x + e * kThreads;
        if (idx < n) dst[idx] = v[e];
    }
}

// Stage 1, one column: digits of gamma_i . x_t with its scale, the scale of
// v_i, and (first column of the CTA only) max |beta|.
template <bool XBF16>
__device__ void stage1_column(const GemvParams &P, const dbf_layer &L, int K, int pitch, int64_t t, int i, int lc,
                              bool with_beta, const Smem &S)
{
    const int cb = col_bytes(P.pitch_max);
    const int lane = threadIdx.x & 31;
    const int nq = (pitch + kGroupWords - 1) / kGroupWords * kGroupWords * 8;   // quads incl. padding
    const uint16_t *gp = L.gamma + static_cast<int64_t>(i) * K;
    const int64_t xb = t * K;
    if (threadIdx.x == 0) {
        S.col[lc].amax = 0u;
        S.col[lc].qsum = 0;
        S.col[lc].qabs = 0;
        if (with_beta) *S.bmax = 0u;
    }
    __syncthreads();
    const bool one_round = nq <= kQuadsPerRound * kThreads;
    float4 u[kQuadsPerRound];
    float m = 0.f, mb = 0.f;
    for (int Q0 = threadIdx.x; Q0 < nq; Q0 += kQuadsPerRound * kThreads) {
        float g[kQuadsPerRound][4], xv[kQuadsPerRound][4];
        float bvals[kBetaPerRound];
        // ---- issue every load of the round before any use
#pragma unroll
        for (int e = 0; e < kQuadsPerRound; ++e) {
            const int k0 = quad_k0(Q0 + e * kThreads);
            const int ks[4] = {k0, k0 + 16, k0 + 1, k0 + 17};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int kk = ks[c] < K ? ks[c] : K - 1;
                g[e][c] = ldg_h(gp + kk);
                xv[e][c] = ldg_x<XBF16>(P.x, xb + kk);
            }
        }
        if (with_beta && Q0 == static_cast<int>(threadIdx.x)) {
            const int nb = L.R * L.ell;
#pragma unroll
            for (int e = 0; e < kBetaPerRound; ++e) {
                const int idx = threadIdx.x + e * kThreads;
                bvals[e] = ldg_h(L.beta + (idx < nb ? idx : nb - 1));
            }
        }
        // ---- use
#pragma unroll
        for (int e = 0; e < kQuadsPerRound; ++e) {
            const int Q = Q0 + e * kThreads;
            const int k0 = quad_k0(Q);
            const bool qok = Q < nq;
            float a[4];
            const int ks[4] = {k0, k0 + 16, k0 + 1, k0 + 17};
#pragma unroll
            for (int c = 0; c < 4; ++c) a[c] = (qok && ks[c] < K) ? g[e][c] * xv[e][c] : 0.f;
            u[e] = make_float4(a[0], a[1], a[2], a[3]);
            m = fmaxf(m, fmaxf(fmaxf(fabsf(a[0]), fabsf(a[1])), fmaxf(fabsf(a[2]), fabsf(a[3]))));
            if (!one_round && qok) S.ubuf[Q] = u[e];
        }
        if (with_beta && Q0 == static_cast<int>(threadIdx.x)) {
            const int nb = L.R * L.ell;
#pragma unroll
            for (int e = 0; e < kBetaPerRound; ++e)
                if (threadIdx.x + e * kThreads < nb) mb = fmaxf(mb, fabsf(bvals[e]));
            // ranks beyond the first round: 8 independent loads per step
            for (int base = threadIdx.x + kBetaPerRound * kThreads; base < nb; base += 8 * kThreads) {
                float w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int idx = base + e * kThreads;
                    w[e] = ldg_h(L.beta + (idx < nb ? idx : nb - 1));
                }
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (base + e * kThreads < nb) mb = fmaxf(mb, fabsf(w[e]));
            }
        }
    }
    const unsigned mw = warp_max(__float_as_uint(m));
    if (lane == 0) atomicMax(&S.col[lc].amax, mw);
    if (with_beta) {
        const unsigned bw = warp_max(__float_as_uint(mb));
        if (lane == 0) atomicMax(S.bmax, bw);
    }
    __syncthreads();
    const int sh = scale_exponent(__uint_as_float(S.col[lc].amax));
    const bool plain = sh >= -126 && sh <= 126;
    const float scale = plain ? exp2i(sh) : 0.f;
    char *plane0 = S.digits + static_cast<size_t>(kPlanes * lc) * cb;
    int sq = 0, sa = 0;
    for (int Q0 = threadIdx.x, r = 0; Q0 < nq; Q0 += kQuadsPerRound * kThreads, ++r) {
#pragma unroll
        for (int e = 0; e < kQuadsPerRound; ++e) {
            const int Q = Q0 + e * kThreads;
            if (Q < nq) {
                const float4 v = one_round ? u[e] : S.ubuf[Q];
                const int q0 = quantize(v.x, scale, sh, plain), q1 = quantize(v.y, scale, sh, plain);
                const int q2 = quantize(v.z, scale, sh, plain), q3 = quantize(v.w, scale, sh, plain);
                sq += q0 + q1 + q2 + q3;
                sa += abs(q0) + abs(q1) + abs(q2) + abs(q3);
                store_quad(plane0, cb, digit_offset(quad_k0(Q)), q0, q1, q2, q3);
            }
        }
    }
    const long long sq64 = warp_sum64(sq), sa64 = warp_sum64(sa);
    if (lane == 0) {
        atomicAdd(reinterpret_cast<unsigned long long *>(&S.col[lc].qsum), static_cast<unsigned long long>(sq64));
        atomicAdd(reinterpret_cast<unsigned long long *>(&S.col[lc].qabs), static_cast<unsigned long long>(sa64));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        S.col[lc].sh = sh;
        // |v_r| = |beta_r h_r| <= max|beta| sum|q| 2^-sh; the factor covers
        // the fp32 roundings of h and beta h
        const float bound = __uint_as_float(*S.bmax) * scale_pow2(static_cast<float>(S.col[lc].qabs), -sh) *
                            (1.0f + 1.0f / 1024.0f);
        S.col[lc].sh_next = scale_exponent(bound);
    }
}

// Two packed words (2t, 2t+1 of an 8-word group) of one row, zero past the row.
template <bool SMEM>
__device__ __forceinline__ uint2 load_pair(const uint32_t *row, int w, int pitch, bool even, bool valid)
{
    uint2 r = make_uint2(0u, 0u);
    if (!valid) return r;
    if (even) {   // pitch even and 8-byte aligned rows: one 8-byte load
        if (w < pitch)
            r = SMEM ? *reinterpret_cast<const uint2 *>(row + w) : __ldg(reinterpret_cast<const uint2 *>(row + w));
    } else {
        if (w < pitch) r.x = SMEM ? row[w] : __ldg(row + w);
        if (w + 1 < pitch) r.y = SMEM ? row[w + 1] : __ldg(row + w + 1);
    }
    return r;
}

// One warp: 8-word groups [u0, u1) of one row block (rows read through pa =
// row g, pb = row g+8), one MMA column group per sweep so that only the eight
// mask accumulators are live. Exact int32 results are added into the shared
// tile.
template <bool SMEM>
__device__ __noinline__ void warp_run(const uint32_t *pa, const uint32_t *pb, bool va, bool vb, int pitch,
                                         bool even, int u0, int u1, const char *dig, const char *zero_col,
                                         int ngroups, int bcols, int cb, int *tile)
{
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;
    const int t = lane & 3;
    for (int q = 0; q < ngroups; ++q) {
        int acc[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0;
        const int col = q * 8 + g;
        const char *colp = (col < bcols ? dig + col * cb : zero_col) + t * 8;
        for (int u = u0; u < u1; ++u) {
            const int w = u * kGroupWords + 2 * t;
            const uint2 A = load_pair<SMEM>(pa, w, pitch, even, va);
            const uint2 B = load_pair<SMEM>(pb, w, pitch, even, vb);
            const char *bp = colp + u * 256;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t m = 0x01010101u << j;
                const uint2 bv = *reinterpret_cast<const uint2 *>(bp + j * 32);
                mma_u8s8(acc[j], A.x & m, B.x & m, A.y & m, B.y & m, bv.x, bv.y);
            }
        }
        // fold the mask weights 2^j (exact: acc[j] is a multiple of 2^j)
        int f[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            f[e] = acc[0][e];
#pragma unroll
            for (int j = 1; j < 8; ++j) f[e] += acc[j][e] >> j;
        }
        atomicAdd(&tile[g * kMaxBcols + q * 8 + 2 * t], f[0]);
        atomicAdd(&tile[g * kMaxBcols + q * 8 + 2 * t + 1], f[1]);
        atomicAdd(&tile[(g + 8) * kMaxBcols + q * 8 + 2 * t], f[2]);
        atomicAdd(&tile[(g + 8) * kMaxBcols + q * 8 + 2 * t + 1], f[3]);
    }
}

// sum_k b_k q_k of one (row, column) from the three digit-plane tiles
__device__ __forceinline__ long long plane_sum(const int *tr, int lc)
{
    return static_cast<long long>(tr[kPlanes * lc]) + 256LL * tr[kPlanes * lc + 1] + 65536LL * tr[kPlanes * lc + 2];
}

__device__ __forceinline__ bool wait_flag(const Smem &S, int which, uint32_t parity, int32_t *status)
{
    // one thread waits (bounded); the outcome is shared through the flag
    if (threadIdx.x == 0) {
        const bool ok = bar_wait(&S.bar[which], parity);
        *S.flag = ok ? 1 : 0;
        if (!ok) set_status(status, DBF_ERR_TIMEOUT);
    }
    __syncthreads();
    return *S.flag != 0;
}

template <int STAGE, bool SEG>
__global__ void __launch_bounds__(kThreads, 2) gemv_kernel(const GemvParams P)
{
    extern __shared__ __align__(128) char smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // let the next kernel in the stream start its own weight prefetch now
    pdl_trigger();
    // Reads of anything the preceding kernel may have written (segment tables,
    // descriptors, activations, the v image) and every global write come
    // after the wait. Only with static weights does the sign copy start first.
    const bool early = !SEG && (P.flags & DBF_WEIGHTS_STATIC);
    if (P.pdl_wait && !early) pdl_wait();

    // ---- which layer and tokens this CTA serves
    dbf_layer L = P.layer;
    int64_t t0 = 0, t1 = P.T;
    bool active = true;
    if (SEG) {
        const int s = blockIdx.y;
        t0 = P.seg_off[s];
        t1 = P.seg_off[s + 1];
        const int a = P.seg_adp[s];
        const bool bad_range = t0 < 0 || t1 < t0 || t1 > P.T;
        if (bad_range || a < -1 || a >= P.num_adapters) {
            if (threadIdx.x == 0 && blockIdx.x == 0) set_status(P.status, DBF_ERR_INVALID_ARG);
            active = false;
        } else if (a == -1) {
            // no adapter: zero branch (stage 2 writes zeros unless accumulating)
            if (STAGE == 2 && !(P.flags & DBF_ACCUMULATE)) {
                const int64_t n_el = (t1 - t0) * P.N;
                for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n_el;
                     idx += static_cast<int64_t>(gridDim.x) * blockDim.x)
                    store_act(P.y, P.yd, t0 * P.N + idx, 0.0f);
            }
            active = false;
        } else {
            L = P.adapters[a];
            if (L.M != P.M || L.N != P.N || L.R < 1 || L.R > P.max_R || L.ell < 1 || L.ell > P.max_ell ||
                L.ell > kMaxEll) {
                if (threadIdx.x == 0 && blockIdx.x == 0) set_status(P.status, DBF_ERR_INVALID_ARG);
                active = false;
            }
        }
    }
    if (!active || t1 <= t0) return;
    const int ell = L.ell;
    const int K = STAGE == 1 ? L.M : L.R;
    const int rows = STAGE == 1 ? L.R : L.N;
    const int nrb = (rows + kRows - 1) / kRows;
    const int rb_begin = static_cast<int>(static_cast<int64_t>(nrb) * blockIdx.x / gridDim.x);
    const int rb_end = static_cast<int>(static_cast<int64_t>(nrb) * (blockIdx.x + 1) / gridDim.x);
    const uint32_t *Sg = STAGE == 1 ? L.b2_packed : L.b1_packed;
    const int pitch = static_cast<int>(pitch_words(K));
    const bool even = (pitch % 2 == 0) && ((reinterpret_cast<uintptr_t>(Sg) & 7u) == 0);
    const bool vec = (pitch % 4 == 0) && ((reinterpret_cast<uintptr_t>(Sg) & 15u) == 0);
    const int ngrp = (pitch + kGroupWords - 1) / kGroupWords;
    const int cb = col_bytes(P.pitch_max);
    const int tpp = P.ncl_pass / ell;   // tokens per pass

    Smem S;
    S.digits = smem + P.off_digits;
    S.zero_col = S.digits + static_cast<size_t>(kPlanes) * P.ncl_pass * cb;
    S.col = reinterpret_cast<ColInfo *>(smem + P.off_colinfo);
    S.bmax = reinterpret_cast<unsigned *>(S.col + kMaxNcl);
    S.rscale = reinterpret_cast<float *>(smem + P.off_rscale);
    S.tiles = reinterpret_cast<int *>(smem + P.off_tiles);
    S.bar = reinterpret_cast<uint64_t *>(smem + P.off_bar);
    S.flag = reinterpret_cast<int *>(smem + P.off_bar + 16);
    S.signs = reinterpret_cast<uint32_t *>(smem);   // slice at offset 0
    S.ubuf = reinterpret_cast<float4 *>(smem + P.off_ubuf);

    // ---- sign slice -> shared memory (one bulk copy, all of it in flight now)
    const int row_lo = rb_begin * kRows;
    const int row_hi = min(rb_end * kRows, rows);
    const int nrows = row_hi > row_lo ? row_hi - row_lo : 0;
    const bool use_slice = vec && nrows > 0 && nrows <= P.prefetch_rows;
    if (threadIdx.x == 0) {
        bar_init(&S.bar[0], 1);
        bar_init(&S.bar[1], 1);
        if (use_slice) {
            const uint32_t bytes = static_cast<uint32_t>(nrows) * pitch * 4u;
            bar_expect_tx(&S.bar[0], bytes);
            bulk_copy(S.signs, Sg + static_cast<int64_t>(row_lo) * pitch, bytes, &S.bar[0]);
        }
    }
    for (int i = threadIdx.x; i < cb / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(S.zero_col)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (P.pdl_wait && early) pdl_wait();
    // scales of this CTA's rows for the epilogue
    if (nrows > 0)
        load_row_scales(STAGE == 1 ? L.beta : L.alpha, STAGE == 1 ? L.R : L.N, ell, row_lo, nrows, S.rscale);

    bool slice_ready = !use_slice;
    int pass = 0;
    for (int64_t tg = t0; tg < t1; tg += tpp, ++pass) {
        const int ntok = static_cast<int>((t1 - tg) < tpp ? (t1 - tg) : tpp);
        const int ncl = ntok * ell;
        const int bcols = kPlanes * ncl;
        const int ngroups = (bcols + 7) / 8;
        if (STAGE == 1) {
            for (int lc = 0; lc < ncl; ++lc) {
                const int tok = lc / ell, i = lc - tok * ell;
                if (P.xd == DBF_BF16)
                    stage1_column<true>(P, L, K, pitch, tg + tok, i, lc, pass == 0 && lc == 0, S);
                else
                    stage1_column<false>(P, L, K, pitch, tg + tok, i, lc, pass == 0 && lc == 0, S);
            }
            __syncthreads();
        } else {
            // the v digit image written by stage 1 (one bulk copy per column);
            // the sums of q are the stage-1 CTA partials
            if (threadIdx.x == 0) {
                // order the previous pass's reads of the digits before the async writes
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                bar_expect_tx(&S.bar[1], static_cast<uint32_t>(ncl * kPlanes * cb));
                for (int lc = 0; lc < ncl; ++lc) {
                    const int tok = lc / ell, i = lc - tok * ell;
                    const int64_t c = (tg + tok) * P.ell_cap + i;
                    bulk_copy(S.digits + static_cast<size_t>(kPlanes) * lc * cb,
                              P.img + static_cast<size_t>(c) * kPlanes * P.cb2, static_cast<uint32_t>(kPlanes) * cb,
                              &S.bar[1]);
                }
            }
            for (int lc = warp; lc < ncl; lc += kWarps) {
                const int tok = lc / ell, i = lc - tok * ell;
                const int64_t c = (tg + tok) * P.ell_cap + i;
                long long part[kMaxCtas / 32];
#pragma unroll
                for (int e = 0; e < kMaxCtas / 32; ++e) {
                    const int k = lane + 32 * e;
                    part[e] = k < P.stage1_ctas ? __ldg(P.qpart + static_cast<int64_t>(k) * P.T * P.ell_cap + c) : 0;
                }
                long long sq = 0;
#pragma unroll
                for (int e = 0; e < kMaxCtas / 32; ++e) sq += part[e];
                sq = warp_sum64(sq);
                if (lane == 0) {
                    S.col[lc].qsum = sq;
                    S.col[lc].sh = __ldg(P.sh2 + c);
                }
            }
            if (!wait_flag(S, 1, pass & 1, P.status)) return;
        }
        if (!slice_ready) {
            if (!wait_flag(S, 0, 0, P.status)) return;
            slice_ready = true;
        }
        long long qpart_local[kMaxNcl];
#pragma unroll
        for (int lc = 0; lc < kMaxNcl; ++lc) qpart_local[lc] = 0;
        for (int rbb = rb_begin; rbb < rb_end; rbb += P.nb_max) {
            const int nb = min(P.nb_max, rb_end - rbb);
            for (int i = threadIdx.x; i < nb * kRows * kMaxBcols; i += blockDim.x) S.tiles[i] = 0;
            __syncthreads();
            // units (row block, 8-word group) split contiguously over the warps;
            // a warp accumulates its run in registers until the row block changes
            const int units = nb * ngrp;
            int u = units * warp / kWarps;
            const int uend = units * (warp + 1) / kWarps;
            while (u < uend) {
                const int b = u / ngrp;
                const int g0 = u - b * ngrp;
                const int g1 = min(ngrp, g0 + (uend - u));
                const int row0 = (rbb + b) * kRows;
                const int g = lane >> 2;
                const bool va = row0 + g < rows, vb = row0 + g + 8 < rows;
                if (use_slice) {
                    const uint32_t *base = S.signs + static_cast<int64_t>(row0 + g - row_lo) * pitch;
                    warp_run<true>(base, base + 8 * pitch, va, vb, pitch, even, g0, g1, S.digits, S.zero_col,
                                   ngroups, bcols, cb, S.tiles + b * kRows * kMaxBcols);
                } else {
                    const uint32_t *base = Sg + static_cast<int64_t>(row0 + g) * pitch;
                    warp_run<false>(base, base + 8 * pitch, va, vb, pitch, even, g0, g1, S.digits, S.zero_col,
                                    ngroups, bcols, cb, S.tiles + b * kRows * kMaxBcols);
                }
                u += g1 - g0;
            }
            __syncthreads();
            // ---- epilogue
            if (STAGE == 1) {
                // v = beta . h, digitised with the scale fixed above, into the image
                for (int idx = threadIdx.x; idx < nb * kRows * ncl; idx += blockDim.x) {
                    const int row = idx % (nb * kRows);
                    const int lc = idx / (nb * kRows);
                    const int r = rbb * kRows + row;
                    if (r >= rows) continue;
                    const ColInfo &ci = S.col[lc];
                    const float h = scale_pow2(__ll2float_rn(ci.qsum - 2 * plane_sum(S.tiles + row * kMaxBcols, lc)), -ci.sh);
                    const int tok = lc / ell, i = lc - tok * ell;
                    const float v = S.rscale[i * nrows + (r - row_lo)] * h;
                    const int sh2 = ci.sh_next;
                    const bool plain = sh2 >= -126 && sh2 <= 126;
                    const int q = quantize(v, plain ? exp2i(sh2) : 0.f, sh2, plain);
                    const uint32_t db = digit_bytes(q);
                    char *img = P.img + static_cast<size_t>((tg + tok) * P.ell_cap + i) * kPlanes * P.cb2 + digit_offset(r);
                    img[0] = static_cast<char>(db & 255u);
                    img[P.cb2] = static_cast<char>((db >> 8) & 255u);
                    img[2 * P.cb2] = static_cast<char>(db >> 16);
#pragma unroll
                    for (int c = 0; c < kMaxNcl; ++c)
                        if (c == lc) qpart_local[c] += q;
                }
            } else {
                for (int idx = threadIdx.x; idx < nb * kRows * ntok; idx += blockDim.x) {
                    const int row = idx % (nb * kRows);
                    const int tok = idx / (nb * kRows);
                    const int n = rbb * kRows + row;
                    if (n >= rows) continue;
                    const int64_t t = tg + tok;
                    float yv = (P.flags & DBF_ACCUMULATE) ? load_act(P.y, P.yd, t * P.N + n) : 0.f;
                    for (int i = 0; i < ell; ++i) {
                        const int lc = tok * ell + i;
                        const ColInfo &ci = S.col[lc];
                        const float z =
                            scale_pow2(__ll2float_rn(ci.qsum - 2 * plane_sum(S.tiles + row * kMaxBcols, lc)), -ci.sh);
                        yv += S.rscale[i * nrows + (n - row_lo)] * z;
                    }
                    store_act(P.y, P.yd, t * P.N + n, yv);
                }
            }
            __syncthreads();
        }
        if (STAGE == 1) {
            // zero the image past the rank (up to the padded length) and publish
            // this CTA's partial sums of q and the scale of v
            const int kp2 = P.cb2 - 32;
            if (rb_end == nrb) {
                for (int idx = threadIdx.x; idx < ncl * (kp2 - L.R); idx += blockDim.x) {
                    const int lc = idx / (kp2 - L.R);
                    const int r = L.R + idx % (kp2 - L.R);
                    const int tok = lc / ell, i = lc - tok * ell;
                    char *img = P.img + static_cast<size_t>((tg + tok) * P.ell_cap + i) * kPlanes * P.cb2 + digit_offset(r);
                    img[0] = 0;
                    img[P.cb2] = 0;
                    img[2 * P.cb2] = 0;
                }
            }
            long long *red = reinterpret_cast<long long *>(S.tiles);
            for (int lc = threadIdx.x; lc < ncl; lc += blockDim.x) red[lc] = 0;
            __syncthreads();
            for (int lc = 0; lc < ncl; ++lc) {
                long long v = 0;
#pragma unroll
                for (int c = 0; c < kMaxNcl; ++c)
                    if (c == lc) v = qpart_local[c];
                v = warp_sum64(v);
                if (lane == 0) atomicAdd(reinterpret_cast<unsigned long long *>(&red[lc]), static_cast<unsigned long long>(v));
            }
            __syncthreads();
            for (int lc = threadIdx.x; lc < ncl; lc += blockDim.x) {
                const int tok = lc / ell, i = lc - tok * ell;
                const int64_t c = (tg + tok) * P.ell_cap + i;
                P.qpart[static_cast<int64_t>(blockIdx.x) * P.T * P.ell_cap + c] = red[lc];
                if (blockIdx.x == 0) P.sh2[c] = S.col[lc].sh_next;
            }
            __syncthreads();
        }
    }
}

int num_sms() { return device_sms(); }

int quads_of(int pitch) { return (pitch + kGroupWords - 1) / kGroupWords * kGroupWords * 8; }

// Shared-memory plan for one stage; false if no plan fits.
bool plan(GemvParams &P, int stage, int K, int rows_max, int ctas, int max_ell, int64_t T, size_t &smem)
{
    const int pitch = static_cast<int>(pitch_words(K));
    const int nrb = (rows_max + kRows - 1) / kRows;
    const int rb_per_cta = (nrb + ctas - 1) / ctas;
    if (rb_per_cta * kRows * max_ell > kScalesPerThread * kThreads) return false;
    P.pitch_max = pitch;
    if (kMaxNcl < max_ell) return false;
    const int64_t tok_cap = kMaxNcl / max_ell;
    int ncl = static_cast<int>((T < tok_cap ? T : tok_cap) * max_ell);
    auto carve = [&](int prefetch_rows, int nb, int ncl_pass, bool commit) -> size_t {
        size_t off = align_up(static_cast<size_t>(prefetch_rows) * pitch * 4, 128);
        const size_t o_dig = off;
        off += static_cast<size_t>(kPlanes * ncl_pass + 1) * col_bytes(pitch);   // + zero column
        off = align_up(off, 16);
        const size_t o_col = off;
        off += static_cast<size_t>(kMaxNcl) * sizeof(ColInfo) + 16;
        off = align_up(off, 16);
        const size_t o_tiles = off;
        off += static_cast<size_t>(nb > 1 ? nb : 1) * kRows * kMaxBcols * 4;
        off = align_up(off, 16);
        const size_t o_bar = off;
        off += 32;   // two mbarriers + wait flag
        const size_t o_rs = off;
        off += static_cast<size_t>(rb_per_cta) * kRows * max_ell * 4;
        off = align_up(off, 16);
        const size_t o_ubuf = off;
        if (stage == 1 && quads_of(pitch) > kQuadsPerRound * kThreads) off += static_cast<size_t>(quads_of(pitch)) * 16;
        if (commit) {
            P.off_digits = static_cast<int>(o_dig);
            P.off_colinfo = static_cast<int>(o_col);
            P.off_tiles = static_cast<int>(o_tiles);
            P.off_bar = static_cast<int>(o_bar);
            P.off_rscale = static_cast<int>(o_rs);
            P.off_ubuf = static_cast<int>(o_ubuf);
            P.prefetch_rows = prefetch_rows;
            P.nb_max = nb;
            P.ncl_pass = ncl_pass;
        }
        return off;
    };
    int nb = rb_per_cta < 16 ? rb_per_cta : 16;
    if (nb < 1) nb = 1;
    int prefetch_rows = rb_per_cta * kRows;
    if (static_cast<size_t>(prefetch_rows) * pitch * 4 > kPrefetchCap || pitch % 4 != 0) prefetch_rows = 0;
    while (true) {
        if (carve(prefetch_rows, nb, ncl, false) <= kSmemCap) {
            smem = carve(prefetch_rows, nb, ncl, true);
            return true;
        }
        if (ncl > max_ell) --ncl;
        else if (nb > 1) nb = nb / 2;
        else if (prefetch_rows > 0) prefetch_rows = 0;
        else return false;
    }
}

template <int STAGE, bool SEG>
cudaError_t launch(GemvParams P, int K, int rows_max, int nseg, int ctas, int max_ell, cudaStream_t s)
{
    size_t smem = 0;
    if (!plan(P, STAGE, K, rows_max, ctas, max_ell, P.T, smem)) return cudaErrorInvalidValue;
    {
        // one carve-out for both stages: no L1/shared reconfiguration between
        // them, and a stage-2 CTA fits beside a stage-1 CTA
        cudaError_t e = allow_smem(reinterpret_cast<const void *>(gemv_kernel<STAGE, SEG>), static_cast<int>(smem), true);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctas, nseg);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    P.pdl_wait = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_kernel<STAGE, SEG>, P);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

struct WsLayout {
    size_t img, qpart, sh2, total;
};

WsLayout ws_layout(int64_t R, int64_t ell, int64_t T)
{
    WsLayout w;
    const int64_t cols = T * ell;
    const size_t cb2 = static_cast<size_t>(col_bytes(static_cast<int>(pitch_words(R))));
    w.img = 0;
    w.qpart = align_up(static_cast<size_t>(cols) * kPlanes * cb2, 256);
    w.sh2 = w.qpart + align_up(static_cast<size_t>(kMaxCtas) * cols * sizeof(long long), 256);
    w.total = w.sh2 + align_up(static_cast<size_t>(cols) * sizeof(int), 256);
    return w;
}

void bind_workspace(GemvParams &P, int max_R, int max_ell, void *ws)
{
    const WsLayout w = ws_layout(max_R, max_ell, P.T);
    char *body = static_cast<char *>(ws) + kWsHeaderBytes;
    P.img = body + w.img;
    P.qpart = reinterpret_cast<long long *>(body + w.qpart);
    P.sh2 = reinterpret_cast<int *>(body + w.sh2);
    P.cb2 = col_bytes(static_cast<int>(pitch_words(max_R)));
}

template <bool SEG>
cudaError_t run_both(GemvParams P, int M, int max_R, int N, int nseg, int budget, int max_ell, void *ws, cudaStream_t s)
{
    bind_workspace(P, max_R, max_ell, ws);
    // CTAs per segment: the budget, at least enough that a CTA's row scales
    // fit the loader, never more than there are row blocks
    auto ctas_for = [&](int rows) {
        const int nrb = (rows + kRows - 1) / kRows;
        const int per = kScalesPerThread * kThreads / (kRows * max_ell);   // row blocks per CTA at most
        int c = budget;
        if (c < (nrb + per - 1) / per) c = (nrb + per - 1) / per;
        if (c > nrb) c = nrb;
        return c < 1 ? 1 : c;
    };
    int c1 = ctas_for(max_R);
    if (c1 > kMaxCtas) c1 = kMaxCtas;
    const int c2 = ctas_for(N);
    P.stage1_ctas = c1;
    cudaError_t e = launch<1, SEG>(P, M, max_R, nseg, c1, max_ell, s);
    if (e != cudaSuccess) return e;
    return launch<2, SEG>(P, max_R, N, nseg, c2, max_ell, s);
}

}  // namespace

size_t gemv_workspace_bytes(int64_t R, int64_t ell, int64_t T)
{
    // either kernel: the two launches here or the single launch
    const size_t a = kWsHeaderBytes + ws_layout(R, ell, T).total;
    const size_t b = multi_segmented_workspace_bytes(static_cast<int32_t>(R), static_cast<int32_t>(ell), T);
    return a > b ? a : b;
}

size_t gemv_layer_workspace_bytes(const dbf_layer &L, int64_t T)
{
    const size_t a = gemv_workspace_bytes(L.R, L.ell, T), b = decode_workspace_bytes(L, T);
    const size_t c = multi_workspace_bytes(L, T);
    return std::max(a, std::max(b, c));
}

int gemv_launches(const dbf_layer &L, int64_t T) { return (decode_fits(L, T) || multi_fits(L, T)) ? 1 : 2; }

cudaError_t gemv_forward(const dbf_layer &L, const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                         int flags, void *ws, cudaStream_t s)
{
    // one launch (grid barrier) when the call fits one of the single-launch kernels
    if (decode_fits(L, T)) return decode_forward(L, x, xd, y, yd, T, flags, ws, s);
    if (multi_fits(L, T)) return multi_forward(L, x, xd, y, yd, T, flags, ws, s);
    GemvParams P{};
    P.layer = L;
    P.M = L.M;
    P.N = L.N;
    P.max_R = L.R;
    P.max_ell = L.ell;
    P.x = x;
    P.xd = xd;
    P.y = y;
    P.yd = yd;
    P.flags = flags;
    P.ell_cap = L.ell;
    P.R_cap = L.R;
    P.T = T;
    return run_both<false>(P, L.M, L.R, L.N, 1, num_sms(), L.ell, ws, s);
}

cudaError_t gemv_forward_segmented(const dbf_layer *adapters, int32_t num_adapters, const int32_t *seg_off,
                                   const int32_t *seg_adp, int32_t S, int32_t max_R, int32_t max_ell, int32_t M,
                                   int32_t N, const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                                   int flags, void *ws, int32_t *status, cudaStream_t s)
{
    // one launch when the call fits it
    if (multi_segmented_fits(S, max_R, max_ell, M, N, T))
        return multi_forward_segmented(adapters, num_adapters, seg_off, seg_adp, S, max_R, max_ell, M, N, x, xd, y,
                                       yd, T, flags, ws, status, s);
    GemvParams P{};
    P.adapters = adapters;
    P.num_adapters = num_adapters;
    P.seg_off = seg_off;
    P.seg_adp = seg_adp;
    P.M = M;
    P.N = N;
    P.max_R = max_R;
    P.max_ell = max_ell;
    P.x = x;
    P.xd = xd;
    P.y = y;
    P.yd = yd;
    P.flags = flags;
    P.ell_cap = max_ell;
    P.R_cap = max_R;
    P.T = T;
    P.status = status;
    const int per_seg = max(1, (2 * num_sms() + S - 1) / S);
    return run_both<true>(P, M, max_R, N, S, per_seg, max_ell, ws, s);
}

}  // namespace dbf
