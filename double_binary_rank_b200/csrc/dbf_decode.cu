// Decode-regime forward in one launch, for calls of one layer whose
// (token, envelope) columns number at most eight (the decode step itself);
// longer calls and segmented adapters take dbf_decode_multi.cu.
//
// LoRDBA page, section 2 ("Kernel de Inferencia"): the forward is two
// sign-accumulation products with per-channel scaling between them; DBF page,
// section 2 ("Inferencia"): with binary factors the dense product becomes
// additions and scalar-vector products. Stage 1 computes
// v_i = beta_i . (B2 (gamma_i . x)), stage 2 y = [acc] y + sum_i alpha_i . (B1 v_i).
//
// Arithmetic. A sign is s = 1 - 2b with b in {0, 1} the packed bit, so
//   sum_k s_k a_k = sum_k a_k - 2 sum_k b_k a_k .
// Every activation column a (one token and envelope) becomes the integers
// q_k = round(a_k 2^sh), |q| <= 2^22, with one power-of-two scale per column
// (q is exact whenever a is a small dyadic value), written as three balanced
// base-256 int8 digits. mma.sync m16n8k32 u8 x s8 accumulates sum_k b_k d_k
// exactly in int32: masking a packed word with 0x01010101 << j gives four
// bytes in {0, 2^j} (bits j, j+8, j+16, j+24), so the eight masks j = 0..7
// of the words feed eight MMAs whose accumulators carry the weight 2^j and
// are folded with exact right shifts. The digits are laid out to match: in
// each 256-column group (8 packed words), mask j and MMA thread t read 8
// bytes at j*32 + t*8, the digits of words 2t and 2t+1 at bits j + 8i. The
// three digit columns are recombined in int64 and converted once:
// (sum q - 2 sum b q) 2^-sh. Sums are exact integers, so the result does not
// depend on how K is split across warps.
//
// Stage 1: every CTA digitises gamma.x itself (one warp per packed word, one
// lane per column), runs its 16-row blocks of B2, and writes v = beta.h as
// digits into an image in the workspace, plus its share of sum q. The scale
// of v is fixed in advance from the bound |v_r| <= max|beta| sum_m |q_m| 2^-sh
// (integers and bit patterns only, so every CTA derives the same value
// without an exchange). A grid barrier publishes the image; stage 2 copies it
// into shared memory and runs its 16-row blocks of B1.
//
// Data movement. One CTA per SM (cooperative launch, so the whole grid is
// co-resident). At entry one warp issues bulk asynchronous copies of the
// CTA's slices of B2 and B1 into shared memory (row strides of 8 or 24 words
// modulo 32, so the A-fragment loads of a half warp hit distinct banks);
// with static weights they start before the previous kernel in the stream
// has finished (programmatic dependent launch). Activations, the workspace
// and y wait for it.
//
// Grid barrier (workspace header, 8 bytes: arrivals in the low word, an epoch
// in the high word). A CTA reads the epoch, then adds its arrival with an
// acquire-release atomic; the arrival that brings the count to the grid size
// stores (epoch + 1, count 0) with release semantics, and every other CTA
// polls (bounded by a time limit counted from the CTA's entry) until it sees
// the full count or the new epoch. The epoch can change only after every CTA has arrived, so
// a CTA that starts late still reads the current epoch; the count is zero
// again once the last CTA has arrived, whatever happened to the waits. A wait that runs out of
// time stores DBF_ERR_TIMEOUT in the header's status word and the CTA skips
// its stage-2 rows.
#include "dbf_internal.cuh"

#include <mutex>

namespace dbf {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kDigits = 3;               // int8 digits per activation value
constexpr int kMaxCols = 8;              // (token, envelope) columns of one call
constexpr int kGroupWords = 8;           // packed words per MMA unit (256 columns of K)
constexpr int kMaxWordsPerWarp = 32;     // M <= 8192
constexpr int kSmemCap = 227 * 1024;
constexpr int kMaxGrid = 160;            // CTAs at most (sizes the per-CTA sums in the workspace)
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;   // 2 s

struct DecodeParams {
    dbf_layer L;
    const void *x;
    void *y;
    dbf_dtype xd, yd;
    int T, C;                     // tokens, columns (T * ell)
    int flags;
    unsigned long long *sync;     // header word: arrivals (low 32 bits), epoch (high 32 bits)
    int32_t *status;              // header: sticky status of the call's kernels
    char *img;                    // digits of v: [C][kDigits][cb2]
    long long *qpart;             // sum of q of v per CTA: [G][C]
    int cb1, cb2;                 // bytes per digit column of u (stage 1) and v (stage 2)
    int nrb1, nrb2;               // 16-row blocks of B2 and B1
    int pitch1, pitch2;           // packed words per row of B2, B1
    int stride1, stride2;         // words per row in the shared-memory slices
    int ng1, ng2;                 // 256-column groups of K in stage 1, stage 2
    int max_rb1, max_rb2;         // row blocks of the largest CTA
    int bulk1, bulk2;             // slices copied by bulk asynchronous copies
    int bulk_g, bulk_x;           // gamma and x staged by bulk copies (else element by element)
    int gs_bytes, xs_bytes;       // staged gamma, and one token's x buffer (16-byte rounded)
    int gpitch;                   // values per staged gamma row (M rounded up to 8)
    int tile_ld;                  // int32 per row of the partial-sum tile (8 per column group, plus 1)
    int off_s2, off_dig, off_tile, off_misc, off_rs1, off_rs2;   // shared-memory offsets
    unsigned long long wait_ns;   // limit of the grid-barrier wait
};

struct Misc {
    uint64_t bar[5];              // slice 1, slice 2, gamma, x buffers 0 and 1 arrived
    unsigned long long t_entry;   // %globaltimer at the CTA's entry
    int flag;
    unsigned e0;                  // epoch read at entry
    unsigned bmax;                // max |beta| (fp32 bits)
    unsigned amax[kMaxCols];      // max |gamma . x| per column (fp32 bits)
    int sh_u[kMaxCols], sh_v[kMaxCols];
    long long qsum_u[kMaxCols], qabs_u[kMaxCols], qsum_v[kMaxCols];
    long long wq[kWarps][kMaxCols], wa[kWarps][kMaxCols];   // per-warp partial sums
};

// ---- small device helpers ----------------------------------------------------
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
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
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

// One thread waits for phase 0 of a slice barrier (bounded by the default
// limit, whatever the grid barrier's limit is, so that no copy is cut
// short); the outcome is shared through the flag. False on timeout
// (recorded in the status word).
__device__ __forceinline__ bool slice_wait(uint64_t *bar, const DecodeParams &P, Misc *ms)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned long long t0 = global_ns();
        bool ok = true;
        while (!bar_try(bar, 0)) {
            if (global_ns() - t0 > kDefaultWaitNs) {
                ok = false;
                atomicExch(P.status, static_cast<int32_t>(DBF_ERR_TIMEOUT));
                break;
            }
        }
        ms->flag = ok ? 1 : 0;
    }
    __syncthreads();
    return ms->flag != 0;
}

// Wait until token t's x (buffer t & 1, its (t / 2)-th copy) and, for the
// first token, gamma are in shared memory: bulk copies are waited for by
// thread 0 (bounded by the default limit), element copies by the barrier.
__device__ __forceinline__ void token_wait(const DecodeParams &P, Misc *ms, int t)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned long long t0 = global_ns();
        const uint32_t par = static_cast<uint32_t>(t >> 1) & 1u;
        while ((t == 0 && P.bulk_g && !bar_try(&ms->bar[2], 0)) || (P.bulk_x && !bar_try(&ms->bar[3 + (t & 1)], par))) {
            if (global_ns() - t0 > kDefaultWaitNs) {
                atomicExch(P.status, static_cast<int32_t>(DBF_ERR_TIMEOUT));
                break;
            }
        }
    }
    __syncthreads();
}

// gamma_env[col] x_t[col] and the same at col + 1 (col even) from the
// staged copies, exact in fp32; zero at and past m
__device__ __forceinline__ float2 stage_u2(const uint16_t *gc, const unsigned char *xs, dbf_dtype xd, int col, int m)
{
    float2 x, g;
    if (col + 1 < m) {
        const __half2 gh = *reinterpret_cast<const __half2 *>(gc + col);
        g = __half22float2(gh);
        x = xd == DBF_BF16 ? __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(xs + 2 * col))
                           : *reinterpret_cast<const float2 *>(xs + 4 * col);
    } else if (col < m) {
        g = make_float2(__half2float(__ushort_as_half(gc[col])), 0.f);
        x = make_float2(xd == DBF_BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(xs)[col])
                                       : reinterpret_cast<const float *>(xs)[col],
                        0.f);
    } else {
        return make_float2(0.f, 0.f);
    }
    return make_float2(g.x * x.x, g.y * x.y);
}

__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Column of a packed word that bit i holds (bits p and 16 + p: columns 2p, 2p + 1).
__device__ __forceinline__ int col_of_bit(int i) { return i < 16 ? 2 * i : 2 * (i - 16) + 1; }

// Byte of the digit layout that holds bit 'bit' of packed word 'w' (see the
// file comment): group w / 8, mask bit % 8, MMA thread (w % 8) / 2, half
// w % 2, byte bit / 8.
__device__ __forceinline__ int digit_byte(int w, int bit)
{
    const int wi = w & 7;
    return (w >> 3) * 256 + (bit & 7) * 32 + (wi >> 1) * 8 + (wi & 1) * 4 + (bit >> 3);
}

// The byte of column k of K in the digit layout.
__device__ __forceinline__ int digit_offset(int k)
{
    const int j = k & 31;
    return digit_byte(k >> 5, (j & 1) ? 16 + (j >> 1) : (j >> 1));
}

// exact 2^e for |e| <= 126
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

__device__ __forceinline__ float scale_pow2(float v, int e)
{
    return (e >= -126 && e <= 126) ? v * exp2i(e) : ldexpf(v, e);
}

// |q| <= 2^22 for every value of magnitude below 'bound': sh = 22 - e with bound < 2^e
__device__ __forceinline__ int scale_exponent(float bound) { return bound > 0.f ? 22 - (ilogbf(bound) + 1) : 0; }

// q = round-to-nearest-even(u 2^sh) for |u 2^sh| < 2^22, through the fp32
// adder when 2^sh is a normal float: 1.5 * 2^23 + v has an ulp of 1.
__device__ __forceinline__ int quantize(float u, int sh)
{
    if (sh >= -126 && sh <= 126) return __float_as_int(fmaf(u, exp2i(sh), 12582912.0f)) - 0x4B400000;
    return __float2int_rn(ldexpf(u, sh));
}

// The three balanced base-256 digits of q (|q| <= 2^22) as int8 bytes 0..2:
// the bytes of q + 0x808080 are d_i + 128, and xor 0x80 gives the int8 bits of d_i.
__device__ __forceinline__ uint32_t digit_bytes(int q) { return static_cast<uint32_t>(q + 0x808080) ^ 0x808080u; }

__device__ __forceinline__ float ldg_h(const uint16_t *p) { return __half2float(__ushort_as_half(__ldg(p))); }

__device__ __forceinline__ long long warp_sum64(long long v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Exact warp sum of per-thread int32 values: 16-bit halves summed separately
// (one reduction instruction each).
__device__ __forceinline__ long long warp_sum_exact(int v)
{
    const unsigned lo = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(v) & 0xFFFFu);
    const int hi = __reduce_add_sync(0xffffffffu, v >> 16);
    return static_cast<long long>(hi) * 65536 + lo;
}

// Copy rows [0, n) of a packed matrix slice into shared memory with row
// stride 'stride': bulk copies issued by one warp (one copy when unpadded).
__device__ __forceinline__ void slice_bulk(uint32_t *dst, const uint32_t *src, int n, int pitch, int stride,
                                           uint64_t *bar)
{
    const int lane = threadIdx.x & 31;
    if (n <= 0) return;
    if (stride == pitch) {
        if (lane == 0) {
            const uint32_t bytes = static_cast<uint32_t>(n) * pitch * 4u;
            for (uint32_t off = 0; off < bytes; off += 65536u)
                bulk_g2s(reinterpret_cast<char *>(dst) + off, reinterpret_cast<const char *>(src) + off,
                         min(65536u, bytes - off), bar);
        }
        return;
    }
    for (int r = lane; r < n; r += 32)
        bulk_g2s(dst + static_cast<int64_t>(r) * stride, src + static_cast<int64_t>(r) * pitch,
                 static_cast<uint32_t>(pitch) * 4u, bar);
}

// The same with plain loads by the whole CTA (rows that are not whole 16-byte units).
__device__ __forceinline__ void slice_plain(uint32_t *dst, const uint32_t *src, int n, int pitch, int stride)
{
    for (int i = threadIdx.x; i < n * pitch; i += blockDim.x) {
        const int r = i / pitch, w = i - r * pitch;
        dst[r * stride + w] = __ldg(src + static_cast<int64_t>(r) * pitch + w);
    }
}

// Words [pitch, stride) of every row and every word of rows [n, rows) are
// zero: the MMA units read whole 8-word groups, and rows past the matrix
// contribute nothing.
__device__ __forceinline__ void slice_pad(uint32_t *dst, int n, int rows, int pitch, int stride)
{
    const int padw = stride - pitch;
    for (int i = threadIdx.x; i < n * padw; i += blockDim.x) {
        const int r = i / padw;
        dst[r * stride + pitch + (i - r * padw)] = 0u;
    }
    for (int i = n * stride + threadIdx.x; i < rows * stride; i += blockDim.x) dst[i] = 0u;
}

// Grid barrier on the header word (see the file comment); false on timeout.
__device__ bool grid_sync(const DecodeParams &P, Misc *ms)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        bool ok = true;
        // the release half of the arrival covers the CTA's writes, ordered
        // before it by the barrier above
        unsigned ticket;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                     : "=r"(ticket)
                     : "l"(reinterpret_cast<unsigned *>(P.sync))
                     : "memory");
        if (ticket == gridDim.x - 1) {
            const unsigned long long next = static_cast<unsigned long long>(ms->e0 + 1u) << 32;
            asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(P.sync), "l"(next) : "memory");
        } else {
            // every CTA has arrived once the count reaches the grid size (seen
            // before the last arrival resets it) or the epoch has moved on;
            // relaxed polls, then one acquire fence. The limit counts from
            // the CTA's entry and is checked before each poll.
            while (true) {
                if (global_ns() - ms->t_entry > P.wait_ns) {
                    ok = false;
                    atomicExch(P.status, static_cast<int32_t>(DBF_ERR_TIMEOUT));
                    break;
                }
                unsigned long long v;
                asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(P.sync) : "memory");
                if (static_cast<unsigned>(v >> 32) != ms->e0 || static_cast<unsigned>(v) >= gridDim.x) break;
            }
            asm volatile("fence.acq_rel.gpu;" ::: "memory");
        }
        ms->flag = ok ? 1 : 0;
    }
    __syncthreads();
    return ms->flag != 0;
}

// Sign sums of the CTA's row blocks: tile[row][col] += sum_k b[row, k] d[col, k]
// for the digit columns col < ndcol (column groups of eight; digit columns at
// or past ndcol read the zero column). The (row block, K group) units are
// split contiguously over the warps; a warp keeps its run of units of one
// row block in eight mask accumulators and adds the folded sums to the tile.
__device__ __noinline__ void sign_sums(const uint32_t *slice, int stride, int nrb, int ng, const char *dig, int cb,
                                       int ndcol, int *tile, int tile_ld)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int units = nrb * ng;
    const int u_begin = units * warp / kWarps, u_end = units * (warp + 1) / kWarps;
    const int ncg = (ndcol + 7) / 8;
    const char *zero = dig + static_cast<size_t>(ndcol) * cb;
    for (int u = u_begin; u < u_end;) {
        const int rb = u / ng;
        const int g0 = u - rb * ng;
        const int g1 = min(ng, g0 + (u_end - u));
        const uint32_t *pa = slice + (rb * 16 + g) * stride + 2 * t;
        const uint32_t *pb = pa + 8 * stride;
        for (int q = 0; q < ncg; ++q) {
            const int col = q * 8 + g;
            const char *colp = (col < ndcol ? dig + static_cast<size_t>(col) * cb : zero) + t * 8;
            int acc[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0;
            for (int gr = g0; gr < g1; ++gr) {
                const uint2 A = *reinterpret_cast<const uint2 *>(pa + gr * kGroupWords);
                const uint2 B = *reinterpret_cast<const uint2 *>(pb + gr * kGroupWords);
                const char *bp = colp + gr * 256;
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
            int *tr = tile + (rb * 16 + g) * tile_ld + q * 8 + 2 * t;
            atomicAdd(tr, f[0]);
            atomicAdd(tr + 1, f[1]);
            atomicAdd(tr + 8 * tile_ld, f[2]);
            atomicAdd(tr + 8 * tile_ld + 1, f[3]);
        }
        u += g1 - g0;
    }
}

// sum_k b_k q_k of one (row, column) from the three digit columns of the tile
__device__ __forceinline__ long long digit_sum(const int *tr, int c)
{
    return static_cast<long long>(tr[kDigits * c]) + 256LL * tr[kDigits * c + 1] + 65536LL * tr[kDigits * c + 2];
}

// ---- the kernel -----------------------------------------------------------------
// Every phase that runs once per call is a rolled loop: the kernel runs once
// per CTA per call, so its instructions are fetched cold each time, and the
// length of the code it executes, not its arithmetic, sets the time of those
// phases. Inputs of the digit build (x and gamma) are staged in shared memory
// by bulk copies, so those loops do not wait on global loads.
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const __grid_constant__ DecodeParams P)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, b = blockIdx.x;
    const dbf_layer &L = P.L;
    const int ell = L.ell, C = P.C, ndcol = kDigits * C;

    pdl_trigger();   // the next kernel in the stream may start its own weight copies
    const bool early = (P.flags & DBF_WEIGHTS_STATIC) != 0;
    if (!early) pdl_wait();

    // ---- this CTA's 16-row blocks: stage 1 [r1b, r1e), stage 2 [r2b, r2e)
    const int r1b = static_cast<int>(static_cast<int64_t>(P.nrb1) * b / G);
    const int r1e = static_cast<int>(static_cast<int64_t>(P.nrb1) * (b + 1) / G);
    const int r2b = static_cast<int>(static_cast<int64_t>(P.nrb2) * b / G);
    const int r2e = static_cast<int>(static_cast<int64_t>(P.nrb2) * (b + 1) / G);
    const int lo1 = r1b * 16, rows1 = (r1e - r1b) * 16;
    const int n1 = max(0, min(r1e * 16, L.R) - lo1);   // rows of B2 in the slice
    const int lo2 = r2b * 16, rows2 = (r2e - r2b) * 16;
    const int n2 = max(0, min(r2e * 16, L.N) - lo2);

    uint32_t *s1 = reinterpret_cast<uint32_t *>(smem);
    uint32_t *s2 = reinterpret_cast<uint32_t *>(smem + P.off_s2);
    // x and gamma are staged where the B1 slice goes; that slice is copied
    // once the digits of gamma . x are built
    const uint16_t *gs = reinterpret_cast<const uint16_t *>(smem + P.off_s2);
    char *dig = reinterpret_cast<char *>(smem + P.off_dig);
    int *tile = reinterpret_cast<int *>(smem + P.off_tile);
    Misc *ms = reinterpret_cast<Misc *>(smem + P.off_misc);
    float *rs1 = reinterpret_cast<float *>(smem + P.off_rs1);   // beta_i of the CTA's stage-1 rows
    float *rs2 = reinterpret_cast<float *>(smem + P.off_rs2);   // alpha_i of its stage-2 rows

    if (tid < kMaxCols) {
        ms->amax[tid] = 0u;
        ms->qsum_v[tid] = 0;
    }
    if (tid == 0) {
        ms->t_entry = global_ns();
        for (int i = 0; i < 5; ++i) bar_init(&ms->bar[i], 1);
        ms->bmax = 0u;
    }
    __syncthreads();
    // ---- the B2 slice and gamma -> shared memory, in flight from here on
    if (tid == 0) {
        if (P.bulk1 && n1 > 0) bar_expect_tx(&ms->bar[0], static_cast<uint32_t>(n1) * P.pitch1 * 4u);
        if (P.bulk_g) {
            bar_expect_tx(&ms->bar[2], static_cast<uint32_t>(P.gs_bytes));
            bulk_g2s(smem + P.off_s2, L.gamma, static_cast<uint32_t>(P.gs_bytes), &ms->bar[2]);
        }
    }
    if (warp == 0) {
        __syncwarp();
        if (P.bulk1) slice_bulk(s1, L.b2_packed + static_cast<int64_t>(lo1) * P.pitch1, n1, P.pitch1, P.stride1, &ms->bar[0]);
    }
    slice_pad(s1, n1, rows1, P.pitch1, P.stride1);
    if (!P.bulk1) slice_plain(s1, L.b2_packed + static_cast<int64_t>(lo1) * P.pitch1, n1, P.pitch1, P.stride1);
    if (!P.bulk_g) {
        // element by element, rows padded to a multiple of 8 values
        uint16_t *g = reinterpret_cast<uint16_t *>(smem + P.off_s2);
#pragma unroll 1
        for (int i = tid; i < ell * L.M; i += kThreads) {
            const int e = i / L.M;
            g[e * P.gpitch + (i - e * L.M)] = __ldg(L.gamma + i);
        }
    }
    // ---- weight-side scales: the CTA's beta and alpha rows, max |beta|. The
    // first round of all three is loaded together (one memory round trip for
    // the usual sizes); any rest follows in rolled loops.
    {
        // fp16 magnitudes order like their bit patterns: the maximum is taken on
        // the bits, two at a time (16-byte loads when beta is 16-byte aligned)
        const int nb = L.R * ell;
        const int nv = (reinterpret_cast<uintptr_t>(L.beta) & 15u) == 0 ? nb / 8 : 0;
        const uint4 *bp = reinterpret_cast<const uint4 *>(L.beta);
        constexpr int kV = 4;   // 16-byte beta loads per thread in the first round
        uint4 w[kV];
#pragma unroll
        for (int e = 0; e < kV; ++e) {
            const int i = tid + e * kThreads;
            w[e] = i < nv ? __ldg(bp + i) : make_uint4(0u, 0u, 0u, 0u);
        }
        auto scale1 = [&](int i) {
            const int e = i / rows1, r = i - e * rows1;
            return r < n1 ? ldg_h(L.beta + static_cast<int64_t>(e) * L.R + lo1 + r) : 0.f;
        };
        auto scale2 = [&](int i) {
            const int e = i / rows2, r = i - e * rows2;
            return r < n2 ? ldg_h(L.alpha + static_cast<int64_t>(e) * L.N + lo2 + r) : 0.f;
        };
        const float v1 = tid < rows1 * ell ? scale1(tid) : 0.f;
        const float v2 = tid < rows2 * ell ? scale2(tid) : 0.f;
        unsigned m2 = 0u;
#pragma unroll
        for (int e = 0; e < kV; ++e) {
            m2 = __vmaxu2(m2, w[e].x & 0x7FFF7FFFu);
            m2 = __vmaxu2(m2, w[e].y & 0x7FFF7FFFu);
            m2 = __vmaxu2(m2, w[e].z & 0x7FFF7FFFu);
            m2 = __vmaxu2(m2, w[e].w & 0x7FFF7FFFu);
        }
        if (tid < rows1 * ell) rs1[tid] = v1;
        if (tid < rows2 * ell) rs2[tid] = v2;
#pragma unroll 1
        for (int i = tid + kThreads; i < rows1 * ell; i += kThreads) rs1[i] = scale1(i);
#pragma unroll 1
        for (int i = tid + kThreads; i < rows2 * ell; i += kThreads) rs2[i] = scale2(i);
#pragma unroll 1
        for (int i = tid + kV * kThreads; i < nv; i += kThreads) {
            const uint4 u = __ldg(bp + i);
            m2 = __vmaxu2(__vmaxu2(m2, u.x & 0x7FFF7FFFu), __vmaxu2(u.y & 0x7FFF7FFFu, u.z & 0x7FFF7FFFu));
            m2 = __vmaxu2(m2, u.w & 0x7FFF7FFFu);
        }
#pragma unroll 1
        for (int i = nv * 8 + tid; i < nb; i += kThreads) m2 = max(m2, static_cast<unsigned>(__ldg(L.beta + i)) & 0x7FFFu);
        m2 = max(m2 & 0xFFFFu, m2 >> 16);
        for (int o = 16; o; o >>= 1) m2 = max(m2, __shfl_xor_sync(0xffffffffu, m2, o));
        if (lane == 0) atomicMax(&ms->bmax, __float_as_uint(__half2float(__ushort_as_half(static_cast<unsigned short>(m2)))));
    }
    // the zero digit column of stage 1 (digit columns past 3C of an MMA column group)
#pragma unroll 1
    for (int i = tid; i < P.cb1 / 16; i += kThreads)
        reinterpret_cast<uint4 *>(dig + static_cast<size_t>(ndcol) * P.cb1)[i] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
    for (int i = tid; i < rows1 * P.tile_ld; i += kThreads) tile[i] = 0;

    // ---- activations: x, one token at a time, into two shared-memory buffers
    // (the next token's copy is in flight while a token is digitised)
    if (early) pdl_wait();
    if (tid == 0) {
        unsigned long long v;
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(P.sync) : "memory");
        ms->e0 = static_cast<unsigned>(v >> 32);
    }
    const int xsize = P.xd == DBF_BF16 ? 2 : 4;
    auto stage_token = [&](int t) {
        unsigned char *dst = smem + P.off_s2 + P.gs_bytes + (t & 1) * P.xs_bytes;
        const unsigned char *src = static_cast<const unsigned char *>(P.x) + static_cast<int64_t>(t) * L.M * xsize;
        if (P.bulk_x) {
            if (tid == 0) {
                // the buffer's previous token was read by generic loads: order
                // them before the asynchronous write
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                bar_expect_tx(&ms->bar[3 + (t & 1)], static_cast<uint32_t>(L.M * xsize));
                bulk_g2s(dst, src, static_cast<uint32_t>(L.M * xsize), &ms->bar[3 + (t & 1)]);
            }
        } else if (xsize == 2) {
#pragma unroll 1
            for (int i = tid; i < L.M; i += kThreads)
                reinterpret_cast<uint16_t *>(dst)[i] = reinterpret_cast<const uint16_t *>(src)[i];
        } else {
#pragma unroll 1
            for (int i = tid; i < L.M; i += kThreads)
                reinterpret_cast<uint32_t *>(dst)[i] = reinterpret_cast<const uint32_t *>(src)[i];
        }
    };
    stage_token(0);
    if (P.T > 1) stage_token(1);

    // ---- stage 1 operand: digits of q = round(gamma_i . x_t 2^sh) per column.
    // A half warp takes one packed word per step: lane p (of 16) the columns
    // 2p and 2p + 1, which bits p and 16 + p stand for. Two passes over
    // shared memory: the column's max |gamma . x|, then its digits.
    const bool do1 = n1 > 0;
    const int nwp = P.ng1 * kGroupWords / 2;   // word pairs, up to the last 256-column group
    const int hp = lane & 15, hw = lane >> 4;
#pragma unroll 1
    for (int tok = 0; tok < P.T; ++tok) {
        token_wait(P, ms, tok);
        const unsigned char *xs = smem + P.off_s2 + P.gs_bytes + (tok & 1) * P.xs_bytes;
#pragma unroll 1
        for (int env = 0; env < ell; ++env) {
            const int c = tok * ell + env;
            const uint16_t *gc = gs + static_cast<int64_t>(env) * P.gpitch;
            float m = 0.f;
            // unrolled by four: the iterations' shared-memory loads overlap
#pragma unroll 4
            for (int wp = warp; wp < nwp; wp += kWarps) {
                const int col = 64 * wp + 32 * hw + 2 * hp;
                const float2 u = stage_u2(gc, xs, P.xd, col, L.M);
                m = fmaxf(m, fmaxf(fabsf(u.x), fabsf(u.y)));
            }
            for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) atomicMax(&ms->amax[c], __float_as_uint(m));
            __syncthreads();
            const int sh = scale_exponent(__uint_as_float(ms->amax[c]));
            int sq = 0, sa = 0;
            char *d0 = dig + static_cast<size_t>(kDigits * c) * P.cb1;
#pragma unroll 4
            for (int wp = warp; wp < nwp; wp += kWarps) {
                const int w = 2 * wp + hw;
                const float2 u = stage_u2(gc, xs, P.xd, 32 * w + 2 * hp, L.M);
                const int q0 = quantize(u.x, sh), q1 = quantize(u.y, sh);
                sq += q0 + q1;
                sa += abs(q0) + abs(q1);
                const uint32_t d0b = digit_bytes(q0), d1b = digit_bytes(q1);
                const int off = digit_byte(w, hp);   // bit hp; bit 16 + hp is two bytes on
                d0[off] = static_cast<char>(d0b & 255u);
                d0[off + 2] = static_cast<char>(d1b & 255u);
                d0[P.cb1 + off] = static_cast<char>((d0b >> 8) & 255u);
                d0[P.cb1 + off + 2] = static_cast<char>((d1b >> 8) & 255u);
                d0[2 * P.cb1 + off] = static_cast<char>(d0b >> 16);
                d0[2 * P.cb1 + off + 2] = static_cast<char>(d1b >> 16);
            }
            // per-warp partial sums through shared memory (no 64-bit shared atomics)
            const long long sq64 = warp_sum_exact(sq), sa64 = warp_sum_exact(sa);
            if (lane == 0) {
                ms->wq[warp][c] = sq64;
                ms->wa[warp][c] = sa64;
            }
            if (tid == 0) ms->sh_u[c] = sh;
        }
        if (tok + 2 < P.T) {
            __syncthreads();   // every read of this token's buffer is done
            stage_token(tok + 2);
        }
    }
    __syncthreads();
    // ---- the B1 slice -> shared memory (over the staged x and gamma, which
    // are no longer read: the generic reads are ordered before the copy)
    if (warp == 0) {
        if (lane == 0) {
            if (P.bulk2 && n2 > 0) bar_expect_tx(&ms->bar[1], static_cast<uint32_t>(n2) * P.pitch2 * 4u);
        }
        __syncwarp();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (P.bulk2) slice_bulk(s2, L.b1_packed + static_cast<int64_t>(lo2) * P.pitch2, n2, P.pitch2, P.stride2, &ms->bar[1]);
    }
    slice_pad(s2, n2, rows2, P.pitch2, P.stride2);
    if (!P.bulk2) slice_plain(s2, L.b1_packed + static_cast<int64_t>(lo2) * P.pitch2, n2, P.pitch2, P.stride2);
    if (tid < C) {
        long long sq = 0, sa = 0;
        for (int w = 0; w < kWarps; ++w) {
            sq += ms->wq[w][tid];
            sa += ms->wa[w][tid];
        }
        ms->qsum_u[tid] = sq;
        ms->qabs_u[tid] = sa;
        // |v_r| = |beta_r h_r| <= max|beta| sum|q| 2^-sh; the factor covers the
        // fp32 roundings of h and of beta h
        const float bound = __uint_as_float(ms->bmax) * scale_pow2(static_cast<float>(sa), -ms->sh_u[tid]) *
                            (1.0f + 1.0f / 1024.0f);
        ms->sh_v[tid] = scale_exponent(bound);
    }

    // ---- stage 1: h = B2 u for the CTA's row blocks, then v = beta . h as digits into the image
    // (one (row, column) per thread and step; each thread's sums of q of v per
    // column are reduced per warp and summed through shared memory)
    int qv[kMaxCols];
#pragma unroll
    for (int c = 0; c < kMaxCols; ++c) qv[c] = 0;
    if (do1) {
        const bool ok1 = P.bulk1 ? slice_wait(&ms->bar[0], P, ms) : true;
        if (ok1) {
            sign_sums(s1, P.stride1, rows1 / 16, P.ng1, dig, P.cb1, ndcol, tile, P.tile_ld);
            __syncthreads();
#pragma unroll 1
            for (int i = tid; i < n1 * C; i += kThreads) {
                const int c = i / n1, lr = i - c * n1;
                const int env = c - (c / ell) * ell;
                const long long s = digit_sum(tile + lr * P.tile_ld, c);
                const float h = scale_pow2(__ll2float_rn(ms->qsum_u[c] - 2 * s), -ms->sh_u[c]);
                const int q = quantize(rs1[env * rows1 + lr] * h, ms->sh_v[c]);
                const uint32_t db = digit_bytes(q);
                char *im = P.img + static_cast<size_t>(kDigits * c) * P.cb2 + digit_offset(lo1 + lr);
                im[0] = static_cast<char>(db & 255u);
                im[P.cb2] = static_cast<char>((db >> 8) & 255u);
                im[2 * P.cb2] = static_cast<char>(db >> 16);
#pragma unroll
                for (int cc = 0; cc < kMaxCols; ++cc)
                    if (cc == c) qv[cc] += q;
            }
        }
    }
    // digits of v past the rank, up to the last 256-column group, are zero
    if (r1e == P.nrb1 && r1e > r1b) {
        const int tail = P.ng2 * 256 - L.R;
#pragma unroll 1
        for (int i = tid; i < C * tail; i += kThreads) {
            const int c = i / tail, r = L.R + (i - c * tail);
            char *im = P.img + static_cast<size_t>(kDigits * c) * P.cb2 + digit_offset(r);
            im[0] = 0;
            im[P.cb2] = 0;
            im[2 * P.cb2] = 0;
        }
    }
    __syncthreads();   // the digit build's partial sums have been read
#pragma unroll
    for (int c = 0; c < kMaxCols; ++c) {
        if (c < C) {
            const long long w = warp_sum_exact(qv[c]);
            if (lane == 0) ms->wq[warp][c] = w;
        }
    }
    __syncthreads();
    if (tid < C) {
        long long sum = 0;
        for (int w = 0; w < kWarps; ++w) sum += ms->wq[w][tid];
        P.qpart[static_cast<int64_t>(b) * C + tid] = sum;
    }

    // ---- every CTA's digits of v and its sums are written
    const bool passed = grid_sync(P, ms);
    const bool do2 = n2 > 0;
    if (!passed || !do2) {
        if (do2 && P.bulk2) slice_wait(&ms->bar[1], P, ms);   // no copy left in flight
        return;
    }

    // ---- stage 2: the digits of v (coherent 16-byte loads: other CTAs wrote
    // them in this kernel) and the sums of q of v, their loads in flight
    // together, then the CTA's rows of y
    {
        constexpr int kP = (kMaxGrid + 31) / 32;
        long long part[kP];
        if (warp < C) {
#pragma unroll
            for (int e = 0; e < kP; ++e) {
                const int k = lane + 32 * e;
                part[e] = k < G ? __ldcg(P.qpart + static_cast<int64_t>(k) * C + warp) : 0;
            }
        }
        const int n16 = ndcol * P.cb2 / 16;
        const uint4 *src = reinterpret_cast<const uint4 *>(P.img);
        uint4 *dst = reinterpret_cast<uint4 *>(dig);
        constexpr int kLoads = 8;
#pragma unroll 1
        for (int i0 = tid; i0 < n16; i0 += kLoads * kThreads) {
            uint4 v[kLoads];
#pragma unroll
            for (int e = 0; e < kLoads; ++e) {
                const int i = i0 + e * kThreads;
                v[e] = i < n16 ? __ldcg(src + i) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int e = 0; e < kLoads; ++e)
                if (i0 + e * kThreads < n16) dst[i0 + e * kThreads] = v[e];
        }
        if (warp < C) {
            long long sum = 0;
#pragma unroll
            for (int e = 0; e < kP; ++e) sum += part[e];
            sum = warp_sum64(sum);
            if (lane == 0) ms->qsum_v[warp] = sum;
        }
    }
#pragma unroll 1
    for (int i = tid; i < P.cb2 / 16; i += kThreads)
        reinterpret_cast<uint4 *>(dig + static_cast<size_t>(ndcol) * P.cb2)[i] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
    for (int i = tid; i < rows2 * P.tile_ld; i += kThreads) tile[i] = 0;
    if (P.bulk2) {
        if (!slice_wait(&ms->bar[1], P, ms)) return;
    } else {
        __syncthreads();
    }
    sign_sums(s2, P.stride2, rows2 / 16, P.ng2, dig, P.cb2, ndcol, tile, P.tile_ld);
    __syncthreads();
    // ---- y = [acc] y + sum_i alpha_i . z_i, one (token, row) per thread
#pragma unroll 1
    for (int i = tid; i < P.T * n2; i += kThreads) {
        const int tok = i / n2, lr = i - tok * n2;
        const int64_t yi = static_cast<int64_t>(tok) * L.N + lo2 + lr;
        float yv = (P.flags & DBF_ACCUMULATE) ? load_act(P.y, P.yd, yi) : 0.f;
#pragma unroll 1
        for (int env = 0; env < ell; ++env) {
            const int c = tok * ell + env;
            const long long s = digit_sum(tile + lr * P.tile_ld, c);
            const float z = scale_pow2(__ll2float_rn(ms->qsum_v[c] - 2 * s), -ms->sh_v[c]);
            yv += rs2[env * rows2 + lr] * z;
        }
        store_act(P.y, P.yd, yi, yv);
    }
}

// ---- host side ----------------------------------------------------------------

// Row stride of a slice: whole 8-word groups, and a stride of 8 or 24 words
// modulo 32 so that the 8-byte A-fragment loads of rows g = 0..3 (a half
// warp) fall on four different bank octets.
int slice_stride(int pitch)
{
    const int r8 = (pitch + kGroupWords - 1) / kGroupWords * kGroupWords;
    return (r8 % 16 == 0) ? r8 + 8 : r8;
}

// Bytes per digit column: 256 per group of 8 packed words, plus 32 so that
// consecutive columns start 32 bytes apart modulo 128 (the 8-byte B-fragment
// loads of a half warp, columns g = 0..3 and threads t = 0..3, then cover
// the 32 banks once).
int col_bytes(int ng) { return ng * 256 + 32; }

size_t img_bytes(int C, int ng2) { return align_up(static_cast<size_t>(kDigits) * C * col_bytes(ng2), 256); }

std::mutex g_coop_lock;
int g_coop_ok[64];   // per device: 0 unknown, 1 cooperative + PDL accepted, 2 refused

// Plan of the single-launch decode for this call; false when the call is
// outside its range (more than kMaxCols columns, M above 8192, or shared
// memory).
bool decode_plan(const dbf_layer &L, int64_t T, int sms, DecodeParams *out, size_t *smem_out, int *grid_out)
{
    const int64_t C = T * L.ell;
    if (T < 1 || C > kMaxCols || L.M > kMaxWordsPerWarp * kWarps * 32) return false;
    DecodeParams P{};
    P.L = L;
    P.T = static_cast<int>(T);
    P.C = static_cast<int>(C);
    P.pitch1 = static_cast<int>(pitch_words(L.M));
    P.pitch2 = static_cast<int>(pitch_words(L.R));
    P.stride1 = slice_stride(P.pitch1);
    P.stride2 = slice_stride(P.pitch2);
    P.ng1 = (P.pitch1 + kGroupWords - 1) / kGroupWords;
    P.ng2 = (P.pitch2 + kGroupWords - 1) / kGroupWords;
    P.cb1 = col_bytes(P.ng1);
    P.cb2 = col_bytes(P.ng2);
    P.nrb1 = (L.R + 15) / 16;
    P.nrb2 = (L.N + 15) / 16;
    int G = sms < kMaxGrid ? sms : kMaxGrid;
    const int nrb = P.nrb1 > P.nrb2 ? P.nrb1 : P.nrb2;
    if (G > nrb) G = nrb;
    if (G < 1) G = 1;
    P.max_rb1 = (P.nrb1 + G - 1) / G;
    P.max_rb2 = (P.nrb2 + G - 1) / G;
    P.bulk1 = P.pitch1 % 4 == 0;
    P.bulk2 = P.pitch2 % 4 == 0;
    P.tile_ld = 8 * ((kDigits * P.C + 7) / 8) + 1;   // odd: the epilogue's row-per-lane reads hit distinct banks
    const int rows1 = P.max_rb1 * 16, rows2 = P.max_rb2 * 16;
    const int cbm = P.cb1 > P.cb2 ? P.cb1 : P.cb2;
    // gamma and x are staged in the B1 slice's region (fp32 x: 4 bytes per value)
    P.gpitch = (L.M + 7) / 8 * 8;
    P.gs_bytes = static_cast<int>(static_cast<size_t>(L.ell) * P.gpitch * 2);
    P.xs_bytes = static_cast<int>(align_up(static_cast<size_t>(L.M) * 4, 16));   // fp32 x at most
    const size_t s2_bytes = static_cast<size_t>(rows2) * P.stride2 * 4;
    const size_t stage_bytes = static_cast<size_t>(P.gs_bytes) + 2 * static_cast<size_t>(P.xs_bytes);
    size_t off = align_up(static_cast<size_t>(rows1) * P.stride1 * 4, 128);
    P.off_s2 = static_cast<int>(off);
    off = align_up(off + (s2_bytes > stage_bytes ? s2_bytes : stage_bytes), 128);
    P.off_dig = static_cast<int>(off);
    off = align_up(off + static_cast<size_t>(kDigits * P.C + 1) * cbm, 16);
    P.off_tile = static_cast<int>(off);
    off = align_up(off + static_cast<size_t>(rows1 > rows2 ? rows1 : rows2) * P.tile_ld * 4, 16);
    P.off_misc = static_cast<int>(off);
    off = align_up(off + sizeof(Misc), 16);
    P.off_rs1 = static_cast<int>(off);
    off = align_up(off + static_cast<size_t>(rows1) * L.ell * 4, 16);
    P.off_rs2 = static_cast<int>(off);
    off = align_up(off + static_cast<size_t>(rows2) * L.ell * 4, 16);
    if (off > static_cast<size_t>(kSmemCap)) return false;
    *out = P;
    *smem_out = off;
    *grid_out = G;
    return true;
}

}  // namespace

size_t decode_workspace_bytes(const dbf_layer &L, int64_t T)
{
    DecodeParams P;
    size_t smem;
    int G;
    if (!decode_plan(L, T, kMaxGrid, &P, &smem, &G)) return 0;
    return kWsHeaderBytes + img_bytes(P.C, P.ng2) + static_cast<size_t>(kMaxGrid) * P.C * sizeof(long long);
}

bool decode_fits(const dbf_layer &L, int64_t T)
{
    DecodeParams P;
    size_t smem;
    int G;
    return decode_plan(L, T, device_sms(), &P, &smem, &G);
}

cudaError_t decode_forward(const dbf_layer &L, const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                           int flags, void *ws, cudaStream_t s)
{
    DecodeParams P;
    size_t smem;
    int G;
    if (!decode_plan(L, T, device_sms(), &P, &smem, &G)) return cudaErrorInvalidValue;
    P.x = x;
    P.y = y;
    P.xd = xd;
    P.yd = yd;
    P.flags = flags;
    char *w = static_cast<char *>(ws);
    P.sync = reinterpret_cast<unsigned long long *>(w);
    P.status = reinterpret_cast<int32_t *>(w + kWsStatusOffset);
    P.img = w + kWsHeaderBytes;
    P.qpart = reinterpret_cast<long long *>(w + kWsHeaderBytes + img_bytes(P.C, P.ng2));
    P.wait_ns = decode_wait_ns();
    // staged inputs by bulk copies when whole 16-byte units (x is 16-byte
    // aligned by the call's contract; gamma only 2-byte)
    P.bulk_x = (static_cast<size_t>(L.M) * (xd == DBF_BF16 ? 2 : 4)) % 16 == 0;
    P.bulk_g = (reinterpret_cast<uintptr_t>(L.gamma) & 15u) == 0 && L.M % 8 == 0;   // rows unpadded
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(decode_kernel), static_cast<int>(smem), true);
    if (e != cudaSuccess) return e;

    int dev = 0;
    cudaGetDevice(&dev);
    int coop = 1;
    if (dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> guard(g_coop_lock);
        coop = g_coop_ok[dev] != 2;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = coop ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, decode_kernel, P);
    if (e != cudaSuccess && coop) {
        // the cooperative attribute together with programmatic dependent
        // launch was refused: launch without it, the grid being no larger
        // than one CTA per SM with every SM able to hold one (checked here)
        (void)cudaGetLastError();
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel, kThreads, smem) != cudaSuccess ||
            per_sm < 1 || G > device_sms())
            return cudaErrorCooperativeLaunchTooLarge;
        if (dev >= 0 && dev < 64) {
            std::lock_guard<std::mutex> guard(g_coop_lock);
            g_coop_ok[dev] = 2;
        }
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, decode_kernel, P);
    } else if (e == cudaSuccess && coop && dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> guard(g_coop_lock);
        g_coop_ok[dev] = 1;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace dbf
