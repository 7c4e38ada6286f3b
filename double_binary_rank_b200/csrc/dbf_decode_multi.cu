// Decode-regime forward in one launch for many tokens (more than one chunk
// of columns) and for many adapters routed by token segments. Calls of one
// layer whose columns make a single chunk take the kernel in dbf_decode.cu.
//
// LoRDBA page, section 2 ("Kernel de Inferencia"): the forward is two
// sign-accumulation products with per-channel scaling between them; DBF page,
// section 2 ("Inferencia"): with binary factors the dense product becomes
// additions and scalar-vector products. Stage 1 computes
// v_i = beta_i . (B2 (gamma_i . x)), stage 2 y = [acc] y + sum_i alpha_i . (B1 v_i).
// LoRDBA page, section 1: many adapters are served in one batch, each token
// segment through its own adapter.
//
// Arithmetic. A sign is s = 1 - 2b with b in {0, 1} the packed bit, so
//   sum_k s_k a_k = sum_k a_k - 2 sum_k b_k a_k .
// Every activation column a (one token and envelope) becomes the integers
// q_k = round(a_k 2^sh), |q| <= 2^22, with one power-of-two scale per column
// (q is exact whenever a is a small dyadic value), written as three balanced
// base-256 int8 digits. mma.sync m16n8k32 u8 x s8 accumulates sum_k b_k d_k
// exactly in int32: masking a packed word with 0x01010101 << j gives four
// bytes in {0, 2^j} (bits j, j + 8, j + 16, j + 24), so the eight masks
// j = 0..7 of a group of eight words feed eight MMAs whose accumulators carry
// the weight 2^j and are folded with exact right shifts. The digits are laid
// out to match: in each 256-column group, mask j and MMA thread t read 8
// bytes at j * 32 + t * 8, the digits of words 2t and 2t + 1 at bits j + 8i.
// The three digit columns are recombined in int64 and converted once:
// (sum q - 2 sum b q) 2^-sh. Every sum is an exact integer, so the result does
// not depend on how K is split.
//
// Work. The (token, envelope) columns are cut into chunks of at most eight
// columns (whole tokens of one segment). Stage-1 items are (chunk, range of
// rows of B2), stage-2 items (chunk, range of rows of B1); each CTA takes a
// contiguous run of items of each stage, so a long rank is split over CTAs
// by rows and many tokens by chunks. A stage-1 item digitises its chunk's
// gamma . x (unless the previous item had the same chunk), runs its rows of
// B2 and writes v = beta . h as digits into an image in the workspace, with
// its share of sum q. The scale of v is fixed in advance from the bound
// |v_r| <= max|beta| sum_m |q_m| 2^-sh (integers and bit patterns only, so
// every item of a chunk derives the same value without an exchange). A grid
// barrier publishes the image; a stage-2 item copies its chunk's digits of v
// into shared memory and runs its rows of B1.
//
// Data movement. One CTA per SM at most (cooperative launch, so the whole
// grid is co-resident). The rows of an item's slice are copied into shared
// memory by bulk asynchronous copies (whole 8-word groups per row, and a row
// stride of 8 or 24 words modulo 32 so that the A-fragment loads of a half
// warp hit distinct banks: one copy when the pitch already has that form,
// else one per row); for one layer with static weights the first stage-1 slice and gamma
// are in flight before the previous kernel in the stream has finished
// (programmatic dependent launch). Activations are staged one token at a
// time into two shared buffers (the next token's copy in flight while a token
// is digitised); the first stage-2 slice is copied over them once the CTA
// has built its last digits.
//
// Grid barrier (workspace header, 8 bytes: arrivals in the low word, an epoch
// in the high word). A CTA reads the epoch, then adds its arrival with an
// acquire-release atomic; the arrival that brings the count to the grid size
// stores (epoch + 1, count 0) with release semantics, and every other CTA
// polls (bounded by a time limit counted from the CTA's entry) until it sees
// the full count or the new epoch. The epoch can change only after every CTA has arrived, so a CTA that
// starts late still reads the current epoch; the count is zero again once
// the last CTA has arrived, whatever happened to the waits. A wait that runs
// out of time stores DBF_ERR_TIMEOUT in the header's status word and the CTA
// skips its stage-2 items.
#include "dbf_internal.cuh"

#include <algorithm>
#include <cmath>
#include <mutex>

namespace dbf {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kDigits = 3;               // int8 digits per activation value
constexpr int kChunkCols = 8;            // (token, envelope) columns per chunk at most
constexpr int kGroupWords = 8;           // packed words per MMA unit (256 columns of K)
constexpr int kMaxM = 8192;              // inputs at most (digit-build registers)
constexpr int kSmemCap = 227 * 1024;
constexpr int kMaxGrid = 160;
constexpr int kMaxSegments = 512;        // segments of one call (shared-memory chunk table)
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;   // 2 s

struct DecodeParams {
    dbf_layer L;                  // one layer (segmented == 0)
    const dbf_layer *adapters;    // segmented calls: adapter table (device)
    const int32_t *seg_off;       // segmented calls: [S + 1] token offsets (device)
    const int32_t *seg_adp;       // segmented calls: [S] adapter ids (device)
    int32_t *seg_status;          // segmented calls: optional sticky status for bad tables
    int segmented, S, num_adapters;
    int M, N, max_R, ell_cap;     // ell_cap: image columns per token (the largest ell)
    const void *x;
    void *y;
    dbf_dtype xd, yd;
    int T;
    int flags;
    unsigned long long *sync;     // header word: arrivals (low 32 bits), epoch (high 32 bits)
    int32_t *status;              // header: sticky status of the call's kernels
    char *img;                    // digits of v: [T * ell_cap][kDigits][cb2]
    long long *qpart;             // sums of q of v: [T * ell_cap][P1]
    int32_t *sh2;                 // scale exponents of v: [T * ell_cap]
    int tpc;                      // tokens per chunk
    int P1, P2;                   // row ranges per chunk in stage 1 (rows of B2) and stage 2 (rows of B1)
    int pitch1;                   // packed words per row of B2
    int stride1, stride2;         // words per row of the shared slices (stride2 for the largest rank)
    int cb1, cb2;                 // bytes per digit column of u (stage 1) and v (stage 2)
    int rows1, rows2;             // rows of an item at most (multiples of 16)
    int tile_ld;                  // int32 per tile row (8 per MMA column group, plus 1)
    int gpitch, gs_bytes, xs_bytes;   // staged gamma (values per row, bytes) and one token's x buffer
    int stage_g;                  // gamma staged in shared memory (else read from global memory: no room)
    int word2;                    // stage 2 in the per-word layout (small ranks, see digit_offset_word)
    int off_s2, off_dig, off_tile, off_misc, off_rs1, off_rs2, off_seg;   // shared-memory offsets
    unsigned long long wait_ns;   // limit of the grid-barrier wait
};

struct Misc {
    uint64_t bar[5];              // stage-1 slice, stage-2 slice, gamma, x buffers 0 and 1
    unsigned long long t_entry;   // %globaltimer at the CTA's entry
    int flag;
    unsigned e0;                  // epoch read at entry
    unsigned bmax;                // max |beta| of the current adapter (fp32 bits)
    int Q;                        // chunks of the call
    unsigned amax[kChunkCols];    // max |gamma . x| per chunk column (fp32 bits)
    int sh_u[kChunkCols], sh_v[kChunkCols];
    long long qsum_u[kChunkCols], qsum_v[kChunkCols];
    long long wq[kWarps][kChunkCols], wa[kWarps][kChunkCols];   // per-warp partial sums
};

// One chunk: its tokens [t0, t0 + ntok) of segment s, served by adapter a
// (-1: no adapter, the branch is zero).
struct Chunk {
    int s, t0, ntok, a;
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

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

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

// Every thread: wait until phase 'parity' of a copy barrier has completed.
// Thread 0 polls, bounded by the default limit whatever the grid barrier's
// limit is (no copy is cut short); a timeout is recorded in the status word
// and the CTA carries on.
__device__ __noinline__ void copy_wait(uint64_t *bar, uint32_t parity, int32_t *status)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned long long t0 = global_ns();
        while (!bar_try(bar, parity)) {
            if (global_ns() - t0 > kDefaultWaitNs) {
                atomicExch(status, static_cast<int32_t>(DBF_ERR_TIMEOUT));
                break;
            }
        }
    }
    __syncthreads();
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

__device__ __forceinline__ uint2 lds64(uint32_t a)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

// Digit layout (see the file comment): unit (word w, mask j < 8) holds the
// digits of bits j, j + 8, j + 16, j + 24 (bytes 0..3) of word w in its
// 256-byte group: group w / 8, mask j, MMA thread (w % 8) / 2, half w % 2.
__device__ __forceinline__ int unit_offset(int w, int j)
{
    return (w >> 3) * 256 + j * 32 + ((w & 7) >> 1) * 8 + (w & 1) * 4;
}

// The byte of column k of K: in-word column 2p sits at bit p, 2p + 1 at bit 16 + p.
__device__ __forceinline__ int digit_offset(int k)
{
    const int kk = k & 31;
    const int bit = (kk & 1) ? 16 + (kk >> 1) : (kk >> 1);
    return unit_offset(k >> 5, bit & 7) + (bit >> 3);
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

// gamma[col] x[col] and the same at col + 1 (col even), exact in fp32; zero
// at and past m. gamma is read through a generic pointer (shared or global).
__device__ __forceinline__ float2 gamma_x2(const uint16_t *gc, const unsigned char *xs, dbf_dtype xd, int col, int m)
{
    float2 x, g;
    if (col + 1 < m) {
        g = (reinterpret_cast<uintptr_t>(gc + col) & 3u) == 0
                ? __half22float2(*reinterpret_cast<const __half2 *>(gc + col))
                : make_float2(__half2float(__ushort_as_half(gc[col])), __half2float(__ushort_as_half(gc[col + 1])));
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

// Exact warp sum of per-thread int32 values: 16-bit halves summed separately.
__device__ __forceinline__ long long warp_sum_exact(int v)
{
    const unsigned lo = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(v) & 0xFFFFu);
    const int hi = __reduce_add_sync(0xffffffffu, v >> 16);
    return static_cast<long long>(hi) * 65536 + lo;
}

// Exact warp sum of per-thread int64 values of magnitude below 2^46: three
// 16-bit pieces and a signed top (each piece summed exactly in 32 bits).
__device__ __forceinline__ long long warp_sum_exact64(long long v)
{
    const unsigned p0 = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(v & 0xFFFF));
    const unsigned p1 = __reduce_add_sync(0xffffffffu, static_cast<unsigned>((v >> 16) & 0xFFFF));
    const int p2 = __reduce_add_sync(0xffffffffu, static_cast<int>(v >> 32));
    return static_cast<long long>(p2) * 4294967296LL + static_cast<long long>(p1) * 65536 + p0;
}

// 256-column groups of K in a row of 'pitch' packed words
__host__ __device__ inline int groups_of(int pitch) { return (pitch + kGroupWords - 1) / kGroupWords; }

// Row stride of a slice: whole 8-word groups, and 8 or 24 words modulo 32 so
// that the 8-byte A-fragment loads of rows g = 0..3 (a half warp) fall on
// four different bank octets.
__host__ __device__ inline int slice_stride(int pitch)
{
    const int r8 = groups_of(pitch) * kGroupWords;
    return (r8 % 16 == 0) ? r8 + 8 : r8;
}

// Bytes per digit column: 256 per group, plus 32 so that consecutive columns
// start 32 bytes apart modulo 128 (the 8-byte B-fragment loads of a half
// warp, columns g = 0..3 and threads t = 0..3, then cover the 32 banks once).
__host__ __device__ inline int col_bytes(int pitch) { return groups_of(pitch) * 256 + 32; }

// Stage 2 of small ranks (at most four packed words per row of B1) uses a
// per-word layout instead of whole groups, so that no MMA runs on padding:
// one MMA per packed word, MMA thread t taking bits t + 8i of the word for
// its first four K slots and bits t + 4 + 8i for its other four
// ((word >> t) & 0x01010101 and (word >> (t + 4)) & 0x01010101, bytes in
// {0, 1}); the digits of unit (word w, bit j) sit at
// w * 32 + (j % 4) * 8 + (j / 4) * 4, thread t's eight bytes at w * 32 + 8t.
constexpr int kWordPitchMax = 4;
__host__ __device__ inline bool word_layout(int pitch) { return pitch <= kWordPitchMax; }
__device__ __forceinline__ int digit_offset_word(int k)
{
    const int kk = k & 31;
    const int bit = (kk & 1) ? 16 + (kk >> 1) : (kk >> 1);
    return (k >> 5) * 32 + ((bit & 7) & 3) * 8 + ((bit & 7) >> 2) * 4 + (bit >> 3);
}
// row stride 4 modulo 8 words (the eight rows of a half MMA tile read one
// word each from distinct banks); digit columns of whole 4-word units, 32
// bytes apart modulo 128
__host__ __device__ inline int slice_stride_word(int pitch) { return pitch + ((12 - pitch % 8) % 8); }
__host__ __device__ inline int col_bytes_word(int pitch) { return (pitch + 3) / 4 * 4 * 32 + 32; }
// Stage-2 layout: chosen once per call from the largest rank (every adapter
// of a segmented call uses it). Row stride, bytes per digit column, and the
// packed words of K that stage 2 reads per row (whole groups, or the words).
__host__ __device__ inline int stride2_of(bool word, int pitch) { return word ? slice_stride_word(pitch) : slice_stride(pitch); }
__host__ __device__ inline int cb2_of(bool word, int pitch) { return word ? col_bytes_word(pitch) : col_bytes(pitch); }
__host__ __device__ inline int kwords2_of(bool word, int pitch) { return word ? pitch : groups_of(pitch) * kGroupWords; }

// Rows [0, n) of a packed matrix (pitch words per row) into a shared slice of
// 'stride' words per row: bulk copies issued by warp 0 with completion on
// 'bar' (rows of whole 16-byte units), else plain loads by the CTA. Words
// [pitch, stride) of every row and rows [n, rows) are zeroed (the MMA units
// read whole groups). True if the caller has to wait on 'bar'.
__device__ __noinline__ bool slice_load(uint32_t *dst, const uint32_t *src, int n, int rows, int pitch, int stride,
                                       uint64_t *bar, bool pad)
{
    const bool bulk = n > 0 && pitch % 4 == 0 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
    if (bulk) {
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            if (lane == 0) {
                fence_proxy_async();   // earlier generic reads of the slice come first
                bar_expect_tx(bar, static_cast<uint32_t>(n) * pitch * 4u);
            }
            __syncwarp();
            if (stride == pitch) {
                if (lane == 0) {
                    const uint32_t bytes = static_cast<uint32_t>(n) * pitch * 4u;
                    for (uint32_t off = 0; off < bytes; off += 65536u)
                        bulk_g2s(reinterpret_cast<char *>(dst) + off, reinterpret_cast<const char *>(src) + off,
                                 min(65536u, bytes - off), bar);
                }
            } else {
                for (int r = lane; r < n; r += 32)
                    bulk_g2s(dst + static_cast<int64_t>(r) * stride, src + static_cast<int64_t>(r) * pitch,
                             static_cast<uint32_t>(pitch) * 4u, bar);
            }
        }
    } else {
        for (int i = threadIdx.x; i < n * pitch; i += kThreads) {
            const int r = i / pitch, w = i - r * pitch;
            dst[r * stride + w] = __ldg(src + static_cast<int64_t>(r) * pitch + w);
        }
    }
    const int padw = pad ? stride - pitch : 0;
    for (int i = threadIdx.x; i < n * padw; i += kThreads) {
        const int r = i / padw;
        dst[r * stride + pitch + (i - r * padw)] = 0u;
    }
    for (int i = n * stride + threadIdx.x; i < rows * stride; i += kThreads) dst[i] = 0u;
    return bulk;
}

// Grid barrier on the header word (see the file comment); false on timeout.
__device__ __noinline__ bool grid_sync(const DecodeParams &P, Misc *ms)
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

// Sign sums of the slice's row blocks: tile[row][col] += sum_k b[row, k] d[col, k]
// for digit columns col < ndcol over 'ng' groups of K (tile columns from
// ndcol to the end of the last column group receive sums of column 0 and are
// never read). The (row block, group) units are split contiguously over the
// warps; for each column group a warp runs its units of one row block twice,
// masks 0..3 and then 4..7 (four mask accumulators live at a time), and adds
// the folded sums to the tile. Shared memory is addressed by 32-bit offsets.
__device__ __noinline__ void sign_sums(uint32_t slice, int stride, int nrb, int ng, uint32_t dig, int cb,
                                          int ndcol, int *tile, int tile_ld)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int units = nrb * ng;
    const int u_begin = static_cast<int>(static_cast<int64_t>(units) * warp / kWarps);
    const int u_end = static_cast<int>(static_cast<int64_t>(units) * (warp + 1) / kWarps);
    const int ncg = (ndcol + 7) >> 3;
    for (int u = u_begin; u < u_end;) {
        const int rb = u / ng;
        const int g0 = u - rb * ng;
        const int g1 = min(ng, g0 + (u_end - u));
        const uint32_t pa = slice + static_cast<uint32_t>(((rb * 16 + g) * stride + 2 * t + g0 * kGroupWords) * 4);
        const uint32_t pb = pa + static_cast<uint32_t>(8 * stride * 4);
        for (int q = 0; q < ncg; ++q) {
            const int col = q * 8 + g;
            const uint32_t colp = dig + static_cast<uint32_t>((col < ndcol ? col : 0) * cb + t * 8 + g0 * 256);
            int f[4] = {0, 0, 0, 0};
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                int acc[4][4];
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0;
                for (int gr = 0; gr < g1 - g0; ++gr) {
                    const uint2 A = lds64(pa + gr * kGroupWords * 4);
                    const uint2 B = lds64(pb + gr * kGroupWords * 4);
                    const uint32_t bp = colp + gr * 256 + half * 128;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t m = 0x01010101u << (4 * half + j);
                        const uint2 bv = lds64(bp + j * 32);
                        mma_u8s8(acc[j], A.x & m, B.x & m, A.y & m, B.y & m, bv.x, bv.y);
                    }
                }
                // fold the mask weights 2^j (exact: acc[j] is a multiple of 2^j)
#pragma unroll
                for (int e = 0; e < 4; ++e)
#pragma unroll
                    for (int j = 0; j < 4; ++j) f[e] += acc[j][e] >> (4 * half + j);
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

// The same in the per-word layout (stage 2 of small ranks): K = 'pitch'
// packed words, one MMA per word and column group.
__device__ __noinline__ void sign_sums_word(uint32_t slice, int stride, int nrb, int pitch, uint32_t dig, int cb,
                                           int ndcol, int *tile, int tile_ld)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int units = nrb * pitch;
    const int u_begin = static_cast<int>(static_cast<int64_t>(units) * warp / kWarps);
    const int u_end = static_cast<int>(static_cast<int64_t>(units) * (warp + 1) / kWarps);
    const int ncg = (ndcol + 7) >> 3;
    for (int q = 0; q < ncg; ++q) {
        const int col = q * 8 + g;
        const uint32_t cp = dig + static_cast<uint32_t>((col < ndcol ? col : 0) * cb + t * 8);
        for (int u = u_begin; u < u_end;) {
            const int rb = u / pitch;
            const int w0 = u - rb * pitch;
            const int w1 = min(pitch, w0 + (u_end - u));
            const uint32_t ra = slice + static_cast<uint32_t>((rb * 16 + g) * stride * 4);
            const uint32_t rb8 = ra + static_cast<uint32_t>(8 * stride * 4);
            int acc[4] = {0, 0, 0, 0};
            for (int w = w0; w < w1; ++w) {
                uint32_t wa, wb;
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wa) : "r"(ra + w * 4));
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wb) : "r"(rb8 + w * 4));
                const uint2 bv = lds64(cp + w * 32);
                mma_u8s8(acc, (wa >> t) & 0x01010101u, (wb >> t) & 0x01010101u, (wa >> (t + 4)) & 0x01010101u,
                         (wb >> (t + 4)) & 0x01010101u, bv.x, bv.y);
            }
            int *tr = tile + (rb * 16 + g) * tile_ld + q * 8 + 2 * t;
            atomicAdd(tr, acc[0]);
            atomicAdd(tr + 1, acc[1]);
            atomicAdd(tr + 8 * tile_ld, acc[2]);
            atomicAdd(tr + 8 * tile_ld + 1, acc[3]);
            u += w1 - w0;
        }
    }
}

// sum_k b_k q_k of one (row, chunk column) from the three digit columns of the tile


__device__ __forceinline__ long long digit_sum(const int *tr, int l)
{
    return static_cast<long long>(tr[kDigits * l]) + 256LL * tr[kDigits * l + 1] + 65536LL * tr[kDigits * l + 2];
}

// Scale rows [lo, lo + n) of each of 'ell' envelopes (fp16, row stride ld)
// into dst[e * rows + r] as fp32, zero past n.
__device__ __noinline__ void load_scales(float *dst, const uint16_t *src, int ld, int ell, int lo, int n, int rows)
{
    // eight loads per thread in flight before their stores
    constexpr int kBatch = 8;
    const int total = rows * ell;
    for (int base = threadIdx.x; base < total; base += kBatch * kThreads) {
        float v[kBatch];
#pragma unroll
        for (int e = 0; e < kBatch; ++e) {
            const int i = base + e * kThreads;
            const int env = i / rows, r = i - env * rows;
            v[e] = (i < total && r < n) ? ldg_h(src + static_cast<int64_t>(env) * ld + lo + r) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < kBatch; ++e) {
            const int i = base + e * kThreads;
            if (i < total) dst[i] = v[e];
        }
    }
}

// max |beta| over all rows and envelopes of an adapter, into *out (fp32 bits;
// zero beforehand, read after a barrier). fp16 magnitudes order like their
// bit patterns, so the maximum is taken on the bits.
__device__ __noinline__ void beta_max(const dbf_layer &A, unsigned *out)
{
    const int nb = A.R * A.ell;
    unsigned m2 = 0u;
    if ((reinterpret_cast<uintptr_t>(A.beta) & 15u) == 0) {
        const uint4 *bp = reinterpret_cast<const uint4 *>(A.beta);
        for (int i = threadIdx.x; i < nb / 8; i += kThreads) {
            const uint4 u = __ldg(bp + i);
            m2 = __vmaxu2(__vmaxu2(m2, u.x & 0x7FFF7FFFu), __vmaxu2(u.y & 0x7FFF7FFFu, u.z & 0x7FFF7FFFu));
            m2 = __vmaxu2(m2, u.w & 0x7FFF7FFFu);
        }
        for (int i = nb / 8 * 8 + threadIdx.x; i < nb; i += kThreads)
            m2 = max(m2, static_cast<unsigned>(__ldg(A.beta + i)) & 0x7FFFu);
    } else {
        for (int i = threadIdx.x; i < nb; i += kThreads) m2 = max(m2, static_cast<unsigned>(__ldg(A.beta + i)) & 0x7FFFu);
    }
    m2 = max(m2 & 0xFFFFu, m2 >> 16);
    m2 = __reduce_max_sync(0xffffffffu, m2);
    if ((threadIdx.x & 31) == 0)
        atomicMax(out, __float_as_uint(__half2float(__ushort_as_half(static_cast<unsigned short>(m2)))));
}

// ---- chunks ----------------------------------------------------------------------
// Segment table in shared memory (segmented calls): cs[s] = first chunk of
// segment s (cs[S] = chunk count), then t0[s], t1[s] and the adapter id
// (-1: none; segments with a bad range, id or adapter shape contribute no
// chunks and are reported). One layer: a single segment [0, T).
__device__ __noinline__ void build_chunk_table(const DecodeParams &P, int *tab, Misc *ms)
{
    int *cs = tab, *st0 = tab + P.S + 1, *st1 = st0 + P.S, *sad = st1 + P.S;
    for (int s = threadIdx.x; s < P.S; s += kThreads) {
        const int t0 = P.seg_off[s], t1 = P.seg_off[s + 1], a = P.seg_adp[s];
        bool ok = t0 >= 0 && t1 >= t0 && t1 <= P.T && a >= -1 && a < P.num_adapters;
        if (ok && a >= 0) {
            const dbf_layer &A = P.adapters[a];
            ok = A.M == P.M && A.N == P.N && A.R >= 1 && A.R <= P.max_R && A.ell >= 1 && A.ell <= P.ell_cap;
        }
        if (!ok && blockIdx.x == 0 && P.seg_status) atomicExch(P.seg_status, static_cast<int32_t>(DBF_ERR_INVALID_ARG));
        st0[s] = t0;
        st1[s] = t1;
        sad[s] = ok ? a : -2;
        cs[s] = ok ? (t1 - t0 + P.tpc - 1) / P.tpc : 0;
    }
    __syncthreads();
    // exclusive scan of the chunk counts (one warp; S <= kMaxSegments)
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int carry = 0;
        for (int base = 0; base < P.S; base += 32) {
            const int s = base + lane;
            const int v = s < P.S ? cs[s] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (s < P.S) cs[s] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            cs[P.S] = carry;
            ms->Q = carry;
        }
    }
    __syncthreads();
}

__device__ __forceinline__ Chunk chunk_of(const DecodeParams &P, const int *tab, int q)
{
    Chunk c;
    if (!P.segmented) {
        c.s = 0;
        c.t0 = q * P.tpc;
        c.ntok = min(P.tpc, P.T - c.t0);
        c.a = 0;
        return c;
    }
    const int *cs = tab, *st0 = tab + P.S + 1, *st1 = st0 + P.S, *sad = st1 + P.S;
    // the last segment s with cs[s] <= q (segments without chunks share
    // their start with the next one)
    int lo = 0, hi = P.S;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cs[mid] <= q) lo = mid;
        else hi = mid;
    }
    c.s = lo;
    c.t0 = st0[lo] + (q - cs[lo]) * P.tpc;
    c.ntok = min(P.tpc, st1[lo] - c.t0);
    c.a = sad[lo];
    return c;
}

__device__ __forceinline__ dbf_layer adapter_of(const DecodeParams &P, int a)
{
    return P.segmented ? P.adapters[a] : P.L;
}

// One activation column of a chunk: q = round(gamma . x 2^sh) with sh from
// the column's max |gamma . x|, as three digit columns at d0 (cb bytes
// apart), in two rolled passes over the staged values (maximum, then
// digits). A thread takes units (packed word w, mask j): the columns that
// bits j, j + 8, j + 16 and j + 24 of word w stand for (2j, 2j + 16, 2j + 1
// and 2j + 17 of the word) make one 32-bit word per digit. Returns sh; the
// warp's sums of q and |q| go to wq and wa (per-warp partials).
__device__ __noinline__ int digit_column(const uint16_t *gc, const unsigned char *xs, dbf_dtype xd, int m, int nunits,
                                         char *d0, int cb, unsigned *amax, long long *wq, long long *wa)
{
    const int lane = threadIdx.x & 31;
    float mx = 0.f;
#pragma unroll 1
    for (int unit = threadIdx.x; unit < nunits; unit += kThreads) {
        const int col = 32 * (unit >> 3) + 2 * (unit & 7);
        const float2 a = gamma_x2(gc, xs, xd, col, m), h = gamma_x2(gc, xs, xd, col + 16, m);
        mx = fmaxf(fmaxf(mx, fmaxf(fabsf(a.x), fabsf(a.y))), fmaxf(fabsf(h.x), fabsf(h.y)));
    }
    // magnitudes order like their fp32 bit patterns
    const unsigned mw = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
    if (lane == 0) atomicMax(amax, mw);
    __syncthreads();
    const int sh = scale_exponent(__uint_as_float(*amax));
    int sq = 0, sa = 0;   // |sum| < 2^31 per thread for M <= 8192
#pragma unroll 1
    for (int unit = threadIdx.x; unit < nunits; unit += kThreads) {
        const int col = 32 * (unit >> 3) + 2 * (unit & 7);
        const float2 a = gamma_x2(gc, xs, xd, col, m), h = gamma_x2(gc, xs, xd, col + 16, m);
        const int q0 = quantize(a.x, sh), q1 = quantize(h.x, sh), q2 = quantize(a.y, sh), q3 = quantize(h.y, sh);
        sq += (q0 + q1) + (q2 + q3);
        sa += (abs(q0) + abs(q1)) + (abs(q2) + abs(q3));
        const uint32_t D0 = digit_bytes(q0), D1 = digit_bytes(q1), D2 = digit_bytes(q2), D3 = digit_bytes(q3);
        // byte k of digit word i = byte i of Dk
        const uint32_t lo01 = __byte_perm(D0, D1, 0x5140), lo23 = __byte_perm(D2, D3, 0x5140);
        const uint32_t hi01 = __byte_perm(D0, D1, 0x0062), hi23 = __byte_perm(D2, D3, 0x0062);
        char *dp = d0 + unit_offset(unit >> 3, unit & 7);
        *reinterpret_cast<uint32_t *>(dp) = __byte_perm(lo01, lo23, 0x5410);
        *reinterpret_cast<uint32_t *>(dp + cb) = __byte_perm(lo01, lo23, 0x7632);
        *reinterpret_cast<uint32_t *>(dp + 2 * cb) = __byte_perm(hi01, hi23, 0x5410);
    }
    const long long q64 = warp_sum_exact(sq), a64 = warp_sum_exact(sa);
    if (lane == 0) {
        *wq = q64;
        *wa = a64;
    }
    return sh;
}

// ---- the kernel -----------------------------------------------------------------
// Phases that run once per item are rolled loops and shared helpers called
// out of line: the kernel's instructions are fetched cold each call, so the
// length of the code a call executes sets the time of those phases. Per-warp
// partial sums go through shared memory as plain stores.
//
// An item's slice and scale rows are reloaded only when its (adapter, row
// range) differs from the previous item's, its digits only when its chunk
// does. Stage-1 items run chunk by chunk (it = q * P1 + p: a CTA's items of
// one chunk share the digits), stage-2 items range by range
// (it = p * Q + q: a CTA's items of one adapter share the slice).
__global__ void __launch_bounds__(kThreads, 2) decode_multi_kernel(const __grid_constant__ DecodeParams P)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, b = blockIdx.x;

    pdl_trigger();   // the next kernel in the stream may start its own weight copies
    const bool early = !P.segmented && (P.flags & DBF_WEIGHTS_STATIC) != 0;
    if (!early) pdl_wait();

    uint32_t *s1 = reinterpret_cast<uint32_t *>(smem);
    uint32_t *s2 = reinterpret_cast<uint32_t *>(smem + P.off_s2);
    uint16_t *gs = reinterpret_cast<uint16_t *>(smem + P.off_s2);            // staged gamma (stage 1)
    unsigned char *xbuf = smem + P.off_s2 + (P.stage_g ? P.gs_bytes : 0);    // two x buffers (stage 1)
    char *dig = reinterpret_cast<char *>(smem + P.off_dig);
    int *tile = reinterpret_cast<int *>(smem + P.off_tile);
    Misc *ms = reinterpret_cast<Misc *>(smem + P.off_misc);
    float *rs1 = reinterpret_cast<float *>(smem + P.off_rs1);                 // beta of the stage-1 rows
    float *rs2 = reinterpret_cast<float *>(smem + P.off_rs2);                 // alpha of the stage-2 rows
    int *tab = reinterpret_cast<int *>(smem + P.off_seg);
    const int xsize = P.xd == DBF_BF16 ? 2 : 4;

    if (tid == 0) {
        ms->t_entry = global_ns();
        ms->bmax = 0u;
        for (int i = 0; i < 5; ++i) bar_init(&ms->bar[i], 1);
    }
    __syncthreads();

    uint32_t n_s1 = 0, n_s2 = 0, n_g = 0, n_x = 0;   // copy-barrier phases used (the same in every thread)
    int Q = P.segmented ? 0 : (P.T + P.tpc - 1) / P.tpc;
    int it1b = 0, it1e = 0, it2b = 0, it2e = 0;
    auto item_ranges = [&]() {
        const int I1 = Q * P.P1, I2 = Q * P.P2;
        it1b = static_cast<int>(static_cast<int64_t>(I1) * b / G);
        it1e = static_cast<int>(static_cast<int64_t>(I1) * (b + 1) / G);
        it2b = static_cast<int>(static_cast<int64_t>(I2) * b / G);
        it2e = static_cast<int>(static_cast<int64_t>(I2) * (b + 1) / G);
    };
    // loaded contexts: slice and scale rows per (adapter, range), gamma and
    // max |beta| per adapter
    int s1_a = -1, s1_p = -1, r1_a = -1, r1_p = -1, s2_a = -1, s2_p = -1, r2_a = -1, r2_p = -1;
    int g_a = -1, bmax_a = -1;
    bool s1_pending = false, s2_pending = false, g_pending = false;

    // row range p of a rank split into P ranges of 16-row blocks
    auto range_of = [](int rows_total, int parts, int p, int &lo, int &rows, int &n) {
        const int nrb = (rows_total + 15) / 16;
        const int blo = nrb * p / parts, bhi = nrb * (p + 1) / parts;
        lo = blo * 16;
        rows = (bhi - blo) * 16;
        n = max(0, min(bhi * 16, rows_total) - lo);
    };
    auto load_s1 = [&](const dbf_layer &A, int a, int p) {
        int lo, rows, n;
        range_of(A.R, P.P1, p, lo, rows, n);
        s1_pending = slice_load(s1, A.b2_packed + static_cast<int64_t>(lo) * P.pitch1, n, rows, P.pitch1, P.stride1,
                                &ms->bar[0], true);
        s1_a = a;
        s1_p = p;
    };
    auto load_r1 = [&](const dbf_layer &A, int a, int p) {
        int lo, rows, n;
        range_of(A.R, P.P1, p, lo, rows, n);
        load_scales(rs1, A.beta, A.R, A.ell, lo, n, rows);
        r1_a = a;
        r1_p = p;
    };
    auto load_s2 = [&](const dbf_layer &A, int a, int p) {
        int lo, rows, n;
        range_of(P.N, P.P2, p, lo, rows, n);
        const int pitch2 = static_cast<int>(pitch_words(A.R));
        s2_pending = slice_load(s2, A.b1_packed + static_cast<int64_t>(lo) * pitch2, n, rows, pitch2,
                                stride2_of(P.word2, pitch2), &ms->bar[1], !P.word2);
        s2_a = a;
        s2_p = p;
    };
    auto load_r2 = [&](const dbf_layer &A, int a, int p) {
        int lo, rows, n;
        range_of(P.N, P.P2, p, lo, rows, n);
        load_scales(rs2, A.alpha, P.N, A.ell, lo, n, rows);
        r2_a = a;
        r2_p = p;
    };
    // gamma of an adapter into rows of gpitch values: one bulk copy when its
    // rows are whole 16-byte units at a 16-byte address, else plain copies
    // (visible after the next barrier)
    auto stage_gamma = [&](const dbf_layer &A, int a) {
        if ((reinterpret_cast<uintptr_t>(A.gamma) & 15u) == 0 && P.M % 8 == 0) {
            if (tid == 0) {
                const uint32_t bytes = static_cast<uint32_t>(A.ell) * P.M * 2u;
                fence_proxy_async();
                bar_expect_tx(&ms->bar[2], bytes);
                for (uint32_t off = 0; off < bytes; off += 65536u)
                    bulk_g2s(reinterpret_cast<char *>(gs) + off, reinterpret_cast<const char *>(A.gamma) + off,
                             min(65536u, bytes - off), &ms->bar[2]);
            }
            g_pending = true;
        } else {
            for (int i = tid; i < A.ell * P.M; i += kThreads) {
                const int e = i / P.M;
                gs[e * P.gpitch + (i - e * P.M)] = A.gamma[i];
            }
        }
        g_a = a;
    };
    auto wait_gamma = [&]() {
        if (g_pending) {
            copy_wait(&ms->bar[2], n_g & 1u, P.status);
            ++n_g;
            g_pending = false;
        }
    };
    // the CTA's first items: slice of stage 1, gamma, scale rows of both
    // stages, max |beta| (one layer with static weights: before the previous
    // kernel has finished)
    auto first_items = [&]() {
        if (it1b < it1e) {
            const Chunk ch = chunk_of(P, tab, it1b / P.P1);
            if (ch.a >= 0) {
                const dbf_layer A = adapter_of(P, ch.a);
                load_s1(A, ch.a, it1b % P.P1);
                if (P.stage_g) stage_gamma(A, ch.a);
                load_r1(A, ch.a, it1b % P.P1);
                beta_max(A, &ms->bmax);
                bmax_a = ch.a;
            }
        }
        if (it2b < it2e) {
            const Chunk ch = chunk_of(P, tab, it2b % Q);
            if (ch.a >= 0) load_r2(adapter_of(P, ch.a), ch.a, it2b / Q);
        }
    };
    if (!P.segmented) item_ranges();
    if (early) {
        first_items();
        pdl_wait();
    }
    if (P.segmented) {
        build_chunk_table(P, tab, ms);
        Q = ms->Q;
        item_ranges();
    }
    if (!early) first_items();
    if (tid == 0) {
        unsigned long long v;
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(P.sync) : "memory");
        ms->e0 = static_cast<unsigned>(v >> 32);
    }
    // the first stage-2 slice goes over the staging buffers once the CTA's
    // last digits are built (or at once, with no stage-1 items)
    bool s2_issued = false;
    auto issue_first_s2 = [&]() {
        wait_gamma();
        __syncthreads();
        if (it2b < it2e) {
            const Chunk ch = chunk_of(P, tab, it2b % Q);
            if (ch.a >= 0) load_s2(adapter_of(P, ch.a), ch.a, it2b / Q);
        }
        s2_issued = true;
    };
    if (it1b >= it1e) issue_first_s2();
    const int q_last1 = it1e > it1b ? (it1e - 1) / P.P1 : -1;

    // ================= stage 1 =================
    int dig_q = -1;
    for (int it = it1b; it < it1e; ++it) {
        const int q = it / P.P1, p = it % P.P1;
        const Chunk ch = chunk_of(P, tab, q);
        if (ch.a < 0) continue;   // no adapter: stage 2 writes the zero branch
        const dbf_layer A = adapter_of(P, ch.a);
        const int ell = A.ell, cc = ch.ntok * ell, ndcol = kDigits * cc;
        int lo, rows, n1;
        range_of(A.R, P.P1, p, lo, rows, n1);
        if (s1_a != ch.a || s1_p != p) {
            __syncthreads();   // the previous item's reads of the slice are done
            load_s1(A, ch.a, p);
        }
        // ---- digits of gamma . x for the chunk's columns (l = token * ell + i)
        if (dig_q != q) {
            __syncthreads();   // earlier reads of the staging buffers and digits are done
            dig_q = q;
            const uint16_t *gsrc = A.gamma;
            int gld = P.M;
            if (P.stage_g) {
                if (g_a != ch.a) stage_gamma(A, ch.a);
                wait_gamma();
                gsrc = gs;
                gld = P.gpitch;
            }
            if (bmax_a != ch.a) {
                __syncthreads();   // earlier reads of the maximum are done
                if (tid == 0) ms->bmax = 0u;
                __syncthreads();
                beta_max(A, &ms->bmax);
                bmax_a = ch.a;
            }
            if (tid < kChunkCols) ms->amax[tid] = 0u;
            // tokens one at a time through the two x buffers
            const bool xbulk = (P.M * xsize) % 16 == 0;
            auto stage_token = [&](int tok, uint32_t seq) {
                unsigned char *dst = xbuf + (seq & 1u) * P.xs_bytes;
                const unsigned char *src =
                    static_cast<const unsigned char *>(P.x) + static_cast<int64_t>(ch.t0 + tok) * P.M * xsize;
                if (xbulk) {
                    if (tid == 0) {
                        fence_proxy_async();   // the buffer's earlier generic reads come first
                        bar_expect_tx(&ms->bar[3 + (seq & 1u)], static_cast<uint32_t>(P.M * xsize));
                        bulk_g2s(dst, src, static_cast<uint32_t>(P.M * xsize), &ms->bar[3 + (seq & 1u)]);
                    }
                } else {
                    for (int i = tid; i < P.M * xsize / 2; i += kThreads)
                        reinterpret_cast<uint16_t *>(dst)[i] = reinterpret_cast<const uint16_t *>(src)[i];
                }
            };
            const uint32_t x0 = n_x;
            stage_token(0, x0);
            if (ch.ntok > 1) stage_token(1, x0 + 1);
            const int nunits = groups_of(P.pitch1) * kGroupWords * 8;   // (word, mask) units of whole groups
#pragma unroll 1
            for (int tok = 0; tok < ch.ntok; ++tok) {
                const uint32_t seq = x0 + tok;
                if (xbulk) copy_wait(&ms->bar[3 + (seq & 1u)], (seq >> 1) & 1u, P.status);
                else __syncthreads();
                const unsigned char *xs = xbuf + (seq & 1u) * P.xs_bytes;
#pragma unroll 1
                for (int i = 0; i < ell; ++i) {
                    const int l = tok * ell + i;
                    const int sh = digit_column(gsrc + static_cast<int64_t>(i) * gld, xs, P.xd, P.M, nunits,
                                                dig + static_cast<size_t>(kDigits * l) * P.cb1, P.cb1, &ms->amax[l],
                                                &ms->wq[warp][l], &ms->wa[warp][l]);
                    if (tid == 0) ms->sh_u[l] = sh;
                }
                if (tok + 2 < ch.ntok) {
                    __syncthreads();   // every read of this token's buffer is done
                    stage_token(tok + 2, seq + 2);
                }
            }
            n_x = x0 + ch.ntok;
            __syncthreads();
            if (tid < cc) {
                long long sq = 0, sa = 0;
                for (int w = 0; w < kWarps; ++w) {
                    sq += ms->wq[w][tid];
                    sa += ms->wa[w][tid];
                }
                ms->qsum_u[tid] = sq;
                // |v_r| = |beta_r h_r| <= max|beta| sum|q| 2^-sh; the factor
                // covers the fp32 roundings of h and of beta h
                const float bound = __uint_as_float(ms->bmax) * scale_pow2(static_cast<float>(sa), -ms->sh_u[tid]) *
                                    (1.0f + 1.0f / 1024.0f);
                ms->sh_v[tid] = scale_exponent(bound);
            }
            if (!s2_issued && q == q_last1) issue_first_s2();
        }
        // ---- beta of the item's rows, the tile, then the sign sums
        if (r1_a != ch.a || r1_p != p) {
            __syncthreads();   // the previous item's reads of the rows are done
            load_r1(A, ch.a, p);
        }
        for (int i = tid; i < rows * P.tile_ld; i += kThreads) tile[i] = 0;
        if (s1_pending) {
            copy_wait(&ms->bar[0], n_s1 & 1u, P.status);
            ++n_s1;
            s1_pending = false;
        } else {
            __syncthreads();
        }
        if (n1 > 0)
            sign_sums(smem_u32(s1), P.stride1, rows / 16, groups_of(P.pitch1), smem_u32(dig), P.cb1, ndcol, tile,
                      P.tile_ld);
        __syncthreads();
        // ---- v = beta . h as digits into the image (stage-2 layout); sums of q of v per column
        const int pitch2 = static_cast<int>(pitch_words(A.R));
        int qv[kChunkCols];
#pragma unroll
        for (int c = 0; c < kChunkCols; ++c) qv[c] = 0;
#pragma unroll 1
        for (int i = tid; i < n1 * cc; i += kThreads) {
            const int l = i / n1, r = i - l * n1;
            const int tok = l / ell, env = l - tok * ell;
            const long long sm = digit_sum(tile + r * P.tile_ld, l);
            const float h = scale_pow2(__ll2float_rn(ms->qsum_u[l] - 2 * sm), -ms->sh_u[l]);
            const int qq = quantize(rs1[env * rows + r] * h, ms->sh_v[l]);
            const uint32_t db = digit_bytes(qq);
            const int64_t c = static_cast<int64_t>(ch.t0 + tok) * P.ell_cap + env;
            char *im = P.img + static_cast<size_t>(c) * kDigits * P.cb2 +
                       (P.word2 ? digit_offset_word(lo + r) : digit_offset(lo + r));
            im[0] = static_cast<char>(db & 255u);
            im[P.cb2] = static_cast<char>((db >> 8) & 255u);
            im[2 * P.cb2] = static_cast<char>(db >> 16);
#pragma unroll
            for (int c2 = 0; c2 < kChunkCols; ++c2)
                if (c2 == l) qv[c2] += qq;
        }
        // digits of v past the rank, to the end of the K words stage 2 reads,
        // are zero (whatever the padding bits of B1)
        if (lo + rows >= A.R) {
            const int tail = kwords2_of(P.word2, pitch2) * 32 - A.R;
#pragma unroll 1
            for (int i = tid; i < cc * tail; i += kThreads) {
                const int l = i / tail, k = A.R + (i - l * tail);
                const int tok = l / ell, env = l - tok * ell;
                const int64_t c = static_cast<int64_t>(ch.t0 + tok) * P.ell_cap + env;
                char *im = P.img + static_cast<size_t>(c) * kDigits * P.cb2 +
                           (P.word2 ? digit_offset_word(k) : digit_offset(k));
                im[0] = 0;
                im[P.cb2] = 0;
                im[2 * P.cb2] = 0;
            }
        }
#pragma unroll
        for (int l = 0; l < kChunkCols; ++l) {
            if (l < cc) {
                const long long w = warp_sum_exact(qv[l]);
                if (lane == 0) ms->wq[warp][l] = w;
            }
        }
        __syncthreads();
        if (tid < cc) {
            long long sum = 0;
            for (int w = 0; w < kWarps; ++w) sum += ms->wq[w][tid];
            const int tok = tid / ell, env = tid - tok * ell;
            const int64_t c = static_cast<int64_t>(ch.t0 + tok) * P.ell_cap + env;
            P.qpart[c * P.P1 + p] = sum;
            if (n1 > 0) P.sh2[c] = ms->sh_v[tid];   // the same value from every item of the chunk
        }
    }
    if (!s2_issued) issue_first_s2();
    wait_gamma();   // no copy left in flight

    // ---- every CTA's digits of v and its sums are written
    const bool passed = grid_sync(P, ms);
    if (!passed) {
        if (s2_pending) copy_wait(&ms->bar[1], n_s2 & 1u, P.status);   // no copy left in flight
        return;
    }

    // ================= stage 2 =================
    int img_q = -1;
    for (int it = it2b; it < it2e; ++it) {
        const int p = it / Q, q = it % Q;
        const Chunk ch = chunk_of(P, tab, q);
        int lo, rows, n2;
        range_of(P.N, P.P2, p, lo, rows, n2);
        if (ch.a < 0) {
            // no adapter: the branch is zero
            if (!(P.flags & DBF_ACCUMULATE)) {
                for (int i = tid; i < ch.ntok * n2; i += kThreads) {
                    const int tok = i / n2, r = i - tok * n2;
                    store_act(P.y, P.yd, static_cast<int64_t>(ch.t0 + tok) * P.N + lo + r, 0.f);
                }
            }
            continue;
        }
        const dbf_layer A = adapter_of(P, ch.a);
        const int ell = A.ell, cc = ch.ntok * ell, ndcol = kDigits * cc;
        const int pitch2 = static_cast<int>(pitch_words(A.R));
        if (s2_a != ch.a || s2_p != p) {
            __syncthreads();   // the previous item's reads of the slice are done
            load_s2(A, ch.a, p);
        }
        if (r2_a != ch.a || r2_p != p) {
            __syncthreads();   // the previous item's reads of the rows are done
            load_r2(A, ch.a, p);
        }
        // ---- the chunk's digits of v (coherent 16-byte loads: other CTAs wrote
        // them in this kernel), its sums of q and scales: the first round of
        // both kinds of loads is in flight together
        if (img_q != q) {
            __syncthreads();   // earlier reads of the digits are done
            img_q = q;
            const int n16 = kwords2_of(P.word2, pitch2) * 2;   // 16-byte units of one digit row
            const int nimg = ndcol * n16;
            auto img_unit = [&](int i) {
                const int dc = i / n16, k = i - dc * n16;
                const int l = dc / kDigits, d = dc - l * kDigits;
                const int tok = l / ell, env = l - tok * ell;
                const int64_t c = static_cast<int64_t>(ch.t0 + tok) * P.ell_cap + env;
                return reinterpret_cast<const uint4 *>(P.img + (static_cast<size_t>(c) * kDigits + d) * P.cb2) + k;
            };
            constexpr int kImg = 3, kPart = 6;
            uint4 iv[kImg];
#pragma unroll
            for (int e = 0; e < kImg; ++e) {
                const int i = tid + e * kThreads;
                iv[e] = i < nimg ? __ldcg(img_unit(i)) : make_uint4(0u, 0u, 0u, 0u);
            }
            long long pv[kPart];
            int64_t cw = 0;
            int shv = 0;
            if (warp < cc) {
                const int tok = warp / ell, env = warp - tok * ell;
                cw = static_cast<int64_t>(ch.t0 + tok) * P.ell_cap + env;
#pragma unroll
                for (int e = 0; e < kPart; ++e) {
                    const int k = lane + 32 * e;
                    pv[e] = k < P.P1 ? __ldcg(P.qpart + cw * P.P1 + k) : 0;
                }
                shv = __ldcg(P.sh2 + cw);
            }
#pragma unroll
            for (int e = 0; e < kImg; ++e) {
                const int i = tid + e * kThreads;
                if (i < nimg) reinterpret_cast<uint4 *>(dig + static_cast<size_t>(i / n16) * P.cb2)[i % n16] = iv[e];
            }
#pragma unroll 1
            for (int i = tid + kImg * kThreads; i < nimg; i += kThreads)
                reinterpret_cast<uint4 *>(dig + static_cast<size_t>(i / n16) * P.cb2)[i % n16] = __ldcg(img_unit(i));
            if (warp < cc) {
                long long sum = 0;
#pragma unroll
                for (int e = 0; e < kPart; ++e) sum += pv[e];
                for (int k = lane + 32 * kPart; k < P.P1; k += 32) sum += __ldcg(P.qpart + cw * P.P1 + k);
                sum = warp_sum_exact64(sum);
                if (lane == 0) {
                    ms->qsum_v[warp] = sum;
                    ms->sh_v[warp] = shv;
                }
            }
        }
        for (int i = tid; i < rows * P.tile_ld; i += kThreads) tile[i] = 0;
        if (s2_pending) {
            copy_wait(&ms->bar[1], n_s2 & 1u, P.status);
            ++n_s2;
            s2_pending = false;
        } else {
            __syncthreads();
        }
        if (n2 > 0) {
            if (P.word2)
                sign_sums_word(smem_u32(s2), stride2_of(true, pitch2), rows / 16, pitch2, smem_u32(dig), P.cb2, ndcol,
                               tile, P.tile_ld);
            else
                sign_sums(smem_u32(s2), stride2_of(false, pitch2), rows / 16, groups_of(pitch2), smem_u32(dig), P.cb2,
                          ndcol, tile, P.tile_ld);
        }
        __syncthreads();
        // ---- y = [acc] y + sum_i alpha_i . z_i, one (token, row) per thread
#pragma unroll 1
        for (int i = tid; i < ch.ntok * n2; i += kThreads) {
            const int tok = i / n2, r = i - tok * n2;
            const int64_t yi = static_cast<int64_t>(ch.t0 + tok) * P.N + lo + r;
            float yv = (P.flags & DBF_ACCUMULATE) ? load_act(P.y, P.yd, yi) : 0.f;
#pragma unroll 1
            for (int env = 0; env < ell; ++env) {
                const int l = tok * ell + env;
                const long long sm = digit_sum(tile + r * P.tile_ld, l);
                const float z = scale_pow2(__ll2float_rn(ms->qsum_v[l] - 2 * sm), -ms->sh_v[l]);
                yv += rs2[env * rows + r] * z;
            }
            store_act(P.y, P.yd, yi, yv);
        }
    }
}

// ---- host side ----------------------------------------------------------------

// Workspace: header | image of v | per-range sums of q | scale exponents.
// The per-range sums are sized for the largest number of row ranges any
// plan uses (one per 16-row block of the rank).
struct WsLayout {
    size_t img, qpart, sh2, total;
};

WsLayout ws_layout(int64_t cols, int max_R)
{
    WsLayout w;
    const int pitch2 = static_cast<int>(pitch_words(max_R));
    const int cb2 = cb2_of(word_layout(pitch2), pitch2);
    const int64_t nrb1 = (max_R + 15) / 16;
    w.img = kWsHeaderBytes;
    w.qpart = w.img + align_up(static_cast<size_t>(cols) * kDigits * cb2, 256);
    w.sh2 = w.qpart + align_up(static_cast<size_t>(cols) * nrb1 * sizeof(long long), 256);
    w.total = w.sh2 + align_up(static_cast<size_t>(cols) * sizeof(int32_t), 256);
    return w;
}

std::mutex g_coop_lock;
int g_coop_ok[64];   // per device: 0 unknown, 1 cooperative + PDL accepted, 2 refused

struct CallShape {
    int segmented;
    int M, N, max_R, ell_cap;
    int64_t T;
    int S;
    int xsize;   // bytes per activation (4 when unknown: the larger staging)
};

// Shared-memory offsets of a plan; returns the bytes.
size_t smem_layout(DecodeParams &P)
{
    const int ccmax = P.tpc * P.ell_cap;
    const int cbm = P.cb1 > P.cb2 ? P.cb1 : P.cb2;
    const size_t s1_bytes = static_cast<size_t>(P.rows1) * P.stride1 * 4;
    const size_t s2_bytes = static_cast<size_t>(P.rows2) * P.stride2 * 4;
    const size_t stage_bytes = static_cast<size_t>(P.stage_g ? P.gs_bytes : 0) + 2 * static_cast<size_t>(P.xs_bytes);
    size_t off = align_up(s1_bytes, 128);
    P.off_s2 = static_cast<int>(off);
    off = align_up(off + (s2_bytes > stage_bytes ? s2_bytes : stage_bytes), 128);
    P.off_dig = static_cast<int>(off);
    off = align_up(off + static_cast<size_t>(kDigits) * ccmax * cbm, 128);
    P.off_tile = static_cast<int>(off);
    const int rmax = P.rows1 > P.rows2 ? P.rows1 : P.rows2;
    P.tile_ld = 8 * ((kDigits * ccmax + 7) / 8) + 1;   // odd: the epilogue's row-per-lane reads hit distinct banks
    off = align_up(off + static_cast<size_t>(rmax) * P.tile_ld * 4, 16);
    P.off_misc = static_cast<int>(off);
    off = align_up(off + sizeof(Misc), 16);
    P.off_rs1 = static_cast<int>(off);
    off = align_up(off + static_cast<size_t>(P.rows1) * P.ell_cap * 4, 16);
    P.off_rs2 = static_cast<int>(off);
    off = align_up(off + static_cast<size_t>(P.rows2) * P.ell_cap * 4, 16);
    P.off_seg = static_cast<int>(off);
    if (P.segmented) off = align_up(off + static_cast<size_t>(4 * P.S + 1) * 4, 16);
    return off;
}

// Plan of one call; false when the call is outside the single launch's range
// (M above 8192, too many segments, or no plan fits in shared memory).
// Among the chunk sizes that fit, the one with the lowest estimated time is
// taken (digit build per column, MMAs at the tensor pipe's rate for
// mma.sync, a slice copy per extra item).
bool decode_plan(const CallShape &cs, int sms, DecodeParams *out, size_t *smem_out, int *grid_out)
{
    if (cs.T < 1 || cs.M < 1 || cs.N < 1 || cs.max_R < 1 || cs.ell_cap < 1 || cs.ell_cap > kChunkCols) return false;
    if (cs.M > kMaxM || cs.T > (1 << 28) / cs.ell_cap) return false;
    if (cs.segmented && (cs.S < 1 || cs.S > kMaxSegments)) return false;
    int G = sms < kMaxGrid ? sms : kMaxGrid;
    if (G < 1) G = 1;
    DecodeParams best{};
    size_t best_smem = 0;
    double best_cost = 1e30;
    const int nrb1 = (cs.max_R + 15) / 16, nrb2 = (cs.N + 15) / 16;
    for (int tpc = 1; tpc * cs.ell_cap <= kChunkCols; ++tpc) {
        DecodeParams P{};
        P.segmented = cs.segmented;
        P.S = cs.S;
        P.M = cs.M;
        P.N = cs.N;
        P.max_R = cs.max_R;
        P.ell_cap = cs.ell_cap;
        P.T = static_cast<int>(cs.T);
        P.tpc = tpc;
        P.pitch1 = static_cast<int>(pitch_words(cs.M));
        const int pitch2 = static_cast<int>(pitch_words(cs.max_R));
        P.stride1 = slice_stride(P.pitch1);
        P.word2 = word_layout(pitch2);
        P.stride2 = stride2_of(P.word2, pitch2);
        P.cb1 = col_bytes(P.pitch1);
        P.cb2 = cb2_of(P.word2, pitch2);
        P.gpitch = (cs.M + 7) / 8 * 8;
        P.gs_bytes = static_cast<int>(static_cast<size_t>(cs.ell_cap) * P.gpitch * 2);
        P.xs_bytes = static_cast<int>(align_up(static_cast<size_t>(cs.M) * cs.xsize, 16));
        const int64_t qest64 = cs.segmented ? std::min<int64_t>(cs.T, cs.S + cs.T / tpc) : (cs.T + tpc - 1) / tpc;
        const int Qest = static_cast<int>(qest64 < 1 ? 1 : qest64);
        if (static_cast<int64_t>(Qest) * std::max(nrb1, nrb2) > (int64_t{1} << 30)) continue;   // item indices fit int
        int P1 = Qest >= G ? 1 : std::max(1, std::min(nrb1, G / Qest));
        int P2 = Qest >= G ? 1 : std::max(1, std::min(nrb2, G / Qest));
        size_t smem = 0;
        bool fits = false;
        for (int attempt = 0; attempt < 64; ++attempt) {
            P.P1 = P1;
            P.P2 = P2;
            P.rows1 = (nrb1 + P1 - 1) / P1 * 16;
            P.rows2 = (nrb2 + P2 - 1) / P2 * 16;
            for (int sg = 1; sg >= 0; --sg) {
                P.stage_g = sg;
                smem = smem_layout(P);
                if (smem <= static_cast<size_t>(kSmemCap)) break;
            }
            if (smem <= static_cast<size_t>(kSmemCap)) {
                fits = true;
                break;
            }
            // halve the larger slice
            const size_t b1 = static_cast<size_t>(P.rows1) * P.stride1, b2 = static_cast<size_t>(P.rows2) * P.stride2;
            if (b1 >= b2 && P1 < nrb1) P1 = std::min(nrb1, P1 * 2);
            else if (P2 < nrb2) P2 = std::min(nrb2, P2 * 2);
            else if (P1 < nrb1) P1 = std::min(nrb1, P1 * 2);
            else break;
        }
        if (!fits) continue;
        // estimated microseconds of the busiest CTA
        const int cc = tpc * cs.ell_cap, ncg = (kDigits * cc + 7) / 8;
        const double mma_us = 17.5 / 4 / 1900.0;   // one m16n8k32 per sub-partition every 17.5 cycles
        const int ng1 = groups_of(P.pitch1), ng2 = groups_of(pitch2);
        const int64_t I1 = static_cast<int64_t>(Qest) * P.P1, I2 = static_cast<int64_t>(Qest) * P.P2;
        const double k1 = static_cast<double>((I1 + G - 1) / G), k2 = static_cast<double>((I2 + G - 1) / G);
        const double builds = std::min(k1, std::ceil(k1 / P.P1) + (P.P1 > 1 ? 1 : 0));
        const double c1 = builds * (0.3 + 0.55 * cc * cs.M / 4096.0) + (k1 - 1) * 1.0 +
                          k1 * (P.rows1 / 16) * ng1 * 8 * ncg * mma_us;
        const double mma2 = P.word2 ? pitch2 * 1.4 : ng2 * 8.0;   // per-word MMAs issue about 1.4x slower
        const double c2 = k2 * (0.3 + (P.rows2 / 16) * mma2 * ncg * mma_us) + (k2 - 1) * 1.0;
        const double cost = c1 + c2;
        if (cost < best_cost) {
            best_cost = cost;
            best = P;
            best_smem = smem;
        }
    }
    if (best_cost >= 1e29) return false;
    *out = best;
    *smem_out = best_smem;
    *grid_out = G;
    return true;
}

cudaError_t launch(DecodeParams &P, size_t smem, int G, cudaStream_t s)
{
    P.wait_ns = decode_wait_ns();
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(decode_multi_kernel), static_cast<int>(smem), true);
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
    e = cudaLaunchKernelEx(&cfg, decode_multi_kernel, P);
    if (e != cudaSuccess && coop) {
        // the cooperative attribute together with programmatic dependent
        // launch was refused: launch without it, the grid being no larger
        // than one CTA per SM with every SM able to hold one (checked here)
        (void)cudaGetLastError();
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_multi_kernel, kThreads, smem) != cudaSuccess ||
            per_sm < 1 || G > device_sms())
            return cudaErrorCooperativeLaunchTooLarge;
        if (dev >= 0 && dev < 64) {
            std::lock_guard<std::mutex> guard(g_coop_lock);
            g_coop_ok[dev] = 2;
        }
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, decode_multi_kernel, P);
    } else if (e == cudaSuccess && coop && dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> guard(g_coop_lock);
        g_coop_ok[dev] = 1;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

void set_workspace(DecodeParams &P, void *ws, int64_t cols)
{
    const WsLayout w = ws_layout(cols, P.max_R);
    char *base = static_cast<char *>(ws);
    P.sync = reinterpret_cast<unsigned long long *>(base);
    P.status = reinterpret_cast<int32_t *>(base + kWsStatusOffset);
    P.img = base + w.img;
    P.qpart = reinterpret_cast<long long *>(base + w.qpart);
    P.sh2 = reinterpret_cast<int32_t *>(base + w.sh2);
}

CallShape layer_shape(const dbf_layer &L, int64_t T, int xsize = 4) { return CallShape{0, L.M, L.N, L.R, L.ell, T, 1, xsize}; }

int act_bytes(dbf_dtype d) { return d == DBF_BF16 ? 2 : 4; }

}  // namespace

size_t multi_workspace_bytes(const dbf_layer &L, int64_t T)
{
    // independent of the plan (and so of the device): every call the single
    // launch may take gets its full layout
    if (T < 1 || L.M < 1 || L.M > kMaxM || L.R < 1 || L.ell < 1 || L.ell > kChunkCols) return 0;
    return ws_layout(T * L.ell, L.R).total;
}

bool multi_fits(const dbf_layer &L, int64_t T)
{
    DecodeParams P;
    size_t smem;
    int G;
    return decode_plan(layer_shape(L, T), device_sms(), &P, &smem, &G);
}

cudaError_t multi_forward(const dbf_layer &L, const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                           int flags, void *ws, cudaStream_t s)
{
    DecodeParams P;
    size_t smem;
    int G;
    if (!multi_fits(L, T) || !decode_plan(layer_shape(L, T, act_bytes(xd)), device_sms(), &P, &smem, &G))
        return cudaErrorInvalidValue;
    P.L = L;
    P.x = x;
    P.y = y;
    P.xd = xd;
    P.yd = yd;
    P.flags = flags;
    set_workspace(P, ws, T * L.ell);
    return launch(P, smem, G, s);
}

size_t multi_segmented_workspace_bytes(int32_t max_R, int32_t max_ell, int64_t T)
{
    if (max_R < 1 || max_ell < 1 || T < 0) return 0;
    return ws_layout(T * max_ell, max_R).total;
}

bool multi_segmented_fits(int32_t S, int32_t max_R, int32_t max_ell, int32_t M, int32_t N, int64_t T)
{
    DecodeParams P;
    size_t smem;
    int G;
    return decode_plan(CallShape{1, M, N, max_R, max_ell, T, S, 4}, device_sms(), &P, &smem, &G);
}

cudaError_t multi_forward_segmented(const dbf_layer *adapters, int32_t num_adapters, const int32_t *seg_off,
                                     const int32_t *seg_adp, int32_t S, int32_t max_R, int32_t max_ell, int32_t M,
                                     int32_t N, const void *x, dbf_dtype xd, void *y, dbf_dtype yd, int64_t T,
                                     int flags, void *ws, int32_t *status, cudaStream_t s)
{
    DecodeParams P;
    size_t smem;
    int G;
    if (!multi_segmented_fits(S, max_R, max_ell, M, N, T) ||
        !decode_plan(CallShape{1, M, N, max_R, max_ell, T, S, act_bytes(xd)}, device_sms(), &P, &smem, &G))
        return cudaErrorInvalidValue;
    P.adapters = adapters;
    P.num_adapters = num_adapters;
    P.seg_off = seg_off;
    P.seg_adp = seg_adp;
    P.seg_status = status;
    P.x = x;
    P.y = y;
    P.xd = xd;
    P.yd = yd;
    P.flags = flags;
    set_workspace(P, ws, T * max_ell);
    return launch(P, smem, G, s);
}

}  // namespace dbf
