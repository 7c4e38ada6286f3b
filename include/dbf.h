/*
 * dbf.h -- C ABI of the B200 (sm_100a) double-binary factorised layer forward.
 *
 * The operation (LoRDBA page, section 2 "Arquitetura Central", Delta-W
 * equation; DBF page, section 2, W ~ (a . A . m^T)(B . b^T) with ell = 1):
 *
 *   y[t,:] = [accumulate] y[t,:]
 *            + sum_{i=1..ell} diag(alpha_i) B1 diag(beta_i) B2 diag(gamma_i) x[t,:]
 *
 * with sign matrices B1 in {+-1}^{N x R} and B2 in {+-1}^{R x M} shared by
 * every envelope i, and fp16 per-channel scales alpha_i (N), beta_i (R),
 * gamma_i (M). Following the LoRDBA page's inference-kernel paragraph, it is
 * evaluated as two sign-accumulation products with per-channel scaling
 * between them: h = B2 (gamma . x), v = beta . h, z = B1 v, y += alpha . z.
 * The DBF_ACCUMULATE flag adds the branch into an existing output, the
 * unmerged adapter mode of the LoRDBA page (sections 1, 3 and 5); a
 * full-weight replacement layer (DBF page, section 2 "Inferencia") calls
 * without it.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every data pointer is a DEVICE pointer owned by the caller. The library
 *   allocates nothing, never synchronises the device and enqueues all work on
 *   'stream' (a cudaStream_t; NULL = the legacy default stream). The only
 *   device state that outlives a call is the workspace header described
 *   below, in memory the caller owns; host-side, the library caches per
 *   device the SM count and the kernel attributes it has set.
 * - Workspace header: every workspace (dbf_forward, dbf_backward,
 *   dbf_forward_segmented, dbf_forward_segmented_planned, dbf_mbok_forward)
 *   starts with DBF_WS_HEADER_BYTES bytes that must be zero before its first
 *   use (cudaMemsetAsync once after allocating it); the rest is scratch.
 *     bytes 0..7   the grid-barrier word of the single-launch decode kernel
 *                  (arrival count and epoch); every call leaves it valid for
 *                  the next, also when a wait timed out.
 *     bytes 8..11  int32 device status of the calls made on the workspace:
 *                  a kernel whose bounded wait expired (a grid barrier or a
 *                  pipeline stage not reached within its time limit) stores
 *                  DBF_ERR_TIMEOUT there, and the output of that call is
 *                  incomplete. The library never clears it: read it (and
 *                  zero it if wanted) by a copy once the calls are done.
 *   Calls that share a workspace must be ordered on the GPU (one stream, or
 *   events).
 * - Arguments are checked on the host before any launch; a failed check
 *   returns an error status and launches nothing. Data-dependent faults
 *   found by a kernel (NaN latents, bad segment tables) are reported through
 *   an optional device status word: the kernel stores the dbf_status code
 *   there; it is never cleared by the library.
 * - Matrices are row-major. x is T x M (token-major), y is T x N.
 * - Packed sign layout (one bit per weight; LoRDBA page section 2 storage
 *   efficiency, DBF page section 2): a rows x k sign matrix is stored as rows
 *   of ceil(k/32) little-endian 32-bit words with no other padding. In word w
 *   of a row, bit p (0 <= p < 16) holds column k = 32w + 2p and bit 16 + p
 *   holds column k = 32w + 2p + 1. A set bit is the sign -1, a clear bit +1.
 *   Bits past the last column are zero. B1 is packed along R (N rows of
 *   ceil(R/32) words), B2 along M (R rows of ceil(M/32) words), so both are
 *   packed along their contraction dimension.
 * - Scales are fp16 bit patterns, laid out [ell][len].
 */
#ifndef DBF_H_
#define DBF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DBF_OK = 0,
    DBF_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad enum, bad table */
    DBF_ERR_UNSUPPORTED = 2,   /* valid arguments the requested path cannot serve */
    DBF_ERR_ALIGNMENT = 3,     /* a pointer misses its required alignment */
    DBF_ERR_WORKSPACE = 4,     /* workspace null or smaller than *_workspace_bytes */
    DBF_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
    DBF_ERR_TIMEOUT = 6        /* a bounded device-side wait expired */
} dbf_status;

typedef enum { DBF_F32 = 0, DBF_BF16 = 1, DBF_F16 = 2, DBF_I8 = 3 } dbf_dtype;

#define DBF_WS_HEADER_BYTES 256
#define DBF_WS_STATUS_OFFSET 8

/* Flags of dbf_forward / dbf_forward_segmented (bitwise or).
 * DBF_ACCUMULATE: y += branch instead of y = branch.
 * DBF_WEIGHTS_STATIC: the caller promises that the layer's weights (the
 *   packed sign matrices and the alpha, beta, gamma scales) are not written
 *   by the work enqueued just before this call on the stream. The kernels
 *   are launched as programmatic dependents of the preceding kernel; with
 *   this flag they start reading weights before that kernel has finished
 *   (activations, the workspace, segment tables and every write still wait
 *   for it). Without it nothing is read early. */
enum { DBF_ACCUMULATE = 1, DBF_WEIGHTS_STATIC = 2 };

/* GEMV: the decode kernel (few tokens, bandwidth bound, any shape).
 * GEMM: the prefill kernel (tcgen05 tensor cores; needs M % 128 == 0 and
 *       R % 128 == 0; any N).
 * AUTO: GEMM when the shape allows it and T is at least
 *       dbf_gemm_min_tokens(L) (from measured time models of both paths on
 *       B200; about 13 tokens for a 4096 x 11008 layer at rank 5888, about 80
 *       at 4096 x 4096 rank 1024, never for small adapter ranks), else GEMV. */
typedef enum { DBF_PATH_AUTO = 0, DBF_PATH_GEMV = 1, DBF_PATH_GEMM = 2 } dbf_path;

/* One layer or adapter. All pointers are device pointers, caller owned.
 * b1_packed: N rows x ceil(R/32) words; b2_packed: R rows x ceil(M/32) words;
 * both 16-byte aligned. alpha: fp16 [ell][N]; beta: fp16 [ell][R];
 * gamma: fp16 [ell][M]; each 2-byte aligned. 1 <= ell <= 8. */
typedef struct {
    int32_t M, N, R, ell;
    const uint32_t *b1_packed;
    const uint32_t *b2_packed;
    const uint16_t *alpha;
    const uint16_t *beta;
    const uint16_t *gamma;
} dbf_layer;

/* Bytes of a packed rows x k sign matrix: rows * ceil(k/32) * 4. */
size_t dbf_packed_bytes(int64_t rows, int64_t k);

/* Pack a rows x k sign source into the packed layout (LoRDBA page, section 2
 * training pipeline step 2: B = sign(H)).
 * src: device, rows x k, row-major, dtype DBF_I8 (any value < 0 is -1, others
 *      +1), or DBF_F32 / DBF_BF16 / DBF_F16 latents H where H < 0 gives -1 and
 *      H >= 0 (including -0.0) gives +1.
 * dst: device, dbf_packed_bytes(rows, k) bytes, 4-byte aligned.
 * status_dev: optional device int32; a NaN latent stores DBF_ERR_INVALID_ARG
 *      there (its bit is packed as +1).
 * Errors: DBF_ERR_INVALID_ARG (null, rows or k <= 0, bad dtype, dst_bytes too
 *      small), DBF_ERR_ALIGNMENT, DBF_ERR_CUDA. */
dbf_status dbf_pack_signs(const void *src, dbf_dtype src_dtype, int64_t rows, int64_t k,
                          uint32_t *dst, size_t dst_bytes, int32_t *status_dev, void *stream);

/* Unpack to int8 +-1 (rows x k, row-major). Inverse of dbf_pack_signs on
 * sign matrices. Errors as dbf_pack_signs. */
dbf_status dbf_unpack_signs(const uint32_t *src, int64_t rows, int64_t k, int8_t *dst,
                            void *stream);

/* Transpose of a packed sign matrix: src is rows x k packed along k, dst
 * becomes k x rows packed along rows, in the same layout (bit set = -1,
 * pair-interleaved bits, zero padding). The backward (dbf_backward) needs
 * B1^T and B2^T in this form: its transposed contractions then read packed
 * rows like the forward does. Bit-exact; no arithmetic.
 * src, dst: device, 4-byte aligned; dst_bytes >= dbf_packed_bytes(k, rows).
 * Errors: DBF_ERR_INVALID_ARG, DBF_ERR_ALIGNMENT, DBF_ERR_CUDA. */
dbf_status dbf_transpose_signs(const uint32_t *src, int64_t rows, int64_t k, uint32_t *dst,
                               size_t dst_bytes, void *stream);

/* Straight-through estimator for latent weights H whose signs form a sign
 * matrix B = sign(H) (LoRDBA page, section 2, training pipeline: the signs
 * are trained through an STE; the pages do not give its surrogate, so the
 * caller picks it): dH = dB * s'(H), elementwise over count values, with
 *   tau > 0:  s(H) = tanh(H / tau), s'(H) = (1 - tanh^2(H / tau)) / tau;
 *   tau <= 0: s = identity clipped to |H| <= 1 (s' = 1 there, else 0).
 * dB: device fp32 (e.g. db1 or db2 of dbf_backward); H: device fp32, fp16 or
 * bf16, same shape; dH: device fp32, overwritten or added to with
 * flags = DBF_ACCUMULATE. Errors: DBF_ERR_INVALID_ARG (also tau NaN),
 * DBF_ERR_ALIGNMENT, DBF_ERR_CUDA. */
dbf_status dbf_ste_backward(const float *db, const void *h, dbf_dtype h_dtype, int64_t count, float tau,
                            float *dh, int flags, void *stream);

/* Sign-value-independent decomposition of a dense fp32 matrix X (n x m,
 * row-major): X ~ sign(X) . (s_out s_in^T), s_out s_in^T the best rank-1
 * approximation of |X|, split evenly between the two vectors (DBF page,
 * section 2: the SVID projection inside the factorisation; Multi-Boolean
 * Architectures page, section 2: a boolean kernel with its scales, and
 * successive extraction of further kernels from the residual). The rank-1
 * factor comes from at most `iters` power iterations from the all-positive
 * start: when m is a multiple of 4 and at most 12288 (the single-read path)
 * they stop early once two successive unit iterates agree to 1e-6 in every
 * element (the remaining iterations would move the result by less than that).
 * signs: device, packed sign(X) (bit set = -1, sign(0) = +1), n rows with
 *    signs_ld_words words each (>= ceil(m/32); a larger pitch places the
 *    kernel inside a wider packed matrix, e.g. one block of an MBOK layer).
 * s_out [n], s_in [m]: device fp16 outputs.
 * subtract != 0: X is replaced by the residual X - sign(X) . (s_out s_in^T)
 *    computed with the stored fp16 scales (the next kernel of a successive
 *    extraction); else X is only read.
 * scratch: dbf_svid_scratch_bytes(n, m, iters) bytes, 256-byte aligned.
 * Errors: DBF_ERR_INVALID_ARG, DBF_ERR_ALIGNMENT, DBF_ERR_WORKSPACE,
 *    DBF_ERR_CUDA. */
size_t dbf_svid_scratch_bytes(int64_t n, int64_t m, int32_t iters);
dbf_status dbf_svid(float *X, int64_t n, int64_t m, int32_t iters, int subtract, uint32_t *signs,
                    int64_t signs_ld_words, uint16_t *s_out, uint16_t *s_in, void *scratch,
                    size_t scratch_bytes, void *stream);

/* The number of power iterations (1 .. iters) that the last dbf_svid call
 * given this scratch, n, m and iters ran (it is kept in the scratch). A
 * synchronous device-to-host copy that waits for all work on the device: for
 * tests and measurement, not the hot path. Errors: DBF_ERR_INVALID_ARG,
 * DBF_ERR_ALIGNMENT (scratch not 256-byte aligned), DBF_ERR_CUDA. */
dbf_status dbf_svid_iterations(void *scratch, int64_t n, int64_t m, int32_t iters, int32_t *out);

/* Double binary factorisation of a dense fp32 weight W (n x m, row-major):
 * W ~ (a . A . mid^T)(B . b^T) with sign matrices A (n x k), B (k x m) and
 * scale vectors a [n], mid [k], b [m] (DBF page, section 2: the
 * factorisation by alternating minimisation with ADMM and the SVID
 * projection; the page gives no update formulas, and this is the plainest
 * reading, unweighted). With U = diag(a) A diag(m1), V = diag(m2) B diag(b),
 * mid = m1 . m2, each outer iteration runs admm_iters scaled-form ADMM steps
 * on U with V fixed,
 *     U <- (W V^T + rho (Z - L)) (V V^T + rho I)^-1,
 *     Z <- SVID(U + L),  L <- L + U - Z     (Z from the current U, L = 0),
 * the factor becoming Z, then the same on V with U fixed (operands
 * transposed); rho = rho_rel * trace(Gram) / k; SVID as in dbf_svid with
 * at most svid_iters power iterations.
 * W [n x m], U0 [n x k], V0 [k x m]: device fp32, row-major, read only; the
 *    start is the SVID projection of (U0, V0) (e.g. a truncated SVD split
 *    evenly, or any seeded matrices).
 * outer >= 0 (0 returns the projected start), admm_iters >= 1,
 *    1 <= svid_iters <= 1000, rho_rel > 0.
 * Outputs (device, caller-owned): a_signs = A packed (n rows of ceil(k/32)
 *    words), b_signs = B packed (k rows of ceil(m/32) words), fp16 alpha = a
 *    [n], beta = mid [k], gamma = b [m]: exactly a one-envelope dbf_layer
 *    with M = m, N = n, R = k (b1 = a_signs, b2 = b_signs).
 * objective: optional device fp32 [outer + 1]: |W - U V|_F of the projected
 *    start and after each outer iteration (fp32 scales; costs one n x m x k
 *    product per entry). NULL skips it.
 * ws: dbf_factorize_workspace_bytes(n, m, k, outer, svid_iters) bytes,
 *    256-byte aligned, scratch. Arithmetic is fp32: each product runs on the
 *    tensor cores as three TF32 products per operand pair (fp32
 *    accumulation; about 2^-20 relative per product, plus an accumulation
 *    bias of about K/8 units of 2^-24) when its operands' row pitches are
 *    multiples of 4 floats and its K is at least 32 (n, m and k multiples
 *    of 4 make every product qualify), else as fp32 FMA; the k x k inverse
 *    by an in-place blocked Gauss-Jordan sweep. A tensor-core wait that
 *    expires (1 s) makes alpha, beta and gamma NaN.
 * U0 and V0 must not be zero (a zero Gram matrix gives rho = 0 and NaN).
 * Errors: DBF_ERR_INVALID_ARG, DBF_ERR_ALIGNMENT, DBF_ERR_WORKSPACE,
 *    DBF_ERR_UNSUPPORTED (a dimension above 65535 * 32), DBF_ERR_CUDA. */
size_t dbf_factorize_workspace_bytes(int64_t n, int64_t m, int64_t k, int32_t outer, int32_t svid_iters);
dbf_status dbf_factorize(const float *W, int64_t n, int64_t m, int64_t k, const float *U0, const float *V0,
                         int32_t outer, int32_t admm_iters, int32_t svid_iters, float rho_rel,
                         uint32_t *a_signs, uint32_t *b_signs, uint16_t *alpha, uint16_t *beta,
                         uint16_t *gamma, float *objective, void *ws, size_t ws_bytes, void *stream);

/* Smallest T for which DBF_PATH_AUTO takes the GEMM path on layer L; -1
 * when it never does (shape outside the GEMM path, or the decode kernels
 * stay faster at any T) or L is malformed. Host only, no device access. */
int64_t dbf_gemm_min_tokens(const dbf_layer *L);

/* Workspace bytes dbf_forward needs for this layer, T and path (AUTO is
 * resolved as dbf_forward resolves it). Returns 0 for invalid input. */
size_t dbf_workspace_bytes(const dbf_layer *L, int64_t T, dbf_path path);

/* How many kernels one dbf_forward call with this layer, T and path
 * launches: 3 on the GEMM path (operand pre-pass, stage 1, stage 2); on the
 * GEMV path 1 when T * ell <= 8 and the call fits one pass (single-launch
 * kernel with a grid barrier), else 2. 0 for invalid input or T == 0. Host
 * only; it reads the device's SM count. */
int32_t dbf_forward_launches(const dbf_layer *L, int64_t T, dbf_path path);

/* The forward of one layer (host-side descriptor L).
 * x: device T x M, DBF_F32 or DBF_BF16, 16-byte aligned.
 * y: device T x N, DBF_F32 or DBF_BF16, 16-byte aligned; read first when
 *    flags has DBF_ACCUMULATE. Results are rounded to nearest-even into y's
 *    dtype.
 * flags: DBF_ACCUMULATE | DBF_WEIGHTS_STATIC (see above); other bits must be 0.
 * ws: device workspace of at least dbf_workspace_bytes(L, T, path) bytes,
 *    256-byte aligned, starting with the header described above (zero before
 *    first use; its status word reports device-side timeouts).
 * T == 0 is a no-op. Paths: the GEMV path runs one kernel when T * ell <= 8
 * and M, R <= 8192 (binary tensor-core products with a grid barrier, one CTA
 * per SM, launched cooperatively), else two. Numerics: the GEMV path turns
 * each activation column (gamma.x, then beta.h) into 22-bit fixed point with
 * one power-of-two scale per column and accumulates sign sums exactly in
 * integers (relative error about 2^-22 of the column's largest value per
 * element); the GEMM path rounds gamma.x and beta.h to fp16 operands
 * (|values| below 65504) and accumulates in fp32.
 * Errors: DBF_ERR_INVALID_ARG, DBF_ERR_ALIGNMENT, DBF_ERR_WORKSPACE,
 *    DBF_ERR_UNSUPPORTED (path GEMM on a shape it does not serve), DBF_ERR_CUDA. */
dbf_status dbf_forward(const dbf_layer *L, const void *x, dbf_dtype x_dtype, void *y,
                       dbf_dtype y_dtype, int64_t T, int flags, dbf_path path, void *ws,
                       size_t ws_bytes, void *stream);

/* Workspace bytes dbf_backward needs (0 for invalid input or a shape the
 * backward does not serve); with_sign_grads != 0 when db1 or db2 is wanted. */
size_t dbf_backward_workspace_bytes(const dbf_layer *L, int64_t T, int with_sign_grads);

/* Gradients of a loss through dbf_forward, given dy = dL/dy (LoRDBA page,
 * section 2, training pipeline: quantisation-aware training differentiates
 * this forward; the pages give no formula, these are the forward's
 * derivatives by the chain rule). With u_i = gamma_i.x, h_i = B2 u_i,
 * v_i = beta_i.h_i, z_i = B1 v_i, a_i = alpha_i.dy, g_i = B1^T a_i,
 * e_i = B2^T (beta_i.g_i), per token:
 *   dx      = sum_i gamma_i . e_i                     (T x M)
 *   dalpha_i = sum_t dy . z_i,  dbeta_i = sum_t g_i . h_i,
 *   dgamma_i = sum_t x . e_i                          ([ell][N], [ell][R], [ell][M])
 * Runs on the tensor cores as four sign GEMMs (needs M, N, R multiples of
 * 128; any T); u_i, alpha_i.dy, beta_i.h_i and beta_i.g_i are fp16 operands
 * (|values| below 65504; apply loss scaling to tiny dy), fp32 accumulation.
 * L: the layer (device pointers as in dbf_forward).
 * b1t_packed: B1^T (R x N, packed along N), b2t_packed: B2^T (M x R, packed
 *    along R), both from dbf_transpose_signs, 16-byte aligned.
 * x: T x M and dy: T x N, DBF_F32 or DBF_BF16, 16-byte aligned.
 * dx, dalpha, dbeta, dgamma: device fp32 outputs, each optional (NULL skips
 *    it; dalpha's GEMM and the dx/dgamma GEMM are skipped when not wanted).
 * db1 (N x R), db2 (R x M): optional fp32 gradients with respect to the sign
 *    matrices taken as real variables, dB1 = sum_{t,i} a_i v_i^T and
 *    dB2 = sum_{t,i} (beta_i.g_i) u_i^T: what a straight-through estimator
 *    passes to the latent weights (the estimator's own shape is the caller's;
 *    see dbf_ste_backward). Dense fp16 x fp16 tensor-core products over the
 *    tokens; they need a larger workspace (with_sign_grads).
 *    Every output is overwritten, or added to with flags = DBF_ACCUMULATE.
 * ws: dbf_backward_workspace_bytes(L, T) bytes, 256-byte aligned, header as
 *    in dbf_forward.
 * Errors: DBF_ERR_INVALID_ARG, DBF_ERR_ALIGNMENT, DBF_ERR_WORKSPACE,
 *    DBF_ERR_UNSUPPORTED (shape), DBF_ERR_CUDA. */
dbf_status dbf_backward(const dbf_layer *L, const uint32_t *b1t_packed, const uint32_t *b2t_packed,
                        const void *x, dbf_dtype x_dtype, const void *dy, dbf_dtype dy_dtype, int64_t T,
                        float *dx, float *dalpha, float *dbeta, float *dgamma, float *db1, float *db2,
                        int flags, void *ws, size_t ws_bytes, void *stream);

/* Segmented serving planned on the host (LoRDBA page, section 1: many
 * adapters served at once): the same routing as dbf_forward_segmented, but
 * the segment tables and adapter descriptors are HOST arrays, as a serving
 * scheduler that built the batch has them. Segments whose adapter is on a
 * shape the tensor-core GEMM serves (M, R multiples of 128) run as grouped
 * GEMM launches: adapters of equal (R, ell), up to 48 per launch, share one
 * pre-pass and two GEMM launches whose tiles cover all their segments. Other
 * segments run as their own dbf_forward (decode kernels). All on one stream
 * and one workspace; segments with adapter id -1 get a zero branch.
 * adapters_host: host array of num_adapters descriptors (device pointers
 *    inside), each with the given M and N. seg_offsets_host: host int32
 *    [S+1], nondecreasing within [0, T]; seg_adapter_host: host int32 [S],
 *    each in [-1, num_adapters). x, y, flags as in dbf_forward; every
 *    segment's rows must be 16-byte aligned (M and N times the element size
 *    multiples of 16 bytes, else DBF_ERR_ALIGNMENT).
 * ws: dbf_forward_segmented_planned_workspace_bytes bytes, 256-byte
 *    aligned, header as in dbf_forward.
 * Errors: DBF_ERR_INVALID_ARG (bad tables or descriptors, checked on the
 *    host before any launch), DBF_ERR_ALIGNMENT, DBF_ERR_WORKSPACE,
 *    DBF_ERR_CUDA. */
size_t dbf_forward_segmented_planned_workspace_bytes(const dbf_layer *adapters_host, int32_t num_adapters,
                                                     const int32_t *seg_offsets_host,
                                                     const int32_t *seg_adapter_host, int32_t S, int32_t M,
                                                     int32_t N, int64_t T);
dbf_status dbf_forward_segmented_planned(const dbf_layer *adapters_host, int32_t num_adapters,
                                         const int32_t *seg_offsets_host, const int32_t *seg_adapter_host,
                                         int32_t S, int32_t M, int32_t N, const void *x, dbf_dtype x_dtype,
                                         void *y, dbf_dtype y_dtype, int64_t T, int flags, void *ws,
                                         size_t ws_bytes, void *stream);

/* Multi-boolean-kernel layer (Multi-Boolean Architectures page, section 2):
 * W ~ sum_{k=1..K} W_bool^[k] . (s_out^[k] s_in^[k]^T), K boolean kernels
 * with per-kernel input and output scales; a single-stage sign contraction
 * (no rank-R intermediate), served by the same tensor-core GEMM. */
typedef struct {
    int32_t M, N, K;             /* in, out, number of boolean kernels (1 .. 64) */
    const uint32_t *w_packed;    /* N x (K M) signs packed along the K M columns: row n holds
                                    W^[1][n, :], ..., W^[K][n, :] side by side (bit set = -1) */
    const uint16_t *s_in;        /* fp16 [K][M] */
    const uint16_t *s_out;       /* fp16 [K][N] */
} dbf_mbok_layer;

/* Workspace bytes dbf_mbok_forward needs (0 for invalid input or a shape it
 * does not serve). */
size_t dbf_mbok_workspace_bytes(const dbf_mbok_layer *L, int64_t T);

/* y = [acc] y + sum_k s_out^[k] . (W^[k] (s_in^[k] . x)) for T tokens.
 * L: host descriptor of device arrays (w_packed 16-byte aligned; pack the
 *    N x (K M) int8 sign matrix with dbf_pack_signs). Needs M % 128 == 0.
 * x: T x M, y: T x N, DBF_F32 or DBF_BF16, 16-byte aligned; flags:
 *    DBF_ACCUMULATE or 0. Numerics: s_in . x rounded to fp16 operands,
 *    exact +-s_out fp16 sign operands, fp32 accumulation.
 * ws: dbf_mbok_workspace_bytes bytes, 256-byte aligned, header as in
 *    dbf_forward. Errors: DBF_ERR_INVALID_ARG, DBF_ERR_UNSUPPORTED,
 *    DBF_ERR_ALIGNMENT, DBF_ERR_WORKSPACE, DBF_ERR_CUDA. */
dbf_status dbf_mbok_forward(const dbf_mbok_layer *L, const void *x, dbf_dtype x_dtype, void *y,
                            dbf_dtype y_dtype, int64_t T, int flags, void *ws, size_t ws_bytes,
                            void *stream);

/* Workspace bytes dbf_forward_segmented needs. */
size_t dbf_segmented_workspace_bytes(int32_t max_R, int32_t max_ell, int64_t T);

/* Many adapters served in one call (LoRDBA page, section 1: multi-adapter
 * serving as in S-LoRA / Punica). Tokens are pre-sorted into S segments:
 * tokens seg_offsets_dev[s] .. seg_offsets_dev[s+1]-1 use adapter
 * seg_adapter_dev[s]. An adapter id of -1 means no adapter: those rows get a
 * zero branch (y is left as is when accumulating, else set to 0).
 * adapters_dev: device array of num_adapters dbf_layer descriptors, each with
 *    the given M and N, R <= max_R and ell <= max_ell (ell <= 8).
 * seg_offsets_dev: device int32 [S+1], nondecreasing, from 0 to T.
 * seg_adapter_dev: device int32 [S].
 * x, y, flags as in dbf_forward (decode-path numerics; DBF_WEIGHTS_STATIC
 *    has no effect here because the segment tables are read first).
 * status_dev: optional device int32. A segment whose adapter id is outside
 *    [-1, num_adapters) or whose descriptor does not match M, N, max_R,
 *    max_ell, or an offsets table that is not nondecreasing within [0, T],
 *    stores DBF_ERR_INVALID_ARG there and that segment is skipped.
 * Errors: as dbf_forward. */
dbf_status dbf_forward_segmented(const dbf_layer *adapters_dev, int32_t num_adapters,
                                 const int32_t *seg_offsets_dev, const int32_t *seg_adapter_dev,
                                 int32_t S, int32_t max_R, int32_t max_ell, int32_t M, int32_t N,
                                 const void *x, dbf_dtype x_dtype, void *y, dbf_dtype y_dtype,
                                 int64_t T, int flags, void *ws, size_t ws_bytes,
                                 int32_t *status_dev, void *stream);

/* Decode forward without a caller workspace. The papers have no counterpart
 * to this entry point; it exists for callers that cannot allocate device
 * memory (a framework or serving runtime that owns every allocation, or a
 * thread that must not call cudaMalloc because it may synchronise the device
 * or fail under a memory cap). It runs the same decode (GEMV) kernels as
 * dbf_forward with DBF_PATH_GEMV, taking its scratch memory from a fixed
 * 1 MiB device array inside the library (one copy on every GPU that loads
 * the library, held until the process exits). It allocates nothing and
 * calls no allocating routine.
 * Arguments as dbf_forward, without path and workspace.
 * Limit: the decode workspace of the call (dbf_workspace_bytes(L, T,
 * DBF_PATH_GEMV)) must be at most 1 MiB (1048576 bytes), else
 * DBF_ERR_WORKSPACE; that is ell*T <= 55 at R = 5888, M = 4096.
 * The first call on each device looks the array's device address up once
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture. Every call on a device shares the array and it
 * keeps the last call's contents; its workspace header (see dbf_forward)
 * starts at zero because the array is zero-initialised static storage, and
 * every call leaves it valid. Calls whose work overlaps on the GPU race on
 * the array and must be ordered by the caller. Errors: as dbf_forward, and
 * DBF_ERR_CUDA if the address lookup fails. */
dbf_status dbf_forward_decode_noalloc(const dbf_layer *L, const void *x, dbf_dtype x_dtype, void *y,
                                      dbf_dtype y_dtype, int64_t T, int flags, void *stream);

/* Reads the workspace header of the fixed array that
 * dbf_forward_decode_noalloc uses on the current device: the grid-barrier
 * word (arrival count in the low 32 bits, epoch in the high 32 bits) into
 * *barrier_word and the int32 device status into *status. A synchronous
 * device-to-host copy: it waits for all work on the device. For tests and
 * diagnosis (the count is zero between calls; the status holds
 * DBF_ERR_TIMEOUT after a call whose wait expired); not for the hot path.
 * Errors: DBF_ERR_INVALID_ARG for a null pointer, DBF_ERR_CUDA if the
 * address lookup or the copy fails. */
dbf_status dbf_debug_noalloc_header(uint64_t *barrier_word, int32_t *status);

/* The schedule dbf_forward's prefill path would use for layer *L (shapes
 * only: no pointer is read) and T tokens when 'pairs' CTA pairs can be
 * resident: tiles[0] stage-1 tiles, tiles[1] stage-2 tiles, tiles[2] of them
 * split in two halves of K; makespan[0] and makespan[1] the claim-order
 * model's makespans (in K steps) without and with those splits. Host only,
 * for tests of the model. DBF_ERR_UNSUPPORTED when the layer does not take
 * the one-launch forward (a stage under 32 K steps, or M or R not a multiple
 * of 128); DBF_ERR_INVALID_ARG for null pointers or non-positive sizes. */
dbf_status dbf_debug_fused_schedule(const dbf_layer *L, int64_t T, int32_t pairs, int32_t *tiles,
                                    double *makespan);

/* Time limit of the grid-barrier wait of the single-launch decode kernel
 * for the calls made after this one, in this process, counted from each
 * CTA's start and checked before every poll: ns > 0 sets it, 0 restores the
 * default of 2 s (its waits for its own weight copies always keep the
 * default). For tests of the timeout path: with a limit shorter than the time
 * a CTA takes to reach the barrier, every CTA but the last to arrive gives up, stores
 * DBF_ERR_TIMEOUT in the workspace status word and skip their share of stage
 * 2 (y is left incomplete); the workspace stays usable, and a later call with
 * the default limit is correct. Not for production use; not synchronised with
 * calls in flight on other host threads. */
void dbf_debug_set_decode_wait_ns(uint64_t ns);

/* Static description of a status code. */
const char *dbf_status_string(dbf_status s);

/* Library version string. */
const char *dbf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DBF_H_ */
