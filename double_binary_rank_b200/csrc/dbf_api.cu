// Host entry points of the C ABI declared in include/dbf.h: argument checks
// (no launch on a failed check), path choice and the workspace contract.
#include "dbf_internal.cuh"

#include <cmath>
#include <vector>

namespace {

using namespace dbf;


bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

dbf_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DBF_OK : DBF_ERR_CUDA; }

bool act_dtype_ok(dbf_dtype d) { return d == DBF_F32 || d == DBF_BF16; }

dbf_status check_layer(const dbf_layer *L)
{
    if (!L) return DBF_ERR_INVALID_ARG;
    if (L->M <= 0 || L->N <= 0 || L->R <= 0 || L->ell < 1 || L->ell > kMaxEll)
        return DBF_ERR_INVALID_ARG;
    if (!L->b1_packed || !L->b2_packed || !L->alpha || !L->beta || !L->gamma)
        return DBF_ERR_INVALID_ARG;
    if (!aligned(L->b1_packed, 16) || !aligned(L->b2_packed, 16) || !aligned(L->alpha, 2) ||
        !aligned(L->beta, 2) || !aligned(L->gamma, 2))
        return DBF_ERR_ALIGNMENT;
    return DBF_OK;
}

// Smallest T at which the tcgen05 GEMM path beats the decode kernels on
// this shape (INT64_MAX if it never does or the shape cannot take it), from
// two linear time models fit to B200 sweeps over T on four shapes:
//   decode:  15 us + 8.4e-8 us per sign-MAC of the call, T ell R (M + N);
//   GEMM:    65 us + 4.5e-7 us per packed sign bit R (M + N) (the expansion
//            of the weights into tiles) + the flops 2 T ell R (M + N) at
//            0.9 PFLOP/s.
int64_t gemm_min_tokens(const dbf_layer &L)
{
    if (!gemm_shape_ok(L)) return INT64_MAX;
    const double w = static_cast<double>(L.R) * (static_cast<double>(L.M) + L.N);
    const double per_tok_gemv = 8.4e-8 * L.ell * w, per_tok_gemm = 2.0 * L.ell * w / 9e8;
    if (per_tok_gemv <= per_tok_gemm) return INT64_MAX;
    const double t = (65.0 - 15.0 + 4.5e-7 * w) / (per_tok_gemv - per_tok_gemm);
    return t >= 9.0e18 ? INT64_MAX : static_cast<int64_t>(std::ceil(t));
}

// The path dbf_forward takes; DBF_PATH_GEMM only when the shape allows it.
dbf_path resolve(const dbf_layer &L, int64_t T, dbf_path p)
{
    if (p == DBF_PATH_AUTO) return T >= gemm_min_tokens(L) ? DBF_PATH_GEMM : DBF_PATH_GEMV;
    return p;
}

}  // namespace

extern "C" {

size_t dbf_packed_bytes(int64_t rows, int64_t k)
{
    if (rows <= 0 || k <= 0) return 0;
    return static_cast<size_t>(rows) * static_cast<size_t>(pitch_words(k)) * 4u;
}

dbf_status dbf_pack_signs(const void *src, dbf_dtype src_dtype, int64_t rows, int64_t k,
                          uint32_t *dst, size_t dst_bytes, int32_t *status_dev, void *stream)
{
    if (!src || !dst || rows <= 0 || k <= 0) return DBF_ERR_INVALID_ARG;
    if (src_dtype != DBF_I8 && src_dtype != DBF_F32 && src_dtype != DBF_BF16 && src_dtype != DBF_F16)
        return DBF_ERR_INVALID_ARG;
    if (dst_bytes < dbf_packed_bytes(rows, k)) return DBF_ERR_INVALID_ARG;
    const uintptr_t esz = src_dtype == DBF_I8 ? 1 : (src_dtype == DBF_F32 ? 4 : 2);
    if (!aligned(src, esz) || !aligned(dst, 4) || (status_dev && !aligned(status_dev, 4)))
        return DBF_ERR_ALIGNMENT;
    return from_cuda(launch_pack(src, src_dtype, rows, k, dst, status_dev,
                                 static_cast<cudaStream_t>(stream)));
}

dbf_status dbf_unpack_signs(const uint32_t *src, int64_t rows, int64_t k, int8_t *dst, void *stream)
{
    if (!src || !dst || rows <= 0 || k <= 0) return DBF_ERR_INVALID_ARG;
    if (!aligned(src, 4)) return DBF_ERR_ALIGNMENT;
    return from_cuda(launch_unpack(src, rows, k, dst, static_cast<cudaStream_t>(stream)));
}

dbf_status dbf_transpose_signs(const uint32_t *src, int64_t rows, int64_t k, uint32_t *dst, size_t dst_bytes,
                               void *stream)
{
    if (!src || !dst || rows <= 0 || k <= 0) return DBF_ERR_INVALID_ARG;
    if (dst_bytes < dbf_packed_bytes(k, rows)) return DBF_ERR_INVALID_ARG;
    if (!aligned(src, 4) || !aligned(dst, 4)) return DBF_ERR_ALIGNMENT;
    return from_cuda(launch_transpose(src, rows, k, dst, static_cast<cudaStream_t>(stream)));
}

dbf_status dbf_ste_backward(const float *db, const void *h, dbf_dtype h_dtype, int64_t count, float tau,
                            float *dh, int flags, void *stream)
{
    if (count < 0 || (h_dtype != DBF_F32 && h_dtype != DBF_F16 && h_dtype != DBF_BF16) ||
        (flags & ~DBF_ACCUMULATE) || !(tau == tau))
        return DBF_ERR_INVALID_ARG;
    if (count == 0) return DBF_OK;
    if (!db || !h || !dh) return DBF_ERR_INVALID_ARG;
    if (!aligned(db, 4) || !aligned(dh, 4) || !aligned(h, h_dtype == DBF_F32 ? 4 : 2)) return DBF_ERR_ALIGNMENT;
    return from_cuda(launch_ste(db, h, h_dtype, count, tau, dh, (flags & DBF_ACCUMULATE) ? 1 : 0,
                                static_cast<cudaStream_t>(stream)));
}

size_t dbf_svid_scratch_bytes(int64_t n, int64_t m, int32_t iters)
{
    if (n <= 0 || m <= 0 || iters < 1 || iters > 1000) return 0;
    return svid_scratch_bytes(n, m, iters);
}

dbf_status dbf_svid(float *X, int64_t n, int64_t m, int32_t iters, int subtract, uint32_t *signs,
                    int64_t signs_ld_words, uint16_t *s_out, uint16_t *s_in, void *scratch, size_t scratch_bytes,
                    void *stream)
{
    if (!X || !signs || !s_out || !s_in || n <= 0 || m <= 0 || iters < 1 || iters > 1000 ||
        signs_ld_words < pitch_words(m))
        return DBF_ERR_INVALID_ARG;
    if (!aligned(X, 4) || !aligned(signs, 4) || !aligned(s_out, 2) || !aligned(s_in, 2)) return DBF_ERR_ALIGNMENT;
    if (!scratch || scratch_bytes < svid_scratch_bytes(n, m, iters)) return DBF_ERR_WORKSPACE;
    if (!aligned(scratch, 256)) return DBF_ERR_ALIGNMENT;
    return from_cuda(svid_run(X, n, m, iters, subtract ? 1 : 0, signs, signs_ld_words, s_out, s_in, scratch,
                              static_cast<cudaStream_t>(stream)));
}

dbf_status dbf_svid_iterations(void *scratch, int64_t n, int64_t m, int32_t iters, int32_t *out)
{
    if (!scratch || !out || n <= 0 || m <= 0 || iters < 1 || iters > 1000) return DBF_ERR_INVALID_ARG;
    if (!aligned(scratch, 256)) return DBF_ERR_ALIGNMENT;
    return from_cuda(cudaMemcpy(out, svid_count_slot(scratch, n, m, iters), 4, cudaMemcpyDeviceToHost));
}

namespace {
constexpr int64_t kFactorMaxDim = int64_t(65535) * 32;   // transpose grids of 32-row tiles stay <= 65535

bool factor_args_ok(int64_t n, int64_t m, int64_t k, int32_t outer, int32_t svid_iters)
{
    return n > 0 && m > 0 && k > 0 && outer >= 0 && outer <= 100000 && svid_iters >= 1 && svid_iters <= 1000;
}
}  // namespace

size_t dbf_factorize_workspace_bytes(int64_t n, int64_t m, int64_t k, int32_t outer, int32_t svid_iters)
{
    if (!factor_args_ok(n, m, k, outer, svid_iters) || n > kFactorMaxDim || m > kFactorMaxDim || k > kFactorMaxDim)
        return 0;
    return factorize_workspace_bytes(n, m, k, outer, svid_iters);
}

dbf_status dbf_factorize(const float *W, int64_t n, int64_t m, int64_t k, const float *U0, const float *V0,
                         int32_t outer, int32_t admm_iters, int32_t svid_iters, float rho_rel, uint32_t *a_signs,
                         uint32_t *b_signs, uint16_t *alpha, uint16_t *beta, uint16_t *gamma, float *objective,
                         void *ws, size_t ws_bytes, void *stream)
{
    if (!W || !U0 || !V0 || !a_signs || !b_signs || !alpha || !beta || !gamma ||
        !factor_args_ok(n, m, k, outer, svid_iters) || admm_iters < 1 || admm_iters > 1000 ||
        !(rho_rel > 0.f) || !std::isfinite(rho_rel))
        return DBF_ERR_INVALID_ARG;
    if (n > kFactorMaxDim || m > kFactorMaxDim || k > kFactorMaxDim) return DBF_ERR_UNSUPPORTED;
    if (!aligned(W, 4) || !aligned(U0, 4) || !aligned(V0, 4) || !aligned(a_signs, 4) || !aligned(b_signs, 4) ||
        !aligned(alpha, 2) || !aligned(beta, 2) || !aligned(gamma, 2) || (objective && !aligned(objective, 4)))
        return DBF_ERR_ALIGNMENT;
    if (!ws || ws_bytes < factorize_workspace_bytes(n, m, k, outer, svid_iters)) return DBF_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return DBF_ERR_ALIGNMENT;
    return from_cuda(factorize_run(W, n, m, k, U0, V0, outer, admm_iters, svid_iters, rho_rel, a_signs, b_signs,
                                   alpha, beta, gamma, objective, ws, static_cast<cudaStream_t>(stream)));
}

int64_t dbf_gemm_min_tokens(const dbf_layer *L)
{
    if (!L || L->M <= 0 || L->N <= 0 || L->R <= 0 || L->ell < 1 || L->ell > kMaxEll) return -1;
    const int64_t t = gemm_min_tokens(*L);
    return t == INT64_MAX ? -1 : t;
}

void dbf_debug_set_decode_wait_ns(uint64_t ns) { set_decode_wait_ns(ns); }

size_t dbf_workspace_bytes(const dbf_layer *L, int64_t T, dbf_path path)
{
    if (!L || L->M <= 0 || L->N <= 0 || L->R <= 0 || L->ell < 1 || L->ell > kMaxEll || T < 0)
        return 0;
    if (path != DBF_PATH_AUTO && path != DBF_PATH_GEMV && path != DBF_PATH_GEMM) return 0;
    const dbf_path p = resolve(*L, T, path);
    if (p == DBF_PATH_GEMM) return gemm_shape_ok(*L) ? gemm_workspace_bytes(*L, T) : 0;
    return gemv_layer_workspace_bytes(*L, T);
}

int32_t dbf_forward_launches(const dbf_layer *L, int64_t T, dbf_path path)
{
    if (!L || L->M <= 0 || L->N <= 0 || L->R <= 0 || L->ell < 1 || L->ell > kMaxEll || T < 0)
        return 0;
    if (path != DBF_PATH_AUTO && path != DBF_PATH_GEMV && path != DBF_PATH_GEMM) return 0;
    if (T == 0) return 0;
    const dbf_path p = resolve(*L, T, path);
    if (p == DBF_PATH_GEMM) return gemm_shape_ok(*L) ? gemm_forward_launches(*L) : 0;
    return gemv_launches(*L, T);
}

dbf_status dbf_forward(const dbf_layer *L, const void *x, dbf_dtype x_dtype, void *y,
                       dbf_dtype y_dtype, int64_t T, int flags, dbf_path path, void *ws,
                       size_t ws_bytes, void *stream)
{
    dbf_status st = check_layer(L);
    if (st != DBF_OK) return st;
    if (T < 0 || !act_dtype_ok(x_dtype) || !act_dtype_ok(y_dtype)) return DBF_ERR_INVALID_ARG;
    if (flags & ~(DBF_ACCUMULATE | DBF_WEIGHTS_STATIC)) return DBF_ERR_INVALID_ARG;
    if (path != DBF_PATH_AUTO && path != DBF_PATH_GEMV && path != DBF_PATH_GEMM)
        return DBF_ERR_INVALID_ARG;
    if (T == 0) return DBF_OK;
    if (!x || !y) return DBF_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16)) return DBF_ERR_ALIGNMENT;
    const dbf_path p = resolve(*L, T, path);
    if (p == DBF_PATH_GEMM && !gemm_shape_ok(*L)) return DBF_ERR_UNSUPPORTED;
    const size_t need = dbf_workspace_bytes(L, T, p);
    if (need > 0 && (!ws || ws_bytes < need)) return DBF_ERR_WORKSPACE;
    if (ws && !aligned(ws, 256)) return DBF_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p == DBF_PATH_GEMM) return from_cuda(gemm_forward(*L, x, x_dtype, y, y_dtype, T, flags, ws, s));
    return from_cuda(gemv_forward(*L, x, x_dtype, y, y_dtype, T, flags, ws, s));
}

size_t dbf_backward_workspace_bytes(const dbf_layer *L, int64_t T, int with_sign_grads)
{
    if (!L || L->M <= 0 || L->N <= 0 || L->R <= 0 || L->ell < 1 || L->ell > kMaxEll || T < 0)
        return 0;
    if (!gemm_backward_shape_ok(*L)) return 0;
    return gemm_backward_workspace_bytes(*L, T, with_sign_grads != 0);
}

dbf_status dbf_backward(const dbf_layer *L, const uint32_t *b1t_packed, const uint32_t *b2t_packed,
                        const void *x, dbf_dtype x_dtype, const void *dy, dbf_dtype dy_dtype, int64_t T,
                        float *dx, float *dalpha, float *dbeta, float *dgamma, float *db1, float *db2,
                        int flags, void *ws, size_t ws_bytes, void *stream)
{
    dbf_status st = check_layer(L);
    if (st != DBF_OK) return st;
    if (T < 0 || !act_dtype_ok(x_dtype) || !act_dtype_ok(dy_dtype)) return DBF_ERR_INVALID_ARG;
    if (flags & ~DBF_ACCUMULATE) return DBF_ERR_INVALID_ARG;
    if (!gemm_backward_shape_ok(*L)) return DBF_ERR_UNSUPPORTED;
    if (T == 0) return DBF_OK;
    if (!b1t_packed || !b2t_packed || !x || !dy) return DBF_ERR_INVALID_ARG;
    if (!aligned(b1t_packed, 16) || !aligned(b2t_packed, 16) || !aligned(x, 16) || !aligned(dy, 16) ||
        (dbeta && !aligned(dbeta, 4)) || (dx && !aligned(dx, 4)) || (dalpha && !aligned(dalpha, 4)) ||
        (dgamma && !aligned(dgamma, 4)) || (db1 && !aligned(db1, 4)) || (db2 && !aligned(db2, 4)))
        return DBF_ERR_ALIGNMENT;
    const size_t need = gemm_backward_workspace_bytes(*L, T, db1 || db2);
    if (!ws || ws_bytes < need) return DBF_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return DBF_ERR_ALIGNMENT;
    return from_cuda(gemm_backward(*L, b1t_packed, b2t_packed, x, x_dtype, dy, dy_dtype, T, dx, dalpha, dbeta,
                                   dgamma, db1, db2, flags, ws, static_cast<cudaStream_t>(stream)));
}

// Host-planned segmented forward: validation shared by the size query and the call.
static dbf_status check_plan(const dbf_layer *adapters, int32_t num_adapters, const int32_t *offs,
                             const int32_t *ids, int32_t S, int32_t M, int32_t N, int64_t T)
{
    if (num_adapters < 0 || S < 0 || M <= 0 || N <= 0 || T < 0) return DBF_ERR_INVALID_ARG;
    if (S == 0) return DBF_OK;
    if (!offs || !ids || (num_adapters > 0 && !adapters)) return DBF_ERR_INVALID_ARG;
    if (offs[0] < 0 || offs[S] > T) return DBF_ERR_INVALID_ARG;
    for (int32_t q = 0; q < S; ++q) {
        if (offs[q + 1] < offs[q] || ids[q] < -1 || ids[q] >= num_adapters) return DBF_ERR_INVALID_ARG;
        if (ids[q] >= 0) {
            const dbf_status st = check_layer(&adapters[ids[q]]);
            if (st != DBF_OK) return st;
            if (adapters[ids[q]].M != M || adapters[ids[q]].N != N) return DBF_ERR_INVALID_ARG;
        }
    }
    return DBF_OK;
}

// Segments served by a grouped GEMM launch: an adapter on a shape the GEMM
// serves; they are grouped by (R, ell).
static bool grouped_ok(const dbf_layer &L) { return gemm_shape_ok(L); }

size_t dbf_forward_segmented_planned_workspace_bytes(const dbf_layer *adapters_host, int32_t num_adapters,
                                                     const int32_t *seg_offsets_host,
                                                     const int32_t *seg_adapter_host, int32_t S, int32_t M,
                                                     int32_t N, int64_t T)
{
    if (check_plan(adapters_host, num_adapters, seg_offsets_host, seg_adapter_host, S, M, N, T) != DBF_OK) return 0;
    size_t need = kWsHeaderBytes;
    for (int32_t q = 0; q < S; ++q) {
        const int64_t n = static_cast<int64_t>(seg_offsets_host[q + 1]) - seg_offsets_host[q];
        if (seg_adapter_host[q] < 0 || n <= 0) continue;
        const dbf_layer &L = adapters_host[seg_adapter_host[q]];
        // grouped: the pre-pass and v buffers span all T token rows
        const size_t b = grouped_ok(L) ? gemm_workspace_bytes(L, T) : dbf_workspace_bytes(&L, n, DBF_PATH_AUTO);
        if (b > need) need = b;
    }
    return need;
}

dbf_status dbf_forward_segmented_planned(const dbf_layer *adapters_host, int32_t num_adapters,
                                         const int32_t *seg_offsets_host, const int32_t *seg_adapter_host,
                                         int32_t S, int32_t M, int32_t N, const void *x, dbf_dtype x_dtype,
                                         void *y, dbf_dtype y_dtype, int64_t T, int flags, void *ws,
                                         size_t ws_bytes, void *stream)
{
    dbf_status st = check_plan(adapters_host, num_adapters, seg_offsets_host, seg_adapter_host, S, M, N, T);
    if (st != DBF_OK) return st;
    if (!act_dtype_ok(x_dtype) || !act_dtype_ok(y_dtype) || (flags & ~(DBF_ACCUMULATE | DBF_WEIGHTS_STATIC)))
        return DBF_ERR_INVALID_ARG;
    if (T == 0 || S == 0) return DBF_OK;
    if (!x || !y) return DBF_ERR_INVALID_ARG;
    const size_t xe = x_dtype == DBF_F32 ? 4 : 2, ye = y_dtype == DBF_F32 ? 4 : 2;
    // every segment's rows must start on a 16-byte boundary
    if (!aligned(x, 16) || !aligned(y, 16) || (static_cast<size_t>(M) * xe) % 16 || (static_cast<size_t>(N) * ye) % 16)
        return DBF_ERR_ALIGNMENT;
    const size_t need = dbf_forward_segmented_planned_workspace_bytes(adapters_host, num_adapters, seg_offsets_host,
                                                                      seg_adapter_host, S, M, N, T);
    if (!ws || ws_bytes < need) return DBF_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return DBF_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // adapters the GEMM serves: one grouped launch per (R, ell) class, up to
    // kMaxGroupsPerLaunch segments each
    std::vector<char> done(static_cast<size_t>(S), 0);
    for (int32_t q0 = 0; q0 < S; ++q0) {
        const int32_t a0 = seg_adapter_host[q0];
        if (done[q0] || a0 < 0 || seg_offsets_host[q0 + 1] <= seg_offsets_host[q0] || !grouped_ok(adapters_host[a0]))
            continue;
        const int R0 = adapters_host[a0].R, ell0 = adapters_host[a0].ell;
        std::vector<const dbf_layer *> ls;
        std::vector<int> offs, ns;
        for (int32_t q = q0; q < S; ++q) {
            const int32_t a = seg_adapter_host[q];
            if (done[q] || a < 0 || seg_offsets_host[q + 1] <= seg_offsets_host[q]) continue;
            const dbf_layer &L = adapters_host[a];
            if (!grouped_ok(L) || L.R != R0 || L.ell != ell0) continue;
            done[q] = 1;
            ls.push_back(&L);
            offs.push_back(seg_offsets_host[q]);
            ns.push_back(seg_offsets_host[q + 1] - seg_offsets_host[q]);
            if (static_cast<int>(ls.size()) == kMaxGroupsPerLaunch) {
                if (gemm_forward_grouped(ls.data(), offs.data(), ns.data(), static_cast<int>(ls.size()), x, x_dtype,
                                         y, y_dtype, T, flags, ws, s) != cudaSuccess)
                    return DBF_ERR_CUDA;
                ls.clear();
                offs.clear();
                ns.clear();
            }
        }
        if (!ls.empty() && gemm_forward_grouped(ls.data(), offs.data(), ns.data(), static_cast<int>(ls.size()), x,
                                                x_dtype, y, y_dtype, T, flags, ws, s) != cudaSuccess)
            return DBF_ERR_CUDA;
    }
    for (int32_t q = 0; q < S; ++q) {
        const int64_t off = seg_offsets_host[q], n = static_cast<int64_t>(seg_offsets_host[q + 1]) - off;
        if (n <= 0 || done[q]) continue;
        char *yq = static_cast<char *>(y) + off * N * ye;
        if (seg_adapter_host[q] < 0) {
            // no adapter: a zero branch
            if (!(flags & DBF_ACCUMULATE) && cudaMemsetAsync(yq, 0, static_cast<size_t>(n) * N * ye, s) != cudaSuccess)
                return DBF_ERR_CUDA;
            continue;
        }
        st = dbf_forward(&adapters_host[seg_adapter_host[q]], static_cast<const char *>(x) + off * M * xe, x_dtype, yq,
                         y_dtype, n, flags, DBF_PATH_AUTO, ws, ws_bytes, stream);
        if (st != DBF_OK) return st;
    }
    return DBF_OK;
}

size_t dbf_mbok_workspace_bytes(const dbf_mbok_layer *L, int64_t T)
{
    if (!L || T < 0 || !mbok_shape_ok(L->M, L->N, L->K)) return 0;
    return mbok_workspace_bytes(L->M, L->K, T);
}

dbf_status dbf_mbok_forward(const dbf_mbok_layer *L, const void *x, dbf_dtype x_dtype, void *y, dbf_dtype y_dtype,
                            int64_t T, int flags, void *ws, size_t ws_bytes, void *stream)
{
    if (!L || L->M <= 0 || L->N <= 0 || L->K < 1 || T < 0 || !act_dtype_ok(x_dtype) || !act_dtype_ok(y_dtype))
        return DBF_ERR_INVALID_ARG;
    if (flags & ~DBF_ACCUMULATE) return DBF_ERR_INVALID_ARG;
    if (!mbok_shape_ok(L->M, L->N, L->K)) return DBF_ERR_UNSUPPORTED;
    if (T == 0) return DBF_OK;
    if (!L->w_packed || !L->s_in || !L->s_out || !x || !y) return DBF_ERR_INVALID_ARG;
    if (!aligned(L->w_packed, 16) || !aligned(L->s_in, 2) || !aligned(L->s_out, 2) || !aligned(x, 16) ||
        !aligned(y, 16))
        return DBF_ERR_ALIGNMENT;
    if (!ws || ws_bytes < mbok_workspace_bytes(L->M, L->K, T)) return DBF_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return DBF_ERR_ALIGNMENT;
    return from_cuda(mbok_forward(L->M, L->N, L->K, L->w_packed, L->s_in, L->s_out, x, x_dtype, y, y_dtype, T,
                                  flags, ws, static_cast<cudaStream_t>(stream)));
}

size_t dbf_segmented_workspace_bytes(int32_t max_R, int32_t max_ell, int64_t T)
{
    if (max_R <= 0 || max_ell < 1 || max_ell > kMaxEll || T < 0) return 0;
    return gemv_workspace_bytes(max_R, max_ell, T);
}

dbf_status dbf_forward_segmented(const dbf_layer *adapters_dev, int32_t num_adapters,
                                 const int32_t *seg_offsets_dev, const int32_t *seg_adapter_dev,
                                 int32_t S, int32_t max_R, int32_t max_ell, int32_t M, int32_t N,
                                 const void *x, dbf_dtype x_dtype, void *y, dbf_dtype y_dtype,
                                 int64_t T, int flags, void *ws, size_t ws_bytes,
                                 int32_t *status_dev, void *stream)
{
    if (num_adapters < 0 || S < 0 || max_R <= 0 || max_ell < 1 || max_ell > kMaxEll || M <= 0 ||
        N <= 0 || T < 0 || !act_dtype_ok(x_dtype) || !act_dtype_ok(y_dtype) ||
        (flags & ~(DBF_ACCUMULATE | DBF_WEIGHTS_STATIC)))
        return DBF_ERR_INVALID_ARG;
    if (S > 65535) return DBF_ERR_UNSUPPORTED;
    if (T == 0 || S == 0) return DBF_OK;
    if (!seg_offsets_dev || !seg_adapter_dev || !x || !y || (num_adapters > 0 && !adapters_dev))
        return DBF_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(seg_offsets_dev, 4) ||
        !aligned(seg_adapter_dev, 4) || (adapters_dev && !aligned(adapters_dev, 8)) ||
        (status_dev && !aligned(status_dev, 4)))
        return DBF_ERR_ALIGNMENT;
    const size_t need = dbf_segmented_workspace_bytes(max_R, max_ell, T);
    if (!ws || ws_bytes < need) return DBF_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return DBF_ERR_ALIGNMENT;
    return from_cuda(gemv_forward_segmented(adapters_dev, num_adapters, seg_offsets_dev,
                                            seg_adapter_dev, S, max_R, max_ell, M, N, x, x_dtype,
                                            y, y_dtype, T, flags, ws, status_dev,
                                            static_cast<cudaStream_t>(stream)));
}

const char *dbf_status_string(dbf_status s)
{
    switch (s) {
    case DBF_OK: return "ok";
    case DBF_ERR_INVALID_ARG: return "invalid argument";
    case DBF_ERR_UNSUPPORTED: return "unsupported shape or path";
    case DBF_ERR_ALIGNMENT: return "misaligned pointer";
    case DBF_ERR_WORKSPACE: return "workspace missing or too small";
    case DBF_ERR_CUDA: return "CUDA error";
    case DBF_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

const char *dbf_version(void) { return "dbf-b200 0.1 (sm_100a)"; }

}  // extern "C"
