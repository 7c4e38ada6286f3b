// Decode forward for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device memory for a workspace: code
// running inside a framework that owns every allocation (a graph executor or
// a serving runtime with a fixed memory plan), or a host thread that must not
// call cudaMalloc because cudaMalloc may synchronise the device or fail under
// a memory cap. For them this file provides one entry point that runs the
// decode (GEMV) forward with its scratch memory taken from a fixed device
// array compiled into the library instead of from a caller workspace.
//
// The array is a file-scope __device__ object of kNoallocScratchBytes bytes;
// every GPU that loads this library holds one copy until the process exits.
// Host code cannot use the array's name as a device address, so on the first
// call on each device (with that device current) the entry point looks the
// address up once with cudaGetSymbolAddress and keeps it. That first call
// should therefore come before any stream capture.
//
// All calls on a device share the one array and it keeps whatever the last
// call left in it. Only its first bytes, the workspace header that holds the
// single-launch decode kernel's barrier counter, must start at zero; static
// device storage is zero-initialised and every call leaves the header valid.
// Every other location the decode kernels read is written earlier by the same
// call. Calls whose work overlaps on the GPU (different streams, or work that
// runs concurrently) race on the array; callers must order them.
#include "dbf_internal.cuh"

#include <cstring>
#include <mutex>

namespace dbf {
namespace {

constexpr size_t kNoallocScratchBytes = 1u << 20;   // 1 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_lock;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool is_aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace dbf

extern "C" {

dbf_status dbf_forward_decode_noalloc(const dbf_layer *L, const void *x, dbf_dtype x_dtype, void *y,
                                      dbf_dtype y_dtype, int64_t T, int flags, void *stream)
{
    using namespace dbf;
    if (!L || L->M <= 0 || L->N <= 0 || L->R <= 0 || L->ell < 1 || L->ell > kMaxEll) return DBF_ERR_INVALID_ARG;
    if (!L->b1_packed || !L->b2_packed || !L->alpha || !L->beta || !L->gamma) return DBF_ERR_INVALID_ARG;
    if (!is_aligned(L->b1_packed, 16) || !is_aligned(L->b2_packed, 16) || !is_aligned(L->alpha, 2) ||
        !is_aligned(L->beta, 2) || !is_aligned(L->gamma, 2))
        return DBF_ERR_ALIGNMENT;
    if (T < 0 || (x_dtype != DBF_F32 && x_dtype != DBF_BF16) || (y_dtype != DBF_F32 && y_dtype != DBF_BF16))
        return DBF_ERR_INVALID_ARG;
    if (flags & ~(DBF_ACCUMULATE | DBF_WEIGHTS_STATIC)) return DBF_ERR_INVALID_ARG;
    if (T == 0) return DBF_OK;
    if (!x || !y) return DBF_ERR_INVALID_ARG;
    if (!is_aligned(x, 16) || !is_aligned(y, 16)) return DBF_ERR_ALIGNMENT;
    // the fixed scratch must hold this call's decode workspace
    if (gemv_layer_workspace_bytes(*L, T) > kNoallocScratchBytes) return DBF_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return DBF_ERR_CUDA;
    return gemv_forward(*L, x, x_dtype, y, y_dtype, T, flags, scratch, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? DBF_OK
               : DBF_ERR_CUDA;
}

dbf_status dbf_debug_noalloc_header(uint64_t *barrier_word, int32_t *status)
{
    using namespace dbf;
    if (!barrier_word || !status) return DBF_ERR_INVALID_ARG;
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return DBF_ERR_CUDA;
    unsigned char h[kWsStatusOffset + sizeof(int32_t)];
    if (cudaMemcpy(h, scratch, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return DBF_ERR_CUDA;
    std::memcpy(barrier_word, h, sizeof(uint64_t));
    std::memcpy(status, h + kWsStatusOffset, sizeof(int32_t));
    return DBF_OK;
}

}  // extern "C"
