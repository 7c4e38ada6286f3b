// Prefill-regime forward (tcgen05 tensor cores). Placeholder until the
// kernel lands: no shape is served, so DBF_PATH_AUTO takes the GEMV path.
#include "dbf_internal.cuh"

namespace dbf {
bool gemm_shape_ok(const dbf_layer &) { return false; }
size_t gemm_workspace_bytes(const dbf_layer &, int64_t) { return 0; }
cudaError_t gemm_forward(const dbf_layer &, const void *, dbf_dtype, void *, dbf_dtype, int64_t, int,
                         void *, cudaStream_t)
{
    return cudaErrorNotSupported;
}
}  // namespace dbf
