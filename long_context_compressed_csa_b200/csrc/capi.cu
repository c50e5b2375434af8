// Status strings, version and workspace helpers of the C ABI.
#include "common.cuh"

extern "C" const char* csa_status_string(int status)
{
    switch (status) {
        case CSA_OK: return "CSA_OK";
        case CSA_ERR_ARG: return "CSA_ERR_ARG: null pointer, negative or inconsistent size";
        case CSA_ERR_ALIGN: return "CSA_ERR_ALIGN: pointer or stride not 16-byte aligned";
        case CSA_ERR_DTYPE: return "CSA_ERR_DTYPE: unknown dtype or output type";
        case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE: workspace missing or too small";
        case CSA_ERR_CUDA: return "CSA_ERR_CUDA: CUDA launch or runtime error";
        case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED: shape not implemented";
        case CSA_ERR_TIMEOUT: return "CSA_ERR_TIMEOUT: a bounded device-side wait gave up";
        default: return "CSA_ERR_UNKNOWN";
    }
}

extern "C" int csa_version(void) { return 100; }

extern "C" int csa_workspace_zero(void* workspace, size_t bytes, csa_stream_t stream)
{
    if (bytes == 0) return CSA_OK;
    if (!workspace) return CSA_ERR_ARG;
    cudaError_t e = cudaMemsetAsync(workspace, 0, bytes, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

namespace {
__global__ void store_i64(int64_t* p, int64_t v) { *p = v; }
}  // namespace

extern "C" int csa_workspace_set_wait_budget(void* workspace, int64_t cycles, csa_stream_t stream)
{
    if (!workspace || cycles < 0) return CSA_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return CSA_ERR_ALIGN;
    store_i64<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<int64_t*>(static_cast<char*>(workspace) + 8), cycles);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}
