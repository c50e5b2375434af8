// csa_indexer_topk without a caller-provided workspace.
//
// Some callers have no way to obtain device memory for scratch: a serving engine that
// reserved all of HBM up front for its own cache pool and hands kernels no allocator,
// a foreign-language plugin that only receives tensor pointers, or a latency-critical
// path that must not pay for an allocation.  This entry point lets them run the indexer
// and top-k with scratch that already lives in the library: a fixed, file-scope device
// array.  It computes exactly what csa_indexer_topk computes, by calling it.
#include <mutex>

#include "indexer.cuh"

namespace csa {
namespace {

// 8 MiB per GPU, resident from the moment the library's device code is loaded on that
// GPU until the process exits.  Holds the indexer workspace (status word, histograms,
// counters, fp32 scores and candidate lists: about 20 B per compressed entry per query
// plus 33 KB per query).
constexpr size_t kScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_indexer_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices];  // device address of g_indexer_scratch, per device

// Device address of the scratch array on the current device.  In host code the array's
// name is only a host-side handle, so the address is looked up once per device (with
// that device current) and cached.
int scratch_address(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return CSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_indexer_scratch) != cudaSuccess || !p) return CSA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return CSA_OK;
}

}  // namespace
}  // namespace csa

extern "C" int csa_indexer_topk_noalloc(const void* qI, const float* wI, const void* KI,
                                        const int64_t* t, int B, int nq, int64_t N_cap, int n_hI,
                                        int cI, int m, int k, int32_t* idx_out, float* scores_out,
                                        int dtype, csa_stream_t stream)
{
    using namespace csa;
    if (B < 0 || nq < 0 || N_cap < 0 || N_cap >= (int64_t(1) << 31)) return CSA_ERR_ARG;
    if (B == 0 || nq == 0) return CSA_OK;
    if ((int64_t)B * nq > 65535) return CSA_ERR_UNSUPPORTED;  // before any size arithmetic
    const size_t need = csa_indexer_topk_workspace_size(B, nq, N_cap, k);
    if (need == 0 || need > kScratchBytes) return CSA_ERR_WORKSPACE;  // beyond the fixed scratch
    void* scratch = nullptr;
    int st = scratch_address(&scratch);
    if (st != CSA_OK) return st;
    // Every argument error is reported here, before anything is enqueued on the stream.
    st = indexer_topk_check(qI, wI, KI, t, B, nq, N_cap, n_hI, cI, m, k, idx_out, scores_out, scratch,
                            kScratchBytes, dtype);
    if (st != CSA_OK) return st;
    // The array keeps whatever the previous call left; the histograms, counters and the
    // status word (which a previous call's timeout may have set) must start at zero.
    const size_t zero = topk_ws_layout(nullptr, B * nq, N_cap).zero_bytes;
    if (cudaMemsetAsync(scratch, 0, zero, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return CSA_ERR_CUDA;
    return csa_indexer_topk(qI, wI, KI, t, B, nq, N_cap, n_hI, cI, m, k, idx_out, scores_out, scratch,
                            kScratchBytes, dtype, stream);
}

extern "C" int csa_indexer_topk_noalloc_status(csa_stream_t stream)
{
    using namespace csa;
    void* scratch = nullptr;
    const int st = scratch_address(&scratch);
    if (st != CSA_OK) return st;
    uint32_t word = 0;  // the status word: the first 4 bytes of the scratch
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return CSA_ERR_CUDA;
    return word ? CSA_ERR_TIMEOUT : CSA_OK;
}
