// tcgen05 indexer scan (bf16): placeholder until the tensor-core kernel lands.
#include "indexer.cuh"

namespace csa {

bool indexer_tc_supported(int n_hI, int cI)
{
    (void)n_hI;
    (void)cI;
    return false;
}

int launch_scan_tc(const void*, const float*, const void*, const int64_t*, int, int, int64_t,
                   int, int, int, int, const TopkWs&, cudaStream_t)
{
    return CSA_ERR_UNSUPPORTED;
}

}  // namespace csa
