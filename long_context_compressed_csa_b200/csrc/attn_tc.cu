// tcgen05 attention (bf16): placeholder until the tensor-core kernel lands.
#include "attn.cuh"

namespace csa {

bool attn_tc_supported(int n_h, int c)
{
    (void)n_h;
    (void)c;
    return false;
}

AttnPlan attn_plan_tc(int G, int n_h, int c, int64_t entries)
{
    (void)c;
    return attn_plan_cuda_core(G, n_h, entries);
}

int launch_attn_tc(const AttnArgs&, const AttnPlan&, cudaStream_t) { return CSA_ERR_UNSUPPORTED; }

}  // namespace csa
