// Internal interface of the attention kernels (split-KV partials + combine).
#pragma once
#include "common.cuh"

namespace csa {

constexpr int kMaxC = 512;        // widest compressed entry the kernels hold on chip
constexpr int kMaxSplits = 1024;  // splits per query the combine kernel accepts
constexpr int kCcHeads = 16;      // CUDA-core kernel: heads per CTA
constexpr int kCcChunk = 32;      // CUDA-core kernel: entries per shared-memory chunk
constexpr int kCombineThreads = 256;
constexpr int kCombineCols = 128;  // output columns per combine CTA

struct AttnArgs {
    const void* q;        // [G][n_h][c]
    const void* cache;    // [B][N_cap][c]
    const int32_t* idx;   // sparse: [G][k]
    const int64_t* t;     // dense: [G] query positions (device)
    int B, nq, n_h, c;
    int64_t N_cap;
    int k, m_prime;
    int dense;
    // sliding-window branch (win == null: none): window entries of tokens
    // max(0, t - n_win + 1) .. t (t from the array t above, also for the sparse path),
    // token p at row p % win_cap of win [B][win_cap][c]
    const void* win;
    int n_win, win_cap;
    float scale_log2;     // softmax scale * log2(e)
    int splits;
    int64_t per_split;    // list positions per split
    void* part_o;         // [G][splits][n_h][c]: fp32 O_i (CUDA-core path) or bf16 O_i / l_i (tcgen05 path)
    float2* part_ml;      // [G][splits][n_h] (max, sum) of 2^(scaled logit)
    // direct = 1 (tcgen05 path with one split per query): the split kernel writes the final
    // output out [G][n_h][c] (fp32, or bf16 when out_bf16) and lse [G][n_h] itself
    int direct;
    void* out;
    int out_bf16;
    float* lse;
};

struct AttnPlan {
    int splits = 1;
    int64_t per_split = 1;
    int head_groups = 1;
    int kernel = 0;  // 0: CUDA cores; 1: tcgen05, full-width splits (attn_tc.cu); 2: tcgen05 CTA pairs (attn_pair.cu)
};

AttnPlan attn_plan_cuda_core(int G, int n_h, int64_t entries);
AttnPlan attn_plan_tc(int G, int n_h, int c, int64_t entries);
bool attn_tc_supported(int n_h, int c);
size_t attn_ws_bytes(int G, int n_h, int c, int splits);
int launch_attn_tc(const AttnArgs& a, const AttnPlan& plan, uint32_t* status, cudaStream_t stream);
int launch_attn_pair(const AttnArgs& a, const AttnPlan& plan, uint32_t* status, cudaStream_t stream);
// normalized: part_o holds bf16 O_i / l_i (tcgen05 path) instead of fp32 O_i.
int launch_attn_combine(const AttnArgs& a, bool normalized, void* out, int out_bf16, float* lse,
                        cudaStream_t stream);

}  // namespace csa

extern "C" size_t csa_attn_workspace_size(int B, int nq, int n_h, int c, int64_t max_entries);
