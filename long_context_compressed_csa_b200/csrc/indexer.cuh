// Internal interface between the indexer scan kernels and the top-k select kernel.
#pragma once
#include "common.cuh"

namespace csa {

constexpr int kBins = 4096;  // 12-bit radix digits
// per query: [0] emitted, [1] candidates, [2] ticket, [3] arrivals at the first grid
// meeting of the in-place select, [4] at its second, [5] nonzero when the workspace needs a
// full reset (a timed-out wait or an aborted scan)
constexpr int kCtrs = 8;
constexpr int kCtrDirty = 5;

// Slot of a 12-bit digit in a 4096-bin histogram.  Bins are stored transposed
// ([16][256]) so that the threshold search, in which thread t reads the 16 consecutive
// bins 16u .. 16u + 15 (u = 255 - t), touches 32 different banks per warp access.
CSA_DEV uint32_t hist_slot(uint32_t bin) { return (bin & 15u) * 256u + (bin >> 4); }

// Workspace of csa_indexer_topk, carved from one caller buffer.
struct TopkWs {
    uint32_t* status; // 256-byte status block: word 0 the sticky device status (nonzero after
                      // a bounded wait timed out); bytes 8-15 an int64 wait budget (SM cycles)
                      // for the in-place select's grid meeting, 0 for the default
    uint32_t* hist0;  // [G][kBins] digit-0 histogram (zero between calls)
    uint32_t* ctr;    // [G][kCtrs] counters (zero between calls)
    float* scores;    // [G][ld] fp32 scores of the visible entries
    uint2* cand;      // [G][ld] (score key, index) candidates
    uint2* cand2;     // [G][ld] second candidate buffer
    int64_t ld;       // per-query stride of scores / cand (N_cap rounded up to 64)
    size_t bytes;     // total bytes used
    size_t zero_bytes;  // leading bytes that must be zero before a call
};

TopkWs topk_ws_layout(void* base, int G, int64_t N_cap);

bool indexer_tc_supported(int n_hI, int cI);
// tcgen05 scan; *fused is set when the scan kernel also performed the top-k select
// (idx_out / scores_out written), otherwise launch_topk_select must follow.
int launch_scan_tc(const void* qI, const float* wI, const void* KI, const int64_t* t, int B,
                   int nq, int64_t N_cap, int n_hI, int cI, int m, int k, const TopkWs& ws,
                   int32_t* idx_out, float* scores_out, bool* fused, cudaStream_t stream);
// E4M3 keys (k_scale: one fp32 scale per key) with bf16 queries quantised per head.
bool indexer_e4m3_supported(int n_hI, int cI);
int launch_scan_tc_e4m3(const void* qI, const float* wI, const void* KI8, const float* k_scale,
                        const int64_t* t, int B, int nq, int64_t N_cap, int n_hI, int cI, int m, int k,
                        const TopkWs& ws, int32_t* idx_out, float* scores_out, bool* fused,
                        cudaStream_t stream);
// E2M1 keys (two codes per byte, k_scale one fp32 scale per key) with bf16 queries
// quantised here per head to E4M3: kind::f8f6f4 with an E2M1 A operand, the codes
// unpacked by the TMA into the 16-byte-aligned layout that operand reads.
bool indexer_e2m1_supported(int n_hI, int cI);
int launch_scan_tc_e2m1(const void* qI, const float* wI, const void* KI4, const float* k_scale,
                        const int64_t* t, int B, int nq, int64_t N_cap, int n_hI, int cI, int m, int k,
                        const TopkWs& ws, int32_t* idx_out, float* scores_out, bool* fused,
                        cudaStream_t stream);
// Many queries of one batch row at once (chunked prefill): tcgen05 scores of a resident
// block of queries against streamed key tiles, into ws.scores; the stand-alone select
// with self_hist follows.
constexpr int kMqMinQueries = 16;
bool indexer_mq_eligible(const void* qI, const void* KI, int B, int nq, int64_t N_cap, int n_hI, int cI);
int launch_scan_mq(const void* qI, const float* wI, const void* KI, const int64_t* t, int B, int nq,
                   int64_t N_cap, int n_hI, int cI, int m, const TopkWs& ws, cudaStream_t stream);
int launch_scan_cuda_core(const void* qI, const float* wI, const void* KI, const int64_t* t,
                          int B, int nq, int64_t N_cap, int n_hI, int cI, int m, int k,
                          const TopkWs& ws, int dtype, cudaStream_t stream);
// Every error csa_indexer_topk reports before a launch (CSA_OK when the call may run).
int indexer_topk_check(const void* qI, const float* wI, const void* KI, const int64_t* t, int B, int nq,
                       int64_t N_cap, int n_hI, int cI, int m, int k, const int32_t* idx_out,
                       const float* scores_out, const void* workspace, size_t ws_bytes, int dtype);
// self_hist: one CTA per query, which builds the digit-0 histogram from the scores itself
// (after a scan that leaves ws.hist0 untouched).
int launch_topk_select(const TopkWs& ws, const int64_t* t, int G, int m, int k, int64_t N_cap,
                       int32_t* idx_out, float* scores_out, cudaStream_t stream, bool self_hist = false);

}  // namespace csa
