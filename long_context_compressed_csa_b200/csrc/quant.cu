// Per-row E4M3 quantisation of indexer keys (csa_quantize_e4m3) and the E4M3 indexer
// entry point (csa_indexer_topk_e4m3).  Reading of the pages' low-precision indexer
// ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch", section 6.4: the indexer runs
// in FP4, which has the peak of FP8 on current hardware, section 12; no block-scale
// format is given): E4M3 codes with one fp32 scale per row, scale = max|x| / 448.
#include "e4m3.cuh"
#include "indexer.cuh"

namespace csa {
namespace {

constexpr int kQuantThreads = 256;  // 8 warps, one row per warp at a time

// One warp per row: the row's largest magnitude, its scale, then the codes.  cols is a
// multiple of 4; lanes own 4 consecutive columns at a time.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
quant_rows_e4m3(const T* __restrict__ x, int64_t rows, int cols, int64_t ld, uint8_t* __restrict__ codes,
                float* __restrict__ scales)
{
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kQuantThreads / 32);
    for (int64_t r = (int64_t)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
        const T* xr = x + r * ld;
        float amax = 0.f;
        for (int c = lane * 4; c < cols; c += 128)
#pragma unroll
            for (int u = 0; u < 4; ++u) amax = fmaxf(amax, fabsf(to_f32(xr[c + u])));
#pragma unroll
        for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float f = e4m3_factor(amax);
        for (int c = lane * 4; c < cols; c += 128) {
            const float a = to_f32(xr[c]), b = to_f32(xr[c + 1]), d = to_f32(xr[c + 2]), e = to_f32(xr[c + 3]);
            *reinterpret_cast<uint32_t*>(codes + r * cols + c) = e4m3x2(a, b, f) | (e4m3x2(d, e, f) << 16);
        }
        if (lane == 0) scales[r] = e4m3_scale(amax);
    }
}

// E2M1 codes of one row per warp: lanes own 8 consecutive columns (one 32-bit word of
// codes) at a time.  cols is a multiple of 8.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads)
quant_rows_e2m1(const T* __restrict__ x, int64_t rows, int cols, int64_t ld, uint8_t* __restrict__ codes,
                float* __restrict__ scales)
{
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kQuantThreads / 32);
    for (int64_t r = (int64_t)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
        const T* xr = x + r * ld;
        float amax = 0.f;
        for (int c = lane * 8; c < cols; c += 256)
#pragma unroll
            for (int u = 0; u < 8; ++u) amax = fmaxf(amax, fabsf(to_f32(xr[c + u])));
#pragma unroll
        for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float f = e2m1_factor(amax);
        for (int c = lane * 8; c < cols; c += 256) {
            uint32_t w = 0;
#pragma unroll
            for (int u = 0; u < 8; u += 2) w |= e2m1x2(to_f32(xr[c + u]), to_f32(xr[c + u + 1]), f) << (4 * u);
            *reinterpret_cast<uint32_t*>(codes + r * (cols / 2) + c / 2) = w;
        }
        if (lane == 0) scales[r] = e2m1_scale(amax);
    }
}

}  // namespace
}  // namespace csa

extern "C" int csa_quantize_e2m1(const void* x, int64_t rows, int cols, int64_t ld, void* codes, float* scales,
                                 int dtype, csa_stream_t stream_)
{
    using namespace csa;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (dtype != CSA_BF16 && dtype != CSA_F32) return CSA_ERR_DTYPE;
    if (rows < 0 || cols <= 0 || cols % 8 != 0 || ld < cols) return CSA_ERR_ARG;
    if (rows == 0) return CSA_OK;
    if (!x || !codes || !scales) return CSA_ERR_ARG;
    if (((uintptr_t)x & (uintptr_t)(elem_bytes(dtype) - 1)) || ((uintptr_t)codes & 3) || ((uintptr_t)scales & 3))
        return CSA_ERR_ALIGN;
    int64_t blocks = (rows + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
    if (blocks > 8 * kNumSMs) blocks = 8 * kNumSMs;
    if (dtype == CSA_BF16)
        launch_pdl(quant_rows_e2m1<__nv_bfloat16>, dim3((unsigned)blocks), dim3(kQuantThreads), 0, stream,
                   static_cast<const __nv_bfloat16*>(x), rows, cols, ld, static_cast<uint8_t*>(codes), scales);
    else
        launch_pdl(quant_rows_e2m1<float>, dim3((unsigned)blocks), dim3(kQuantThreads), 0, stream,
                   static_cast<const float*>(x), rows, cols, ld, static_cast<uint8_t*>(codes), scales);
    return launch_status();
}

extern "C" int csa_quantize_e4m3(const void* x, int64_t rows, int cols, int64_t ld, void* codes, float* scales,
                                 int dtype, csa_stream_t stream_)
{
    using namespace csa;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (dtype != CSA_BF16 && dtype != CSA_F32) return CSA_ERR_DTYPE;
    if (rows < 0 || cols <= 0 || cols % 4 != 0 || ld < cols) return CSA_ERR_ARG;
    if (rows == 0) return CSA_OK;
    if (!x || !codes || !scales) return CSA_ERR_ARG;
    if (((uintptr_t)x & (uintptr_t)(elem_bytes(dtype) - 1)) || ((uintptr_t)codes & 3) || ((uintptr_t)scales & 3))
        return CSA_ERR_ALIGN;
    int64_t blocks = (rows + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
    if (blocks > 8 * kNumSMs) blocks = 8 * kNumSMs;
    if (dtype == CSA_BF16)
        launch_pdl(quant_rows_e4m3<__nv_bfloat16>, dim3((unsigned)blocks), dim3(kQuantThreads), 0, stream,
                   static_cast<const __nv_bfloat16*>(x), rows, cols, ld, static_cast<uint8_t*>(codes), scales);
    else
        launch_pdl(quant_rows_e4m3<float>, dim3((unsigned)blocks), dim3(kQuantThreads), 0, stream,
                   static_cast<const float*>(x), rows, cols, ld, static_cast<uint8_t*>(codes), scales);
    return launch_status();
}

extern "C" int csa_indexer_topk_e4m3(const void* qI, const float* wI, const void* KI8, const float* KI_scale,
                                     const int64_t* t, int B, int nq, int64_t N_cap, int n_hI, int cI, int m,
                                     int k, int32_t* idx_out, float* scores_out, void* workspace,
                                     size_t ws_bytes, csa_stream_t stream_)
{
    using namespace csa;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (B < 0 || nq < 0 || N_cap < 0 || N_cap >= (int64_t(1) << 31) || n_hI <= 0 || cI <= 0 || m <= 0 || k <= 0)
        return CSA_ERR_ARG;
    if (!indexer_e4m3_supported(n_hI, cI)) return CSA_ERR_UNSUPPORTED;
    if (B == 0 || nq == 0) return CSA_OK;
    if ((int64_t)B * nq > 65535) return CSA_ERR_UNSUPPORTED;  // one grid row per query
    if (!qI || !wI || !KI8 || !KI_scale || !t || !idx_out) return CSA_ERR_ARG;
    if (((uintptr_t)wI & 3) || ((uintptr_t)KI_scale & 3) || ((uintptr_t)t & 7) || ((uintptr_t)idx_out & 3) ||
        ((uintptr_t)scores_out & 3) || !aligned16(workspace))
        return CSA_ERR_ALIGN;
    if (!workspace || ws_bytes < csa_indexer_topk_workspace_size(B, nq, N_cap, k)) return CSA_ERR_WORKSPACE;
    TopkWs ws = topk_ws_layout(workspace, B * nq, N_cap);
    bool fused = false;
    const int st = launch_scan_tc_e4m3(qI, wI, KI8, KI_scale, t, B, nq, N_cap, n_hI, cI, m, k, ws, idx_out,
                                       scores_out, &fused, stream);
    if (st != CSA_OK || fused) return st;
    return launch_topk_select(ws, t, B * nq, m, k, N_cap, idx_out, scores_out, stream);
}

extern "C" int csa_indexer_topk_e2m1(const void* qI, const float* wI, const void* KI4, const float* KI_scale,
                                     const int64_t* t, int B, int nq, int64_t N_cap, int n_hI, int cI, int m,
                                     int k, int32_t* idx_out, float* scores_out, void* workspace,
                                     size_t ws_bytes, csa_stream_t stream_)
{
    using namespace csa;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (B < 0 || nq < 0 || N_cap < 0 || N_cap >= (int64_t(1) << 31) || n_hI <= 0 || cI <= 0 || m <= 0 || k <= 0)
        return CSA_ERR_ARG;
    if (!indexer_e2m1_supported(n_hI, cI)) return CSA_ERR_UNSUPPORTED;
    if (B == 0 || nq == 0) return CSA_OK;
    if ((int64_t)B * nq > 65535) return CSA_ERR_UNSUPPORTED;  // one grid row per query
    if (!qI || !wI || !KI4 || !KI_scale || !t || !idx_out) return CSA_ERR_ARG;
    if (((uintptr_t)KI4 & 31) || !aligned16(qI) || ((uintptr_t)wI & 3) || ((uintptr_t)KI_scale & 3) ||
        ((uintptr_t)t & 7) || ((uintptr_t)idx_out & 3) || ((uintptr_t)scores_out & 3) || !aligned16(workspace))
        return CSA_ERR_ALIGN;
    if (!workspace || ws_bytes < csa_indexer_topk_workspace_size(B, nq, N_cap, k)) return CSA_ERR_WORKSPACE;
    TopkWs ws = topk_ws_layout(workspace, B * nq, N_cap);
    bool fused = false;
    const int st = launch_scan_tc_e2m1(qI, wI, KI4, KI_scale, t, B, nq, N_cap, n_hI, cI, m, k, ws, idx_out,
                                       scores_out, &fused, stream);
    if (st != CSA_OK || fused) return st;
    return launch_topk_select(ws, t, B * nq, m, k, N_cap, idx_out, scores_out, stream);
}
