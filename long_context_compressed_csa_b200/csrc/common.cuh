// Shared device helpers for the sm_100a CSA / HCA kernels (not part of the public ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/csa.h"

#define CSA_DEV __device__ __forceinline__

namespace csa {

constexpr int kNumSMs = 148;  // B200: 2 dies x 74 SMs
constexpr float kLog2e = 1.4426950408889634f;

// 16 bytes of one row: 8 bf16 or 4 fp32 elements, widened to fp32 in registers.
template <typename T>
struct Vec;

template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    CSA_DEV static void load(const __nv_bfloat16* p, float* f)
    {
        uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));  // streaming: read once
        unpack(u, f);
    }
    CSA_DEV static void load_cached(const __nv_bfloat16* p, float* f)
    {
        uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        unpack(u, f);
    }
    CSA_DEV static void unpack(uint4 u, float* f)
    {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    CSA_DEV static void store(__nv_bfloat16* p, const float* f)
    {
        uint4 u;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        u.x = w[0]; u.y = w[1]; u.z = w[2]; u.w = w[3];
        *reinterpret_cast<uint4*>(p) = u;
    }
};

template <>
struct Vec<float> {
    static constexpr int N = 4;
    CSA_DEV static void load(const float* p, float* f)
    {
        float4 v = __ldcs(reinterpret_cast<const float4*>(p));
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    }
    CSA_DEV static void load_cached(const float* p, float* f)
    {
        float4 v = __ldg(reinterpret_cast<const float4*>(p));
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    }
    CSA_DEV static void store(float* p, const float* f)
    {
        *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
    }
};

CSA_DEV float to_f32(float x) { return x; }
CSA_DEV float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
CSA_DEV T from_f32(float x);
template <>
CSA_DEV float from_f32<float>(float x) { return x; }
template <>
CSA_DEV __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Order-preserving map fp32 -> uint32 (larger float <-> larger key); -0 maps like +0.
CSA_DEV uint32_t order_key(float f)
{
    uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
CSA_DEV float key_to_float(uint32_t k)
{
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// Programmatic dependent launch: every kernel lets the next kernel in the stream start
// launching at once, and waits for the previous kernel's results (completion and memory
// visibility) before its first global-memory access.  Both are no-ops for a kernel that
// was launched without the attribute.
CSA_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
CSA_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch with programmatic stream serialisation, so the kernel's launch and prologue
// overlap the tail of the previous kernel on the stream.
template <typename... P, typename... A>
inline cudaError_t launch_pdl(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              A&&... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

// The same launch with thread-block clusters of two CTAs along x (CTA pairs).
inline void pair_launch_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute (&attr)[2], dim3 grid, dim3 block,
                               size_t smem, cudaStream_t stream)
{
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
}
template <typename... P, typename... A>
inline cudaError_t launch_pdl_pairs(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                    A&&... args)
{
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[2];
    pair_launch_config(cfg, attr, grid, block, smem, stream);
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}
// CTA pairs of `kern` that fit on the device at once (0 if none, or on error).
template <typename... P>
inline int max_resident_pairs(void (*kern)(P...), dim3 block, size_t smem)
{
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[2];
    pair_launch_config(cfg, attr, dim3(2), block, smem, nullptr);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline int elem_bytes(int dtype) { return dtype == CSA_BF16 ? 2 : 4; }

inline int launch_status()
{
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa
