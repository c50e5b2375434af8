// Device helpers shared by the two tcgen05 attention kernels (attn_tc.cu: full-width
// splits; attn_pair.cu: CTA pairs splitting c): 16-byte gathers and the TMEM -> shared
// memory staging of an output half for its TMA stores.
#pragma once
#include "tc_utils.cuh"

namespace csa {
namespace atc {

constexpr int kC = 512;        // entry width handled by the tensor-core kernels
constexpr int kHalf = 256;     // output columns owned by each CTA of a split
constexpr int kHeads = 128;    // M: one query's heads
constexpr int kBoxCols = 64;             // one output box: 128 rows x 64 bf16 columns (128 B)
constexpr int kBoxBytes = kHeads * 128;  // 16 KB
constexpr float kRescaleThreshold = 8.0f;  // lazy O rescaling, log2 units

CSA_DEV void cp_async16(uint32_t dst, const void* src, bool valid)
{
    const int n = valid ? 16 : 0;  // 0 bytes read -> 16 zero bytes written
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
CSA_DEV void cp_async_wait_all() { asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory"); }
CSA_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
CSA_DEV void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }  // all but the newest group

// Copy columns [col0, col0 + ncols) of row h of the output half from TMEM (o_taddr: this
// warp's lane quarter, first O column), scaled by inv = 1 / l, into the staging boxes as
// bf16: four 128-row x 64-column boxes in the 128-byte swizzled layout of the output
// tensor map.  The TMEM loads of a row are issued two at a time before one wait.
CSA_DEV void stage_o_cols(uint8_t* stage, uint32_t o_taddr, int h, int col0, float inv, int ncols)
{
#pragma unroll 1
    for (int c0 = col0; c0 < col0 + ncols; c0 += 32) {
        uint32_t r[32];
        tc::tmem_ld32_async(o_taddr + c0, r);
        tc::tmem_wait_ld_regs(r);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
            w[i] = *reinterpret_cast<uint32_t*>(&pr);
        }
        uint8_t* row = stage + (c0 / kBoxCols) * kBoxBytes + h * 128;
        const int q0 = (c0 % kBoxCols) / 8;  // 16-byte chunk of the 128-byte box row
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(row + (((q0 + i) ^ (h & 7)) << 4)) =
                make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
}

// The same for an fp32 output: eight 128-row x 32-column boxes (128 B rows).
CSA_DEV void stage_o_cols_f32(uint8_t* stage, uint32_t o_taddr, int h, int col0, float inv, int ncols)
{
#pragma unroll 1
    for (int c0 = col0; c0 < col0 + ncols; c0 += 32) {
        uint32_t r[32];
        tc::tmem_ld32_async(o_taddr + c0, r);
        tc::tmem_wait_ld_regs(r);
        uint8_t* row = stage + (c0 / 32) * kBoxBytes + h * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            *reinterpret_cast<float4*>(row + ((i ^ (h & 7)) << 4)) =
                make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                            __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv);
    }
}

}  // namespace atc
}  // namespace csa
