// Shared-KV MQA over compressed entries on the 5th-generation tensor cores
// ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch", section 8 sparse over the
// top-k entries, section 10 dense over all visible entries; key = value = entry).
//
// For one query, S = Q C^T (128 heads x entries, K = c = 512) and O = softmax(S) C
// (128 heads x 512) are dense contractions against entries shared by every head, so
// both run on tcgen05 with the heads as the M = 128 dimension.  The fp32 accumulator of
// O for all 512 columns would fill the whole 512-column TMEM, leaving no room for S,
// so a CTA owns one half of the output columns (N = 256) and recomputes S: work per
// entry is 1.5x the minimum, which is cheap next to the entry traffic.
//
// CTA = (split of the entry list, output half, query).  Entries stream through in
// chunks of 32 rows, gathered by index with 16-byte cp.async into a double-buffered
// 128-byte-swizzled tile; the same bytes serve as the K-major B operand of S and as
// the MN-major B operand of P C.
//   warps 0-3 loaders  : q (once) and the entry chunks -> shared memory
//   warps 4-7 softmax  : S rows from TMEM, online softmax with lazy rescaling (O is
//                        rescaled in TMEM only when the running max grows by > 2^8),
//                        P (bf16) -> shared memory; final O half -> partials
//   warp 8    MMA      : S(j+1) is issued before P(j) C so the tensor core keeps busy
// Partials (O unnormalised, running max and sum in base 2) are merged by the combine
// kernel of attn.cu.  Every barrier wait is bounded; a timeout sets the workspace
// status word and the CTA drains and exits.
#include "attn.cuh"
#include "tc_utils.cuh"

namespace csa {
namespace {

constexpr int kC = 512;             // entry width handled by this kernel
constexpr int kHalf = 256;          // output columns per CTA
constexpr int kHeads = 128;         // M
constexpr int kE = 32;              // entries per chunk (N of S)
constexpr int kLoaders = 128;
constexpr int kThreads = 288;       // 4 loader warps, 4 softmax warps, 1 MMA warp
constexpr int kQBytes = kHeads * kC * 2;          // 128 KB, 8 panels of 16 KB
constexpr int kCBytes = kE * kC * 2;              // 32 KB, 8 panels of 4 KB
constexpr int kPBytes = kHeads * 128;             // 16 KB (64 B of each 128 B row used)
constexpr int kMaxIds = 1024;                     // entry ids of a CTA's range staged in smem
constexpr int kSmem = 1024 + kQBytes + 2 * kCBytes + kPBytes + 256 + kMaxIds * 4;
constexpr float kRescaleThreshold = 8.0f;         // log2 units

CSA_DEV void cp_async16(uint32_t dst, const void* src, bool valid)
{
    const int n = valid ? 16 : 0;  // 0 bytes read -> 16 zero bytes written
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
CSA_DEV void cp_async_wait_all()
{
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(AttnArgs a, uint32_t* status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sC0 = sQ + kQBytes;  // chunk buffer `buf` at sC0 + buf * kCBytes
    uint8_t* sP = sQ + kQBytes + 2 * kCBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sP + kPBytes);
    uint64_t* Cfull = bars;        // [2] loaders -> MMA      (count 128)
    uint64_t* Cempty = bars + 2;   // [2] MMA commit -> loaders
    uint64_t* Sfull = bars + 4;    // [2] MMA commit -> softmax
    uint64_t* Sempty = bars + 6;   // [2] softmax -> MMA      (count 128)
    uint64_t* Pfull = bars + 8;    // softmax -> MMA          (count 128)
    uint64_t* PVdone = bars + 9;   // MMA commit -> softmax
    uint64_t* idsready = bars + 10; // loaders -> softmax: entry ids staged (count 128)
    uint64_t* staged = bars + 11;   // softmax warps: output half staged (count 128)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    int* s_ids = reinterpret_cast<int*>(sP + kPBytes + 256);  // [kMaxIds]

    pdl_launch_dependents();
    const int split = blockIdx.x, half = blockIdx.y, g = blockIdx.z;
    const int64_t b = g / a.nq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&Cfull[i], kLoaders);
            tc::mbar_init(&Cempty[i], 1);
            tc::mbar_init(&Sfull[i], 1);
            tc::mbar_init(&Sempty[i], kHeads);
        }
        tc::mbar_init(Pfull, kHeads);
        tc::mbar_init(PVdone, 1);
        tc::mbar_init(idsready, kLoaders);
        tc::mbar_init(staged, kHeads);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 8) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // only shared memory and TMEM were touched so far (overlaps the previous kernel)
    pdl_wait();
    int64_t count;
    if (a.dense) {
        const int64_t tt = a.t[g];
        const int64_t v = tt < 0 ? 0 : tt / a.m_prime;
        count = v < a.N_cap ? v : a.N_cap;
    } else {
        count = a.k;
    }
    const int64_t p_begin = (int64_t)split * a.per_split;
    const int64_t p_end = min(count, p_begin + a.per_split);
    const int nchunks = p_end > p_begin ? (int)((p_end - p_begin + kE - 1) / kE) : 0;
    const size_t prow = ((size_t)g * a.splits + split) * kHeads;  // partial row of head 0
    const __nv_bfloat16* cache = static_cast<const __nv_bfloat16*>(a.cache) + b * a.N_cap * kC;

    // entry id of list position p (-1: padding or outside the cache).  Sparse ranges of
    // up to kMaxIds positions are staged in shared memory once by the loaders, so the
    // gathers and the softmax masks make no dependent global loads per chunk.
    const bool ids_staged = !a.dense && (p_end - p_begin) <= kMaxIds;
    auto entry_global = [&](int64_t p) -> int64_t {
        if (p >= p_end) return -1;
        if (a.dense) return p;
        const int32_t v = __ldg(&a.idx[(int64_t)g * a.k + p]);
        return (v >= 0 && v < a.N_cap) ? v : -1;
    };
    auto entry_of = [&](int64_t p) -> int64_t {
        if (ids_staged) return p < p_end ? (int64_t)s_ids[p - p_begin] : -1;
        return entry_global(p);
    };

    if (nchunks == 0) {
        // empty range: an empty partial (max -inf, sum 0) that the combine skips
        if (half == 0 && threadIdx.x < kHeads) a.part_ml[prow + threadIdx.x] = make_float2(-INFINITY, 0.f);
    } else if (warp < 4) {
        // ------------------------------------------------------------ loaders
        const int lt = threadIdx.x;
        const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q) + (int64_t)g * kHeads * kC;
        const uint32_t q0 = tc::smem_u32(sQ);
        for (int i = lt; i < kHeads * (kC / 8); i += kLoaders) {
            const int row = i >> 6, cc = i & 63;
            cp_async16(q0 + (cc >> 3) * (kHeads * 128) + tc::sw128_offset(row, cc & 7), qg + row * kC + cc * 8, true);
        }
        if (ids_staged)
            for (int64_t i = lt; i < p_end - p_begin; i += kLoaders) s_ids[i] = (int)entry_global(p_begin + i);
        tc::mbar_arrive(idsready);
        asm volatile("bar.sync 2, 128;" ::: "memory");  // loader warps: ids visible to each other
        for (int j = 0; j < nchunks; ++j) {
            const int buf = j & 1;
            if (*abort_flag) break;
            if (!tc::mbar_wait(&Cempty[buf], ((j >> 1) & 1) ^ 1, tc::kWaitBudget)) {
                *abort_flag = 1;
                break;
            }
            const uint32_t c0 = tc::smem_u32(sC0 + buf * kCBytes);
            const int64_t p0 = p_begin + (int64_t)j * kE;
#pragma unroll 4
            for (int i = lt; i < kE * (kC / 8); i += kLoaders) {
                const int row = i >> 6, cc = i & 63;
                const int64_t e = entry_of(p0 + row);
                const __nv_bfloat16* src = cache + (e >= 0 ? e : 0) * kC + cc * 8;
                cp_async16(c0 + (cc >> 3) * (kE * 128) + tc::sw128_offset(row, cc & 7), src, e >= 0);
            }
            cp_async_wait_all();
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(&Cfull[buf]);
        }
        cp_async_wait_all();
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax
        const int quarter = warp & 3;
        const int h = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = tc::mbar_wait(idsready, 0, tc::kWaitBudget);
        for (int j = 0; j < nchunks && ok; ++j) {
            const int buf = j & 1;
            if (*abort_flag || !tc::mbar_wait(&Sfull[buf], (j >> 1) & 1, tc::kWaitBudget)) {
                *abort_flag = 1;
                ok = false;
                break;
            }
            tc::fence_after_sync();
            float s[kE];
            tc::tmem_ld16(tmem + lane_base + buf * kE, s);
            tc::tmem_ld16(tmem + lane_base + buf * kE + 16, s + 16);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            tc::mbar_arrive(&Sempty[buf]);
            const int64_t p0 = p_begin + (int64_t)j * kE;
            const unsigned vmask = __ballot_sync(0xffffffffu, entry_of(p0 + lane) >= 0);
            float cmax = -INFINITY;
#pragma unroll
            for (int e = 0; e < kE; ++e) {
                s[e] = ((vmask >> e) & 1u) ? s[e] * a.scale_log2 : -INFINITY;
                cmax = fmaxf(cmax, s[e]);
            }
            if (j > 0) {
                // P buffer and O are free once the previous chunk's P C has finished
                if (!tc::mbar_wait(PVdone, (j - 1) & 1, tc::kWaitBudget)) {
                    *abort_flag = 1;
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const bool need = cmax > m_run + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    const float f = need ? (m_run == -INFINITY ? 0.f : exp2f(m_run - cmax)) : 1.f;
                    const uint32_t ob = tmem + lane_base + kHalf;
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalf; c0 += 16) {
                        float o[16];
                        tc::tmem_ld16(ob + c0, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] *= f;
                        tc::tmem_st16(ob + c0, o);
                    }
                    tc::tmem_wait_st();
                    if (need) {
                        l_run *= f;
                        m_run = cmax;
                    }
                }
            } else {
                m_run = cmax;
            }
            float psum = 0.f;
            uint32_t packed[kE / 2];
#pragma unroll
            for (int e = 0; e < kE; e += 2) {
                const float p0f = (s[e] == -INFINITY) ? 0.f : exp2f(s[e] - m_run);
                const float p1f = (s[e + 1] == -INFINITY) ? 0.f : exp2f(s[e + 1] - m_run);
                psum += p0f + p1f;
                __nv_bfloat162 pr = __floats2bfloat162_rn(p0f, p1f);
                packed[e / 2] = *reinterpret_cast<uint32_t*>(&pr);
            }
            l_run += psum;
#pragma unroll
            for (int qc = 0; qc < kE / 8; ++qc) {
                uint4 v = make_uint4(packed[4 * qc], packed[4 * qc + 1], packed[4 * qc + 2], packed[4 * qc + 3]);
                *reinterpret_cast<uint4*>(sP + tc::sw128_offset(h, qc)) = v;
            }
            tc::fence_proxy_async_smem();
            tc::fence_before_sync();
            tc::mbar_arrive(Pfull);
        }
        if (ok && !*abort_flag && tc::mbar_wait(PVdone, (nchunks - 1) & 1, tc::kWaitBudget)) {
            tc::fence_after_sync();
            // The last P C has completed, so every MMA reading q has too: the q tile (128 KB)
            // is free and stages the 128 x 256 fp32 output half.  Rows are written with the
            // 16-byte units XOR-swizzled by (row & 7), then copied out row by row with
            // coalesced 16-byte stores (one thread per row would scatter 16 B pieces 1 KB
            // apart).
            float4* stage = reinterpret_cast<float4*>(sQ);  // [128 rows][64 float4]
            const uint32_t ob = tmem + lane_base + kHalf;
#pragma unroll 1
            for (int c0 = 0; c0 < kHalf; c0 += 16) {
                float o[16];
                tc::tmem_ld16(ob + c0, o);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; i += 4) {
                    const int q4 = (c0 + i) >> 2;
                    stage[h * 64 + (q4 ^ (h & 7))] = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
                }
            }
            if (half == 0) a.part_ml[prow + h] = make_float2(m_run, l_run);
            tc::mbar_arrive(staged);
            if (tc::mbar_wait(staged, 0, tc::kWaitBudget)) {
                const int st = threadIdx.x - 128;  // 0..127
                float* po = a.part_o + prow * a.c + half * kHalf;
#pragma unroll 4
                for (int i = st; i < kHeads * 64; i += 128) {
                    const int r = i >> 6, q4 = i & 63;
                    *reinterpret_cast<float4*>(po + (size_t)r * a.c + q4 * 4) = stage[r * 64 + (q4 ^ (r & 7))];
                }
            } else {
                *abort_flag = 1;
            }
        } else {
            tc::mbar_arrive(staged);
            *abort_flag = 1;
            if (half == 0) a.part_ml[prow + h] = make_float2(-INFINITY, 0.f);
        }
    } else {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescS = tc::idesc_bf16_f32(kHeads, kE, false, false);
            constexpr uint32_t kIdescPV = tc::idesc_bf16_f32(kHeads, kHalf, false, true);
            const uint32_t q0 = tc::smem_u32(sQ);
            const uint32_t p0 = tc::smem_u32(sP);
            auto issue_S = [&](int j) -> bool {
                const int buf = j & 1;
                if (!tc::mbar_wait(&Cfull[buf], (j >> 1) & 1, tc::kWaitBudget) ||
                    !tc::mbar_wait(&Sempty[buf], ((j >> 1) & 1) ^ 1, tc::kWaitBudget))
                    return false;
                tc::fence_after_sync();
                const uint32_t c0 = tc::smem_u32(sC0 + buf * kCBytes);
#pragma unroll
                for (int p = 0; p < kC / 64; ++p) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = tc::smem_desc_sw128(q0 + p * (kHeads * 128) + kk * 32, 16, 1024);
                        const uint64_t bd = tc::smem_desc_sw128(c0 + p * (kE * 128) + kk * 32, 16, 1024);
                        tc::mma_bf16_ss(tmem + buf * kE, ad, bd, kIdescS, (p | kk) ? 1u : 0u);
                    }
                }
                tc::mma_commit(&Sfull[buf]);
                return true;
            };
            bool ok = issue_S(0);
            for (int j = 0; j < nchunks && ok; ++j) {
                if (*abort_flag) break;
                if (j + 1 < nchunks && !issue_S(j + 1)) {
                    ok = false;
                    break;
                }
                if (!tc::mbar_wait(Pfull, j & 1, tc::kWaitBudget)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const int buf = j & 1;
                const uint32_t c0 = tc::smem_u32(sC0 + buf * kCBytes) + half * 4 * (kE * 128);
#pragma unroll
                for (int kk = 0; kk < kE / 16; ++kk) {
                    const uint64_t ad = tc::smem_desc_sw128(p0 + kk * 32, 16, 1024);
                    const uint64_t bd = tc::smem_desc_sw128(c0 + kk * 16 * 128, kE * 128, 1024);
                    tc::mma_bf16_ss(tmem + kHalf, ad, bd, kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc::mma_commit(&Cempty[buf]);
                tc::mma_commit(PVdone);
            }
            if (!ok) *abort_flag = 1;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) atomicExch(status, 1u);
    if (warp == 8) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

}  // namespace

bool attn_tc_supported(int n_h, int c) { return n_h == kHeads && c == kC; }

AttnPlan attn_plan_tc(int G, int n_h, int c, int64_t entries)
{
    (void)n_h;
    (void)c;
    AttnPlan p;
    const int64_t chunks = (entries + kE - 1) / kE;
    int64_t splits = kNumSMs / (2 * (int64_t)G);
    if (splits < 1) splits = 1;
    if (splits > chunks) splits = chunks;
    if (splits < 1) splits = 1;
    const int64_t per_chunks = (chunks + splits - 1) / splits;
    p.per_split = per_chunks * kE;
    if (p.per_split < kE) p.per_split = kE;
    p.splits = (int)((entries + p.per_split - 1) / p.per_split);
    if (p.splits < 1) p.splits = 1;
    p.head_groups = 1;
    return p;
}

int launch_attn_tc(const AttnArgs& a, const AttnPlan& plan, uint32_t* status, cudaStream_t stream)
{
    if (!aligned16(a.q) || !aligned16(a.cache)) return CSA_ERR_ALIGN;
    cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    dim3 grid((unsigned)plan.splits, 2u, (unsigned)(a.B * a.nq));
    launch_pdl(attn_tc_kernel, grid, dim3(kThreads), kSmem, stream, a, status);
    return launch_status();
}

}  // namespace csa
