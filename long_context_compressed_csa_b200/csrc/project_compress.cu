// Fused HCA projection + compression on tcgen05 ("DeepSeek-V4 Hybrid Attention: CSA and
// HCA from Scratch", section 10: one KV stream C = H W^KV and its pooling logits
// Z = H W^Z, then the boxed per-column softmax over the m' = 128 tokens of an entry and
// the weighted sum; section 3 states the projections H W for the CSA streams).
//
// The projections are a dense GEMM over the model width d, and the pooling only needs,
// per output column, the 128 values of C and Z of one entry.  The products are computed
// transposed, columns on the MMA M dimension and tokens on N:
//   D_C[j, r] = sum_k W_C[j, k] H[r, k],   D_Z[j, r] = sum_k W_Z[j, k] H[r, k]
// so that TMEM lane j holds a whole entry's C and Z values of column j and the softmax
// over the entry's tokens runs inside one thread, with no cross-thread reduction.
//
//   warp 0    TMA producer: per 64-wide K panel, a 128 x 64 tile of W_C and of W_Z and
//             a 256 x 64 tile of H (two entries' tokens), 128-byte swizzle, into a ring;
//   warp 1    MMA issuer: M = 128 columns, N = 256 tokens, K = 16, two accumulators
//             (C in TMEM columns 0-255, Z in 256-511);
//   warps 2-9 epilogue: thread = column of one of the tile's two entries (warps 2-5 the
//             first, 6-9 the second); an online softmax over the entry's 128 tokens (32
//             at a time from TMEM), then one bf16 entry value.
// CTAs are persistent over tiles (token block, column block) with the column blocks of
// one token block consecutive, so the CTAs running at the same time share H tiles in L2.
// C and Z never leave the chip.  Every wait is bounded; a timeout sets the workspace
// status word and every role drains and exits.
#include "common.cuh"
#include "tc_utils.cuh"
#include "cluster.cuh"

namespace csa {
namespace {

constexpr int kPcThreads = 320;                  // TMA warp, MMA warp, 8 epilogue warps
constexpr int kPcCols = 128;                     // output columns per tile (MMA M)
constexpr int kPcMp = 128;                       // tokens per entry (m')
constexpr int kPcTokens = 2 * kPcMp;             // tokens per tile (MMA N): two entries
constexpr int kPcWBytes = kPcCols * 128;         // one 128 x 64 weight panel: 16 KB
constexpr int kPcHBytes = kPcTokens * 128;       // one 256 x 64 H panel: 32 KB
constexpr int kPcStage = 2 * kPcWBytes + kPcHBytes;  // 64 KB
constexpr int kPcStages = 3;
constexpr int kPcSmem = 1024 + kPcStages * kPcStage + 256;
static_assert((2 * kPcStages + 3) * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit 256 bytes");

struct PcArgs {
    int64_t rows_per_batch;  // H rows of one batch in the buffer (ld_batch / ld_row)
    int64_t tok0;            // token of buffer row 0 of each batch
    int d;                   // model width (K)
    int c;                   // output columns
    const float* bias;       // [m'][c] or null
    __nv_bfloat16* out;      // entry i of batch b at out + b * out_ld_batch + i * c
    int64_t out_ld_batch;
    int64_t e0, e1;          // entries [e0, e1) of every batch
    int n_cb;                // column blocks of 128
    int64_t n_tb;            // token blocks (two entries) per batch
    int64_t tiles;           // B * n_tb * n_cb
    uint32_t* status;
};

CSA_DEV void pc_tile(const PcArgs& a, int64_t t, int& b, int64_t& tb, int& cb)
{
    cb = (int)(t % a.n_cb);
    const int64_t r = t / a.n_cb;
    tb = r % a.n_tb;
    b = (int)(r / a.n_tb);
}

// One HCA entry for one epilogue thread (TMEM lane = output column j): the online
// softmax over the entry's 128 tokens, 32 at a time from TMEM (Z at column offset
// kPcTokens), in base-2 logit units so that every exponential is one ex2 of the
// multi-function unit (relative error about 2^-22, far inside the entry's bf16 rounding).
CSA_DEV float hca_entry(uint32_t taddr_entry, const float* bias, int c, int j, bool use_bias)
{
    constexpr float kLog2e = 1.4426950408889634f;
    float m = -INFINITY, l = 0.f, acc = 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < kPcMp; c0 += 32) {
        uint32_t zr[32], cr[32];
        tc::tmem_ld32_async(taddr_entry + kPcTokens + c0, zr);
        tc::tmem_ld32_async(taddr_entry + c0, cr);
        tc::tmem_wait_ld_regs(zr);
        tc::tmem_wait_ld_regs(cr);
        float z[32];
        float cmax = -INFINITY;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const float b = use_bias ? __ldg(&bias[(int64_t)(c0 + u) * c + j]) : 0.f;
            z[u] = (__uint_as_float(zr[u]) + b) * kLog2e;
            cmax = fmaxf(cmax, z[u]);
        }
        const float mn = fmaxf(m, cmax);
        const float f = tc::ex2_approx(m - mn);  // 0 on the first chunk (m = -inf)
        l *= f;
        acc *= f;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
            const float p = tc::ex2_approx(z[u] - mn);
            l += p;
            acc = fmaf(p, __uint_as_float(cr[u]), acc);
        }
        m = mn;
    }
    return acc * tc::rcp_approx(l);
}

__global__ void __launch_bounds__(kPcThreads, 1)
hca_project_compress_kernel(const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ CUtensorMap tmap_wc,
                            const __grid_constant__ CUtensorMap tmap_wz, PcArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned; an offset from the __shared__ array keeps every derived pointer in
    // the shared window, so its accesses compile to shared-memory instructions
    uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPcStages * kPcStage);
    uint64_t* empty = full + kPcStages;
    uint64_t* tfull = empty + kPcStages;   // MMA -> epilogue: the tile's accumulators are complete
    uint64_t* tempty = tfull + 1;          // epilogue -> MMA: TMEM read out (count 128)
    uint64_t* done = tempty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kPcStages; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        tc::mbar_init(tfull, 1);
        tc::mbar_init(tempty, kPcThreads - 64);
        tc::mbar_init(done, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tmap_h);
        tc::tma_prefetch_desc(&tmap_wc);
        tc::tma_prefetch_desc(&tmap_wz);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();

    const int kpanels = a.d / 64;
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int it = 0;
            bool stop = false;
            for (int64_t t = blockIdx.x; t < a.tiles && !stop; t += gridDim.x) {
                int b, cb;
                int64_t tb;
                pc_tile(a, t, b, tb, cb);
                const int hrow = (int)(b * a.rows_per_batch + kPcMp * (a.e0 + 2 * tb) - a.tok0);
                const int wrow = cb * kPcCols;
                for (int kp = 0; kp < kpanels; ++kp, ++it) {
                    const int s = it % kPcStages;
                    const uint32_t ph = (it / kPcStages) & 1;
                    if (*abort_flag || !tc::mbar_wait(&empty[s], ph ^ 1, tc::kWaitBudget)) {
                        *abort_flag = 1;
                        stop = true;
                        break;
                    }
                    uint8_t* st = smem + s * kPcStage;
                    tc::mbar_arrive_expect_tx(&full[s], kPcStage);
                    tc::tma_load_2d(st, &tmap_wc, &full[s], kp * 64, wrow);
                    tc::tma_load_2d(st + kPcWBytes, &tmap_wz, &full[s], kp * 64, wrow);
                    tc::tma_load_2d(st + 2 * kPcWBytes, &tmap_h, &full[s], kp * 64, hrow);
                }
            }
            // drain: every issued load has landed before the CTA may exit
            for (int j = it - kPcStages < 0 ? 0 : it - kPcStages; j < it; ++j)
                if (!tc::mbar_wait(&full[j % kPcStages], (j / kPcStages) & 1, tc::kWaitBudget)) *abort_flag = 1;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdesc = tc::idesc_bf16_f32(kPcCols, kPcTokens, false, false);
            int it = 0, nt = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < a.tiles && ok; t += gridDim.x, ++nt) {
                if (!tc::mbar_wait(tempty, (nt & 1) ^ 1, tc::kWaitBudget)) {  // TMEM read out
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                for (int kp = 0; kp < kpanels; ++kp, ++it) {
                    const int s = it % kPcStages;
                    const uint32_t ph = (it / kPcStages) & 1;
                    if (*abort_flag || !tc::mbar_wait(&full[s], ph, tc::kWaitBudget)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t wc = tc::smem_u32(smem + s * kPcStage);
                    const uint32_t wz = wc + kPcWBytes;
                    const uint32_t hh = wc + 2 * kPcWBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bd = tc::smem_desc_sw128(hh + kk * 32, 16, 1024);
                        const uint32_t acc = (kp | kk) ? 1u : 0u;
                        tc::mma_bf16_ss(tmem, tc::smem_desc_sw128(wc + kk * 32, 16, 1024), bd, kIdesc, acc);
                        tc::mma_bf16_ss(tmem + kPcTokens, tc::smem_desc_sw128(wz + kk * 32, 16, 1024), bd, kIdesc, acc);
                    }
                    tc::mma_commit(&empty[s]);  // the stage is free once these MMAs finish
                }
                if (!ok) break;
                tc::mma_commit(tfull);          // the tile's C and Z accumulators are complete
            }
            if (!ok) *abort_flag = 1;
            tc::mma_commit(done);               // all issued MMAs complete before TMEM is freed
            if (!tc::mbar_wait(done, 0, tc::kWaitBudget)) *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;        // TMEM lanes this warp may read
        const int ent = (warp - 2) >> 2;     // which of the tile's two entries
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16);
        int nt = 0;
        for (int64_t t = blockIdx.x; t < a.tiles; t += gridDim.x, ++nt) {
            if (*abort_flag || !tc::mbar_wait(tfull, nt & 1, tc::kWaitBudget)) {
                *abort_flag = 1;
                break;
            }
            tc::fence_after_sync();
            int b, cb;
            int64_t tb;
            pc_tile(a, t, b, tb, cb);
            const int j = cb * kPcCols + quarter * 32 + lane;  // this thread's output column
            const float res = hca_entry(taddr + ent * kPcMp, a.bias, a.c, j, a.bias != nullptr);
            tc::fence_before_sync();
            tc::mbar_arrive(tempty);  // TMEM read out: the next tile's MMAs may start
            const int64_t i = a.e0 + 2 * tb + ent;
            if (i < a.e1) a.out[(int64_t)b * a.out_ld_batch + i * a.c + j] = __float2bfloat16_rn(res);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) atomicExch(a.status, 1u);
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------------
// CSA form ([P1] sections 3-5): four projections C^a = H W_a^KV, C^b = H W_b^KV,
// Z^a = H W_a^Z, Z^b = H W_b^Z, then for entry i and column j the softmax over the 2m = 8
// logits Z^a of block i (+ B^a) and Z^b of block i - 1 (+ B^b), and the weighted sum of
// the matching C^a and C^b values; entry 0 has no b-part.
//
// With m = 4 a tile of 256 tokens holds 64 blocks.  Block 0 only serves as the b-part of
// the tile's first entry, so a tile yields 63 entries and consecutive tiles overlap by
// one block.  A tile covers 256 output columns on a CTA pair (a cluster of two) with one
// cta_group::2 MMA per step: M = 256 columns (128 per CTA) by N = 256 tokens, whose H
// rows are split 128 per CTA.  Per 64-wide K panel each SM thus loads its two 16 KB
// weight panels and only half of the H panel, 48 KB, and the ring has four stages.
// Only two accumulators of 256 tokens fit a CTA's 512 TMEM columns, so each tile runs
// two passes over K (C in TMEM columns 0-255, Z in 256-511):
//   pass b   C^b and Z^b: per block, the softmax statistics of its four b-logits, kept in
//            the epilogue threads' registers as (value, base-2 log of the weight sum)
//               v_b = sum_r 2^{zl_r - mx} C_r / sum_r 2^{zl_r - mx},
//               s_b = mx + log2(sum_r 2^{zl_r - mx}),   zl = (z + B) log2(e);
//   pass a   C^a and Z^a: per block i, the same sums over its four a-logits, merged with
//            block i - 1's statistics into the softmax over all eight logits, then the
//            bf16 entry.
// The merge is the usual split softmax: with M = max(mx_a, s_b) the entry is
// (2^{mx_a-M} acc_a + 2^{s_b-M} v_b) / (2^{mx_a-M} l_a + 2^{s_b-M}).  Exponentials,
// logarithms and reciprocals are the multi-function unit's approximations (relative
// error about 2^-22), far inside the bf16 rounding of the entry.
// Pass a walks K backwards, so the H panels that pass b read last are re-read first,
// while they are still in L2.  Eight epilogue warps per CTA (two per TMEM lane quarter,
// each owning half of the tile's blocks) keep the TMEM drain between passes short.
//   both CTAs, warp 0    TMA producer into its own shared memory; the bytes complete on
//                        the leader's (rank 0) stage barrier;
//   leader, warp 1       MMA issuer; each commit arrives on both CTAs' barriers;
//   both CTAs, warps 2-9 epilogue of its own columns; each warp then arrives on the
//                        leader's TMEM-free barrier.
// With an odd number of 128-column blocks the last pair's second half reads weight rows
// past c (zero-filled by TMA) and writes nothing.
constexpr int kCsM = 4;                          // tokens per CSA block
constexpr int kCsTokens = kPcTokens;             // tokens per tile (MMA N): 64 blocks
constexpr int kCsEntries = kCsTokens / kCsM - 1; // 63 entries per tile
constexpr int kCsThreads = 64 + 256;             // TMA warp, MMA warp, 8 epilogue warps
constexpr int kCsHBytes = (kCsTokens / 2) * 128;   // this CTA's 128 x 64 half of the H panel: 16 KB
constexpr int kCsStage = 2 * kPcWBytes + kCsHBytes;  // 48 KB per CTA: two weight panels, the H half
constexpr int kCsStages = 4;
constexpr int kCsSmem = 1024 + kCsStages * kCsStage + 256;
static_assert((2 * kCsStages + 3) * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit 256 bytes");

struct CsArgs {
    int64_t rows_per_batch, tok0;
    int d, c;
    const float* ba;         // [m][c] or null
    const float* bb;         // [m][c] or null
    __nv_bfloat16* out;
    int64_t out_ld_batch;
    int64_t e0, e1;
    int n_cb;
    int64_t n_tb;            // tiles of 63 entries per batch
    int64_t tiles;
    uint32_t* status;
};

// Pass b for one epilogue thread.  Half 0 keeps blocks 0-30 (u = kb), half 1 blocks
// 31-62 (u = kb - 31): the b-parts of the a-blocks 1-31 and 32-63 that the same thread
// merges in pass a.  Loads are 16-column aligned, so half 1 starts at token 112.
// Logits are taken in base 2: zl = z log2(e) + bias log2(e) (bl2 holds the scaled bias),
// so every exponential is one ex2 of the multi-function unit.
template <int HALF>
CSA_DEV void cs_pass_b(uint32_t taddr, const float (&bl2)[kCsM], float (&sv)[32], float (&ss)[32],
                       uint32_t tempty_leader)
{
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr int kLo = HALF ? 7 : 0, kHi = HALF ? 15 : 7;
#pragma unroll
    for (int ch = kLo; ch <= kHi; ++ch) {
        uint32_t rc[16], rz[16];
        tc::tmem_ld16_async(taddr + ch * 16, rc);
        tc::tmem_ld16_async(taddr + kCsTokens + ch * 16, rz);
        tc::tmem_wait_ld_regs16(rc, rz);
        if (ch == kHi) {  // this warp's TMEM reads are done
            tc::fence_before_sync();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) cl::mbar_arrive_remote(tempty_leader);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int kb = 4 * ch + q;
            if (HALF == 0 ? kb > 30 : (kb < 31 || kb > 62)) continue;
            const int u = HALF ? kb - 31 : kb;
            float z[kCsM], mx = -INFINITY;
#pragma unroll
            for (int r = 0; r < kCsM; ++r) {
                z[r] = fmaf(__uint_as_float(rz[4 * q + r]), kLog2e, bl2[r]);
                mx = fmaxf(mx, z[r]);
            }
            float l = 0.f, acc = 0.f;
#pragma unroll
            for (int r = 0; r < kCsM; ++r) {
                const float p = tc::ex2_approx(z[r] - mx);
                l += p;
                acc = fmaf(p, __uint_as_float(rc[4 * q + r]), acc);
            }
            sv[u] = acc * tc::rcp_approx(l);  // l in [1, 4]
            ss[u] = mx + tc::lg2_approx(l);
        }
    }
}

// Pass a for one epilogue thread: half 0 writes the entries of a-blocks 1-31, half 1
// those of a-blocks 32-63 (entry first + kb - 1, b-part in sv/ss[u]).
template <int HALF>
CSA_DEV void cs_pass_a(uint32_t taddr, const float (&bl2)[kCsM], const float (&sv)[32], const float (&ss)[32],
                       int64_t first, int64_t e1, int64_t ld_entry, __nv_bfloat16* orow, uint32_t tempty_leader)
{
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr int kLo = HALF ? 8 : 0, kHi = HALF ? 15 : 7;
#pragma unroll
    for (int ch = kLo; ch <= kHi; ++ch) {
        uint32_t rc[16], rz[16];
        tc::tmem_ld16_async(taddr + ch * 16, rc);
        tc::tmem_ld16_async(taddr + kCsTokens + ch * 16, rz);
        tc::tmem_wait_ld_regs16(rc, rz);
        if (ch == kHi) {  // this warp's TMEM reads are done
            tc::fence_before_sync();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) cl::mbar_arrive_remote(tempty_leader);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int kb = 4 * ch + q;
            if (HALF == 0 && kb == 0) continue;
            const int u = HALF ? kb - 32 : kb - 1;
            const int64_t i = first + kb - 1;
            float z[kCsM], mx = -INFINITY;
#pragma unroll
            for (int r = 0; r < kCsM; ++r) {
                z[r] = fmaf(__uint_as_float(rz[4 * q + r]), kLog2e, bl2[r]);
                mx = fmaxf(mx, z[r]);
            }
            float l = 0.f, acc = 0.f;
#pragma unroll
            for (int r = 0; r < kCsM; ++r) {
                const float p = tc::ex2_approx(z[r] - mx);
                l += p;
                acc = fmaf(p, __uint_as_float(rc[4 * q + r]), acc);
            }
            float res;
            if (i > 0) {  // merge with block i - 1's b-part: weights 2^(mx - M) and 2^(s_b - M)
                const float M = fmaxf(mx, ss[u]);
                const float wa = tc::ex2_approx(mx - M), wb = tc::ex2_approx(ss[u] - M);
                res = fmaf(wa, acc, wb * sv[u]) * tc::rcp_approx(fmaf(wa, l, wb));
            } else {      // entry 0 has no b-part
                res = acc * tc::rcp_approx(l);
            }
            if (i < e1) orow[i * ld_entry] = __float2bfloat16_rn(res);
        }
    }
}

__global__ void __launch_bounds__(kCsThreads, 1)
csa_project_compress_kernel(const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ CUtensorMap tmap_wa_kv,
                            const __grid_constant__ CUtensorMap tmap_wb_kv, const __grid_constant__ CUtensorMap tmap_wa_z,
                            const __grid_constant__ CUtensorMap tmap_wb_z, CsArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned; an offset from the __shared__ array keeps every derived pointer in
    // the shared window, so its accesses compile to shared-memory instructions
    uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kCsStages * kCsStage);  // leader's are used
    uint64_t* empty = full + kCsStages;    // each CTA's: its stage may be overwritten
    uint64_t* tfull = empty + kCsStages;   // each CTA's: the pass's accumulators are complete
    uint64_t* tempty = tfull + 1;          // leader's: both CTAs read TMEM out (16 warps)
    uint64_t* done = tempty + 1;           // leader's: every MMA complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cl::cluster_rank();
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kCsStages; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        tc::mbar_init(tfull, 1);
        tc::mbar_init(tempty, 2 * ((kCsThreads - 64) / 32));
        tc::mbar_init(done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        tc::tma_prefetch_desc(&tmap_h);
        tc::tma_prefetch_desc(&tmap_wa_kv);
        tc::tma_prefetch_desc(&tmap_wb_kv);
        tc::tma_prefetch_desc(&tmap_wa_z);
        tc::tma_prefetch_desc(&tmap_wb_z);
    }
    if (warp == 1) {
        cl::tmem_alloc_pair(tmem_slot, 512);
        cl::tmem_relinquish_pair();
    }
    tc::fence_before_sync();
    __syncthreads();
    cl::cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();

    const int kpanels = a.d / 64;
    const int n_cp = (a.n_cb + 1) / 2;  // column pairs
    auto tile_of = [&](int64_t t, int& b, int64_t& tb, int& cp) {
        cp = (int)(t % n_cp);
        const int64_t r = t / n_cp;
        tb = r % a.n_tb;
        b = (int)(r / a.n_tb);
    };
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int it = 0;
            bool stop = false;
            for (int64_t t = pair; t < a.tiles && !stop; t += npairs) {
                int b, cp;
                int64_t tb;
                tile_of(t, b, tb, cp);
                // block 0 of the tile is block (first entry - 1); rows before the batch's
                // first token (entry 0) are read but never used.  This CTA loads tokens
                // 128 rank .. 128 rank + 127 of the tile.
                const int hrow = (int)(b * a.rows_per_batch + kCsM * (a.e0 + kCsEntries * tb - 1) - a.tok0) +
                                 (int)rank * (kCsTokens / 2);
                const int wrow = (2 * cp + (int)rank) * kPcCols;
                for (int pass = 0; pass < 2 && !stop; ++pass) {
                    const CUtensorMap* wkv = pass == 0 ? &tmap_wb_kv : &tmap_wa_kv;
                    const CUtensorMap* wz = pass == 0 ? &tmap_wb_z : &tmap_wa_z;
                    for (int kp = 0; kp < kpanels; ++kp, ++it) {
                        const int s = it % kCsStages;
                        const uint32_t ph = (it / kCsStages) & 1;
                        if (*abort_flag || !tc::mbar_wait(&empty[s], ph ^ 1, tc::kWaitBudget)) {
                            *abort_flag = 1;
                            stop = true;
                            break;
                        }
                        uint8_t* st = smem + s * kCsStage;
                        if (rank == 0) tc::mbar_arrive_expect_tx(&full[s], 2 * kCsStage);  // both CTAs' bytes
                        const uint32_t fb = cl::peer_addr(tc::smem_u32(&full[s]), 0);  // the leader's full[s]
                        // pass a walks K backwards: the H panels pass b read last are
                        // the first ones it needs, while they are still in L2
                        const int kx = (pass == 0 ? kp : kpanels - 1 - kp) * 64;
                        cl::tma_load_2d_pair(st, wkv, fb, kx, wrow);
                        cl::tma_load_2d_pair(st + kPcWBytes, wz, fb, kx, wrow);
                        cl::tma_load_2d_pair(st + 2 * kPcWBytes, &tmap_h, fb, kx, hrow);
                    }
                }
            }
            // drain: this CTA's loads of the last stages were consumed (or the CTA gives up)
            for (int j = it - kCsStages < 0 ? 0 : it - kCsStages; j < it; ++j)
                if (!tc::mbar_wait(&empty[j % kCsStages], (j / kCsStages) & 1, tc::kWaitBudget)) *abort_flag = 1;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t kIdesc = tc::idesc_bf16_f32(2 * kPcCols, kCsTokens, false, false);
            int it = 0, np = 0;
            bool ok = true;
            for (int64_t t = pair; t < a.tiles && ok; t += npairs) {
                for (int pass = 0; pass < 2 && ok; ++pass, ++np) {
                    if (!tc::mbar_wait(tempty, (np & 1) ^ 1, tc::kWaitBudget)) {  // both CTAs' TMEM read out
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    for (int kp = 0; kp < kpanels; ++kp, ++it) {
                        const int s = it % kCsStages;
                        const uint32_t ph = (it / kCsStages) & 1;
                        if (*abort_flag || !tc::mbar_wait(&full[s], ph, tc::kWaitBudget)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after_sync();
                        const uint32_t wc = tc::smem_u32(smem + s * kCsStage);
                        const uint32_t wz = wc + kPcWBytes;
                        const uint32_t hh = wc + 2 * kPcWBytes;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t bd = tc::smem_desc_sw128(hh + kk * 32, 16, 1024);
                            const uint32_t acc = (kp | kk) ? 1u : 0u;
                            cl::mma_bf16_ss_pair(tmem, tc::smem_desc_sw128(wc + kk * 32, 16, 1024), bd, kIdesc, acc);
                            cl::mma_bf16_ss_pair(tmem + kCsTokens, tc::smem_desc_sw128(wz + kk * 32, 16, 1024), bd,
                                                 kIdesc, acc);
                        }
                        cl::mma_commit_pair(&empty[s], 0x3);  // both CTAs' stage s is free
                    }
                    if (!ok) break;
                    cl::mma_commit_pair(tfull, 0x3);          // both CTAs' accumulators are complete
                }
            }
            if (!ok) *abort_flag = 1;
            cl::mma_commit_pair(done, 0x1);
            if (!tc::mbar_wait(done, 0, tc::kWaitBudget)) *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int quarter = warp & 3;               // TMEM lanes this warp may read
        const int half = (warp - 2) >> 2;           // which 32 blocks of the tile
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t tempty0 = cl::peer_addr(tc::smem_u32(tempty), 0);
        float sv[32], ss[32];                       // pass b statistics, carried to pass a
        int np = 0;
        for (int64_t t = pair; t < a.tiles; t += npairs) {
            int b, cp;
            int64_t tb;
            tile_of(t, b, tb, cp);
            const int j = (2 * cp + (int)rank) * kPcCols + quarter * 32 + lane;  // this thread's output column
            const bool live = j < a.c;  // the second half of an odd last column pair has none
            constexpr float kLog2e = 1.4426950408889634f;
            float ba[kCsM], bb[kCsM];  // biases in base-2 logit units
#pragma unroll
            for (int r = 0; r < kCsM; ++r) {
                ba[r] = a.ba && live ? __ldg(&a.ba[r * a.c + j]) * kLog2e : 0.f;
                bb[r] = a.bb && live ? __ldg(&a.bb[r * a.c + j]) * kLog2e : 0.f;
            }
            if (*abort_flag || !tc::mbar_wait(tfull, np & 1, tc::kWaitBudget)) {
                *abort_flag = 1;
                break;
            }
            ++np;
            tc::fence_after_sync();
            if (half == 0) cs_pass_b<0>(taddr, bb, sv, ss, tempty0);
            else cs_pass_b<1>(taddr, bb, sv, ss, tempty0);
            if (*abort_flag || !tc::mbar_wait(tfull, np & 1, tc::kWaitBudget)) {
                *abort_flag = 1;
                break;
            }
            ++np;
            tc::fence_after_sync();
            const int64_t first = a.e0 + kCsEntries * tb;  // entry of tile block 1
            __nv_bfloat16* orow = a.out + (int64_t)b * a.out_ld_batch + j;
            const int64_t e1 = live ? a.e1 : 0;            // a dead column writes nothing
            if (half == 0) cs_pass_a<0>(taddr, ba, sv, ss, first, e1, a.c, orow, tempty0);
            else cs_pass_a<1>(taddr, ba, sv, ss, first, e1, a.c, orow, tempty0);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    cl::cluster_sync();  // the leader's MMAs into this CTA's TMEM are complete
    if (*abort_flag && threadIdx.x == 0) atomicExch(a.status, 1u);
    if (warp == 1) {
        tc::fence_after_sync();
        cl::tmem_dealloc_pair(tmem, 512);
    }
}

}  // namespace
}  // namespace csa

extern "C" int hca_project_compress(const void* H, int64_t ld_row, int64_t ld_batch, int64_t tok0, int64_t n,
                                    const void* Wc, const void* Wz, int d, const float* Bias, void* out,
                                    int64_t out_ld_batch, int B, int c, int m_prime, int64_t entry_begin,
                                    int64_t entry_end, void* workspace, size_t ws_bytes, csa_stream_t stream_)
{
    using namespace csa;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (B < 0 || c <= 0 || d <= 0 || m_prime <= 0 || n < 0 || entry_begin < 0 || entry_end < entry_begin)
        return CSA_ERR_ARG;
    if ((int64_t)m_prime * entry_end > n || tok0 < 0 || tok0 > (int64_t)m_prime * entry_begin)
        return CSA_ERR_ARG;
    if (ld_row < d || ld_batch < (n - tok0) * ld_row || out_ld_batch < entry_end * c) return CSA_ERR_ARG;
    if (m_prime != kPcMp || c % kPcCols != 0 || d % 64 != 0 || ld_row % 8 != 0 || ld_batch % ld_row != 0)
        return CSA_ERR_UNSUPPORTED;
    if (B == 0 || entry_end == entry_begin) return CSA_OK;
    if (!H || !Wc || !Wz || !out || !workspace) return CSA_ERR_ARG;
    if (!aligned16(H) || !aligned16(Wc) || !aligned16(Wz) || !aligned16(workspace) || ((uintptr_t)Bias & 3) ||
        ((uintptr_t)out & 1))
        return CSA_ERR_ALIGN;
    if (ws_bytes < 256) return CSA_ERR_WORKSPACE;
    PcArgs a;
    a.rows_per_batch = ld_batch / ld_row;
    if ((int64_t)B * a.rows_per_batch + kPcTokens >= (int64_t(1) << 31)) return CSA_ERR_UNSUPPORTED;
    a.tok0 = tok0;
    a.d = d;
    a.c = c;
    a.bias = Bias;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.out_ld_batch = out_ld_batch;
    a.e0 = entry_begin;
    a.e1 = entry_end;
    a.n_cb = c / kPcCols;
    a.n_tb = (entry_end - entry_begin + 1) / 2;
    a.status = static_cast<uint32_t*>(workspace);
    CUtensorMap th, twc, twz;
    a.tiles = (int64_t)B * a.n_tb * a.n_cb;
    if (!make_tmap_bf16_2d(&th, H, (uint64_t)B * a.rows_per_batch, d, ld_row, 64, kPcTokens) ||
        !make_tmap_bf16_2d(&twc, Wc, c, d, d, 64, kPcCols) || !make_tmap_bf16_2d(&twz, Wz, c, d, d, 64, kPcCols))
        return CSA_ERR_CUDA;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t grid = a.tiles < sms ? a.tiles : sms;
    cudaFuncSetAttribute(hca_project_compress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPcSmem);
    launch_pdl(hca_project_compress_kernel, dim3((unsigned)grid), dim3(kPcThreads), (size_t)kPcSmem, stream, th, twc,
               twz, a);
    return launch_status();
}

extern "C" int csa_project_compress(const void* H, int64_t ld_row, int64_t ld_batch, int64_t tok0, int64_t n,
                                    const void* Wa_kv, const void* Wb_kv, const void* Wa_z, const void* Wb_z, int d,
                                    const float* Ba, const float* Bb, void* out, int64_t out_ld_batch, int B, int c,
                                    int m, int64_t entry_begin, int64_t entry_end, void* workspace, size_t ws_bytes,
                                    csa_stream_t stream_)
{
    using namespace csa;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (B < 0 || c <= 0 || d <= 0 || m <= 0 || n < 0 || entry_begin < 0 || entry_end < entry_begin || tok0 < 0)
        return CSA_ERR_ARG;
    const int64_t first_row = entry_begin == 0 ? 0 : (int64_t)m * (entry_begin - 1);
    if ((int64_t)m * entry_end > n || (entry_end > entry_begin && tok0 > first_row)) return CSA_ERR_ARG;
    if (ld_row < d || ld_batch < (n - tok0) * ld_row || out_ld_batch < entry_end * c) return CSA_ERR_ARG;
    if (m != kCsM || c % kPcCols != 0 || d % 64 != 0 || ld_row % 8 != 0 || ld_batch % ld_row != 0)
        return CSA_ERR_UNSUPPORTED;
    if (B == 0 || entry_end == entry_begin) return CSA_OK;
    if (!H || !Wa_kv || !Wb_kv || !Wa_z || !Wb_z || !out || !workspace) return CSA_ERR_ARG;
    if (!aligned16(H) || !aligned16(Wa_kv) || !aligned16(Wb_kv) || !aligned16(Wa_z) || !aligned16(Wb_z) ||
        !aligned16(workspace) || (((uintptr_t)Ba | (uintptr_t)Bb) & 3) || ((uintptr_t)out & 1))
        return CSA_ERR_ALIGN;
    if (ws_bytes < 256) return CSA_ERR_WORKSPACE;
    CsArgs a;
    a.rows_per_batch = ld_batch / ld_row;
    if ((int64_t)B * a.rows_per_batch + kCsTokens >= (int64_t(1) << 31)) return CSA_ERR_UNSUPPORTED;
    a.tok0 = tok0;
    a.d = d;
    a.c = c;
    a.ba = Ba;
    a.bb = Bb;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.out_ld_batch = out_ld_batch;
    a.e0 = entry_begin;
    a.e1 = entry_end;
    a.n_cb = c / kPcCols;
    a.n_tb = (entry_end - entry_begin + kCsEntries - 1) / kCsEntries;
    a.tiles = (int64_t)B * a.n_tb * ((a.n_cb + 1) / 2);  // (token tile, pair of 128-column blocks)
    a.status = static_cast<uint32_t*>(workspace);
    CUtensorMap th, tw[4];
    const void* ws4[4] = {Wa_kv, Wb_kv, Wa_z, Wb_z};
    if (!make_tmap_bf16_2d(&th, H, (uint64_t)B * a.rows_per_batch, d, ld_row, 64, kCsTokens / 2)) return CSA_ERR_CUDA;
    for (int w = 0; w < 4; ++w)
        if (!make_tmap_bf16_2d(&tw[w], ws4[w], c, d, d, 64, kPcCols)) return CSA_ERR_CUDA;
    cudaFuncSetAttribute(csa_project_compress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCsSmem);
    const int pairs = max_resident_pairs(csa_project_compress_kernel, dim3(kCsThreads), kCsSmem);
    if (pairs <= 0) return CSA_ERR_CUDA;
    const int64_t np = a.tiles < pairs ? a.tiles : pairs;
    launch_pdl_pairs(csa_project_compress_kernel, dim3((unsigned)(2 * np)), dim3(kCsThreads), (size_t)kCsSmem, stream,
                     th, tw[0], tw[1], tw[2], tw[3], a);
    return launch_status();
}
