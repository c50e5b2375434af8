// Lightning-indexer scores for many queries at once (chunked prefill) on tcgen05
// ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch", section 6.4: the boxed
// score, and the cost paragraph there, by which each of the n queries scores every one
// of the n/m compressed blocks).
//
// With many queries the score is a dense contraction over all of them:
//   D[s, (j, h)] = K^I[s] . q^I[j, h]     (M = 128 keys, N = 256 query-head pairs, K = c^I)
//   I[j, s]      = sum_h w[j, h] ReLU(D[s, (j, h)])
// A CTA keeps one block of 2 x (256 / n_h^I) queries resident in shared memory (two
// N = 256 halves of the B operand) and streams a range of key tiles past it, so every
// key tile is read once per query block instead of once per query:
//
//   warp 0   TMA producer: the query block once, then 128-key tiles (128-byte swizzle)
//            into a ring of as many stages as shared memory allows;
//   warp 1   MMA issuer: per key tile two M = 128, N = 256 accumulations, one into
//            each half of TMEM (columns 0-255 and 256-511), so one half's epilogue
//            overlaps the other half's MMAs;
//   warps 2-17 epilogue, eight warps per half (one per TMEM lane quarter and column
//            half): each thread owns one key row, reads 128 of its dot products,
//            applies ReLU and the head weights and writes one fp32 score per query of
//            its columns.  Two warps per scheduler drain a half, so a half's epilogue
//            fits in the time of the other half's MMAs.
//
// Consecutive CTAs take consecutive query blocks of the same key range, so the key
// tiles they stream are shared in L2.  The scores go to the workspace, together with the
// largest score of every 32 consecutive keys; the row select (one CTA per query)
// follows.  Every wait is bounded; a timeout sets the workspace status word and every
// role drains and exits.
#include "indexer.cuh"
#include "tc_utils.cuh"

namespace csa {
namespace {

constexpr int kMqColParts = 2;                         // epilogue warps per lane quarter and half
constexpr int kMqEpiThreads = 2 * 4 * kMqColParts * 32;  // both halves
constexpr int kMqThreads = 64 + kMqEpiThreads;           // producer, MMA, epilogue warps
constexpr int kMqKeys = 128;     // keys per tile (MMA M)
constexpr int kMqN = 256;        // (query, head) rows per accumulator half (MMA N)
constexpr int kMqSmem = 232448;  // the opt-in shared-memory limit per block

template <int NH, int CI>
struct MqCfg {
    static constexpr int kQPM = kMqN / NH;                     // queries per half
    static constexpr int kQB = 2 * kQPM;                       // queries per CTA
    static constexpr int kPanels = CI / 64;                    // 128-byte column panels
    static constexpr int kQPanel = kMqN * 128;                 // one panel of one half
    static constexpr int kQBytes = 2 * kPanels * kQPanel;      // the resident query block
    static constexpr int kAStage = kMqKeys * CI * 2;           // one key tile
    static constexpr int kTail = kQB * NH * 4 + 256;           // head weights + barriers
    static constexpr int kStagesRaw = (kMqSmem - kQBytes - kTail) / kAStage;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    // what is left for aligning the dynamic shared-memory base up to 1024 bytes
    static constexpr int kSlack = kMqSmem - kQBytes - kStages * kAStage - kTail;
    static_assert(kStages >= 2, "not enough shared memory for a 2-stage ring");
    static_assert((2 * kStages + 6) * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit 256 bytes");
    static_assert(kQPM * NH == kMqN, "heads divide the MMA N");
};

struct MqArgs {
    const float* wI;   // [G][NH]
    const int64_t* t;  // [G]
    int nq;            // queries per batch row
    int64_t N_cap;     // keys per batch row
    int m;             // tokens per compressed entry
    int qblocks;       // query blocks per batch row
    int splits;        // key ranges per query block
    TopkWs ws;
};

CSA_DEV int64_t mq_visible(const int64_t* t, int64_t g, int m, int64_t N_cap)
{
    const int64_t tt = t[g];
    if (tt < 0) return 0;
    const int64_t v = tt / m;
    return v < N_cap ? v : N_cap;
}

template <int NH, int CI>
__global__ void __launch_bounds__(kMqThreads, 1)
scan_mq_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q, MqArgs a)
{
    using Cfg = MqCfg<NH, CI>;
    constexpr int S = Cfg::kStages;
    constexpr int QPM = Cfg::kQPM;
    constexpr int QB = Cfg::kQB;
    // no static shared memory in this kernel, so the dynamic block normally starts on a
    // 1024-byte boundary; the slack covers a base that does not
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t* sQ = smem_raw + pad;                                     // [2 halves][panels][256 rows][128 B]
    uint8_t* sA = sQ + Cfg::kQBytes;                                  // [S][panels][128 keys][128 B]
    float* sw = reinterpret_cast<float*>(sA + S * Cfg::kAStage);      // [QB][NH] head weights
    uint64_t* full = reinterpret_cast<uint64_t*>(sw + QB * NH);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;
    uint64_t* tempty = tfull + 2;
    uint64_t* done = tempty + 2;
    uint64_t* qfull = done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qfull + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    pdl_launch_dependents();
    if (pad > (uint32_t)Cfg::kSlack) {  // the same base for every CTA: the whole grid stops
        pdl_wait();
        if (threadIdx.x == 0) atomicExch(a.ws.status, 2u);
        return;
    }
    const int qb = blockIdx.x, sp = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            tc::mbar_init(&tfull[h], 1);
            tc::mbar_init(&tempty[h], kMqEpiThreads / 2);
        }
        tc::mbar_init(done, 1);
        tc::mbar_init(qfull, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tmap_k);
        tc::tma_prefetch_desc(&tmap_q);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 2 * kMqN);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    // only this CTA's shared memory and TMEM were touched so far; global memory after this
    pdl_wait();
    const int64_t g0 = (int64_t)b * a.nq + (int64_t)qb * QB;  // first query of the block
    const int nvalid = min(QB, a.nq - qb * QB);
    int64_t vmax = 0;
    for (int j = 0; j < nvalid; ++j) vmax = max(vmax, mq_visible(a.t, g0 + j, a.m, a.N_cap));
    const int ntb = (int)((vmax + kMqKeys - 1) / kMqKeys);
    const int tile0 = (int)((int64_t)ntb * sp / a.splits);
    const int tile1 = (int)((int64_t)ntb * (sp + 1) / a.splits);
    const bool active = tile1 > tile0;

    if (!active) {
        // no visible key tile in this CTA's range
    } else if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(qfull, Cfg::kQBytes);
            for (int hf = 0; hf < 2; ++hf)
                for (int p = 0; p < Cfg::kPanels; ++p)
                    tc::tma_load_2d(sQ + (hf * Cfg::kPanels + p) * Cfg::kQPanel, &tmap_q, qfull, 64 * p,
                                    (int)((g0 + hf * QPM) * NH));
            int it = 0;
            for (int tile = tile0; tile < tile1; ++tile, ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1;
                if (*abort_flag) break;
                if (!tc::mbar_wait(&empty[s], ph ^ 1, tc::kWaitBudget)) {
                    *abort_flag = 1;
                    break;
                }
                tc::mbar_arrive_expect_tx(&full[s], Cfg::kAStage);
                const int row0 = (int)((int64_t)b * a.N_cap) + tile * kMqKeys;
#pragma unroll
                for (int p = 0; p < Cfg::kPanels; ++p)
                    tc::tma_load_2d(sA + s * Cfg::kAStage + p * (kMqKeys * 128), &tmap_k, &full[s], 64 * p, row0);
            }
            // drain: every issued load has landed before the CTA may exit
            for (int j = it - S < 0 ? 0 : it - S; j < it; ++j)
                if (!tc::mbar_wait(&full[j % S], (j / S) & 1, tc::kWaitBudget)) *abort_flag = 1;
            if (!tc::mbar_wait(qfull, 0, tc::kWaitBudget)) *abort_flag = 1;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdesc = tc::idesc_bf16_f32(kMqKeys, kMqN, false, false);
            bool ok = tc::mbar_wait(qfull, 0, tc::kWaitBudget);
            if (!ok) *abort_flag = 1;
            int it = 0;
            for (int tile = tile0; ok && tile < tile1; ++tile, ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1;
                if (*abort_flag || !tc::mbar_wait(&full[s], ph, tc::kWaitBudget)) {
                    ok = false;
                    break;
                }
                const uint32_t a0 = tc::smem_u32(sA + s * Cfg::kAStage);
                for (int hf = 0; hf < 2 && ok; ++hf) {
                    if (!tc::mbar_wait(&tempty[hf], (it & 1) ^ 1, tc::kWaitBudget)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t d = tmem_base + hf * kMqN;
                    const uint32_t b0 = tc::smem_u32(sQ + hf * Cfg::kPanels * Cfg::kQPanel);
#pragma unroll
                    for (int p = 0; p < Cfg::kPanels; ++p) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = tc::smem_desc_sw128(a0 + p * (kMqKeys * 128) + kk * 32, 16, 1024);
                            const uint64_t bd = tc::smem_desc_sw128(b0 + p * Cfg::kQPanel + kk * 32, 16, 1024);
                            tc::mma_bf16_ss(d, ad, bd, kIdesc, (p | kk) ? 1u : 0u);
                        }
                    }
                    tc::mma_commit(&tfull[hf]);  // this half's accumulator is ready
                }
                if (!ok) break;
                tc::mma_commit(&empty[s]);       // the key stage is free once both halves finish
            }
            if (!ok) *abort_flag = 1;
            tc::mma_commit(done);                // all issued MMAs complete before TMEM is freed
            if (!tc::mbar_wait(done, 0, tc::kWaitBudget)) *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;
        for (int i = et; i < QB * NH; i += kMqEpiThreads)
            sw[i] = i / NH < nvalid ? __ldg(&a.wI[g0 * NH + i]) : 0.f;
        asm volatile("bar.sync 1, %0;" ::"n"(kMqEpiThreads) : "memory");  // epilogue warps only
        const int quarter = warp & 3;          // TMEM lane quarter this warp may access
        const int hf = ((warp - 2) >> 2) & 1;  // accumulator half: queries hf*QPM .. +QPM-1
        const int cp = (warp - 2) >> 3;        // column part of the half
        const int row = quarter * 32 + lane;   // key row of this thread within a tile
        constexpr int kCols = kMqN / kMqColParts;  // columns of this warp: whole queries
        constexpr int kQW = kCols / NH;             // queries of this warp
        static_assert(kCols % NH == 0, "a column part holds whole queries");
        const int q0 = hf * QPM + cp * kQW;         // first query of this warp in the block
        int vis[kQW];
#pragma unroll
        for (int j = 0; j < kQW; ++j)
            vis[j] = q0 + j < nvalid ? (int)mq_visible(a.t, g0 + q0 + j, a.m, a.N_cap) : 0;
        float* sc_base = a.ws.scores + (g0 + q0) * a.ws.ld;
        // per query, the largest order key of every 32 consecutive keys, for the select's
        // first filter (stored in the query's second candidate buffer, unused until then)
        uint32_t* gm_base = reinterpret_cast<uint32_t*>(a.ws.cand2) + (g0 + q0) * 2 * a.ws.ld;
        const float* wh = sw + q0 * NH;
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + hf * kMqN + cp * kCols;
        // This warp's columns in batches of 32, double buffered: the TMEM load of batch
        // b + 1 is in flight while batch b is summed.  A query's partial sums carry over
        // batches (NH = 64 or 128).
        constexpr int kBatch = 32;
        constexpr int kNB = kCols / kBatch;
        int it = 0;
        for (int tile = tile0; tile < tile1; ++tile, ++it) {
            if (*abort_flag) break;
            if (!tc::mbar_wait(&tfull[hf], it & 1, tc::kWaitBudget)) {
                *abort_flag = 1;
                break;
            }
            tc::fence_after_sync();
            const int sidx = tile * kMqKeys + row;
            // 4 independent chains (heads h = 0, 1, 2, 3 mod 4), two per packed FMA
            float2 p01 = make_float2(0.f, 0.f), p23 = make_float2(0.f, 0.f);
            uint32_t ra[32], rb[32];
            tc::tmem_ld32_async(taddr, ra);
            tc::tmem_wait_ld_regs(ra);
#pragma unroll
            for (int bt = 0; bt < kNB; ++bt) {
                uint32_t(&cur)[32] = (bt & 1) ? rb : ra;
                uint32_t(&nxt)[32] = (bt & 1) ? ra : rb;
                if (bt + 1 < kNB) tc::tmem_ld32_async(taddr + (bt + 1) * kBatch, nxt);
#pragma unroll
                for (int c = 0; c < kBatch; c += 4) {
                    const int col = bt * kBatch + c;  // column within this warp's part
                    const int j = col / NH, h = col % NH;  // query of this warp, head
                    const float4 w4 = *reinterpret_cast<const float4*>(wh + j * NH + h);
                    const float x0 = fmaxf(__uint_as_float(cur[c]), 0.f), x1 = fmaxf(__uint_as_float(cur[c + 1]), 0.f);
                    const float x2 = fmaxf(__uint_as_float(cur[c + 2]), 0.f), x3 = fmaxf(__uint_as_float(cur[c + 3]), 0.f);
                    p01 = tc::fma2(make_float2(x0, x1), make_float2(w4.x, w4.y), p01);
                    p23 = tc::fma2(make_float2(x2, x3), make_float2(w4.z, w4.w), p23);
                    if (h + 4 == NH) {  // query j complete
                        const float sc = (p01.x + p01.y) + (p23.x + p23.y);
                        p01 = p23 = make_float2(0.f, 0.f);
                        const bool valid = sidx < vis[j];
                        if (valid) sc_base[(int64_t)j * a.ws.ld + sidx] = sc;
                        const uint32_t gk = __reduce_max_sync(0xffffffffu, valid ? order_key(sc) : 0u);
                        if (lane == 0 && tile * kMqKeys + quarter * 32 < vis[j])
                            gm_base[(int64_t)j * 2 * a.ws.ld + tile * 4 + quarter] = gk;
                    }
                }
                if (bt + 1 < kNB) tc::tmem_wait_ld_regs(nxt);
                if (bt + 2 == kNB) {  // the last batch is in registers: the MMA may refill the half
                    tc::fence_before_sync();
                    tc::mbar_arrive(&tempty[hf]);
                }
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (active && *abort_flag && threadIdx.x == 0) atomicExch(a.ws.status, 1u);
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem_base, 2 * kMqN);
    }
}

template <int NH, int CI>
int launch_mq(const void* qI, const float* wI, const void* KI, const int64_t* t, int B, int nq,
              int64_t N_cap, int m, const TopkWs& ws, cudaStream_t stream)
{
    using Cfg = MqCfg<NH, CI>;
    CUtensorMap tk, tq;
    if (!make_tmap_bf16_2d(&tk, KI, (uint64_t)B * N_cap, CI, CI, 64, kMqKeys)) return CSA_ERR_CUDA;
    if (!make_tmap_bf16_2d(&tq, qI, (uint64_t)B * nq * NH, CI, CI, 64, kMqN)) return CSA_ERR_CUDA;
    auto kern = scan_mq_kernel<NH, CI>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMqSmem);
    MqArgs a;
    a.wI = wI;
    a.t = t;
    a.nq = nq;
    a.N_cap = N_cap;
    a.m = m;
    a.ws = ws;
    a.qblocks = (nq + Cfg::kQB - 1) / Cfg::kQB;
    // Key ranges per query block: one CTA per SM, so the grid runs in waves of kNumSMs
    // CTAs.  The split count minimises waves x (key tiles per CTA + 3), the 3 standing
    // for a CTA's fixed cost (query block load, pipeline fill) in tile periods.
    const int64_t blocks = (int64_t)B * a.qblocks;
    const int64_t tiles = (N_cap + kMqKeys - 1) / kMqKeys;
    int64_t splits = 1, best = -1;
    for (int64_t sp = 1; sp <= 256 && sp <= tiles; ++sp) {
        const int64_t waves = (blocks * sp + kNumSMs - 1) / kNumSMs;
        const int64_t cost = waves * ((tiles + sp - 1) / sp + 3);
        if (best < 0 || cost < best) {
            best = cost;
            splits = sp;
        }
    }
    a.splits = (int)splits;
    dim3 grid((unsigned)a.qblocks, (unsigned)splits, (unsigned)B);
    launch_pdl(kern, grid, dim3(kMqThreads), (size_t)kMqSmem, stream, tk, tq, a);
    return launch_status();
}

}  // namespace

bool indexer_mq_eligible(const void* qI, const void* KI, int B, int nq, int64_t N_cap, int n_hI, int cI)
{
    const bool shape = (n_hI == 32 || n_hI == 64 || n_hI == 128) && (cI == 64 || cI == 128);
    return shape && nq >= kMqMinQueries && B <= 65535 && N_cap >= kMqKeys &&
           (int64_t)B * N_cap + kMqKeys < (int64_t(1) << 31) &&
           (int64_t)B * nq * n_hI + kMqN < (int64_t(1) << 31) && aligned16(qI) && aligned16(KI);
}

int launch_scan_mq(const void* qI, const float* wI, const void* KI, const int64_t* t, int B, int nq,
                   int64_t N_cap, int n_hI, int cI, int m, const TopkWs& ws, cudaStream_t stream)
{
#define CSA_MQ_CASE(NH_, CI_) \
    if (n_hI == NH_ && cI == CI_) return launch_mq<NH_, CI_>(qI, wI, KI, t, B, nq, N_cap, m, ws, stream);
    CSA_MQ_CASE(32, 64) CSA_MQ_CASE(32, 128) CSA_MQ_CASE(64, 64) CSA_MQ_CASE(64, 128)
    CSA_MQ_CASE(128, 64) CSA_MQ_CASE(128, 128)
#undef CSA_MQ_CASE
    return CSA_ERR_UNSUPPORTED;
}

}  // namespace csa
