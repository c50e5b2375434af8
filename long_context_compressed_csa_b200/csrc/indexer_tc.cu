// Lightning-indexer scan on the 5th-generation tensor cores (tcgen05, bf16 in, fp32 out)
// ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch", section 6.4 boxed score).
//
// For one query the score of every compressed key is sum_h w[h] * ReLU(q[h] . K[s]):
// a dense [keys x c^I] x [c^I x n_h^I] contraction followed by a ReLU-weighted row
// reduction.  At n_h^I = 64 heads it performs 64 flop per byte of key read, six times
// the fp32 CUDA-core ridge of a B200, so the contraction runs on tcgen05:
//
//   warp 0   TMA producer: 128-key tiles of K^I (two 64-column panels for c^I = 128,
//            128-byte swizzle) into a STAGES-deep shared-memory ring;
//   warp 1   MMA issuer: D[128 keys x n_h^I] = K_tile * q^T with M = 128, N = n_h^I,
//            K = 16 per instruction, accumulating in TMEM; two accumulator buffers so
//            the next tile's MMAs overlap the previous tile's epilogue;
//   warps 2-9 epilogue (two groups of four, one per accumulator buffer): one thread
//            per key row reads its n_h^I fp32 dot products from
//            TMEM (tcgen05.ld), applies ReLU and the head weights, writes the fp32
//            score and adds its top-12-bit radix digit to a shared-memory histogram.
//
// q^I (the B operand) is staged once per CTA into the same swizzled layout.  Each CTA
// walks a strided set of key tiles of one query.  Every barrier wait is bounded; a
// timeout sets the workspace status word and every role drains and exits.
//
// Key formats: bf16 (kind::f16); E4M3 codes (kind::f8f6f4, q^I quantised per head to
// E4M3 by the epilogue warps, the key's fp32 scale applied to the score); E2M1 codes,
// two per byte in global memory, which the TMA unpacks into the 16-bytes-per-16-codes
// layout of an E2M1 operand, so the tiles, swizzle and descriptors are the E4M3 ones.
//
// When the query's grid fits in one wave, the same kernel then selects the top k in
// place (section 7): see the in-place top-k below.
#include "indexer.cuh"
#include "e4m3.cuh"
#include "select.cuh"
#include "tc_utils.cuh"

namespace csa {
namespace {

constexpr int kTcThreads = 320;  // producer, MMA, two groups of 4 epilogue warps
constexpr int kTileKeys = 128;
constexpr int kPrefetchTiles = 2;  // key tiles per CTA prefetched into L2 before the dependency wait

// KB: bytes per key / query element (2: bf16, 1: E4M3)
template <int NH, int CI, int KB = 2>
struct ScanCfg {
    static constexpr int kPanels = CI * KB / 128;          // 128-byte column panels of a tile
    static constexpr int kPanelElems = 128 / KB;             // elements per panel row
    static constexpr int kAStage = kTileKeys * CI * KB;     // bytes of one key tile
    static constexpr int kBBytes = NH * CI * KB;            // q^I tile
    static constexpr int kBudget = 220 * 1024;
    static constexpr int kFixed0 = 1024 + kBBytes + NH * 4 + kBins * 4 + 256;
    // scores of the CTA's first kCacheTiles tiles stay in shared memory for the in-place
    // select, when that still leaves a 3-stage ring
    static constexpr int kCacheTiles = (kBudget - kFixed0 - 3 * kAStage) >= 32 * kTileKeys * 4 ? 32 : 0;
    static constexpr int kFixed = kFixed0 + kCacheTiles * kTileKeys * 4;
    static constexpr int kStagesRaw = (kBudget - kFixed) / kAStage;
    // the scan is bound by the bytes in flight per SM (ring depth / HBM latency), so the
    // ring takes what shared memory allows, up to 12 stages (barrier area limit)
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static_assert((2 * kStages + 6) * 8 + 8 <= 256, "barriers, TMEM slot and abort flag fit 256 bytes");
    static constexpr int kSmem = kFixed + kStages * kAStage;
    static constexpr int kTmemCols = (2 * NH) < 32 ? 32 : (2 * NH);
    static_assert(kStages >= 2, "not enough shared memory for a 2-stage ring");
    static_assert((kTmemCols & (kTmemCols - 1)) == 0, "TMEM columns must be a power of 2");
    // the in-place select reuses the ring: the fallback's two lists, the per-bin counts
    // merged before this CTA's, the merged histogram and the threshold bin's candidates
    static constexpr int kOldOff = 2 * sel::kListCap * 8;
    static constexpr int kGhOff = kOldOff + kBins * 4;
    static constexpr int kCandOff = kGhOff + kBins * 4;
    static constexpr int kFastCapRaw = (kStages * kAStage - kCandOff) / 8;
    static constexpr int kFastCap = kFastCapRaw > 4096 ? 4096 : kFastCapRaw;
    static_assert(kFastCap >= 2048 && kFastCap % sel::kSelThreads == 0, "candidate list of the select's fast path");
};

CSA_DEV void red_release_add(uint32_t* p, uint32_t v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
CSA_DEV uint32_t atom_acq_rel_add(uint32_t* p, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
// Bounded wait until *p >= target (acquire, GPU scope); false after `budget` cycles.
CSA_DEV bool wait_count_geq(const uint32_t* p, uint32_t target, long long budget)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    if (v >= target) return true;
    const long long t0 = clock64();
    for (;;) {
        __nanosleep(64);
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        if (v >= target) return true;
        if (clock64() - t0 > budget) return false;
    }
}

CSA_DEV int64_t visible_of(const int64_t* t, int g, int m, int64_t N_cap)
{
    const int64_t tt = t[g];
    if (tt < 0) return 0;
    const int64_t v = tt / m;
    return v < N_cap ? v : N_cap;
}

// Outputs of the in-place top-k select (fused = 0: scores only, for topk_select).
struct SelOut {
    int32_t* idx_out;
    float* scores_out;
    int fused;
};

// KB = 2: bf16 keys and queries (kind::f16).  KB = 1: E4M3 keys with one fp32 scale per
// key (k_scale), bf16 queries quantised here per head to E4M3 (kind::f8f6f4); the score
// is then k_scale[s] * sum_h (w_h * q_scale_h) ReLU(q8_h . k8_s), which equals the boxed
// formula on the dequantised operands because the scales are non-negative.
template <int NH, int CI, int KB, bool KF4 = false>
__global__ void __launch_bounds__(kTcThreads, 1)
scan_tc_kernel(const __grid_constant__ CUtensorMap tmap, const void* __restrict__ tmap_base,
               const __nv_bfloat16* __restrict__ qI, const float* __restrict__ wI, const float* __restrict__ k_scale,
               const int64_t* __restrict__ t, int nq, int64_t N_cap, int m, int k, TopkWs ws, SelOut so)
{
    using Cfg = ScanCfg<NH, CI, KB>;
    constexpr int S = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned; an offset from the __shared__ array keeps every derived pointer in
    // the shared window, so its accesses compile to shared-memory instructions
    uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = smem;
    uint8_t* sB = sA + S * Cfg::kAStage;
    float* s_sc = reinterpret_cast<float*>(sB + Cfg::kBBytes);  // [kCacheTiles * 128] own scores
    float* sw = s_sc + Cfg::kCacheTiles * kTileKeys;
    uint32_t* sh = reinterpret_cast<uint32_t*>(sw + NH);
    uint64_t* full = reinterpret_cast<uint64_t*>(sh + kBins);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;
    uint64_t* tempty = tfull + 2;
    uint64_t* done = tempty + 2;
    uint64_t* qready = done + 1;  // q^I and w^I staged by the epilogue warps
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qready + 1);
    volatile uint32_t* abort_flag = tmem_slot + 1;

    __shared__ sel::Shared ss;  // scalars of the in-place select
    pdl_launch_dependents();
    const int g = blockIdx.y;
    const int64_t b = g / nq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(&tfull[a], 1);
            tc::mbar_init(&tempty[a], 128);
        }
        tc::mbar_init(done, 1);
        tc::mbar_init(qready, 256);
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tmap);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    // Everything above only touched this CTA's own shared memory and TMEM, so it may
    // overlap the previous kernel; global memory is read only after the wait below.  The
    // first key tiles of this CTA (and its query) are prefetched into L2 before it: a
    // hint that returns nothing, safe before the wait because L2 is the device's point of
    // coherence (an entry the previous kernel appends is updated in L2), so their DRAM
    // reads overlap the previous kernel instead of starting the scan.
    if (threadIdx.x == 32) {
        constexpr int kRowBytes = KF4 ? CI / 2 : CI * KB;  // one key in global memory
        const char* kb = static_cast<const char*>(tmap_base) + (size_t)b * N_cap * kRowBytes;
        const int64_t tiles_cap = (N_cap + kTileKeys - 1) / kTileKeys;
        for (int i = 0; i < kPrefetchTiles; ++i) {
            const int64_t tile = blockIdx.x + (int64_t)i * gridDim.x;
            if (tile >= tiles_cap) break;
            const int64_t rows = min((int64_t)kTileKeys, N_cap - tile * kTileKeys);
            tc::prefetch_l2(kb + tile * kTileKeys * kRowBytes, (uint32_t)(rows * kRowBytes));
        }
        tc::prefetch_l2(qI + (int64_t)g * NH * CI, NH * CI * 2);
    }
    pdl_wait();
    // the workspace's wait-budget override, a test hook read by the thread that later runs
    // the select's meetings: issued here, where its round trip overlaps the scan
    long long budget_ov = 0;
    if (threadIdx.x == 64) budget_ov = *reinterpret_cast<const volatile long long*>(ws.status + 2);
    const int64_t vis = visible_of(t, g, m, N_cap);
    const int ntiles = (int)((vis + kTileKeys - 1) / kTileKeys);
    const bool active = (int)blockIdx.x < ntiles;  // otherwise the CTA is idle for this query
    const bool need_hist = active && vis > k;

    if (!active) {
        // no key tile for this CTA: fall through to the TMEM release
    } else if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t stream_policy = tc::l2_evict_first_policy();  // every key is read once
            int it = 0;
            for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1;
                if (*abort_flag) break;
                if (!tc::mbar_wait(&empty[s], ph ^ 1, tc::kWaitBudget)) {
                    *abort_flag = 1;
                    break;
                }
                // packed E2M1 codes count their global bytes (half the unpacked tile)
                tc::mbar_arrive_expect_tx(&full[s], KF4 ? Cfg::kAStage / 2 : Cfg::kAStage);
                const int row0 = (int)(b * N_cap) + tile * kTileKeys;
#pragma unroll
                for (int p = 0; p < Cfg::kPanels; ++p)
                    tc::tma_load_2d_hint(sA + s * Cfg::kAStage + p * (kTileKeys * 128), &tmap, &full[s],
                                         Cfg::kPanelElems * p, row0, stream_policy);
            }
            // drain: every issued load has landed before the CTA may exit
            for (int j = it - S < 0 ? 0 : it - S; j < it; ++j)
                if (!tc::mbar_wait(&full[j % S], (j / S) & 1, tc::kWaitBudget)) *abort_flag = 1;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdesc = KB == 2 ? tc::idesc_bf16_f32(128, NH, false, false)
                                        : KF4   ? tc::idesc_e2m1_e4m3_f32(128, NH)
                                                : tc::idesc_e4m3_f32(128, NH);
            if (!tc::mbar_wait(qready, 0, tc::kWaitBudget)) *abort_flag = 1;
            int it = 0;
            for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
                const int s = it % S;
                const uint32_t ph = (it / S) & 1;
                const int acc = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                if (*abort_flag) break;
                if (!tc::mbar_wait(&tempty[acc], aph ^ 1, tc::kWaitBudget) ||
                    !tc::mbar_wait(&full[s], ph, tc::kWaitBudget)) {
                    *abort_flag = 1;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t d = tmem_base + acc * NH;
                const uint32_t a0 = tc::smem_u32(sA + s * Cfg::kAStage);
                const uint32_t b0 = tc::smem_u32(sB);
#pragma unroll
                for (int p = 0; p < Cfg::kPanels; ++p) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = tc::smem_desc_sw128(a0 + p * (kTileKeys * 128) + kk * 32, 16, 1024);
                        const uint64_t bd = tc::smem_desc_sw128(b0 + p * (NH * 128) + kk * 32, 16, 1024);
                        if constexpr (KB == 2)
                            tc::mma_bf16_ss(d, ad, bd, kIdesc, (p | kk) ? 1u : 0u);
                        else
                            tc::mma_e4m3_ss(d, ad, bd, kIdesc, (p | kk) ? 1u : 0u);
                    }
                }
                tc::mma_commit(&empty[s]);     // smem stage free once these MMAs finish
                tc::mma_commit(&tfull[acc]);   // accumulator ready for the epilogue
            }
            tc::mma_commit(done);              // all issued MMAs complete before TMEM is freed
            if (!tc::mbar_wait(done, 0, tc::kWaitBudget)) *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // first stage q^I (128-byte-swizzled K-major), w^I and the histogram while the
        // producer's first key tiles are already in flight
        {
            const int et = threadIdx.x - 64;  // 0..255
            const __nv_bfloat16* qg = qI + (int64_t)g * NH * CI;
            if constexpr (KB == 2) {
                constexpr int kChunks = NH * CI / 8;  // 16-byte chunks
                constexpr int kPer = (kChunks + 255) / 256;
                uint4 v[kPer];
#pragma unroll
                for (int u = 0; u < kPer; ++u) {  // all loads first: one round trip
                    const int i = et + u * 256;
                    if (i < kChunks) {
                        const int r = i / (CI / 8), cc = i % (CI / 8);
                        v[u] = __ldg(reinterpret_cast<const uint4*>(qg + (int64_t)r * CI + cc * 8));
                    }
                }
#pragma unroll
                for (int u = 0; u < kPer; ++u) {
                    const int i = et + u * 256;
                    if (i < kChunks) {
                        const int r = i / (CI / 8), cc = i % (CI / 8);
                        *reinterpret_cast<uint4*>(sB + (cc / 8) * (NH * 128) + tc::sw128_offset(r, cc % 8)) = v[u];
                    }
                }
                for (int i = et; i < NH; i += 256) sw[i] = wI[(int64_t)g * NH + i];
            } else {
                // one warp per head: E4M3 codes of q_h / scale_h, scale_h = max|q_h| / 448,
                // and the head weight folded with the scale (w_h * scale_h)
                constexpr int V = CI / 32;  // elements per lane (4 or 8)
                constexpr int HW = NH / 8;  // heads per warp
                const int ew = et >> 5, el = et & 31;
                // every load of this warp's heads first (one round trip), V bf16 per head
                // and the head weights
                uint32_t raw[HW][V / 2];
                float wv[HW];
#pragma unroll
                for (int i = 0; i < HW; ++i) wv[i] = __ldg(&wI[(int64_t)g * NH + ew + 8 * i]);
#pragma unroll
                for (int i = 0; i < HW; ++i) {
                    const __nv_bfloat16* src = qg + (int64_t)(ew + 8 * i) * CI + el * V;
                    if constexpr (V == 4) {
                        const uint2 u2 = __ldg(reinterpret_cast<const uint2*>(src));
                        raw[i][0] = u2.x;
                        raw[i][1] = u2.y;
                    } else {
                        const uint4 u4 = __ldg(reinterpret_cast<const uint4*>(src));
                        raw[i][0] = u4.x; raw[i][1] = u4.y; raw[i][2] = u4.z; raw[i][3] = u4.w;
                    }
                }
#pragma unroll
                for (int i = 0; i < HW; ++i) {
                    const int h = ew + 8 * i;
                    float x[V];
#pragma unroll
                    for (int u = 0; u < V / 2; ++u) {
                        x[2 * u] = __uint_as_float(raw[i][u] << 16);
                        x[2 * u + 1] = __uint_as_float(raw[i][u] & 0xffff0000u);
                    }
                    float amax = 0.f;
#pragma unroll
                    for (int u = 0; u < V; ++u) amax = fmaxf(amax, fabsf(x[u]));
#pragma unroll
                    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                    const float sc = e4m3_scale(amax), f = e4m3_factor(amax);
                    uint32_t w[V / 4];
#pragma unroll
                    for (int u = 0; u < V; u += 4)
                        w[u / 4] = e4m3x2(x[u], x[u + 1], f) | (e4m3x2(x[u + 2], x[u + 3], f) << 16);
                    const int byte = el * V;  // column of the first code = byte in the row
                    uint8_t* dst = sB + (byte / 128) * (NH * 128) + tc::sw128_offset(h, (byte % 128) / 16) + byte % 16;
                    if constexpr (V == 4)
                        *reinterpret_cast<uint32_t*>(dst) = w[0];
                    else
                        *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
                    if (el == 0) sw[h] = wv[i] * sc;
                }
            }
            if (need_hist)
                for (int i = et; i < kBins; i += 256) sh[i] = 0;
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(qready);
            asm volatile("bar.sync 1, 256;" ::: "memory");  // epilogue warps only
        }
        // group 0 (warps 2-5) drains accumulator 0 (even tiles), group 1 (warps 6-9)
        // accumulator 1 (odd tiles), so each group has two tile periods per tile
        const int quarter = warp & 3;          // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;
        const int eg = (warp - 2) >> 2;
        float* scores = ws.scores + (int64_t)g * ws.ld;
        int it = eg;
        for (int tile = blockIdx.x + eg * gridDim.x; tile < ntiles; tile += 2 * gridDim.x, it += 2) {
            const int acc = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            const int64_t sidx = (int64_t)tile * kTileKeys + row;
            float ksc = 1.f;  // E4M3 keys: the key's scale, fetched before the wait
            if constexpr (KB == 1) ksc = sidx < vis ? __ldg(&k_scale[b * N_cap + sidx]) : 0.f;
            if (*abort_flag) break;
            if (!tc::mbar_wait(&tfull[acc], aph, tc::kWaitBudget)) {
                *abort_flag = 1;
                break;
            }
            tc::fence_after_sync();
            float v[NH];
            const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * NH;
#pragma unroll
            for (int c0 = 0; c0 < NH; c0 += 16) tc::tmem_ld16(taddr + c0, v + c0);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            tc::mbar_arrive(&tempty[acc]);
            // 4 independent chains (h = 0, 1, 2, 3 mod 4), not one of NH; two per packed FMA
            float2 p01 = make_float2(0.f, 0.f), p23 = make_float2(0.f, 0.f);
#pragma unroll
            for (int h = 0; h < NH; h += 4) {
                const float4 w4 = *reinterpret_cast<const float4*>(sw + h);
                p01 = tc::fma2(make_float2(fmaxf(v[h], 0.f), fmaxf(v[h + 1], 0.f)), make_float2(w4.x, w4.y), p01);
                p23 = tc::fma2(make_float2(fmaxf(v[h + 2], 0.f), fmaxf(v[h + 3], 0.f)), make_float2(w4.z, w4.w), p23);
            }
            float sc = (p01.x + p01.y) + (p23.x + p23.y);
            if constexpr (KB == 1) sc *= ksc;
            if (sidx < vis) {
                if (!so.fused) {
                    scores[sidx] = sc;
                } else if (vis <= k) {  // everything visible is selected, in index order
                    so.idx_out[(int64_t)g * k + sidx] = (int32_t)sidx;
                    if (so.scores_out) so.scores_out[(int64_t)g * k + sidx] = sc;
                } else if (it < Cfg::kCacheTiles) {
                    s_sc[it * kTileKeys + row] = sc;
                } else {
                    scores[sidx] = sc;
                }
            }
            // the digit-0 histogram: one shared atomic per key (aggregating equal digits
            // across the warp first measured slower)
            if (need_hist && sidx < vis) atomicAdd(&sh[hist_slot(order_key(sc) >> 20)], 1u);
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (active && *abort_flag && threadIdx.x == 0) atomicExch(ws.status, 1u);
    if (need_hist) {
        uint32_t* gh = ws.hist0 + (size_t)g * kBins;
        if (so.fused) {
            // the in-place select places its keys from the counts merged before its own
            // (the atomics' return values), kept per bin in the idle ring; every atomic
            // is issued before the first return value is needed
            uint32_t* s_old = reinterpret_cast<uint32_t*>(sA + Cfg::kOldOff);
            constexpr int kM = (kBins + kTcThreads - 1) / kTcThreads;
            uint32_t c[kM], o[kM];
#pragma unroll
            for (int u = 0; u < kM; ++u) {
                const int i = threadIdx.x + u * kTcThreads;
                c[u] = i < kBins ? sh[i] : 0u;
            }
#pragma unroll
            for (int u = 0; u < kM; ++u) o[u] = c[u] ? atomicAdd(&gh[threadIdx.x + u * kTcThreads], c[u]) : 0u;
#pragma unroll
            for (int u = 0; u < kM; ++u)
                if (c[u]) s_old[threadIdx.x + u * kTcThreads] = o[u];
        } else {
            for (int i = threadIdx.x; i < kBins; i += kTcThreads)
                if (sh[i]) atomicAdd(&gh[i], sh[i]);
        }
    }
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
    if (!so.fused) return;
    __syncthreads();  // the arrival below releases every thread's histogram atomics
    if (warp < 2) return;

    // ---------------------------------------------------------------- in-place top-k
    // The epilogue warps (256 threads, named barrier 1) select from this CTA's scores.
    // Every CTA of the query is resident (the launch keeps the grid within one wave), so
    // they can meet at counters; every wait is bounded.
    using Bar = sel::NamedBar<1>;
    constexpr int T = sel::kSelThreads;
    const int tid = threadIdx.x - 64;
    const sel::Query q = sel::query_view(ws, g, k, so.idx_out, so.scores_out);
    if (vis <= k) {  // padding after the visible entries (written by the epilogue above)
        for (int64_t p = vis + (int64_t)blockIdx.x * T + tid; p < k; p += (int64_t)gridDim.x * T) {
            q.idx_out[p] = -1;
            if (q.sc_out) q.sc_out[p] = -INFINITY;
        }
        return;
    }
    const float* scores = ws.scores + (int64_t)g * ws.ld;
    const int my_tiles = active ? (ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    const int npos = my_tiles * kTileKeys;  // CTA-local positions: tile ordinal * 128 + row
    const uint32_t vis32 = (uint32_t)vis;   // < 2^31 (checked by the host)
    // position j = tile ordinal * 128 + row holds key (blockIdx.x + ordinal * gridDim.x) * 128 + row;
    // kSelThreads = 2 tiles, so from one u to the next the key advances by 2 * gridDim.x tiles
    static_assert(T == 2 * kTileKeys, "two tiles per classification step");
    const uint32_t key_step = 2u * gridDim.x * kTileKeys;
    auto load_keys = [&](int base, uint32_t (&key)[sel::kPer], uint32_t (&eidx)[sel::kPer], bool (&valid)[sel::kPer]) {
        const int j0 = base + tid;
        const int ord0 = j0 / kTileKeys;
        const uint32_t s0 = (blockIdx.x + (uint32_t)ord0 * gridDim.x) * kTileKeys + (uint32_t)(j0 % kTileKeys);
#pragma unroll
        for (int u = 0; u < sel::kPer; ++u) {
            const int j = j0 + u * T;
            const uint32_t s = s0 + (uint32_t)u * key_step;
            valid[u] = j < npos && s < vis32;
            eidx[u] = s;
            key[u] = valid[u] ? order_key(ord0 + 2 * u < Cfg::kCacheTiles ? s_sc[j] : __ldcg(&scores[s])) : 0u;
        }
    };

    // first meeting: every CTA's histogram is merged
    // tid 0 (thread 64, which read the override) runs both meetings
    const long long budget = budget_ov > 0 ? budget_ov : tc::kWaitBudget;
    if (tid == 0) {
        red_release_add(&q.ctr[3], 1u);
        const bool ok = wait_count_geq(&q.ctr[3], gridDim.x, budget);
        if (!ok) atomicExch(ws.status, 1u);
        // a timed-out meeting or an aborted scan leaves the query's workspace for the
        // last CTA to clear in full
        if (!ok || *abort_flag) q.ctr[kCtrDirty] = 1u;
        ss.ok = ok;
    }
    Bar::sync();
    const bool ok = ss.ok != 0;
    uint32_t* s_old = reinterpret_cast<uint32_t*>(sA + Cfg::kOldOff);  // the ring is idle now
    uint32_t* s_gh = reinterpret_cast<uint32_t*>(sA + Cfg::kGhOff);
    uint2* s_cand = reinterpret_cast<uint2*>(sA + Cfg::kCandOff);
    bool fast = false;
    if (ok) {
        sel::load_hist(s_gh, q.hist0, tid);
        Bar::sync();
        sel::threshold_and_suffix<Bar>(s_gh, (uint32_t)k, &ss, tid);
        fast = ss.cnt <= (uint32_t)Cfg::kFastCap;  // the same decision in every CTA
    }

    if (fast) {
        // Every key's output slot follows from counts alone.  The merged histogram, turned
        // into per-bin counts of the bins above (s_gh), orders the bins; inside a bin the
        // CTAs are ordered by their merge atomics (s_old: the bin's count merged before
        // this CTA's) and a CTA's own keys by a shared-memory countdown on its local
        // histogram.  Keys above the threshold bin b0 are emitted at once; b0's keys go to
        // the global candidate list at the same kind of slot.  After a second meeting
        // every CTA loads that list (at most kFastCap entries) and ranks a 1/gridDim.x
        // share of it against the whole list: the candidate of rank r (larger score
        // first, ties to the smaller index) is selected when r < k - above and goes to
        // slot above + r.  The last CTA by an atomic ticket (taken after the second
        // meeting, read at the end) clears the counters; each CTA clears its share of the
        // merged histogram.
        const uint32_t b0 = ss.bin, above = ss.above, nb0 = ss.cnt;
        for (int base = 0; base < npos; base += sel::kRound) {
            uint32_t key[sel::kPer], eidx[sel::kPer];
            bool valid[sel::kPer];
            load_keys(base, key, eidx, valid);
#pragma unroll
            for (int u = 0; u < sel::kPer; ++u) {
                const uint32_t d0 = key[u] >> 20;
                if (!valid[u] || d0 < b0) continue;
                const uint32_t sl = hist_slot(d0);
                const uint32_t r = atomicSub(&sh[sl], 1u) - 1u;
                const uint2 kv = make_uint2(key[u], eidx[u]);
                if (d0 > b0) {
                    sel::emit(q, s_gh[sl] + s_old[sl] + r, kv);
                } else {
                    const uint32_t c = s_old[sl] + r;
                    if (c < nb0) q.cand[c] = kv;  // always, unless the scan was aborted
                }
            }
        }
        Bar::sync();  // the arrival below releases every thread's candidate stores
        uint32_t ticket = 0;
        if (tid == 0) {
            red_release_add(&q.ctr[4], 1u);
            const bool ok2 = wait_count_geq(&q.ctr[4], gridDim.x, budget);
            if (!ok2) {
                atomicExch(ws.status, 1u);
                q.ctr[kCtrDirty] = 1u;
            }
            ss.ok = ok2;
            ticket = atom_acq_rel_add(&q.ctr[2], 1u);  // read at the end: the round trip overlaps the rest
        }
        Bar::sync();
        if (ss.ok) {
            // every CTA has read the merged histogram: clear this CTA's share of it
            const uint32_t per4 = (kBins / 4 + gridDim.x - 1) / gridDim.x;
            const uint32_t z0 = blockIdx.x * per4, z1 = min((uint32_t)(kBins / 4), z0 + per4);
            for (uint32_t i = z0 + tid; i < z1; i += T)
                reinterpret_cast<uint4*>(q.hist0)[i] = make_uint4(0, 0, 0, 0);
            constexpr int kLd = Cfg::kFastCap / T;
            uint2 v[kLd];
#pragma unroll
            for (int u = 0; u < kLd; ++u) {
                const uint32_t i = tid + u * T;
                v[u] = i < nb0 ? __ldcg(&q.cand[i]) : make_uint2(0, 0);
            }
#pragma unroll
            for (int u = 0; u < kLd; ++u) {
                const uint32_t i = tid + u * T;
                if (i < nb0) s_cand[i] = v[u];
            }
            Bar::sync();
            const uint32_t need = (uint32_t)k - above;
            const uint32_t per = (nb0 + gridDim.x - 1) / gridDim.x;
            const uint32_t c0 = min(nb0, blockIdx.x * per), c1 = min(nb0, c0 + per);
            const uint32_t wl = (uint32_t)tid & 31u;
            for (uint32_t i = c0 + (uint32_t)(tid >> 5); i < c1; i += T / 32) {  // a warp per candidate
                const uint2 me = s_cand[i];
                uint32_t rank = 0;
                for (uint32_t j = wl; j < nb0; j += 32) {
                    const uint2 o = s_cand[j];
                    rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
                }
                rank = __reduce_add_sync(0xffffffffu, rank);
                if (wl == 0 && rank < need) sel::emit(q, above + rank, me);
            }
        }
        if (tid == 0) {
            ss.last = ticket == gridDim.x - 1;
            ss.nt = ss.last ? __ldcg(&q.ctr[kCtrDirty]) : 0u;  // read before the reset below
        }
        Bar::sync();
        if (ss.last) sel::reset_query(q, tid, ss.nt != 0u);
        return;
    }
    uint2* s_listA = reinterpret_cast<uint2*>(sA);
    uint2* s_listB = s_listA + sel::kListCap;

    // Fallback (a threshold bin of more than kFastCap keys, or a timed-out meeting): each
    // CTA emits its keys above b0 and appends b0's to the candidate list through global
    // counters; the last CTA (atomic ticket) resolves the candidates digit by digit.
    if (ok) {
        const uint32_t b0 = ss.bin;
        for (int base = 0; base < npos; base += sel::kRound) {
            uint32_t key[sel::kPer], eidx[sel::kPer];
            bool valid[sel::kPer];
            load_keys(base, key, eidx, valid);
            sel::classify_round<Bar>(q, key, eidx, valid, b0, s_listA, s_listB, &ss, tid);
        }
    }
    Bar::sync();  // the ticket releases this CTA's candidate writes (and acquires the others')
    if (tid == 0) ss.last = atom_acq_rel_add(&q.ctr[2], 1u) == gridDim.x - 1;
    Bar::sync();
    if (!ss.last) return;
    if (ok) sel::resolve_candidates<Bar>(q, sh, s_listA, s_listB, &ss, tid);
    Bar::sync();
    sel::reset_query(q, tid);
}

template <int NH, int CI, int KB, bool KF4 = false>
int launch_nh_ci(const CUtensorMap& tmap, const void* KI, const void* qI, const float* wI, const float* k_scale, const int64_t* t,
                 int B, int nq, int64_t N_cap, int m, int k, const TopkWs& ws, int32_t* idx_out,
                 float* scores_out, bool* fused, cudaStream_t stream)
{
    using Cfg = ScanCfg<NH, CI, KB>;
    auto kern = scan_tc_kernel<NH, CI, KB, KF4>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    const int G = B * nq;
    const int64_t tiles = (N_cap + kTileKeys - 1) / kTileKeys;
    // The in-place select makes the CTAs of a query wait for one another, so it is used
    // only when the whole grid fits in one wave of resident CTAs.
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kTcThreads, Cfg::kSmem);
    const int64_t resident = (int64_t)sms * per_sm;
    int64_t ctas;
    if (resident >= G) {
        ctas = resident / G;
        *fused = true;
    } else {
        ctas = (kNumSMs + G - 1) / G;
        *fused = false;
    }
    if (ctas > tiles) ctas = tiles;
    if (ctas < 1) ctas = 1;
    SelOut so;
    so.idx_out = idx_out;
    so.scores_out = scores_out;
    so.fused = *fused ? 1 : 0;
    dim3 grid((unsigned)ctas, (unsigned)G);
    launch_pdl(kern, grid, dim3(kTcThreads), Cfg::kSmem, stream, tmap, KI, static_cast<const __nv_bfloat16*>(qI), wI,
               k_scale, t, nq, N_cap, m, k, ws, so);
    return launch_status();
}

}  // namespace

bool indexer_tc_supported(int n_hI, int cI)
{
    return (n_hI == 16 || n_hI == 32 || n_hI == 64 || n_hI == 128) && (cI == 64 || cI == 128 || cI == 256);
}

int launch_scan_tc(const void* qI, const float* wI, const void* KI, const int64_t* t, int B, int nq,
                   int64_t N_cap, int n_hI, int cI, int m, int k, const TopkWs& ws, int32_t* idx_out,
                   float* scores_out, bool* fused, cudaStream_t stream)
{
    *fused = false;
    if (N_cap == 0) return CSA_OK;
    if ((int64_t)B * N_cap + kTileKeys >= (int64_t(1) << 31) || !aligned16(qI) || !aligned16(KI))
        return launch_scan_cuda_core(qI, wI, KI, t, B, nq, N_cap, n_hI, cI, m, k, ws, CSA_BF16, stream);
    CUtensorMap tmap;
    if (!make_tmap_bf16_2d(&tmap, KI, (uint64_t)B * N_cap, cI, cI, 64, kTileKeys)) return CSA_ERR_CUDA;
#define CSA_SCAN_CASE(NH_, CI_) \
    if (n_hI == NH_ && cI == CI_)   \
        return launch_nh_ci<NH_, CI_, 2>(tmap, KI, qI, wI, nullptr, t, B, nq, N_cap, m, k, ws, idx_out, scores_out, fused, stream);
    CSA_SCAN_CASE(16, 64) CSA_SCAN_CASE(16, 128) CSA_SCAN_CASE(16, 256)
    CSA_SCAN_CASE(32, 64) CSA_SCAN_CASE(32, 128) CSA_SCAN_CASE(32, 256)
    CSA_SCAN_CASE(64, 64) CSA_SCAN_CASE(64, 128) CSA_SCAN_CASE(64, 256)
    CSA_SCAN_CASE(128, 64) CSA_SCAN_CASE(128, 128) CSA_SCAN_CASE(128, 256)
#undef CSA_SCAN_CASE
    return CSA_ERR_UNSUPPORTED;
}

bool indexer_e4m3_supported(int n_hI, int cI)
{
    return (n_hI == 16 || n_hI == 32 || n_hI == 64 || n_hI == 128) && (cI == 128 || cI == 256);
}

int launch_scan_tc_e4m3(const void* qI, const float* wI, const void* KI8, const float* k_scale, const int64_t* t,
                        int B, int nq, int64_t N_cap, int n_hI, int cI, int m, int k, const TopkWs& ws,
                        int32_t* idx_out, float* scores_out, bool* fused, cudaStream_t stream)
{
    *fused = false;
    if (N_cap == 0) return CSA_OK;
    if ((int64_t)B * N_cap + kTileKeys >= (int64_t(1) << 31)) return CSA_ERR_UNSUPPORTED;
    if (!aligned16(qI) || !aligned16(KI8)) return CSA_ERR_ALIGN;
    CUtensorMap tmap;  // E4M3 keys [B * N_cap rows][cI bytes], 128 x 128 boxes
    if (!make_tmap_u8_2d(&tmap, KI8, (uint64_t)B * N_cap, cI, cI, 128, kTileKeys)) return CSA_ERR_CUDA;
#define CSA_SCAN8_CASE(NH_, CI_) \
    if (n_hI == NH_ && cI == CI_)   \
        return launch_nh_ci<NH_, CI_, 1>(tmap, KI8, qI, wI, k_scale, t, B, nq, N_cap, m, k, ws, idx_out, scores_out, fused, stream);
    CSA_SCAN8_CASE(16, 128) CSA_SCAN8_CASE(16, 256) CSA_SCAN8_CASE(32, 128) CSA_SCAN8_CASE(32, 256)
    CSA_SCAN8_CASE(64, 128) CSA_SCAN8_CASE(64, 256) CSA_SCAN8_CASE(128, 128) CSA_SCAN8_CASE(128, 256)
#undef CSA_SCAN8_CASE
    return CSA_ERR_UNSUPPORTED;
}

bool indexer_e2m1_supported(int n_hI, int cI)
{
    return (n_hI == 16 || n_hI == 32 || n_hI == 64 || n_hI == 128) && (cI == 128 || cI == 256);
}

int launch_scan_tc_e2m1(const void* qI, const float* wI, const void* KI4, const float* k_scale, const int64_t* t,
                        int B, int nq, int64_t N_cap, int n_hI, int cI, int m, int k, const TopkWs& ws,
                        int32_t* idx_out, float* scores_out, bool* fused, cudaStream_t stream)
{
    *fused = false;
    if (N_cap == 0) return CSA_OK;
    if ((int64_t)B * N_cap + kTileKeys >= (int64_t(1) << 31)) return CSA_ERR_UNSUPPORTED;
    if (!aligned16(qI) || ((uintptr_t)KI4 & 31)) return CSA_ERR_ALIGN;
    CUtensorMap tmap;  // E2M1 codes [B * N_cap rows][cI codes], 128 x 128 boxes, unpacked to 1 byte per code
    if (!make_tmap_e2m1_2d(&tmap, KI4, (uint64_t)B * N_cap, cI, kTileKeys)) return CSA_ERR_CUDA;
#define CSA_SCAN4_CASE(NH_, CI_) \
    if (n_hI == NH_ && cI == CI_)   \
        return launch_nh_ci<NH_, CI_, 1, true>(tmap, KI4, qI, wI, k_scale, t, B, nq, N_cap, m, k, ws, idx_out, scores_out, fused, stream);
    CSA_SCAN4_CASE(16, 128) CSA_SCAN4_CASE(16, 256) CSA_SCAN4_CASE(32, 128) CSA_SCAN4_CASE(32, 256)
    CSA_SCAN4_CASE(64, 128) CSA_SCAN4_CASE(64, 256) CSA_SCAN4_CASE(128, 128) CSA_SCAN4_CASE(128, 256)
#undef CSA_SCAN4_CASE
    return CSA_ERR_UNSUPPORTED;
}

}  // namespace csa
