// Shared-KV MQA over compressed entries on the 5th-generation tensor cores
// ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch", section 8 sparse over the
// top-k entries, section 10 dense over all visible entries; key = value = entry).
//
// For one query, S = Q C^T (128 heads x entries, K = c = 512) and O = softmax(S) C
// (128 heads x 512) are dense contractions against entries shared by every head, so
// both run on tcgen05 with the heads as the M = 128 dimension.  An fp32 accumulator for
// all 512 output columns would fill the whole 512-column TMEM and leave no room for S,
// so each range ("split") of the entry list is worked by two CTAs, one per half of c:
//   - both CTAs hold the whole q (128 KB) and, for each chunk of 32 entries, the whole
//     entry rows, and both compute the full logits S (K = 512) with the same MMAs in
//     the same order, so their S, softmax and (max, sum) are bit-identical and the two
//     CTAs never communicate;
//   - CTA r accumulates only its half of the output, O[:, 256r : 256r+256] += P C[:, half]
//     (N = 256), in TMEM.
// The redundant S costs tensor-pipe time, which a decode query has to spare; in exchange
// no partial logits cross between CTAs, which removes a dependent exchange from every
// chunk and lets the two CTAs run anywhere on the GPU (no cluster).
// Entries are gathered by index with 16-byte cp.async (contiguous dense chunks by TMA)
// into a double-buffered 128-byte-swizzled tile; the same bytes are the K-major B
// operand of S and, for the CTA's four 64-column panels, the MN-major B operand of P C.
//   warps 0-3 loaders  : L2 prefetches, q (once) and the entry chunks -> shared memory;
//                        at the end, output columns 0..127 -> staging; thread 0 issues
//                        the TMA stores of the staged output half
//   warps 4-7, 9-12    : softmax, two groups (entries 0-15 and 16-31 of a chunk, one
//                        thread per row in each): S from TMEM, online softmax with lazy
//                        rescaling (O is rescaled in TMEM only when the running max grows
//                        by more than 2^8), P (bf16) -> shared memory; at the end, output
//                        columns 128..255 -> staging
//   warp 8    MMA      : issues S(j) and P(j) C as soon as each is ready
// A split's partial is its normalised output O_i / l_i, rounded to bf16 (relative error
// at most 2^-9 per element, the same as the bf16 P fed to the tensor core) and written
// by TMA, with its running max and sum in base 2 in fp32; the combine kernel of attn.cu
// merges the splits in fp32.  Every barrier wait is bounded; a
// timeout sets the workspace status word and the CTA drains and exits.
#include "attn.cuh"
#include "attn_tc.cuh"

namespace csa {
namespace {
using namespace atc;

constexpr int kE = 32;              // entries per chunk (N of S, K of P C)
constexpr int kPanels = kC / 64;    // 128-byte column panels of q and of a chunk
constexpr int kLoaders = 128;
constexpr int kThreads = 416;       // 4 loader warps, 4 softmax warps, the MMA warp, 4 softmax warps
constexpr int kMmaWarp = 8;
constexpr int kSoftmax = 256;       // softmax threads: two per row
constexpr int kQBytes = kHeads * kC * 2;          // 128 KB: 8 panels of 128 rows x 128 B
constexpr int kQPanel = kHeads * 128;             // 16 KB
constexpr int kCBytes = kE * kC * 2;              // 32 KB: 8 panels of 32 rows x 128 B
constexpr int kCPanel = kE * 128;                 // 4 KB
constexpr int kPBytes = kHeads * 128;             // 16 KB: 128 rows x 128 B (the first 64 B used)
constexpr int kMaxIds = 1024;                     // entry ids of a range staged in smem
constexpr int kBarBytes = 256;
constexpr int kXBytes = (2 * 2 + 2) * kHeads * 4; // row maxima [2 chunks][2 groups][128], sums [2][128]
constexpr int kSmem = 1024 + kQBytes + 2 * kCBytes + kPBytes + kBarBytes + kMaxIds * 4 + kXBytes;
static_assert(kQBytes >= kHeads * kHalf * 4, "output staging (fp32 included) reuses q");
static_assert(kSmem <= 227 * 1024, "shared memory of one CTA");

__global__ void __launch_bounds__(kThreads, 1)
attn_split_kernel(const __grid_constant__ CUtensorMap tmap_o, const __grid_constant__ CUtensorMap tmap_q,
                  const __grid_constant__ CUtensorMap tmap_c, const __grid_constant__ CUtensorMap tmap_g,
                  const __grid_constant__ CUtensorMap tmap_w, AttnArgs a, uint32_t* status)
{
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned; an offset from the __shared__ array keeps every derived pointer in
    // the shared window, so its accesses compile to shared-memory instructions
    uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sQ = smem;
    uint8_t* sC0 = sQ + kQBytes;                      // chunk buffer b at sC0 + b * kCBytes
    uint8_t* sP = sC0 + 2 * kCBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sP + kPBytes);
    uint64_t* Cfull = bars;         // [2] loaders -> MMA            (count 128)
    uint64_t* Cempty = bars + 2;    // [2] MMA commit -> loaders
    uint64_t* Sfull = bars + 4;     // [2] MMA commit -> softmax
    uint64_t* Sempty = bars + 6;    // [2] softmax -> MMA            (count 256)
    uint64_t* Pfull = bars + 8;     // softmax -> MMA                (count 256)
    uint64_t* PVdone = bars + 9;    // MMA commit -> softmax
    uint64_t* idsready = bars + 10; // loaders -> softmax            (count 128)
    uint64_t* staged = bars + 11;   // output half staged            (count 384: loaders + softmax)
    uint64_t* Ofinal = bars + 12;   // softmax -> loaders: last P C done (count 128)
    uint64_t* Qfull = bars + 13;    // q landed (TMA, count 1 + bytes)
    uint64_t* MXready = bars + 14;  // both softmax groups' row maxima written (count 256)
    uint64_t* Lready = bars + 15;   // both softmax groups' row sums written (count 256)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    int* s_ids = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(bars) + kBarBytes);  // [kMaxIds]
    float* s_inv_l = reinterpret_cast<float*>(sP);  // [128] 1 / l per head, after the last P C
    float* s_mx = reinterpret_cast<float*>(s_ids + kMaxIds);  // [2][2][128] partial row maxima
    float* s_lp = s_mx + 4 * kHeads;                          // [2][128] partial row sums

    pdl_launch_dependents();
    const int split = blockIdx.x, half = blockIdx.y, g = blockIdx.z;
    const int64_t b = g / a.nq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&Cfull[i], kLoaders);
            tc::mbar_init(&Cempty[i], 1);
            tc::mbar_init(&Sfull[i], 1);
            tc::mbar_init(&Sempty[i], kSoftmax);
        }
        tc::mbar_init(Pfull, kSoftmax);
        tc::mbar_init(PVdone, 1);
        tc::mbar_init(idsready, kLoaders);
        tc::mbar_init(MXready, kSoftmax);
        tc::mbar_init(Lready, kSoftmax);
        tc::mbar_init(Ofinal, kHeads);
        tc::mbar_init(staged, kLoaders + kSoftmax);
        tc::mbar_init(Qfull, 1);
        tc::tma_prefetch_desc(&tmap_o);
        tc::tma_prefetch_desc(&tmap_q);
        tc::tma_prefetch_desc(&tmap_c);
        tc::tma_prefetch_desc(&tmap_g);
        if (a.win) tc::tma_prefetch_desc(&tmap_w);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // Only shared memory and TMEM were touched so far (overlaps the previous kernel).  The
    // L2 prefetches of q and of a dense split's whole range (its compressed entries) go
    // out now too, so their DRAM latency overlaps the previous kernel's tail.
    if (threadIdx.x == 32) {
        const char* qp = static_cast<const char*>(a.q) + (size_t)g * kHeads * kC * 2;
#pragma unroll
        for (int i = 0; i < kQBytes / 16384; ++i) tc::prefetch_l2(qp + i * 16384, 16384);
        if (a.dense) {
            const int64_t r0 = (int64_t)split * a.per_split;
            const int64_t r1 = min(r0 + a.per_split, a.N_cap);
            const char* cp = static_cast<const char*>(a.cache) + ((size_t)b * a.N_cap) * kC * 2;
            // the two CTAs of the split prefetch alternate 16-entry blocks
            for (int64_t r = r0 + 16 * half; r < r1; r += 32)
                tc::prefetch_l2(cp + (size_t)r * kC * 2, (uint32_t)(min((int64_t)16, r1 - r) * kC * 2));
        }
    }
    if (threadIdx.x == 64) {
        // the lines of t[g] and of this split's entry ids, likewise (a line the previous
        // kernel writes afterwards is simply updated in L2)
        if (a.t) asm volatile("prefetch.global.L2 [%0];" ::"l"(a.t + g) : "memory");
        if (!a.dense)
            for (int64_t p = (int64_t)split * a.per_split; p < min((int64_t)(split + 1) * a.per_split, (int64_t)a.k);
                 p += 32)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(a.idx + (int64_t)g * a.k + p) : "memory");
    }
    pdl_wait();
    // list positions: [0, ncomp) compressed entries, then [ncomp, count) the sliding-window
    // entries of tokens wlo .. t (when a window is given)
    int64_t ncomp;
    if (a.dense) {
        const int64_t tt = a.t[g];
        const int64_t v = tt < 0 ? 0 : tt / a.m_prime;
        ncomp = v < a.N_cap ? v : a.N_cap;
    } else {
        ncomp = a.k;
    }
    int64_t nwin = 0;
    int wrow0 = 0;  // ring row of the window's first token
    if (a.win) {
        const int64_t tt = a.t[g];
        if (tt >= 0) {
            nwin = tt + 1 < a.n_win ? tt + 1 : a.n_win;
            wrow0 = (int)((tt - nwin + 1) % a.win_cap);
        }
    }
    const int64_t count = ncomp + nwin;
    const int64_t p_begin = (int64_t)split * a.per_split;
    const int64_t p_end = min(count, p_begin + a.per_split);
    const int nchunks = p_end > p_begin ? (int)((p_end - p_begin + kE - 1) / kE) : 0;
    const size_t prow = ((size_t)g * a.splits + split) * kHeads;  // partial (or output) row of head 0
    const bool f32_out = a.direct && !a.out_bf16;                  // final output in fp32
    // Code of list position p: e >= 0 compressed entry e, e <= -2 window row -2 - e, -1
    // padding or outside the cache.  Sparse ranges of up to kMaxIds positions are staged in
    // shared memory once by the loaders.
    const bool ids_staged = !a.dense && (p_end - p_begin) <= kMaxIds;
    auto entry_global = [&](int64_t p) -> int64_t {
        if (p >= p_end) return -1;
        if (p >= ncomp) {  // window position: at most one wrap of the ring (n_win <= win_cap)
            int r = wrow0 + (int)(p - ncomp);
            r = r >= a.win_cap ? r - a.win_cap : r;
            return -2 - (int64_t)r;
        }
        if (a.dense) return p;
        const int32_t v = __ldg(&a.idx[(int64_t)g * a.k + p]);
        return (v >= 0 && v < a.N_cap) ? v : -1;
    };
    auto entry_of = [&](int64_t p) -> int64_t {
        if (ids_staged) return p < p_end ? (int64_t)s_ids[p - p_begin] : -1;
        return entry_global(p);
    };
    const bool plain = a.dense && !a.win;  // position p is entry p
    if (nchunks == 0) {
        if (!a.direct) {
            // empty range: an empty partial (max -inf, sum 0) that the combine skips
            if (half == 0 && threadIdx.x < kHeads) a.part_ml[prow + threadIdx.x] = make_float2(-INFINITY, 0.f);
        } else {
            // nothing visible: output 0 and lse -inf (this CTA's half of every head row)
            for (int i = threadIdx.x; i < kHeads * kHalf; i += kThreads) {
                const size_t o = ((size_t)g * kHeads + i / kHalf) * kC + half * kHalf + i % kHalf;
                if (a.out_bf16)
                    static_cast<__nv_bfloat16*>(a.out)[o] = __float2bfloat16(0.f);
                else
                    static_cast<float*>(a.out)[o] = 0.f;
            }
            if (half == 0 && a.lse && threadIdx.x < kHeads) a.lse[(size_t)g * kHeads + threadIdx.x] = -INFINITY;
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------ loaders
        const int lt = threadIdx.x;
        if (lt == 0) {  // q: eight 128-row x 64-column TMA boxes (128-byte swizzle)
            tc::mbar_arrive_expect_tx(Qfull, kQBytes);
#pragma unroll
            for (int p = 0; p < kPanels; ++p) tc::tma_load_2d(sQ + p * kQPanel, &tmap_q, Qfull, p * 64, g * kHeads);
        }
        if (ids_staged)
            for (int64_t i = lt; i < p_end - p_begin; i += kLoaders) s_ids[i] = (int)entry_global(p_begin + i);
        tc::mbar_arrive(idsready);
        asm volatile("bar.sync 2, 128;" ::: "memory");  // loader warps: ids visible to each other
        // Every chunk arrives by TMA, counted in bytes on Cfull[buf]: chunks 0 and 1 are
        // issued at once (both buffers start free), chunk j >= 2 once P C of chunk j-2 has
        // released its buffer.  The loaders never wait for data themselves.
        for (int j = 0; j < nchunks; ++j) {
            const int buf = j & 1;
            if (*abort_flag) break;
            if (!tc::mbar_wait(&Cempty[buf], ((j >> 1) & 1) ^ 1, tc::kWaitBudget)) {
                *abort_flag = 1;
                break;
            }
            const uint32_t c0 = tc::smem_u32(sC0 + buf * kCBytes);
            const int64_t p0 = p_begin + (int64_t)j * kE;
            if (plain && p0 + kE <= p_end) {
                // a full dense chunk is one contiguous block of cache rows: eight 32 x 64
                // TMA boxes, counted in bytes on Cfull (the other loaders just arrive)
                if (lt == 0) {
                    tc::mbar_arrive_expect_tx(&Cfull[buf], kCBytes);
#pragma unroll
                    for (int p = 0; p < kPanels; ++p)
                        tc::tma_load_2d(sC0 + buf * kCBytes + p * kCPanel, &tmap_c, &Cfull[buf], p * 64,
                                        (int)(b * a.N_cap + p0));
                } else {
                    tc::mbar_arrive(&Cfull[buf]);
                }
                continue;
            }
            // gathered (or partial dense) chunk: one TMA box of 1 row x 64 columns (128 B)
            // per row and column panel, two per loader thread; a padding row (or a row
            // past the range) is loaded from row -1, which TMA fills with zeros
            {
                const int row = lt >> 2, pp = (lt & 3) * 2;
                const int64_t p = p0 + row;
                const int64_t e = plain ? (p < p_end ? p : (int64_t)-1) : entry_of(p);
                const CUtensorMap* m = e <= -2 ? &tmap_w : &tmap_g;
                const int y = e >= 0 ? (int)(b * a.N_cap + e) : (e <= -2 ? (int)(b * a.win_cap + (-2 - e)) : -1);
                uint8_t* dst = sC0 + buf * kCBytes + row * 128;
                tc::mbar_arrive_expect_tx(&Cfull[buf], 2 * 128);
                tc::tma_load_2d(dst + pp * kCPanel, m, &Cfull[buf], pp * 64, y);
                tc::tma_load_2d(dst + (pp + 1) * kCPanel, m, &Cfull[buf], (pp + 1) * 64, y);
            }
        }
        // q has landed before the CTA may move on (its barrier is used once).  The chunks
        // were consumed by the MMA warp on the normal path; after an abort the bounded
        // waits outlast any load in flight by many orders of magnitude.
        if (lt == 0 && !tc::mbar_wait(Qfull, 0, tc::kWaitBudget)) *abort_flag = 1;
        // The output half leaves through TMA: these warps stage columns 0..127 and the
        // softmax warps 128..255 once the last P C has completed (q is dead by then, so
        // its buffer is the staging area), then thread 0 stores the boxes.
        if (!*abort_flag && tc::mbar_wait(Ofinal, 0, tc::kWaitBudget)) {
            tc::fence_after_sync();
            const int h = warp * 32 + lane;
            const uint32_t ot = tmem + ((uint32_t)(warp * 32) << 16) + kHalf;
            if (f32_out)
                stage_o_cols_f32(smem, ot, h, 0, s_inv_l[h], 128);
            else
                stage_o_cols(smem, ot, h, 0, s_inv_l[h], 128);
        } else {
            *abort_flag = 1;
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(staged);
        if (threadIdx.x == 0) {
            if (tc::mbar_wait(staged, 0, tc::kWaitBudget) && !*abort_flag) {
                const int bc = f32_out ? 32 : kBoxCols;  // columns per 128-byte box row
                for (int p = 0; p < kHalf / bc; ++p)
                    tc::tma_store_2d(&tmap_o, smem + p * kBoxBytes, half * kHalf + p * bc, (int)prow);
                tc::bulk_store_commit_wait();
            } else {
                *abort_flag = 1;
            }
        }
    } else if (warp != kMmaWarp) {
        // ------------------------------------------------------------ softmax
        // Two groups of four warps: group sg owns entries [16 sg, 16 sg + 16) of every
        // chunk for all 128 rows (thread = row).  The two threads of a row agree on the
        // row maximum through a double-buffered shared exchange (bounded mbarrier wait),
        // so they keep identical running maxima and rescale decisions; each keeps its own
        // partial sum of the row.
        const int sg = warp > kMmaWarp ? 1 : 0;
        const int quarter = warp & 3;
        const int h = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        constexpr int kEG = kE / 2;  // entries of a chunk per group
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = tc::mbar_wait(idsready, 0, tc::kWaitBudget);
        for (int j = 0; j < nchunks && ok; ++j) {
            const int buf = j & 1;
            const uint32_t ph = (j >> 1) & 1;
            // the validity of this group's 16 entries, read while S is computed
            const int64_t pg = p_begin + (int64_t)j * kE + sg * kEG;  // list position of entry 0 of the group
            const unsigned vm =
                __ballot_sync(0xffffffffu, lane < kEG && (plain ? pg + lane < p_end : entry_of(pg + lane) != -1));
            if (*abort_flag || !tc::mbar_wait(&Sfull[buf], ph, tc::kWaitBudget)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            float s[kEG];
            tc::tmem_ld16(tmem + lane_base + buf * kE + sg * kEG, s);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            tc::mbar_arrive(&Sempty[buf]);
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // 4 chains, not 1
#pragma unroll
            for (int e = 0; e < kEG; ++e) {
                s[e] = ((vm >> e) & 1u) ? s[e] * a.scale_log2 : -INFINITY;
                mx[e & 3] = fmaxf(mx[e & 3], s[e]);
            }
            // the row maximum of the chunk: both groups' partial maxima, same order in both
            float* mxb = s_mx + (j & 1) * 2 * kHeads;
            mxb[sg * kHeads + h] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            tc::mbar_arrive(MXready);
            if (!tc::mbar_wait(MXready, j & 1, tc::kWaitBudget)) {
                ok = false;
                break;
            }
            const float cmax = fmaxf(mxb[h], mxb[kHeads + h]);
            if (j > 0) {
                // P buffer and O are free once the previous chunk's P C has finished
                if (!tc::mbar_wait(PVdone, (j - 1) & 1, tc::kWaitBudget)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const bool need = cmax > m_run + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    // each group rescales its 128 of the 256 output columns of the row
                    const float f = need ? (m_run == -INFINITY ? 0.f : exp2f(m_run - cmax)) : 1.f;
                    const uint32_t ob = tmem + lane_base + kHalf + sg * (kHalf / 2);
#pragma unroll 1
                    for (int c0 = 0; c0 < kHalf / 2; c0 += 16) {
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
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t packed[kEG / 2];
#pragma unroll
            for (int e = 0; e < kEG; e += 2) {
                const float p0f = (s[e] == -INFINITY) ? 0.f : tc::ex2_approx(s[e] - m_run);
                const float p1f = (s[e + 1] == -INFINITY) ? 0.f : tc::ex2_approx(s[e + 1] - m_run);
                ps[(e >> 1) & 3] += p0f + p1f;
                __nv_bfloat162 pr = __floats2bfloat162_rn(p0f, p1f);
                packed[e / 2] = *reinterpret_cast<uint32_t*>(&pr);
            }
            l_run += (ps[0] + ps[1]) + (ps[2] + ps[3]);
#pragma unroll
            for (int qc = 0; qc < kEG / 8; ++qc) {
                uint4 v = make_uint4(packed[4 * qc], packed[4 * qc + 1], packed[4 * qc + 2], packed[4 * qc + 3]);
                *reinterpret_cast<uint4*>(sP + tc::sw128_offset(h, sg * (kEG / 8) + qc)) = v;
            }
            tc::fence_proxy_async_smem();
            tc::fence_before_sync();
            tc::mbar_arrive(Pfull);
        }
        bool fin = ok && !*abort_flag && tc::mbar_wait(PVdone, (nchunks - 1) & 1, tc::kWaitBudget);
        float l_tot = 0.f;
        if (fin) {
            // the row sum: both groups' partial sums, same order in both
            s_lp[sg * kHeads + h] = l_run;
            tc::mbar_arrive(Lready);
            fin = tc::mbar_wait(Lready, 0, tc::kWaitBudget);
            if (fin) l_tot = s_lp[h] + s_lp[kHeads + h];
        } else {
            tc::mbar_arrive(Lready);
        }
        if (fin) {
            // The last P C has completed, so every MMA reading q, the chunks and P has too:
            // the q buffer stages the output half (columns 128..191 by group 0, 192..255 by
            // group 1), and the P buffer passes 1 / l to the loader warps.
            const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
            if (sg == 0) {
                s_inv_l[h] = inv;
                tc::mbar_arrive(Ofinal);
            }
            tc::fence_after_sync();
            if (f32_out)
                stage_o_cols_f32(smem, tmem + lane_base + kHalf, h, 128 + sg * 64, inv, 64);
            else
                stage_o_cols(smem, tmem + lane_base + kHalf, h, 128 + sg * 64, inv, 64);
            if (half == 0 && sg == 0) {
                if (!a.direct)
                    a.part_ml[prow + h] = make_float2(m_run, l_tot);
                else if (a.lse)  // natural-log lse of the scaled logits (m_run, l_tot in base 2)
                    a.lse[(size_t)g * kHeads + h] = l_tot > 0.f ? (m_run + log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
            }
        } else {
            if (sg == 0) tc::mbar_arrive(Ofinal);
            *abort_flag = 1;
            if (half == 0 && sg == 0 && !a.direct) a.part_ml[prow + h] = make_float2(-INFINITY, 0.f);
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(staged);
    } else {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescS = tc::idesc_bf16_f32(kHeads, kE, false, false);
            constexpr uint32_t kIdescPV = tc::idesc_bf16_f32(kHeads, kHalf, false, true);
            const uint32_t q0 = tc::smem_u32(sQ);
            const uint32_t p0 = tc::smem_u32(sP);
            // The issuer runs whichever product is ready: S(j) once chunk j has landed and
            // its TMEM buffer is free, P(j) C once the softmax has written P(j).  Neither
            // waits on the other, so the gather of chunk j + 2 (which needs P(j) C to free
            // its buffer) overlaps the softmax of chunk j + 1.
            auto issue_S = [&](int j) {
                const uint32_t c0 = tc::smem_u32(sC0 + (j & 1) * kCBytes);
#pragma unroll
                for (int p = 0; p < kPanels; ++p) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = tc::smem_desc_sw128(q0 + p * kQPanel + kk * 32, 16, 1024);
                        const uint64_t bd = tc::smem_desc_sw128(c0 + p * kCPanel + kk * 32, 16, 1024);
                        tc::mma_bf16_ss(tmem + (j & 1) * kE, ad, bd, kIdescS, (p | kk) ? 1u : 0u);
                    }
                }
                tc::mma_commit(&Sfull[j & 1]);
            };
            auto issue_PV = [&](int j) {
                // this CTA's four 64-column panels of the chunk, MN-major (64 columns x
                // 8 entries per 1024-byte atom, panels kCPanel apart)
                const uint32_t c0 = tc::smem_u32(sC0 + (j & 1) * kCBytes) + half * (kPanels / 2) * kCPanel;
#pragma unroll
                for (int kk = 0; kk < kE / 16; ++kk) {
                    const uint64_t ad = tc::smem_desc_sw128(p0 + kk * 32, 16, 1024);
                    const uint64_t bd = tc::smem_desc_sw128(c0 + kk * 16 * 128, kCPanel, 1024);
                    tc::mma_bf16_ss(tmem + kHalf, ad, bd, kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc::mma_commit(&Cempty[j & 1]);
                tc::mma_commit(PVdone);
            };
            bool ok = tc::mbar_wait(Qfull, 0, tc::kWaitBudget);
            int nS = 0, nPV = 0;  // products issued so far
            long long t_last = clock64();
            int idle = 0;
            while (ok && nPV < nchunks) {
                bool progressed = false;
                if (nS < nchunks) {
                    const int buf = nS & 1;
                    const uint32_t ph = (nS >> 1) & 1;
                    if (tc::mbar_test(&Cfull[buf], ph) && tc::mbar_test(&Sempty[buf], ph ^ 1)) {
                        tc::fence_after_sync();
                        issue_S(nS++);
                        progressed = true;
                    }
                }
                if (nPV < nS && tc::mbar_test(Pfull, nPV & 1)) {
                    tc::fence_after_sync();
                    issue_PV(nPV++);
                    progressed = true;
                }
                if (progressed) {
                    t_last = clock64();
                    idle = 0;
                } else {
                    if (*abort_flag || clock64() - t_last > tc::kWaitBudget) ok = false;
                    if (++idle >= 8) __nanosleep(32);
                }
            }
            if (!ok) *abort_flag = 1;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) atomicExch(status, 1u);
    if (warp == kMmaWarp) {
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
    p.head_groups = 1;
    int64_t max_splits = kNumSMs / (2 * (int64_t)G);  // two CTAs per split and query
    if (max_splits < 1) max_splits = 1;
    // Short lists (a decode query's top-k): one 32-entry chunk per split on the
    // full-width kernel, whose chain has no exchange.  Longer lists: the CTA-pair kernel
    // of attn_pair.cu over 64-entry chunks, which does half the MMA work per entry.
    const int64_t c32 = (entries + kE - 1) / kE;
    if (c32 <= max_splits) {
        p.kernel = 1;
        p.per_split = kE;
        p.splits = (int)(c32 > 0 ? c32 : 1);
        return p;
    }
    constexpr int kPairE = 64;
    const int64_t chunks = (entries + kPairE - 1) / kPairE;
    int64_t splits = max_splits < chunks ? max_splits : chunks;
    if (splits < 1) splits = 1;
    const int64_t per_chunks = (chunks + splits - 1) / splits;
    p.kernel = 2;
    p.per_split = per_chunks * kPairE;
    p.splits = (int)((entries + p.per_split - 1) / p.per_split);
    if (p.splits < 1) p.splits = 1;
    return p;
}

int launch_attn_tc(const AttnArgs& a, const AttnPlan& plan, uint32_t* status, cudaStream_t stream)
{
    if (plan.kernel == 2) return launch_attn_pair(a, plan, status, stream);
    if (!aligned16(a.q) || !aligned16(a.cache) || (a.win && !aligned16(a.win))) return CSA_ERR_ALIGN;
    cudaFuncSetAttribute(attn_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    // partial outputs [G * splits * 128 rows][512] bf16 in 64 x 128 boxes, or with one
    // split per query the final output [G * 128 rows][512] (bf16 boxes as above, fp32 in
    // 32 x 128 boxes)
    CUtensorMap tmap_o;
    const uint64_t rows = (uint64_t)a.B * a.nq * plan.splits * kHeads;
    bool ok_o;
    if (!a.direct)
        ok_o = make_tmap_bf16_2d(&tmap_o, a.part_o, rows, kC, kC, kBoxCols, kHeads);
    else if (a.out_bf16)
        ok_o = make_tmap_bf16_2d(&tmap_o, a.out, rows, kC, kC, kBoxCols, kHeads);
    else
        ok_o = make_tmap_f32_2d(&tmap_o, a.out, rows, kC, kC, 32, kHeads);
    if (!ok_o) return CSA_ERR_CUDA;
    CUtensorMap tmap_q;  // queries [G * 128 rows][512] bf16, 64 x 128 boxes
    if (!make_tmap_bf16_2d(&tmap_q, a.q, (uint64_t)a.B * a.nq * kHeads, kC, kC, 64, kHeads)) return CSA_ERR_CUDA;
    CUtensorMap tmap_c;  // compressed cache [B * N_cap rows][512] bf16, 64 x 32 boxes (dense chunks)
    if (!make_tmap_bf16_2d(&tmap_c, a.cache, (uint64_t)a.B * (uint64_t)(a.N_cap > 0 ? a.N_cap : 1), kC, kC, 64, kE))
        return CSA_ERR_CUDA;
    CUtensorMap tmap_g;  // the same rows, 64 x 1 boxes (gathered entries)
    if (!make_tmap_bf16_2d(&tmap_g, a.cache, (uint64_t)a.B * (uint64_t)(a.N_cap > 0 ? a.N_cap : 1), kC, kC, 64, 1))
        return CSA_ERR_CUDA;
    CUtensorMap tmap_w = tmap_g;  // sliding-window ring [B * win_cap rows][512] bf16, 64 x 1 boxes
    if (a.win && !make_tmap_bf16_2d(&tmap_w, a.win, (uint64_t)a.B * (uint64_t)a.win_cap, kC, kC, 64, 1))
        return CSA_ERR_CUDA;
    launch_pdl(attn_split_kernel, dim3((unsigned)plan.splits, 2u, (unsigned)(a.B * a.nq)), dim3(kThreads),
               (size_t)kSmem, stream, tmap_o, tmap_q, tmap_c, tmap_g, tmap_w, a, status);
    return launch_status();
}

}  // namespace csa
