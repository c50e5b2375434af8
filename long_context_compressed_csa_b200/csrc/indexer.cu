// Lightning-indexer scoring and top-k selection
// ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch", section 6.4 boxed score,
// section 7 top-k and causal rule s < floor(t/m)).
//
// Pipeline per query g (= b*nq + q):
//   1. scan   : I[s] = sum_h w[h] * ReLU(q[h] . K[s]) for every visible s, written to the
//               fp32 score buffer of the workspace, and a 4096-bin histogram of the top
//               12 bits of each score's order-preserving key (digit 0), accumulated in
//               shared memory and merged into the workspace with one atomic per
//               non-empty bin.  bf16 inputs with tensor-core shapes run on tcgen05
//               (indexer_tc.cu); everything else on CUDA cores (this file).
//   2. select : a multi-CTA radix select.  Every CTA reads the digit-0 histogram, finds
//               the bin holding the k-th largest score, emits its share of scores above
//               that bin, and appends the scores inside it to a candidate list while
//               histogramming their next 12 bits (digit 1).  The last CTA to finish
//               (atomic ticket, no spinning) resolves the candidates digit by digit on
//               the 64-bit key (score key, ~index), so ties go to the smaller index and
//               exactly k indices come out.  It then zeroes the histograms and counters
//               for the next call.
#include "common.cuh"
#include "indexer.cuh"

namespace csa {

// ----------------------------------------------------------------------------------
// workspace layout
// ----------------------------------------------------------------------------------
TopkWs topk_ws_layout(void* base, int G, int64_t N_cap)
{
    TopkWs w;
    const int64_t Np = (int64_t)align_up((size_t)(N_cap > 0 ? N_cap : 1), 64);
    char* p = static_cast<char*>(base);
    w.ld = Np;
    w.status = reinterpret_cast<uint32_t*>(p); p += 256;
    w.hist0 = reinterpret_cast<uint32_t*>(p);  p += (size_t)G * kBins * 4;
    w.hist1 = reinterpret_cast<uint32_t*>(p);  p += (size_t)G * kBins * 4;
    w.ctr = reinterpret_cast<uint32_t*>(p);    p += (size_t)G * kCtrs * 4;
    p = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(p), 256));
    w.scores = reinterpret_cast<float*>(p);    p += (size_t)G * Np * 4;
    w.cand = reinterpret_cast<uint2*>(p);      p += (size_t)G * Np * 8;
    w.cand2 = reinterpret_cast<uint2*>(p);     p += (size_t)G * Np * 8;
    w.bytes = (size_t)(p - static_cast<char*>(base));
    w.zero_bytes = 256 + (size_t)G * (2 * kBins + kCtrs) * 4;
    return w;
}

namespace {

CSA_DEV int64_t visible_count(const int64_t* t, int g, int m, int64_t N_cap)
{
    const int64_t tt = t[g];
    if (tt < 0) return 0;
    const int64_t v = tt / m;
    return v < N_cap ? v : N_cap;
}

// ----------------------------------------------------------------------------------
// CUDA-core scan: one thread per key, q and w staged in shared memory as fp32.
// ----------------------------------------------------------------------------------
constexpr int kScanThreads = 256;
constexpr int kHeadGroup = 32;

template <typename T, int V>
__global__ void __launch_bounds__(kScanThreads)
scan_cuda_core(const T* __restrict__ qI, const float* __restrict__ wI, const T* __restrict__ KI,
               const int64_t* __restrict__ t, int nq, int64_t N_cap, int n_hI, int cI, int m,
               int k, TopkWs ws)
{
    extern __shared__ float sq[];  // [n_hI * cI] q, then [n_hI] w
    __shared__ uint32_t sh[kBins];
    pdl_launch_dependents();
    pdl_wait();
    const int g = blockIdx.y;
    const int64_t b = g / nq;
    const int64_t vis = visible_count(t, g, m, N_cap);
    const int64_t s0 = (int64_t)blockIdx.x * kScanThreads;
    if (s0 >= vis) return;
    const bool need_hist = vis > k;
    float* sw = sq + n_hI * cI;
    for (int i = threadIdx.x; i < n_hI * cI; i += kScanThreads)
        sq[i] = to_f32(qI[(int64_t)g * n_hI * cI + i]);
    for (int i = threadIdx.x; i < n_hI; i += kScanThreads) sw[i] = wI[(int64_t)g * n_hI + i];
    if (need_hist)
        for (int i = threadIdx.x; i < kBins; i += kScanThreads) sh[i] = 0;
    __syncthreads();

    const int64_t s = s0 + threadIdx.x;
    if (s < vis) {
        const T* krow = KI + (b * N_cap + s) * cI;
        float score = 0.f;
        for (int h0 = 0; h0 < n_hI; h0 += kHeadGroup) {
            float acc[kHeadGroup];
#pragma unroll
            for (int hh = 0; hh < kHeadGroup; ++hh) acc[hh] = 0.f;
            for (int j0 = 0; j0 < cI; j0 += V) {
                float kv[V];
                if constexpr (V * sizeof(T) == 16) {
                    Vec<T>::load_cached(krow + j0, kv);
                } else {
#pragma unroll
                    for (int v = 0; v < V; ++v) kv[v] = to_f32(krow[j0 + v]);
                }
#pragma unroll
                for (int hh = 0; hh < kHeadGroup; ++hh) {
                    if (h0 + hh < n_hI) {
                        const float* qr = sq + (h0 + hh) * cI + j0;
#pragma unroll
                        for (int v = 0; v < V; ++v) acc[hh] = fmaf(qr[v], kv[v], acc[hh]);
                    }
                }
            }
#pragma unroll
            for (int hh = 0; hh < kHeadGroup; ++hh)
                if (h0 + hh < n_hI) score = fmaf(sw[h0 + hh], fmaxf(acc[hh], 0.f), score);
        }
        ws.scores[(int64_t)g * ws.ld + s] = score;
        if (need_hist) atomicAdd(&sh[order_key(score) >> 20], 1u);
    }
    if (need_hist) {
        __syncthreads();
        for (int i = threadIdx.x; i < kBins; i += kScanThreads)
            if (sh[i]) atomicAdd(&ws.hist0[(size_t)g * kBins + i], sh[i]);
    }
}

// ----------------------------------------------------------------------------------
// radix select helpers
// ----------------------------------------------------------------------------------
constexpr int kSelThreads = 256;

// Find the bin holding the need-th largest element of hist[0..nbins) (need >= 1 and
// sum(hist) >= need): *bin = that bin, *above = count in bins strictly above it.
// All kSelThreads threads must call; hist is in shared memory.
template <int NBINS>
CSA_DEV void find_threshold_bin(const uint32_t* hist, uint32_t need, uint32_t* s_bin,
                                uint32_t* s_above, uint32_t* s_scratch /* [32] */)
{
    constexpr int PER = NBINS / kSelThreads;  // bins per thread, top bins to thread 0
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hi = NBINS - tid * PER;  // this thread covers [hi - PER, hi)
    uint32_t local = 0;
#pragma unroll
    for (int i = 1; i <= PER; ++i) local += hist[hi - i];
    // inclusive scan over threads in order 0..255 (thread 0 = top bins)
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_scratch[warp] = incl;
    __syncthreads();
    uint32_t warp_base = 0;
    for (int w = 0; w < warp; ++w) warp_base += s_scratch[w];
    const uint32_t excl = warp_base + incl - local;  // count in bins above this thread's range
    if (excl < need && need <= excl + local) {
        uint32_t cum = excl;
        for (int i = 1; i <= PER; ++i) {
            const uint32_t h = hist[hi - i];
            if (cum + h >= need) {
                *s_bin = (uint32_t)(hi - i);
                *s_above = cum;
                break;
            }
            cum += h;
        }
    }
    __syncthreads();
}

// Warp-aggregated append: returns this lane's slot in a list whose length counter is
// *ctr (global or shared), for lanes with pred true.  All lanes of the warp call.
CSA_DEV uint32_t warp_append(uint32_t* ctr, bool pred)
{
    const unsigned mask = __ballot_sync(0xffffffffu, pred);
    if (!mask) return 0;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(mask) - 1;
    uint32_t base = 0;
    if (lane == leader) base = atomicAdd(ctr, (uint32_t)__popc(mask));
    base = __shfl_sync(0xffffffffu, base, leader);
    return base + __popc(mask & ((1u << lane) - 1u));
}

struct SelArgs {
    TopkWs ws;
    const int64_t* t;
    int m, k;
    int64_t N_cap;
    int32_t* idx_out;
    float* scores_out;
    int64_t chunk;  // scores per CTA
};

// 64-bit selection key: score key in the high word, ~index in the low word, so larger
// means "better" and equal scores prefer the smaller index.
CSA_DEV uint32_t digit_of(uint2 kv, int level)
{
    // level 0: key bits 31..20, level 1: key bits 19..8 (12-bit digits);
    // levels 2..6: key bits 7..0, then ~idx bits 31..24, 23..16, 15..8, 7..0.
    switch (level) {
        case 0: return kv.x >> 20;
        case 1: return (kv.x >> 8) & 0xfffu;
        case 2: return kv.x & 0xffu;
        case 3: return (~kv.y >> 24) & 0xffu;
        case 4: return (~kv.y >> 16) & 0xffu;
        case 5: return (~kv.y >> 8) & 0xffu;
        default: return ~kv.y & 0xffu;
    }
}

// Copy a 4096-bin histogram from global to shared memory.  All loads are issued before
// the first store so that the copy costs one round trip (a load-store loop would be
// serialised into one round trip per iteration).
CSA_DEV void load_hist(uint32_t* sh, const uint32_t* gh)
{
    constexpr int kPerThread = kBins / kSelThreads;
    uint32_t v[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) v[u] = __ldcg(&gh[threadIdx.x + u * kSelThreads]);
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) sh[threadIdx.x + u * kSelThreads] = v[u];
}

// Exclusive prefix sum of v over the kSelThreads threads of the block (thread order);
// *total receives the block sum.  s_warp: 32 words of shared scratch.  All threads call.
CSA_DEV uint32_t block_excl_scan(uint32_t v, uint32_t* s_warp, uint32_t* total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    __syncthreads();  // s_warp may still be read by a previous use
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    uint32_t base = 0, sum = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
        const uint32_t x = s_warp[w];
        base += w < warp ? x : 0u;
        sum += x;
    }
    if (threadIdx.x == 0) *total = sum;
    return base + incl - v;
}

constexpr int kListCap = 2048;  // candidates kept in shared memory by the last CTA
constexpr int kPer = 8;         // scores per thread per round of the first pass
constexpr int kRound = kPer * kSelThreads;
static_assert(kRound <= kListCap, "a round's staging must fit the shared lists");
constexpr int kRankMax = 256;   // lists up to this size are finished by exact ranking

// Emit every entry of a list (count entries) into the output slots counted by *s_out.
CSA_DEV void emit_all(const uint2* list, bool in_smem, uint32_t count, uint32_t* s_out, int k,
                      int32_t* idx_out, float* sc_out)
{
    for (uint32_t i = threadIdx.x; i < ((count + 31) & ~31u); i += kSelThreads) {
        const bool in = i < count;
        const uint2 kv = in ? (in_smem ? list[i] : __ldcg(&list[i])) : make_uint2(0, 0);
        const uint32_t pos = warp_append(s_out, in);
        if (in && pos < (uint32_t)k) {
            idx_out[pos] = (int32_t)kv.y;
            if (sc_out) sc_out[pos] = key_to_float(kv.x);
        }
    }
}

// Emit the `need` best entries of a shared-memory list of at most kSelThreads entries:
// each entry counts the entries that beat it (higher score key, or equal key and a
// smaller index) and is selected when fewer than `need` do.
CSA_DEV void emit_by_rank(const uint2* list, uint32_t count, uint32_t need, uint32_t* s_out, int k,
                          int32_t* idx_out, float* sc_out)
{
    const uint32_t i = threadIdx.x;
    const bool in = i < count;
    const uint2 me = in ? list[i] : make_uint2(0, 0);
    uint32_t rank = 0;
    if (in)
        for (uint32_t j = 0; j < count; ++j) {
            const uint2 o = list[j];
            rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
        }
    const bool take = in && rank < need;
    const uint32_t pos = warp_append(s_out, take);
    if (take && pos < (uint32_t)k) {
        idx_out[pos] = (int32_t)me.y;
        if (sc_out) sc_out[pos] = key_to_float(me.x);
    }
}

__global__ void __launch_bounds__(kSelThreads) topk_select(SelArgs a)
{
    extern __shared__ __align__(16) uint8_t sel_smem[];
    uint32_t* sh = reinterpret_cast<uint32_t*>(sel_smem);               // [kBins]
    uint2* s_listA = reinterpret_cast<uint2*>(sel_smem + kBins * 4);    // [kListCap]
    uint2* s_listB = s_listA + kListCap;                                 // [kListCap]
    __shared__ uint32_t s_scr[32];
    __shared__ uint32_t s_bin, s_above, s_last, s_cnt, s_out, s_nt, s_nc, s_bt, s_bc;
    uint2* s_take = s_listA;  // first pass: staged selections
    uint2* s_cand = s_listB;  // first pass: staged candidates
    pdl_launch_dependents();
    pdl_wait();
    const int g = blockIdx.y;
    const int tid = threadIdx.x;
    // the first round's scores, the digit-0 histogram and t go out in one round trip
    const float* scores0 = a.ws.scores + (int64_t)g * a.ws.ld;
    const int64_t s_begin = (int64_t)blockIdx.x * a.chunk;
    const int64_t s_lim = min(a.N_cap, s_begin + a.chunk);
    uint32_t key0[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int64_t s = s_begin + tid + u * kSelThreads;
        key0[u] = s < s_lim ? order_key(__ldcg(&scores0[s])) : 0u;
    }
    load_hist(sh, a.ws.hist0 + (size_t)g * kBins);
    const int64_t vis = visible_count(a.t, g, a.m, a.N_cap);
    const int k = a.k;
    int32_t* idx_out = a.idx_out + (int64_t)g * k;
    float* sc_out = a.scores_out ? a.scores_out + (int64_t)g * k : nullptr;
    const float* scores = a.ws.scores + (int64_t)g * a.ws.ld;
    uint32_t* ctr = a.ws.ctr + (size_t)g * kCtrs;
    uint2* cand = a.ws.cand + (int64_t)g * a.ws.ld;
    uint2* cand2 = a.ws.cand2 + (int64_t)g * a.ws.ld;

    if (vis <= k) {
        // everything visible is selected, in index order, padded with -1
        const int64_t per = (k + gridDim.x - 1) / gridDim.x;
        const int64_t p0 = (int64_t)blockIdx.x * per;
        const int64_t p1 = min((int64_t)k, p0 + per);
        for (int64_t p = p0 + tid; p < p1; p += kSelThreads) {
            idx_out[p] = p < vis ? (int32_t)p : -1;
            if (sc_out) sc_out[p] = p < vis ? scores[p] : -INFINITY;
        }
    } else {
        // ---- digit 0 threshold from the scan's histogram ----
        __syncthreads();
        find_threshold_bin<kBins>(sh, (uint32_t)k, &s_bin, &s_above, s_scr);
        const uint32_t b0 = s_bin;
        __syncthreads();
        for (int i = tid; i < kBins; i += kSelThreads) sh[i] = 0;
        __syncthreads();
        // ---- emit above b0, collect b0 candidates with their digit-1 histogram ----
        // Rounds of kRound scores: every thread loads its kPer scores at once, the
        // selected entries and candidates are staged in shared memory, and one global
        // atomic per list and round reserves their output slots.
        const int64_t s_end = min(vis, s_begin + a.chunk);
        for (int64_t base = s_begin; base < s_end; base += kRound) {
            uint32_t key[kPer];
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int64_t s = base + tid + u * kSelThreads;
                key[u] = base == s_begin ? key0[u] : (s < s_end ? order_key(__ldcg(&scores[s])) : 0u);
            }
            // slots from one block-wide exclusive scan of (selected, candidate) counts
            // packed in 16-bit halves, instead of one shared atomic per element
            uint32_t cnt = 0;
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int64_t s = base + tid + u * kSelThreads;
                const uint32_t d0 = key[u] >> 20;
                if (s < s_end) cnt += d0 > b0 ? 1u : (d0 == b0 ? 0x10000u : 0u);
            }
            uint32_t excl = block_excl_scan(cnt, s_scr, &s_nt);
            uint32_t tp = excl & 0xffffu, cp = excl >> 16;
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int64_t s = base + tid + u * kSelThreads;
                if (s >= s_end) continue;
                const uint32_t d0 = key[u] >> 20;
                if (d0 > b0) {
                    s_take[tp++] = make_uint2(key[u], (uint32_t)s);
                } else if (d0 == b0) {
                    s_cand[cp++] = make_uint2(key[u], (uint32_t)s);
                    atomicAdd(&sh[(key[u] >> 8) & 0xfffu], 1u);
                }
            }
            if (tid == 0) {
                const uint32_t tot = s_nt;
                s_nt = tot & 0xffffu;
                s_nc = tot >> 16;
            }
            __syncthreads();
            if (tid == 0) {  // both reservations in flight together
                const uint32_t bt = s_nt ? atomicAdd(&ctr[0], s_nt) : 0u;
                const uint32_t bc = s_nc ? atomicAdd(&ctr[1], s_nc) : 0u;
                s_bt = bt;
                s_bc = bc;
            }
            __syncthreads();
            for (uint32_t i = tid; i < s_nt; i += kSelThreads) {
                const uint32_t pos = s_bt + i;
                const uint2 kv = s_take[i];
                if (pos < (uint32_t)k) {
                    idx_out[pos] = (int32_t)kv.y;
                    if (sc_out) sc_out[pos] = key_to_float(kv.x);
                }
            }
            for (uint32_t i = tid; i < s_nc; i += kSelThreads)
                if (s_bc + i < (uint32_t)a.ws.ld) cand[s_bc + i] = s_cand[i];
            __syncthreads();
        }
        __syncthreads();
        for (int i = tid; i < kBins; i += kSelThreads)
            if (sh[i]) atomicAdd(&a.ws.hist1[(size_t)g * kBins + i], sh[i]);
    }

    // ---- last CTA of this query finishes the selection and resets the workspace ----
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const uint32_t ticket = atomicAdd(&ctr[2], 1u);
        s_last = ticket == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    if (vis > k) {
        // Resolve the candidates of the digit-0 threshold bin.  Emission slots now come
        // from a shared-memory counter (this CTA is the only writer left); lists that fit
        // are kept in shared memory so the remaining passes make no global round trips.
        if (tid == 0) s_out = __ldcg(&ctr[0]);
        uint32_t count = __ldcg(&ctr[1]);
        load_hist(sh, a.ws.hist1 + (size_t)g * kBins);
        __syncthreads();
        uint32_t need = (uint32_t)k - s_out;
        uint2* list = cand;
        bool in_smem = false;
        if (count <= (uint32_t)kListCap) {
            // bring the candidates into shared memory with one batched round of loads
            constexpr int kPerT = kListCap / kSelThreads;
            uint2 v[kPerT];
#pragma unroll
            for (int u = 0; u < kPerT; ++u) {
                const uint32_t i = tid + u * kSelThreads;
                v[u] = i < count ? __ldcg(&cand[i]) : make_uint2(0, 0);
            }
#pragma unroll
            for (int u = 0; u < kPerT; ++u) {
                const uint32_t i = tid + u * kSelThreads;
                if (i < count) s_listA[i] = v[u];
            }
            __syncthreads();
            list = s_listA;
            in_smem = true;
        }
        for (int level = 1; need > 0; ++level) {
            if (need >= count) {  // every remaining candidate is selected
                emit_all(list, in_smem, count, &s_out, k, idx_out, sc_out);
                break;
            }
            if (in_smem && count <= kRankMax) {  // exact rank among a small list
                emit_by_rank(list, count, need, &s_out, k, idx_out, sc_out);
                break;
            }
            if (level > 6) break;  // unreachable: (score, index) keys are unique
            if (level >= 2) {
                for (int i = tid; i < 256; i += kSelThreads) sh[i] = 0;
                __syncthreads();
                for (uint32_t i = tid; i < count; i += kSelThreads)
                    atomicAdd(&sh[digit_of(in_smem ? list[i] : __ldcg(&list[i]), level)], 1u);
                __syncthreads();
                find_threshold_bin<256>(sh, need, &s_bin, &s_above, s_scr);
            } else {
                find_threshold_bin<kBins>(sh, need, &s_bin, &s_above, s_scr);
            }
            const uint32_t bt = s_bin, above = s_above, keep_n = sh[bt];
            uint2* next;
            bool next_smem = keep_n <= (uint32_t)kListCap;
            if (next_smem)
                next = (list == s_listA) ? s_listB : s_listA;
            else
                next = (list == cand) ? cand2 : cand;
            if (tid == 0) s_cnt = 0;
            __syncthreads();
            for (uint32_t i = tid; i < ((count + kSelThreads - 1) / kSelThreads) * kSelThreads; i += kSelThreads) {
                const bool in = i < count;
                const uint2 kv = in ? (in_smem ? list[i] : __ldcg(&list[i])) : make_uint2(0, 0);
                const uint32_t d = digit_of(kv, level);
                const bool take = in && d > bt;
                const bool keep = in && d == bt;
                const uint32_t pos = warp_append(&s_out, take);
                if (take && pos < (uint32_t)k) {
                    idx_out[pos] = (int32_t)kv.y;
                    if (sc_out) sc_out[pos] = key_to_float(kv.x);
                }
                const uint32_t npos = warp_append(&s_cnt, keep);
                if (keep && npos < (next_smem ? (uint32_t)kListCap : (uint32_t)a.ws.ld)) next[npos] = kv;
            }
            __threadfence_block();
            __syncthreads();
            need -= above;
            count = s_cnt;
            list = next;
            in_smem = next_smem;
            __syncthreads();
        }
    }
    __syncthreads();
    // reset this query's histograms and counters for the next call
    for (int i = tid; i < kBins; i += kSelThreads) {
        a.ws.hist0[(size_t)g * kBins + i] = 0;
        a.ws.hist1[(size_t)g * kBins + i] = 0;
    }
    if (tid < kCtrs) ctr[tid] = 0;
}

}  // namespace

int launch_topk_select(const TopkWs& ws, const int64_t* t, int G, int m, int k, int64_t N_cap,
                       int32_t* idx_out, float* scores_out, cudaStream_t stream)
{
    SelArgs a;
    a.ws = ws; a.t = t; a.m = m; a.k = k; a.N_cap = N_cap;
    a.idx_out = idx_out; a.scores_out = scores_out;
    int64_t ctas = (2 * kNumSMs + G - 1) / G;
    const int64_t by_size = (N_cap + kRound - 1) / kRound;
    if (ctas > by_size) ctas = by_size;
    if (ctas < 1) ctas = 1;
    a.chunk = (N_cap + ctas - 1) / ctas;
    a.chunk = (a.chunk + kRound - 1) / kRound * kRound;  // whole rounds per CTA
    ctas = (N_cap + a.chunk - 1) / a.chunk;
    if (ctas < 1) ctas = 1;
    dim3 grid((unsigned)ctas, (unsigned)G);
    const size_t smem = kBins * 4 + 2 * kListCap * sizeof(uint2);
    cudaFuncSetAttribute(topk_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_pdl(topk_select, grid, dim3(kSelThreads), smem, stream, a);
    return launch_status();
}

int launch_scan_cuda_core(const void* qI, const float* wI, const void* KI, const int64_t* t,
                          int B, int nq, int64_t N_cap, int n_hI, int cI, int m, int k,
                          const TopkWs& ws, int dtype, cudaStream_t stream)
{
    const int G = B * nq;
    dim3 grid((unsigned)((N_cap + kScanThreads - 1) / kScanThreads), (unsigned)G);
    const size_t smem = ((size_t)n_hI * cI + n_hI) * sizeof(float);
    if (smem > 160 * 1024) return CSA_ERR_UNSUPPORTED;
    const bool vec = cI % (16 / elem_bytes(dtype)) == 0 && aligned16(KI);
    if (dtype == CSA_BF16) {
        auto kern = vec ? scan_cuda_core<__nv_bfloat16, 8> : scan_cuda_core<__nv_bfloat16, 1>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_pdl(kern, grid, dim3(kScanThreads), smem, stream, static_cast<const __nv_bfloat16*>(qI), wI,
                   static_cast<const __nv_bfloat16*>(KI), t, nq, N_cap, n_hI, cI, m, k, ws);
    } else {
        auto kern = vec ? scan_cuda_core<float, 4> : scan_cuda_core<float, 1>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_pdl(kern, grid, dim3(kScanThreads), smem, stream, static_cast<const float*>(qI), wI,
                   static_cast<const float*>(KI), t, nq, N_cap, n_hI, cI, m, k, ws);
    }
    return launch_status();
}

}  // namespace csa

extern "C" size_t csa_indexer_topk_workspace_size(int B, int nq, int64_t N_cap, int k)
{
    (void)k;
    if (B <= 0 || nq <= 0 || N_cap < 0) return 0;
    return csa::topk_ws_layout(nullptr, B * nq, N_cap).bytes + 256;
}

extern "C" int csa_indexer_topk(const void* qI, const float* wI, const void* KI,
                                const int64_t* t, int B, int nq, int64_t N_cap, int n_hI,
                                int cI, int m, int k, int32_t* idx_out, float* scores_out,
                                void* workspace, size_t ws_bytes, int dtype,
                                csa_stream_t stream_)
{
    using namespace csa;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (dtype != CSA_BF16 && dtype != CSA_F32) return CSA_ERR_DTYPE;
    if (B < 0 || nq < 0 || N_cap < 0 || N_cap >= (int64_t(1) << 31) || n_hI <= 0 || cI <= 0 ||
        m <= 0 || k <= 0)
        return CSA_ERR_ARG;
    if (B == 0 || nq == 0) return CSA_OK;
    if (!qI || !wI || !KI || !t || !idx_out) return CSA_ERR_ARG;
    const uintptr_t eb = (uintptr_t)elem_bytes(dtype) - 1;
    if ((((uintptr_t)qI | (uintptr_t)KI) & eb) || ((uintptr_t)wI & 3) || ((uintptr_t)t & 7) ||
        ((uintptr_t)idx_out & 3) || ((uintptr_t)scores_out & 3) || !aligned16(workspace))
        return CSA_ERR_ALIGN;
    const int G = B * nq;
    if (!workspace || ws_bytes < csa_indexer_topk_workspace_size(B, nq, N_cap, k))
        return CSA_ERR_WORKSPACE;
    TopkWs ws = topk_ws_layout(workspace, G, N_cap);
    int st;
    if (dtype == CSA_BF16 && indexer_tc_supported(n_hI, cI))
        st = launch_scan_tc(qI, wI, KI, t, B, nq, N_cap, n_hI, cI, m, k, ws, stream);
    else
        st = launch_scan_cuda_core(qI, wI, KI, t, B, nq, N_cap, n_hI, cI, m, k, ws, dtype, stream);
    if (st != CSA_OK) return st;
    return launch_topk_select(ws, t, G, m, k, N_cap, idx_out, scores_out, stream);
}

extern "C" int csa_workspace_status(const void* workspace, csa_stream_t stream)
{
    if (!workspace) return CSA_ERR_ARG;
    uint32_t st = 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return CSA_ERR_CUDA;
    return st ? CSA_ERR_TIMEOUT : CSA_OK;
}
