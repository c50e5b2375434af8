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
#include "select.cuh"

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
    w.ctr = reinterpret_cast<uint32_t*>(p);    p += (size_t)G * kCtrs * 4;
    p = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(p), 256));
    w.scores = reinterpret_cast<float*>(p);    p += (size_t)G * Np * 4;
    w.cand = reinterpret_cast<uint2*>(p);      p += (size_t)G * Np * 8;
    w.cand2 = reinterpret_cast<uint2*>(p);     p += (size_t)G * Np * 8;
    w.bytes = (size_t)(p - static_cast<char*>(base));
    w.zero_bytes = 256 + (size_t)G * (kBins + kCtrs) * 4;
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
        if (need_hist) atomicAdd(&sh[hist_slot(order_key(score) >> 20)], 1u);
    }
    if (need_hist) {
        __syncthreads();
        for (int i = threadIdx.x; i < kBins; i += kScanThreads)
            if (sh[i]) atomicAdd(&ws.hist0[(size_t)g * kBins + i], sh[i]);
    }
}

// ----------------------------------------------------------------------------------
// stand-alone top-k select (after the CUDA-core scan, or when the scan grid cannot
// select in place)
// ----------------------------------------------------------------------------------
using sel::kSelThreads;
using sel::kListCap;
using sel::kPer;
using sel::kRound;

struct SelArgs {
    TopkWs ws;
    const int64_t* t;
    int m, k;
    int64_t N_cap;
    int32_t* idx_out;
    float* scores_out;
    int64_t chunk;  // scores per CTA
};

__global__ void __launch_bounds__(kSelThreads) topk_select(SelArgs a)
{
    using Bar = sel::CtaBar;
    extern __shared__ __align__(16) uint8_t sel_smem[];
    uint32_t* sh = reinterpret_cast<uint32_t*>(sel_smem);               // [kBins]
    uint2* s_listA = reinterpret_cast<uint2*>(sel_smem + kBins * 4);    // [kListCap]
    uint2* s_listB = s_listA + kListCap;                                 // [kListCap]
    __shared__ sel::Shared s;
    pdl_launch_dependents();
    pdl_wait();
    const int g = blockIdx.y;
    const int tid = threadIdx.x;
    // the first round's scores, the digit-0 histogram and t go out in one round trip
    const float* scores = a.ws.scores + (int64_t)g * a.ws.ld;
    const int64_t s_begin = (int64_t)blockIdx.x * a.chunk;
    const int64_t s_lim = min(a.N_cap, s_begin + a.chunk);
    uint32_t key0[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int64_t i = s_begin + tid + u * kSelThreads;
        key0[u] = i < s_lim ? order_key(__ldcg(&scores[i])) : 0u;
    }
    const int64_t vis = visible_count(a.t, g, a.m, a.N_cap);
    const int k = a.k;
    sel::load_hist(sh, a.ws.hist0 + (size_t)g * kBins, tid);
    const sel::Query q = sel::query_view(a.ws, g, k, a.idx_out, a.scores_out);

    if (vis <= k) {
        // everything visible is selected, in index order, padded with -1
        const int64_t per = (k + gridDim.x - 1) / gridDim.x;
        const int64_t p0 = (int64_t)blockIdx.x * per;
        const int64_t p1 = min((int64_t)k, p0 + per);
        for (int64_t p = p0 + tid; p < p1; p += kSelThreads) {
            q.idx_out[p] = p < vis ? (int32_t)p : -1;
            if (q.sc_out) q.sc_out[p] = p < vis ? scores[p] : -INFINITY;
        }
    } else {
        // ---- digit 0 threshold from the scan's histogram ----
        __syncthreads();
        sel::find_threshold_bin<kBins, Bar>(sh, (uint32_t)k, &s, tid);
        const uint32_t b0 = s.bin;
        // ---- emit above b0, collect the candidates inside b0 ----
        const int64_t s_end = min(vis, s_begin + a.chunk);
        for (int64_t base = s_begin; base < s_end; base += kRound) {
            uint32_t key[kPer], eidx[kPer];
            bool valid[kPer];
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int64_t i = base + tid + u * kSelThreads;
                valid[u] = i < s_end;
                eidx[u] = (uint32_t)i;
                key[u] = base == s_begin ? key0[u] : (valid[u] ? order_key(__ldcg(&scores[i])) : 0u);
            }
            sel::classify_round<Bar>(q, key, eidx, valid, b0, s_listA, s_listB, &s, tid);
        }
    }

    // ---- last CTA of this query finishes the selection and resets the workspace ----
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const uint32_t ticket = atomicAdd(&q.ctr[2], 1u);
        s.last = ticket == gridDim.x - 1;
    }
    __syncthreads();
    if (!s.last) return;
    __threadfence();
    if (vis > k) sel::resolve_candidates<Bar>(q, sh, s_listA, s_listB, &s, tid);
    __syncthreads();
    sel::reset_query(q, tid);
}


// One CTA per query, after the many-query scan, which leaves the scores and, per 32
// consecutive keys, their largest order key (in the query's second candidate buffer).
//  1. Filter: at least k groups have a maximum at or above the lower edge T of the
//     digit-0 bin holding the k-th largest group maximum, so at least k keys are >= T
//     and the top k are among them.  (With fewer than k groups, T admits every key.)
//  2. One pass over the scores, eight float4 loads in flight per thread, appends the
//     keys >= T to the candidate list (warp-aggregated slots from a CTA-local counter:
//     no other CTA shares the query) and counts their digits.
//  3. The threshold bin among the candidates; those above it are emitted, those in it
//     are compacted into the second buffer and resolved as in topk_select.
// Per key this costs one compare; only the few candidates touch shared-memory atomics.
__global__ void __launch_bounds__(kSelThreads) topk_select_row(SelArgs a)
{
    using Bar = sel::CtaBar;
    extern __shared__ __align__(16) uint8_t sel_smem[];
    uint32_t* sh = reinterpret_cast<uint32_t*>(sel_smem);               // [kBins]
    uint2* s_listA = reinterpret_cast<uint2*>(sel_smem + kBins * 4);    // [kListCap]
    uint2* s_listB = s_listA + kListCap;                                 // [kListCap]
    __shared__ sel::Shared s;
    constexpr int kVec = 8;  // float4 loads in flight per thread
    pdl_launch_dependents();
    pdl_wait();
    const int g = blockIdx.x;
    const int tid = threadIdx.x;
    const float* scores = a.ws.scores + (int64_t)g * a.ws.ld;
    const int64_t vis = visible_count(a.t, g, a.m, a.N_cap);
    const int k = a.k;
    sel::Query q = sel::query_view(a.ws, g, k, a.idx_out, a.scores_out);
    if (vis <= k) {  // everything visible is selected, in index order, padded with -1
        for (int64_t p = tid; p < k; p += kSelThreads) {
            q.idx_out[p] = p < vis ? (int32_t)p : -1;
            if (q.sc_out) q.sc_out[p] = p < vis ? __ldcg(&scores[p]) : -INFINITY;
        }
        return;
    }
    // ---- 1. filter threshold from the group maxima ----
    const int64_t ng = (vis + 31) >> 5;
    uint32_t T = 0;
    if (ng >= k) {
        // The maxima crowd just below the largest one, M, so their histogram is taken over
        // a window anchored there: distance bins d = (M - key) >> w, the last bin holding
        // everything further down, in slot 4095 - d so that larger keys sit higher.  The
        // first window (w = 12: 1/2048 octave bins, 2 octaves) is widened (w = 16, 20)
        // only if the k-th largest maximum falls into the last bin.
        const uint32_t* gm = reinterpret_cast<const uint32_t*>(q.cand2);
        uint32_t mx = 0;
        for (int64_t i0 = 0; i0 < ng; i0 += 4 * kSelThreads) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t i = i0 + tid + u * kSelThreads;
                if (i < ng) mx = max(mx, __ldcg(&gm[i]));
            }
        }
        mx = __reduce_max_sync(0xffffffffu, mx);
        if ((tid & 31) == 0) s.scr[tid >> 5] = mx;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < kSelThreads / 32; ++w) mx = max(mx, s.scr[w]);
        for (int w = 12;; w += 4) {
            sel::zero_words(sh, kBins, tid);
            __syncthreads();
            for (int64_t i0 = 0; i0 < ng; i0 += 4 * kSelThreads) {
                uint32_t v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int64_t i = i0 + tid + u * kSelThreads;
                    v[u] = i < ng ? __ldcg(&gm[i]) : 0u;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (i0 + tid + u * kSelThreads < ng) {
                        const uint32_t d = min((mx - v[u]) >> w, (uint32_t)(kBins - 1));
                        atomicAdd(&sh[kBins - 1 - d], 1u);
                    }
                }
            }
            __syncthreads();
            sel::find_threshold_bin<kBins, Bar, true>(sh, (uint32_t)k, &s, tid);
            const uint32_t d = kBins - 1 - s.bin;  // distance bin of the k-th largest maximum
            if (d < kBins - 1 || w == 20) {
                const uint64_t below = ((uint64_t)(d + 1) << w) - 1;  // T: lower edge of that bin
                T = below > mx ? 0u : mx - (uint32_t)below;
                break;
            }
        }
    }
    // ---- 2. candidates: every key >= T, with their digit-0 histogram ----
    sel::zero_words(sh, kBins, tid);
    if (tid == 0) s.cnt = 0;
    __syncthreads();
    const uint32_t cap = (uint32_t)q.ld;
    auto keep_if = [&](uint32_t key, uint32_t e, bool in) {
        const bool keep = in && key >= T;
        const uint32_t pos = sel::warp_append(&s.cnt, keep);
        if (keep) {
            if (pos < cap) q.cand[pos] = make_uint2(key, e);
            atomicAdd(&sh[key >> 20], 1u);
        }
    };
    if (ng >= k) {
        // only groups whose maximum reaches T can hold a candidate: each warp takes 32
        // group maxima at a time and reads the scores of the hits, up to 8 groups of 32
        // scores in flight
        const uint32_t* gm = reinterpret_cast<const uint32_t*>(q.cand2);
        const int lane = tid & 31, warp = tid >> 5;
        for (int64_t i0 = (int64_t)warp * 32; i0 < ng; i0 += kSelThreads) {
            const int64_t gi = i0 + lane;
            unsigned hit = __ballot_sync(0xffffffffu, gi < ng && __ldcg(&gm[gi]) >= T);
            while (hit) {
                int64_t si[8];
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    si[u] = -1;
                    if (hit) {
                        si[u] = ((i0 + __ffs(hit) - 1) << 5) + lane;
                        hit &= hit - 1;
                    }
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = si[u] >= 0 && si[u] < vis ? __ldcg(&scores[si[u]]) : 0.f;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (si[u] == -1 && u > 0) break;  // warp-uniform: no more hits in this batch
                    const bool in = si[u] >= 0 && si[u] < vis;
                    keep_if(in ? order_key(v[u]) : 0u, (uint32_t)si[u], in);
                }
            }
        }
    } else {
        const float4* s4 = reinterpret_cast<const float4*>(scores);
        const int64_t n4 = vis >> 2;  // whole float4 groups; the last vis % 4 scores separately
        for (int64_t i0 = 0; i0 < n4; i0 += kVec * kSelThreads) {
            float4 v[kVec];
#pragma unroll
            for (int u = 0; u < kVec; ++u) {
                const int64_t i = i0 + tid + u * kSelThreads;
                v[u] = i < n4 ? __ldcg(&s4[i]) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kVec; ++u) {
                const int64_t i = i0 + tid + u * kSelThreads;
                const bool in = i < n4;
                const uint32_t k0 = order_key(v[u].x), k1 = order_key(v[u].y);
                const uint32_t k2 = order_key(v[u].z), k3 = order_key(v[u].w);
                if (!__any_sync(0xffffffffu, in && max(max(k0, k1), max(k2, k3)) >= T)) continue;
                const uint32_t e = (uint32_t)(i << 2);
                keep_if(k0, e, in);
                keep_if(k1, e + 1, in);
                keep_if(k2, e + 2, in);
                keep_if(k3, e + 3, in);
            }
        }
        if (tid < 32) {  // the last vis % 4 scores (all lanes of warp 0 call)
            const int64_t i = (n4 << 2) + tid;
            keep_if(i < vis ? order_key(__ldcg(&scores[i])) : 0u, (uint32_t)i, i < vis);
        }
    }
    __syncthreads();
    const uint32_t nc = s.cnt;  // >= k; at most vis <= ld
    sel::find_threshold_bin<kBins, Bar, true>(sh, (uint32_t)k, &s, tid);
    const uint32_t b0 = s.bin;
    // ---- 3. emit above b0; compact the b0 candidates into the second buffer ----
    if (tid == 0) {
        s.out = 0;
        s.cnt = 0;
    }
    __syncthreads();
    const uint32_t rounds = (nc + kSelThreads - 1) / kSelThreads;
    for (uint32_t r = 0; r < rounds; ++r) {
        const uint32_t i = r * kSelThreads + tid;
        const bool in = i < nc;
        const uint2 kv = in ? __ldcg(&q.cand[i]) : make_uint2(0, 0);
        const uint32_t d0 = kv.x >> 20;
        const bool take = in && d0 > b0;
        const bool tie = in && d0 == b0;
        const uint32_t pos = sel::warp_append(&s.out, take);
        if (take) sel::emit(q, pos, kv);
        const uint32_t tpos = sel::warp_append(&s.cnt, tie);
        if (tie) q.cand2[tpos] = kv;
    }
    __syncthreads();
    if (tid == 0) {
        q.ctr[0] = s.out;
        q.ctr[1] = s.cnt;
    }
    __threadfence();
    __syncthreads();
    const uint2* tmp = q.cand;  // the tied candidates now sit in the second buffer
    q.cand = q.cand2;
    q.cand2 = const_cast<uint2*>(tmp);
    sel::resolve_candidates<Bar>(q, sh, s_listA, s_listB, &s, tid);
    __syncthreads();
    sel::reset_query(q, tid, false);
}

}  // namespace

int launch_topk_select(const TopkWs& ws, const int64_t* t, int G, int m, int k, int64_t N_cap,
                       int32_t* idx_out, float* scores_out, cudaStream_t stream, bool self_hist)
{
    SelArgs a;
    a.ws = ws; a.t = t; a.m = m; a.k = k; a.N_cap = N_cap;
    a.idx_out = idx_out; a.scores_out = scores_out;
    const size_t smem = kBins * 4 + 2 * kListCap * sizeof(uint2);
    if (self_hist) {
        a.chunk = N_cap;
        cudaFuncSetAttribute(topk_select_row, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_pdl(topk_select_row, dim3((unsigned)G), dim3(kSelThreads), smem, stream, a);
        return launch_status();
    }
    int64_t ctas = (2 * kNumSMs + G - 1) / G;
    const int64_t by_size = (N_cap + kRound - 1) / kRound;
    if (ctas > by_size) ctas = by_size;
    if (ctas < 1) ctas = 1;
    a.chunk = (N_cap + ctas - 1) / ctas;
    a.chunk = (a.chunk + kRound - 1) / kRound * kRound;  // whole rounds per CTA
    ctas = (N_cap + a.chunk - 1) / a.chunk;
    if (ctas < 1) ctas = 1;
    dim3 grid((unsigned)ctas, (unsigned)G);
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

// Host-side validation of csa_indexer_topk's arguments (every error it can return before
// a launch), shared with the no-allocation variant.
int indexer_topk_check(const void* qI, const float* wI, const void* KI, const int64_t* t, int B, int nq,
                       int64_t N_cap, int n_hI, int cI, int m, int k, const int32_t* idx_out,
                       const float* scores_out, const void* workspace, size_t ws_bytes, int dtype)
{
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
    if ((int64_t)B * nq > 65535) return CSA_ERR_UNSUPPORTED;  // one grid row per query
    if (!workspace || ws_bytes < csa_indexer_topk_workspace_size(B, nq, N_cap, k))
        return CSA_ERR_WORKSPACE;
    // the CUDA-core scan stages q^I and w^I of one query in shared memory
    const bool tc_path = dtype == CSA_BF16 && indexer_tc_supported(n_hI, cI);
    if (!tc_path && ((size_t)n_hI * cI + n_hI) * sizeof(float) > 160 * 1024) return CSA_ERR_UNSUPPORTED;
    return CSA_OK;
}

}  // namespace csa

extern "C" size_t csa_indexer_topk_workspace_size(int B, int nq, int64_t N_cap, int k)
{
    (void)k;
    if (B <= 0 || nq <= 0 || N_cap < 0) return 0;
    const int64_t G = (int64_t)B * nq;
    if (G > 65535) return 0;  // beyond the supported number of queries per call
    return csa::topk_ws_layout(nullptr, (int)G, N_cap).bytes + 256;
}

extern "C" int csa_indexer_topk(const void* qI, const float* wI, const void* KI,
                                const int64_t* t, int B, int nq, int64_t N_cap, int n_hI,
                                int cI, int m, int k, int32_t* idx_out, float* scores_out,
                                void* workspace, size_t ws_bytes, int dtype,
                                csa_stream_t stream_)
{
    using namespace csa;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    const int chk = indexer_topk_check(qI, wI, KI, t, B, nq, N_cap, n_hI, cI, m, k, idx_out, scores_out,
                                       workspace, ws_bytes, dtype);
    if (chk != CSA_OK || B == 0 || nq == 0) return chk;
    const int G = B * nq;
    TopkWs ws = topk_ws_layout(workspace, G, N_cap);
    int st;
    bool fused = false;
    if (dtype == CSA_BF16 && indexer_mq_eligible(qI, KI, B, nq, N_cap, n_hI, cI)) {
        st = launch_scan_mq(qI, wI, KI, t, B, nq, N_cap, n_hI, cI, m, ws, stream);
        if (st != CSA_OK) return st;
        return launch_topk_select(ws, t, G, m, k, N_cap, idx_out, scores_out, stream, true);
    }
    if (dtype == CSA_BF16 && indexer_tc_supported(n_hI, cI))
        st = launch_scan_tc(qI, wI, KI, t, B, nq, N_cap, n_hI, cI, m, k, ws, idx_out, scores_out, &fused, stream);
    else
        st = launch_scan_cuda_core(qI, wI, KI, t, B, nq, N_cap, n_hI, cI, m, k, ws, dtype, stream);
    if (st != CSA_OK || fused) return st;
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
