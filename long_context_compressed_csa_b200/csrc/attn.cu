// Shared-KV multi-query attention over compressed entries
// ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch", section 8 for CSA over the
// top-k set, section 10 for HCA over every visible entry; key = value = the entry,
// logits scaled by 1/sqrt(c)).
//
// Split-KV decode: the entry list of each query is cut into `splits` ranges; each CTA
// produces, for its heads, an unnormalised partial output O_i and its (max, sum) in the
// base-2 domain, and a combine kernel merges the splits with the usual log-sum-exp
// rescaling.  bf16 inputs with tensor-core shapes run the tcgen05 kernel (attn_tc.cu);
// everything else (the fp32 exact path, odd shapes) runs the CUDA-core kernel here.
#include "attn.cuh"

namespace csa {

AttnPlan attn_plan_cuda_core(int G, int n_h, int64_t entries)
{
    AttnPlan p;
    p.head_groups = (n_h + kCcHeads - 1) / kCcHeads;
    int64_t want = (2 * kNumSMs + (int64_t)G * p.head_groups - 1) / ((int64_t)G * p.head_groups);
    int64_t max_splits = (entries + kCcChunk - 1) / kCcChunk;
    if (max_splits < 1) max_splits = 1;
    if (want > max_splits) want = max_splits;
    if (want < 1) want = 1;
    p.per_split = (entries + want - 1) / want;
    p.per_split = (p.per_split + kCcChunk - 1) / kCcChunk * kCcChunk;
    if (p.per_split < kCcChunk) p.per_split = kCcChunk;
    p.splits = (int)((entries + p.per_split - 1) / p.per_split);
    if (p.splits < 1) p.splits = 1;
    return p;
}

size_t attn_ws_bytes(int G, int n_h, int c, int splits)
{
    return 256 + align_up((size_t)G * splits * n_h * c * sizeof(float), 256) +
           align_up((size_t)G * splits * n_h * sizeof(float2), 256);
}

namespace {

// ----------------------------------------------------------------------------------
// CUDA-core split kernel.  CTA = (split, head group of kCcHeads heads, query).  The
// chunk of kCcChunk entries is staged in shared memory as fp32 with a padded row
// stride, so that lane-per-entry dot products and lane-per-column accumulation are both
// bank-conflict free.  Each warp owns kCcHeads/8 heads; a lane keeps c/32 output
// columns of each of them in registers.
// ----------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256)
attn_cuda_core(AttnArgs a)
{
    extern __shared__ float smem[];
    constexpr int HPW = kCcHeads / 8;  // heads per warp
    constexpr int CPL = kMaxC / 32;    // output columns per lane
    const int c = a.c;
    const int cs = c + 1;                    // padded row stride
    float* sC = smem;                        // [kCcChunk][cs]
    float* sQ = smem + kCcChunk * cs;        // [kCcHeads][c]
    __shared__ int s_ent[kCcChunk];

    pdl_launch_dependents();
    pdl_wait();
    const int split = blockIdx.x, hg = blockIdx.y, g = blockIdx.z;
    const int64_t b = g / a.nq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h_base = hg * kCcHeads;

    // list positions: [0, ncomp) compressed entries, then the sliding-window entries
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

    // stage q rows of this head group
    const T* qg = static_cast<const T*>(a.q) + ((int64_t)g * a.n_h) * c;
    for (int i = threadIdx.x; i < kCcHeads * c; i += 256) {
        const int hh = i / c, j = i % c;
        sQ[i] = (h_base + hh < a.n_h) ? to_f32(qg[(int64_t)(h_base + hh) * c + j]) : 0.f;
    }

    float m_run[HPW], l_run[HPW], o[HPW][CPL];
#pragma unroll
    for (int x = 0; x < HPW; ++x) {
        m_run[x] = -INFINITY;
        l_run[x] = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) o[x][i] = 0.f;
    }

    const T* cache = static_cast<const T*>(a.cache) + b * a.N_cap * c;
    const T* wcache = a.win ? static_cast<const T*>(a.win) + b * (int64_t)a.win_cap * c : cache;
    for (int64_t p0 = p_begin; p0 < p_end; p0 += kCcChunk) {
        __syncthreads();  // previous chunk fully consumed (and sQ staged on entry)
        if (threadIdx.x < kCcChunk) {
            const int64_t p = p0 + threadIdx.x;
            int e = -1;  // >= 0 compressed entry, <= -2 window row -2 - e, -1 none
            if (p < p_end) {
                if (p >= ncomp) {  // window position: at most one wrap of the ring
                    int r = wrow0 + (int)(p - ncomp);
                    r = r >= a.win_cap ? r - a.win_cap : r;
                    e = -2 - r;
                } else if (a.dense) {
                    e = (int)p;
                } else {
                    const int32_t v = a.idx[(int64_t)g * a.k + p];
                    e = (v >= 0 && v < a.N_cap) ? v : -1;
                }
            }
            s_ent[threadIdx.x] = e;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < kCcChunk * c; i += 256) {
            const int r = i / c, j = i % c;
            const int e = s_ent[r];
            sC[r * cs + j] = e >= 0    ? to_f32(cache[(int64_t)e * c + j])
                             : e <= -2 ? to_f32(wcache[(int64_t)(-2 - e) * c + j])
                                       : 0.f;
        }
        __syncthreads();
        const bool valid = s_ent[lane] != -1;
#pragma unroll
        for (int x = 0; x < HPW; ++x) {
            const int hh = warp * HPW + x;
            const float* qr = sQ + hh * c;
            const float* cr = sC + lane * cs;
            float dot = 0.f;
            for (int j = 0; j < c; ++j) dot = fmaf(qr[j], cr[j], dot);
            const float logit = valid ? dot * a.scale_log2 : -INFINITY;
            float cmax = logit;
#pragma unroll
            for (int off = 16; off; off >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, off));
            const float m_new = fmaxf(m_run[x], cmax);
            if (m_new == -INFINITY) continue;  // nothing valid yet
            const float alpha = exp2f(m_run[x] - m_new);
            const float pl = valid ? exp2f(logit - m_new) : 0.f;
            float psum = pl;
#pragma unroll
            for (int off = 16; off; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
            l_run[x] = l_run[x] * alpha + psum;
            m_run[x] = m_new;
#pragma unroll
            for (int i = 0; i < CPL; ++i) o[x][i] *= alpha;
            for (int e = 0; e < kCcChunk; ++e) {
                const float pe = __shfl_sync(0xffffffffu, pl, e);
                const float* ce = sC + e * cs;
#pragma unroll
                for (int i = 0; i < CPL; ++i) {
                    const int j = lane + 32 * i;
                    if (j < c) o[x][i] = fmaf(pe, ce[j], o[x][i]);
                }
            }
        }
    }

    // write partials: O_i unnormalised, (m, l) in base-2 units of the scaled logits
#pragma unroll
    for (int x = 0; x < HPW; ++x) {
        const int h = h_base + warp * HPW + x;
        if (h >= a.n_h) continue;
        const size_t row = ((size_t)g * a.splits + split) * a.n_h + h;
        float* po = static_cast<float*>(a.part_o) + row * c;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int j = lane + 32 * i;
            if (j < c) po[j] = o[x][i];
        }
        if (lane == 0) a.part_ml[row] = make_float2(m_run[x], l_run[x]);
    }
}

// ----------------------------------------------------------------------------------
// combine: out[g][h] = sum_i 2^(m_i - M) O_i / sum_i 2^(m_i - M) l_i ; lse in natural log.
// Partials are fp32 O_i, or bf16 O_i / l_i, whose weight is then 2^(m_i - M) l_i.
// ----------------------------------------------------------------------------------
template <typename TO>
CSA_DEV void store_out(TO* p, float v);
template <>
CSA_DEV void store_out<float>(float* p, float v) { *p = v; }
template <>
CSA_DEV void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

CSA_DEV float load1(const float* p) { return *p; }
CSA_DEV float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// 16 bytes of partial values as raw bits, streamed (read once); their values as floats
CSA_DEV uint4 load_raw_stream(const void* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
CSA_DEV void raw_to_float(uint4 x, float (&v)[4])
{
    v[0] = __uint_as_float(x.x); v[1] = __uint_as_float(x.y);
    v[2] = __uint_as_float(x.z); v[3] = __uint_as_float(x.w);
}
CSA_DEV void raw_to_float(uint4 x, float (&v)[8])
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);             // low bf16 of the pair
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);  // high bf16
    }
}

// One CTA per (head, slice of kCombineCols output columns, query), so that the partial
// rows are read by ~4 CTAs per head spread over all SMs (a CTA reads at most the SM's
// share of the L2 bandwidth).  Thread (column group of 16 bytes, split group) issues
// its partial loads right after the (max, sum) loads of every split; the weights are
// formed in shared memory meanwhile.  A split whose weight is 0 (empty range, nothing
// written) is excluded by a select, not a multiply.
template <typename TO, typename TP>
__global__ void __launch_bounds__(kCombineThreads)
attn_combine(const TP* __restrict__ part_o, const float2* __restrict__ part_ml, int splits,
             int n_h, int c, TO* __restrict__ out, float* __restrict__ lse)
{
    constexpr bool kNormalized = sizeof(TP) == 2;  // bf16 partials are O_i / l_i
    constexpr int kV = 16 / sizeof(TP);             // partial values per 16-byte load
    constexpr int kBatch = 8;                       // 16-byte loads in flight per thread
    constexpr int kGroups = kCombineCols / kV;      // column groups of a full slice
    static_assert(kCombineThreads % kGroups == 0, "whole split groups");
    pdl_launch_dependents();
    pdl_wait();
    const int h = blockIdx.x, g = blockIdx.y;
    const int c0 = blockIdx.z * kCombineCols;
    const int width = min(kCombineCols, c - c0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ float s_m[kMaxSplits], s_w[kMaxSplits];
    __shared__ float s_red[kCombineThreads / 32];
    __shared__ float s_acc[kV * kCombineThreads];
    const size_t base = (size_t)g * splits * n_h + h;
    TO* orow = out + ((size_t)g * n_h + h) * c + c0;
    const bool vec = c % kV == 0;
    const int ngrp = kCombineThreads / kGroups;     // split groups
    const int cv = tid % kGroups, grp = tid / kGroups;
    const bool worker = vec && cv * kV < width;
    const TP* col = part_o + base * c + c0 + (size_t)cv * kV;
    const size_t split_stride = (size_t)n_h * c;

    float mloc = -INFINITY;
    for (int i = tid; i < splits; i += kCombineThreads) {
        const float2 ml = part_ml[base + (size_t)i * n_h];
        s_m[i] = ml.x;
        s_w[i] = ml.y;
        mloc = fmaxf(mloc, ml.x);
    }
    uint4 raw[kBatch];  // first batch of partial rows, in flight while the weights form
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
        const int i = grp + u * ngrp;
        raw[u] = worker && i < splits ? load_raw_stream(col + (size_t)i * split_stride) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, off));
    if (lane == 0) s_red[warp] = mloc;
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCombineThreads / 32; ++w) M = fmaxf(M, s_red[w]);
    float lloc = 0.f;
    for (int i = tid; i < splits; i += kCombineThreads) {
        const float w = s_m[i] == -INFINITY ? 0.f : exp2f(s_m[i] - M);
        lloc = fmaf(w, s_w[i], lloc);
        s_w[i] = kNormalized ? w * s_w[i] : w;
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) lloc += __shfl_xor_sync(0xffffffffu, lloc, off);
    __syncthreads();
    if (lane == 0) s_red[warp] = lloc;
    __syncthreads();
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kCombineThreads / 32; ++w) L += s_red[w];
    const float inv = L > 0.f ? 1.f / L : 0.f;
    if (tid == 0 && blockIdx.z == 0 && lse)
        lse[(size_t)g * n_h + h] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;

    if (vec) {
        float acc[kV];
#pragma unroll
        for (int e = 0; e < kV; ++e) acc[e] = 0.f;
        for (int i0 = grp; worker && i0 < splits; i0 += kBatch * ngrp) {
            if (i0 != grp) {  // later batches (more than kBatch splits per split group)
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int i = i0 + u * ngrp;
                    raw[u] = i < splits ? load_raw_stream(col + (size_t)i * split_stride) : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int i = i0 + u * ngrp;
                const float w = i < splits ? s_w[i] : 0.f;
                float v[kV];
                raw_to_float(raw[u], v);
#pragma unroll
                for (int e = 0; e < kV; ++e) acc[e] = w != 0.f ? fmaf(w, v[e], acc[e]) : acc[e];
            }
        }
#pragma unroll
        for (int e = 0; e < kV; ++e) s_acc[e * kCombineThreads + tid] = acc[e];
        __syncthreads();
        if (grp == 0 && worker) {
            for (int q = 1; q < ngrp; ++q)
#pragma unroll
                for (int e = 0; e < kV; ++e) acc[e] += s_acc[e * kCombineThreads + q * kGroups + tid];
#pragma unroll
            for (int e = 0; e < kV; ++e) store_out<TO>(orow + cv * kV + e, acc[e] * inv);
        }
    } else {
        for (int j = tid; j < width; j += kCombineThreads) {
            float acc = 0.f;
            for (int i = 0; i < splits; ++i) {
                const float w = s_w[i];
                if (w != 0.f) acc = fmaf(w, load1(&part_o[(base + (size_t)i * n_h) * c + c0 + j]), acc);
            }
            store_out<TO>(orow + j, acc * inv);
        }
    }
}

// Split merge of the tensor-core path (bf16 partials O_i / l_i), one warp per (output row,
// slice of 32 * VPL columns): a lane keeps the (max, sum) of up to four splits in
// registers, the first kBatch partial loads of its columns are in flight before the
// weights are known, and each split's weight reaches the lanes by a shuffle.  The slice
// width adapts the grid to the number of rows, so that one query (128 rows) and many
// queries (thousands of rows) both spread over every SM in one wave.
constexpr int kRowWarps = 4;        // warps per CTA (a lane keeps the weights of up to 4 x 32 splits)

template <int VPL>
struct RowRaw;
template <>
struct RowRaw<4> {
    using T = uint2;
    static CSA_DEV T load(const __nv_bfloat16* p) { return __ldcs(reinterpret_cast<const uint2*>(p)); }
    static CSA_DEV void unpack(T x, float (&v)[4])
    {
        v[0] = __uint_as_float(x.x << 16); v[1] = __uint_as_float(x.x & 0xffff0000u);
        v[2] = __uint_as_float(x.y << 16); v[3] = __uint_as_float(x.y & 0xffff0000u);
    }
};
template <>
struct RowRaw<8> {
    using T = uint4;
    static CSA_DEV T load(const __nv_bfloat16* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
    static CSA_DEV void unpack(T x, float (&v)[8])
    {
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

// kBatch (16 or 32) partial loads are in flight per lane; a split count of at most
// kBatch is merged in one round trip.
template <typename TO, int VPL, int kBatch>
__global__ void __launch_bounds__(32 * kRowWarps)
attn_combine_rows(const __nv_bfloat16* __restrict__ part_o, const float2* __restrict__ part_ml, int splits, int n_h,
                  int c, int items, TO* __restrict__ out, float* __restrict__ lse)
{
    constexpr int W = 32 * VPL;  // columns of one work item
    static_assert(kBatch == 16 || kBatch == 32, "a batch never straddles two weight registers");
    using R = RowRaw<VPL>;
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int item = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    if (item >= items) return;
    const int slices = c / W;
    const int sl = item % slices, row = item / slices;  // row = g * n_h + h
    const int g = row / n_h, h = row - g * n_h;
    const size_t base = (size_t)g * splits * n_h + h;   // partial row of split 0 (splits n_h rows apart)
    const int col = sl * W + lane * VPL;
    const __nv_bfloat16* src = part_o + base * c + col;
    const size_t sstride = (size_t)n_h * c;
    typename R::T raw[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) raw[u] = u < splits ? R::load(src + (size_t)u * sstride) : typename R::T{};
    float m[4], l[4], M = -INFINITY;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int i = lane + 32 * q;
        const float2 ml = i < splits ? part_ml[base + (size_t)i * n_h] : make_float2(-INFINITY, 0.f);
        m[q] = ml.x;
        l[q] = ml.y;
        M = fmaxf(M, ml.x);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float w[4], L = 0.f;  // weight of split lane + 32 q: 2^(m_i - M) l_i (0 for an empty split)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        w[q] = m[q] == -INFINITY ? 0.f : exp2f(m[q] - M) * l[q];
        L += w[q];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    float acc[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[e] = 0.f;
    for (int i0 = 0; i0 < splits; i0 += kBatch) {
        if (i0 > 0) {
#pragma unroll
            for (int u = 0; u < kBatch; ++u)
                raw[u] = i0 + u < splits ? R::load(src + (size_t)(i0 + u) * sstride) : typename R::T{};
        }
        const int q = i0 >> 5;  // the register holding the weights of this batch
        const float wq = q == 0 ? w[0] : q == 1 ? w[1] : q == 2 ? w[2] : w[3];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const float wi = __shfl_sync(0xffffffffu, wq, (i0 + u) & 31);
            if (i0 + u < splits && wi != 0.f) {
                float v[VPL];
                R::unpack(raw[u], v);
#pragma unroll
                for (int e = 0; e < VPL; ++e) acc[e] = fmaf(wi, v[e], acc[e]);
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    TO* dst = out + (size_t)row * c + col;
    if constexpr (sizeof(TO) == 4) {
#pragma unroll
        for (int e = 0; e < VPL; e += 4)
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(dst) + e) =
                make_float4(acc[e] * inv, acc[e + 1] * inv, acc[e + 2] * inv, acc[e + 3] * inv);
    } else {
        uint32_t pk[VPL / 2];
#pragma unroll
        for (int e = 0; e < VPL; e += 2) {
            __nv_bfloat162 pr = __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
            pk[e / 2] = *reinterpret_cast<uint32_t*>(&pr);
        }
        if constexpr (VPL == 8)
            *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        else
            *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
    }
    if (sl == 0 && lane == 0 && lse) lse[row] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

// 128-column slices (32 loads in flight per lane) below 1024 rows, 256-column slices (16
// loads in flight) from there on.  One query (128 rows) keeps the (head, column slice)
// merge instead: its 256-thread CTAs leave room on every SM for the next kernel's CTAs to
// become resident and start their prologue and prefetches, which the 106-register warps
// of this merge do not (measured: the 1M sparse-then-dense pair of calls ~2.6 us slower).
bool combine_rows_wide(const AttnArgs& a) { return a.B * a.nq * a.n_h >= 1024; }
bool combine_rows_fits(const AttnArgs& a)
{
    return a.B * a.nq >= 4 && a.splits <= (combine_rows_wide(a) ? 16 : 32);
}

template <typename TO>
int launch_combine_rows(const AttnArgs& a, TO* out, float* lse, cudaStream_t stream)
{
    const int rows = a.B * a.nq * a.n_h;
    const bool wide = combine_rows_wide(a);
    const int vpl = wide ? 8 : 4;
    const int items = rows * (a.c / (32 * vpl));
    const dim3 grid((unsigned)((items + kRowWarps - 1) / kRowWarps));
    const __nv_bfloat16* po = static_cast<const __nv_bfloat16*>(a.part_o);
    if (wide)
        launch_pdl(attn_combine_rows<TO, 8, 16>, grid, dim3(32 * kRowWarps), 0, stream, po, a.part_ml, a.splits,
                   a.n_h, a.c, items, out, lse);
    else
        launch_pdl(attn_combine_rows<TO, 4, 32>, grid, dim3(32 * kRowWarps), 0, stream, po, a.part_ml, a.splits,
                   a.n_h, a.c, items, out, lse);
    return launch_status();
}

int launch_cuda_core(AttnArgs a, const AttnPlan& plan, int dtype, cudaStream_t stream)
{
    a.splits = plan.splits;
    a.per_split = plan.per_split;
    const int G = a.B * a.nq;
    dim3 grid((unsigned)plan.splits, (unsigned)plan.head_groups, (unsigned)G);
    const size_t smem = ((size_t)kCcChunk * (a.c + 1) + (size_t)kCcHeads * a.c) * sizeof(float);
    if (dtype == CSA_BF16) {
        auto kern = attn_cuda_core<__nv_bfloat16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_pdl(kern, grid, dim3(256), smem, stream, a);
    } else {
        auto kern = attn_cuda_core<float>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_pdl(kern, grid, dim3(256), smem, stream, a);
    }
    return launch_status();
}

}  // namespace

int launch_attn_combine(const AttnArgs& a, bool normalized, void* out, int out_bf16, float* lse,
                        cudaStream_t stream)
{
    const int G = a.B * a.nq;
    dim3 grid((unsigned)a.n_h, (unsigned)G, (unsigned)((a.c + kCombineCols - 1) / kCombineCols));
    dim3 block(kCombineThreads);
    const float2* ml = a.part_ml;
    // bf16 partials of the tensor-core path, widths of whole 256-column slices, and few
    // enough splits for one round of loads: the warp-per-row merge; otherwise the
    // (head, column slice) CTAs below, which spread many splits over their threads
    if (normalized && combine_rows_fits(a) && a.c % 256 == 0 && aligned16(out) && aligned16(a.part_o)) {
        if (out_bf16) return launch_combine_rows(a, static_cast<__nv_bfloat16*>(out), lse, stream);
        return launch_combine_rows(a, static_cast<float*>(out), lse, stream);
    }
    if (normalized) {
        const __nv_bfloat16* po = static_cast<const __nv_bfloat16*>(a.part_o);
        if (out_bf16)
            launch_pdl(attn_combine<__nv_bfloat16, __nv_bfloat16>, grid, block, 0, stream, po, ml, a.splits, a.n_h,
                       a.c, static_cast<__nv_bfloat16*>(out), lse);
        else
            launch_pdl(attn_combine<float, __nv_bfloat16>, grid, block, 0, stream, po, ml, a.splits, a.n_h, a.c,
                       static_cast<float*>(out), lse);
    } else {
        const float* po = static_cast<const float*>(a.part_o);
        if (out_bf16)
            launch_pdl(attn_combine<__nv_bfloat16, float>, grid, block, 0, stream, po, ml, a.splits, a.n_h, a.c,
                       static_cast<__nv_bfloat16*>(out), lse);
        else
            launch_pdl(attn_combine<float, float>, grid, block, 0, stream, po, ml, a.splits, a.n_h, a.c,
                       static_cast<float*>(out), lse);
    }
    return launch_status();
}

// Shared host path of both exports.
int attn_run(AttnArgs a, float scale, void* out, float* lse, void* workspace, size_t ws_bytes,
             int dtype, int out_bf16, int64_t entries, cudaStream_t stream)
{
    if (dtype != CSA_BF16 && dtype != CSA_F32) return CSA_ERR_DTYPE;
    if (out_bf16 && dtype != CSA_BF16) return CSA_ERR_DTYPE;
    if (a.B < 0 || a.nq < 0 || a.n_h <= 0 || a.c <= 0 || a.N_cap < 0 || entries < 0)
        return CSA_ERR_ARG;
    if (a.c > kMaxC) return CSA_ERR_UNSUPPORTED;
    if (a.B == 0 || a.nq == 0) return CSA_OK;
    if (!a.q || !a.cache || !out || (!a.dense && !a.idx) || (a.dense && !a.t)) return CSA_ERR_ARG;
    const uintptr_t eb = (uintptr_t)elem_bytes(dtype) - 1;
    if ((((uintptr_t)a.q | (uintptr_t)a.cache) & eb) || ((uintptr_t)out & (out_bf16 ? 1 : 3)) ||
        ((uintptr_t)lse & 3) || ((uintptr_t)a.idx & 3) || ((uintptr_t)a.t & 7))
        return CSA_ERR_ALIGN;
    const int G = a.B * a.nq;
    if (!workspace || ws_bytes < csa_attn_workspace_size(a.B, a.nq, a.n_h, a.c, entries))
        return CSA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return CSA_ERR_ALIGN;
    a.scale_log2 = (scale > 0.f ? scale : 1.0f / sqrtf((float)a.c)) * kLog2e;

    // the tensor-core kernels address cache and window rows with 32-bit TMA coordinates
    const bool tc = dtype == CSA_BF16 && attn_tc_supported(a.n_h, a.c) &&
                    (int64_t)a.B * a.N_cap < (int64_t(1) << 31) - 64 &&
                    (!a.win || (int64_t)a.B * a.win_cap < (int64_t(1) << 31));
    AttnPlan plan = tc ? attn_plan_tc(G, a.n_h, a.c, entries) : attn_plan_cuda_core(G, a.n_h, entries);
    char* ws = static_cast<char*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws);  // sticky device status word
    ws += 256;
    a.part_o = ws;
    a.part_ml = reinterpret_cast<float2*>(ws + align_up((size_t)G * plan.splits * a.n_h * a.c * sizeof(float), 256));
    a.splits = plan.splits;
    a.per_split = plan.per_split;
    // one split per query (many queries): the tcgen05 kernel writes the final output and
    // lse itself, with no combine pass
    a.direct = tc && plan.splits == 1 && aligned16(out);
    a.out = out;
    a.out_bf16 = out_bf16;
    a.lse = lse;
    int st = tc ? launch_attn_tc(a, plan, status, stream) : launch_cuda_core(a, plan, dtype, stream);
    if (st != CSA_OK || a.direct) return st;
    return launch_attn_combine(a, tc, out, out_bf16, lse, stream);
}

}  // namespace csa

extern "C" size_t csa_attn_workspace_size(int B, int nq, int n_h, int c, int64_t max_entries)
{
    using namespace csa;
    if (B <= 0 || nq <= 0 || n_h <= 0 || c <= 0 || max_entries < 0) return 0;
    const int G = B * nq;
    AttnPlan p1 = attn_plan_cuda_core(G, n_h, max_entries);
    size_t bytes = attn_ws_bytes(G, n_h, c, p1.splits);
    if (attn_tc_supported(n_h, c)) {
        AttnPlan p2 = attn_plan_tc(G, n_h, c, max_entries);
        size_t b2 = attn_ws_bytes(G, n_h, c, p2.splits);
        if (b2 > bytes) bytes = b2;
    }
    return bytes;
}

extern "C" int csa_sparse_attn(const void* q, const void* cache, const int32_t* idx, int B,
                               int nq, int n_h, int c, int64_t N_cap, int k, float scale,
                               void* out, float* lse, void* workspace, size_t ws_bytes,
                               int dtype, int out_bf16, csa_stream_t stream)
{
    using namespace csa;
    if (k < 0) return CSA_ERR_ARG;
    AttnArgs a{};
    a.q = q; a.cache = cache; a.idx = idx; a.t = nullptr;
    a.B = B; a.nq = nq; a.n_h = n_h; a.c = c; a.N_cap = N_cap; a.k = k; a.m_prime = 1;
    a.dense = 0;
    return attn_run(a, scale, out, lse, workspace, ws_bytes, dtype, out_bf16, k,
                    reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int hca_dense_attn(const void* q, const void* cache, const int64_t* t, int B, int nq,
                              int n_h, int c, int64_t N_cap, int m_prime, float scale, void* out,
                              float* lse, void* workspace, size_t ws_bytes, int dtype,
                              int out_bf16, csa_stream_t stream)
{
    using namespace csa;
    if (m_prime <= 0) return CSA_ERR_ARG;
    AttnArgs a{};
    a.q = q; a.cache = cache; a.idx = nullptr; a.t = t;
    a.B = B; a.nq = nq; a.n_h = n_h; a.c = c; a.N_cap = N_cap; a.k = 0; a.m_prime = m_prime;
    a.dense = 1;
    return attn_run(a, scale, out, lse, workspace, ws_bytes, dtype, out_bf16, N_cap,
                    reinterpret_cast<cudaStream_t>(stream));
}

// Sliding-window variants: the same calls with the window entries of tokens
// max(0, t - n_win + 1) .. t joined to the entry set under one softmax.
namespace {
int window_args(csa::AttnArgs& a, const void* win, const int64_t* t, int n_win, int64_t win_cap,
                int dtype)
{
    if (!win || !t || n_win < 1 || win_cap < n_win || win_cap >= (int64_t(1) << 31)) return CSA_ERR_ARG;
    if (((uintptr_t)win & (uintptr_t)(csa::elem_bytes(dtype) - 1)) || ((uintptr_t)t & 7)) return CSA_ERR_ALIGN;
    a.win = win;
    a.t = t;  // the sparse path reads t only for the window
    a.n_win = n_win;
    a.win_cap = (int)win_cap;
    return CSA_OK;
}
}  // namespace

extern "C" int csa_sparse_attn_window(const void* q, const void* cache, const int32_t* idx,
                                      const void* win, const int64_t* t, int B, int nq, int n_h,
                                      int c, int64_t N_cap, int k, int n_win, int64_t win_cap,
                                      float scale, void* out, float* lse, void* workspace,
                                      size_t ws_bytes, int dtype, int out_bf16, csa_stream_t stream)
{
    using namespace csa;
    if (k < 0) return CSA_ERR_ARG;
    AttnArgs a{};
    a.q = q; a.cache = cache; a.idx = idx; a.t = nullptr;
    a.B = B; a.nq = nq; a.n_h = n_h; a.c = c; a.N_cap = N_cap; a.k = k; a.m_prime = 1;
    a.dense = 0;
    const int st = window_args(a, win, t, n_win, win_cap, dtype);
    if (st != CSA_OK) return st;
    return attn_run(a, scale, out, lse, workspace, ws_bytes, dtype, out_bf16, (int64_t)k + n_win,
                    reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int hca_dense_attn_window(const void* q, const void* cache, const int64_t* t, const void* win,
                                     int B, int nq, int n_h, int c, int64_t N_cap, int m_prime,
                                     int n_win, int64_t win_cap, float scale, void* out, float* lse,
                                     void* workspace, size_t ws_bytes, int dtype, int out_bf16,
                                     csa_stream_t stream)
{
    using namespace csa;
    if (m_prime <= 0) return CSA_ERR_ARG;
    AttnArgs a{};
    a.q = q; a.cache = cache; a.idx = nullptr; a.t = t;
    a.B = B; a.nq = nq; a.n_h = n_h; a.c = c; a.N_cap = N_cap; a.k = 0; a.m_prime = m_prime;
    a.dense = 1;
    const int st = window_args(a, win, t, n_win, win_cap, dtype);
    if (st != CSA_OK) return st;
    return attn_run(a, scale, out, lse, workspace, ws_bytes, dtype, out_bf16, N_cap + n_win,
                    reinterpret_cast<cudaStream_t>(stream));
}
