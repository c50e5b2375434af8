// Sequence-dimension compression of the projected KV streams: CSA overlapped 2m-row
// pooling and HCA m'-row pooling.
//
// Both are one operation ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch",
// section 11: HCA is CSA with the b-stream removed and m replaced by m'): for every
// output column a softmax over the candidate rows' logits weights the candidate rows'
// values (section 4 softmax, boxed sums of sections 5 and 10).
//
// Design (HBM-bound streaming, every input row read exactly once):
//   - one thread owns 16 bytes (8 bf16 / 4 fp32 columns) of one compressed entry and
//     walks that entry's candidate rows; a warp covers 512 contiguous bytes of a row,
//     so each row access is a fully coalesced 16-byte-per-lane load;
//   - loads use the streaming cache hint (read once, evict first) and are issued in
//     groups of kUnroll rows (Z and C) before any arithmetic, so each thread keeps
//     2*kUnroll 16-byte requests in flight;
//   - the softmax is computed online with exactly ONE exponential per candidate
//     element: a new maximum rescales the running sums by exp(old - new) instead of
//     weighting the new element by exp(new - new) = 1, so the exp count equals the
//     candidate count and the exp unit never becomes the limit;
//   - fp32 state (running max, sum, weighted sum) per column, output rounded once.
#include "common.cuh"
#include "tc_utils.cuh"

namespace csa {
namespace {

constexpr int kUnroll = 4;
constexpr int kThreads = 256;

struct PoolArgs {
    const void* Xa;  // values, stream a (HCA: the only stream)
    const void* Za;  // logits, stream a
    const void* Xb;  // values, stream b (CSA only), previous block
    const void* Zb;  // logits, stream b
    const float* Ba;
    const float* Bb;
    int64_t ld_row, ld_batch, tok0;
    void* out;
    int64_t out_ld_batch;
    int B, c, m;
    int64_t e0, e1;
    int has_b;
    int64_t n_rows;  // token rows of each batch in the buffers (n - tok0)
};

// Loads of V consecutive elements of one row: one 16-byte streaming load when the row
// group is a full vector (the hot path), element loads otherwise (odd widths).
template <typename T, int V>
struct RowLoad {
    using Raw = float[V];
    CSA_DEV static void load(const T* p, Raw& r)
    {
#pragma unroll
        for (int v = 0; v < V; ++v) r[v] = to_f32(p[v]);
    }
    CSA_DEV static void unpack(const Raw& r, float* f)
    {
#pragma unroll
        for (int v = 0; v < V; ++v) f[v] = r[v];
    }
};

template <>
struct RowLoad<__nv_bfloat16, 8> {
    using Raw = uint4;
    CSA_DEV static void load(const __nv_bfloat16* p, Raw& r) { r = __ldcs(reinterpret_cast<const uint4*>(p)); }
    CSA_DEV static void unpack(const Raw& u, float* f) { Vec<__nv_bfloat16>::unpack(u, f); }
};

template <>
struct RowLoad<float, 4> {
    using Raw = uint4;
    CSA_DEV static void load(const float* p, Raw& r) { r = __ldcs(reinterpret_cast<const uint4*>(p)); }
    CSA_DEV static void unpack(const Raw& u, float* f)
    {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    }
};

struct OnlineSoftmax {
    float mx, sum, acc;
    CSA_DEV void init()
    {
        mx = -INFINITY;
        sum = 0.f;
        acc = 0.f;
    }
    // One candidate (logit l, value x); one exponential either way.
    CSA_DEV void add(float l, float x)
    {
        const float d = l - mx;
        const float e = exp2f(-fabsf(d) * kLog2e);
        if (d > 0.f) {
            sum = fmaf(sum, e, 1.f);
            acc = fmaf(acc, e, x);
            mx = l;
        } else {
            sum += e;
            acc = fmaf(e, x, acc);
        }
    }
};

// Pool `rows` consecutive token rows starting at Z / X (already offset to this
// thread's 16-byte column group) into the running softmax state of V columns.
template <typename T, int V>
CSA_DEV void pool_rows(const T* __restrict__ Z, const T* __restrict__ X,
                       const float* __restrict__ bias, int rows, int64_t ld_row,
                       int c, OnlineSoftmax* st)
{
    for (int r0 = 0; r0 < rows; r0 += kUnroll) {
        typename RowLoad<T, V>::Raw zr[kUnroll], xr[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (r0 + u < rows) {
                RowLoad<T, V>::load(Z + (int64_t)(r0 + u) * ld_row, zr[u]);
                RowLoad<T, V>::load(X + (int64_t)(r0 + u) * ld_row, xr[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (r0 + u < rows) {
                float z[V], x[V];
                RowLoad<T, V>::unpack(zr[u], z);
                RowLoad<T, V>::unpack(xr[u], x);
                if (bias) {
                    const float* bp = bias + (int64_t)(r0 + u) * c;
                    if constexpr (V % 4 == 0) {
#pragma unroll
                        for (int q = 0; q < V / 4; ++q) {
                            float4 b4 = __ldg(reinterpret_cast<const float4*>(bp) + q);
                            z[4 * q] += b4.x; z[4 * q + 1] += b4.y;
                            z[4 * q + 2] += b4.z; z[4 * q + 3] += b4.w;
                        }
                    } else {
#pragma unroll
                        for (int v = 0; v < V; ++v) z[v] += __ldg(bp + v);
                    }
                }
#pragma unroll
                for (int v = 0; v < V; ++v) st[v].add(z[v], x[v]);
            }
        }
    }
}

template <typename T, int V>
__global__ void __launch_bounds__(kThreads) pool_kernel(PoolArgs p)
{
    pdl_launch_dependents();
    pdl_wait();
    const int vecs = p.c / V;
    const int64_t nent = p.e1 - p.e0;
    const int64_t total = (int64_t)p.B * nent * vecs;
    const T* Xa = static_cast<const T*>(p.Xa);
    const T* Za = static_cast<const T*>(p.Za);
    const T* Xb = static_cast<const T*>(p.Xb);
    const T* Zb = static_cast<const T*>(p.Zb);
    T* out = static_cast<T*>(p.out);
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < total;
         w += (int64_t)gridDim.x * blockDim.x) {
        const int vi = (int)(w % vecs);
        const int64_t rest = w / vecs;
        const int64_t i = p.e0 + rest % nent;
        const int64_t b = rest / nent;
        const int col = vi * V;
        OnlineSoftmax st[V];
#pragma unroll
        for (int v = 0; v < V; ++v) st[v].init();

        const int64_t base = b * p.ld_batch + col;
        const int64_t ra = (int64_t)p.m * i - p.tok0;  // first a-row of block i
        pool_rows<T, V>(Za + base + ra * p.ld_row, Xa + base + ra * p.ld_row,
                        p.Ba ? p.Ba + col : nullptr, p.m, p.ld_row, p.c, st);
        if (p.has_b && i > 0) {
            const int64_t rb = (int64_t)p.m * (i - 1) - p.tok0;  // block i-1 via stream b
            pool_rows<T, V>(Zb + base + rb * p.ld_row, Xb + base + rb * p.ld_row,
                            p.Bb ? p.Bb + col : nullptr, p.m, p.ld_row, p.c, st);
        }
        float o[V];
#pragma unroll
        for (int v = 0; v < V; ++v) o[v] = st[v].acc / st[v].sum;
        T* dst = out + b * p.out_ld_batch + i * p.c + col;
        if constexpr (V * sizeof(T) == 16) {
            Vec<T>::store(dst, o);
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v) dst[v] = from_f32<T>(o[v]);
        }
    }
}

// Decode-sized calls (at most one wave of entries): one CTA per (entry, batch row).
// pool_kernel gives a thread one column group and walks the 2m (or m') candidate rows in
// dependent batches of kUnroll; at a block end of a decode that chain of round trips is
// the whole cost.  Here the candidate rows are fetched into L2 before the dependency wait,
// the whole CTA loads a chunk of up to kSmallChunk candidates at once (logits with their
// bias, and values, as fp32 into shared memory), and one thread per column folds the
// chunk's candidates, in pool_kernel's order, into the same online softmax: the result
// is bit-identical to pool_kernel's.
constexpr int kSmallChunk = 32;             // candidates per chunk
constexpr int kSmallSmem = 160 * 1024;      // shared-memory bound of a chunk: [chunk][c] x 2 fp32
constexpr int kSmallItems = 4;              // (candidate, column group) loads per thread per round

template <typename T, int V>
__global__ void __launch_bounds__(1024, 1) pool_small_kernel(PoolArgs p, int chunk)
{
    pdl_launch_dependents();
    extern __shared__ float s_zx[];         // [chunk][c] logits (bias added), then [chunk][c] values
    const int64_t i = p.e0 + blockIdx.x;    // entry
    const int64_t b = blockIdx.y;           // batch row
    const int c = p.c, vecs = c / V;
    const int ncand = p.has_b && i > 0 ? 2 * p.m : p.m;
    const int64_t ra = (int64_t)p.m * i - p.tok0;        // first a-row of block i
    const int64_t rb = (int64_t)p.m * (i - 1) - p.tok0;  // block i-1 via stream b
    const int64_t boff = b * p.ld_batch;
    // candidate q: a-row q for q < m, then b-row q - m (pool_kernel's order)
    auto row_of = [&](const void* sa, const void* sb, int q) -> const T* {
        return q < p.m ? static_cast<const T*>(sa) + boff + (ra + q) * p.ld_row
                       : static_cast<const T*>(sb) + boff + (rb + q - p.m) * p.ld_row;
    };
    if constexpr (V * sizeof(T) == 16) {
        // whole rows into L2 while the previous kernel finishes (16-byte aligned rows of
        // c * sizeof(T) bytes, a multiple of 16, on this path)
        for (int u = threadIdx.x; u < 2 * ncand; u += blockDim.x)
            tc::prefetch_l2(u & 1 ? row_of(p.Xa, p.Xb, u >> 1) : row_of(p.Za, p.Zb, u >> 1), (uint32_t)(c * sizeof(T)));
    }
    pdl_wait();
    float* sz = s_zx;
    float* sx = s_zx + (size_t)chunk * c;
    const int j = threadIdx.x;  // the column this thread folds
    OnlineSoftmax st;
    st.init();
    for (int q0 = 0; q0 < ncand; q0 += chunk) {
        const int nq = min(chunk, ncand - q0);
        const int items = nq * vecs;
        for (int w0 = threadIdx.x; w0 < items; w0 += kSmallItems * blockDim.x) {
            typename RowLoad<T, V>::Raw zr[kSmallItems], xr[kSmallItems];
#pragma unroll
            for (int u = 0; u < kSmallItems; ++u) {
                const int w = w0 + u * blockDim.x;
                if (w < items) {
                    const int q = q0 + w / vecs, col = (w % vecs) * V;
                    RowLoad<T, V>::load(row_of(p.Za, p.Zb, q) + col, zr[u]);
                    RowLoad<T, V>::load(row_of(p.Xa, p.Xb, q) + col, xr[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < kSmallItems; ++u) {
                const int w = w0 + u * blockDim.x;
                if (w < items) {
                    const int q = q0 + w / vecs, col = (w % vecs) * V;
                    float z[V], x[V];
                    RowLoad<T, V>::unpack(zr[u], z);
                    RowLoad<T, V>::unpack(xr[u], x);
                    const float* bias = q < p.m ? (p.Ba ? p.Ba + (int64_t)q * c : nullptr)
                                                : (p.Bb ? p.Bb + (int64_t)(q - p.m) * c : nullptr);
                    const int o = (q - q0) * c + col;
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        sz[o + v] = bias ? z[v] + __ldg(bias + col + v) : z[v];
                        sx[o + v] = x[v];
                    }
                }
            }
        }
        __syncthreads();
        if (j < c)
            for (int q = 0; q < nq; ++q) st.add(sz[q * c + j], sx[q * c + j]);
        __syncthreads();  // the chunk's buffer is rewritten by the next chunk
    }
    if (j < c) static_cast<T*>(p.out)[b * p.out_ld_batch + i * c + j] = from_f32<T>(st.acc / st.sum);
}

// The chunk (candidates held in shared memory at once) of pool_small_kernel, or 0 when
// the call is not decode-sized or its columns exceed one CTA.
int small_pool_chunk(const PoolArgs& p)
{
    const int64_t nent = p.e1 - p.e0;
    if (nent <= 0 || (int64_t)p.B * nent > kNumSMs || p.B > 65535 || p.c > 1024) return 0;
    const int ncand = p.has_b ? 2 * p.m : p.m;
    int chunk = kSmallSmem / (8 * p.c);
    if (chunk > kSmallChunk) chunk = kSmallChunk;
    if (chunk > ncand) chunk = ncand;
    return chunk;
}

// ----------------------------------------------------------------------------------
// TMA-staged streaming path (bf16, c a multiple of 256, prefill-sized calls; CSA with
// m = 4, HCA with m' a multiple of 32).
//
// pool_kernel's per-thread walk keeps only 2 kUnroll 16-byte loads in flight per thread:
// it reaches 0.67 (CSA) and 0.72 (HCA) of the HBM copy rate.  Here a persistent CTA per
// SM streams the rows through a 6-stage ring of 32 KB TMA boxes ({256 columns x R rows}
// of each stream, unswizzled, so row r of a stream is 512 contiguous bytes of shared
// memory), and sixteen compute warps pool them with one thread per column of the
// 256-column slice:
//   CSA   a stage holds 16 rows of Z^a and C^a (the blocks of 4 consecutive entries) and
//         16 rows of Z^b and C^b starting one block earlier, so each of the 4 entries
//         finds its 8 candidates in the same stage; each of the two warp groups takes 2
//         of the 4 entries.  Entry 0's b-rows (before the batch's first token) are loaded
//         but never used.
//   HCA   a stage holds 32 rows of Z and C; an entry of m' rows is m'/32 consecutive
//         stages, pooled online; the two warp groups take alternate entries.
// Logits are taken in base 2 (zl = (z + B) log2 e) and every exponential is the
// multi-function unit's ex2 (relative error about 2^-22).  Each compute warp releases a
// stage with one arrival.  Waits are bounded; after a timeout (never expected) the
// compute threads write NaN into every entry they have not finished, so a failure
// cannot pass for a result.
constexpr int kSpCols = 256;                     // columns per slice: one per compute thread
constexpr int kSpWarps = 16;                     // compute warps: two per column group
constexpr int kSpEntPerThread = 2;               // of a stage's 4 entries
constexpr int kSpThreads = 32 * (kSpWarps + 1);  // + the producer warp
constexpr int kSpStageBytes = 32768;
constexpr int kSpStages = 6;
constexpr int kSpSmem = kSpStages * kSpStageBytes + 128 + 128;
constexpr int kSpCsaEntries = 64;                // CSA entries per work item (16 stages)

struct SpArgs {
    int64_t rows_per_batch, tok0;
    const float* Ba;         // [m][c] or null
    const float* Bb;         // [m][c] or null
    __nv_bfloat16* out;
    int64_t out_ld_batch;
    int c, m;
    int64_t e0, e1;
    int n_slices;
    int64_t groups;          // per (batch, slice): groups of kSpCsaEntries entries
    int64_t items;           // B * groups * n_slices
};

template <bool kCsa>
__global__ void __launch_bounds__(kSpThreads, 1)
stream_pool_kernel(const __grid_constant__ CUtensorMap t0, const __grid_constant__ CUtensorMap t1,
                   const __grid_constant__ CUtensorMap t2, const __grid_constant__ CUtensorMap t3, SpArgs a)
{
    // CSA: t0 = Z^a, t1 = C^a, t2 = Z^b, t3 = C^b.  HCA: t0 = Z, t1 = C.
    constexpr int kStreams = kCsa ? 4 : 2;
    constexpr int kRows = kSpStageBytes / (kStreams * kSpCols * 2);  // CSA 16 rows (4 blocks), HCA 32
    constexpr int kStreamBytes = kRows * kSpCols * 2;
    constexpr float kL2e = 1.4426950408889634f;
    extern __shared__ uint8_t smem_raw[];
    // 128-byte aligned; an offset from the __shared__ array keeps derived pointers in the
    // shared window (shared-memory instructions)
    uint8_t* smem = smem_raw + ((128u - (tc::smem_u32(smem_raw) & 127u)) & 127u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSpStages * kSpStageBytes);
    uint64_t* empty = full + kSpStages;
    volatile uint32_t* abort_flag = reinterpret_cast<uint32_t*>(empty + kSpStages);

    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSpStages; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], kSpWarps);  // every compute warp passes every stage
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&t0);
        tc::tma_prefetch_desc(&t1);
        if (kCsa) {
            tc::tma_prefetch_desc(&t2);
            tc::tma_prefetch_desc(&t3);
        }
    }
    __syncthreads();
    pdl_wait();

    auto item_of = [&](int64_t t, int& b, int& sl, int64_t& g) {
        sl = (int)(t % a.n_slices);
        const int64_t r = t / a.n_slices;
        g = r % a.groups;
        b = (int)(r / a.groups);
    };
    // stages of an item and the entries it covers
    auto item_span = [&](int64_t g, int64_t& ent0, int& nent, int& nst) {
        if (kCsa) {
            ent0 = a.e0 + g * kSpCsaEntries;
            const int64_t left = a.e1 - ent0;
            nent = (int)(left < kSpCsaEntries ? left : kSpCsaEntries);
            nst = (nent + 3) / 4;
        } else {  // one entry of m' rows
            ent0 = a.e0 + g;
            nent = 1;
            nst = a.m / kRows;
        }
    };

    if (warp == kSpWarps) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int it = 0;
            bool stop = false;
            for (int64_t t = blockIdx.x; t < a.items && !stop; t += gridDim.x) {
                int b, sl, nent, nst;
                int64_t g, ent0;
                item_of(t, b, sl, g);
                item_span(g, ent0, nent, nst);
                const int x = sl * kSpCols;
                const int ra = (int)(b * a.rows_per_batch + (int64_t)a.m * ent0 - a.tok0);  // first a-row
                for (int j = 0; j < nst; ++j, ++it) {
                    const int s = it % kSpStages;
                    const uint32_t ph = (it / kSpStages) & 1;
                    if (*abort_flag || !tc::mbar_wait(&empty[s], ph ^ 1, tc::kWaitBudget)) {
                        *abort_flag = 1;
                        stop = true;
                        break;
                    }
                    uint8_t* st = smem + s * kSpStageBytes;
                    tc::mbar_arrive_expect_tx(&full[s], kSpStageBytes);
                    tc::tma_load_2d(st, &t0, &full[s], x, ra + kRows * j);
                    tc::tma_load_2d(st + kStreamBytes, &t1, &full[s], x, ra + kRows * j);
                    if (kCsa) {  // b-rows one block (m = 4 rows) earlier
                        tc::tma_load_2d(st + 2 * kStreamBytes, &t2, &full[s], x, ra - 4 + kRows * j);
                        tc::tma_load_2d(st + 3 * kStreamBytes, &t3, &full[s], x, ra - 4 + kRows * j);
                    }
                }
            }
            // drain: every issued load has landed before the CTA may exit
            for (int j = it - kSpStages < 0 ? 0 : it - kSpStages; j < it; ++j)
                if (!tc::mbar_wait(&full[j % kSpStages], (j / kSpStages) & 1, tc::kWaitBudget)) *abort_flag = 1;
        }
    } else if constexpr (!kCsa) {
        // ------------------------------------------------------------ HCA compute
        // The two warp groups take alternate items (one entry each), so each thread keeps
        // one online softmax state per entry (thread = column); the rows of a stage are
        // pooled 8 at a time: the chunk maximum rescales the state once, then one ex2 per
        // row.  Each group still waits for every stage of the other group's items and
        // releases it at once, so that it observes every phase of every slot in order: a
        // slot's full barrier can then never be a whole phase behind the parity a group
        // waits for (TMA loads of different stages complete in any order), and a slot is
        // refilled only after both groups have passed it.
        const int col = threadIdx.x % kSpCols;
        const int grp = threadIdx.x / kSpCols;
        bool ok = true;
        int64_t t = blockIdx.x, tl = 0;  // tl: the CTA's item ordinal
        for (; t < a.items; t += gridDim.x, ++tl) {
            int b, sl, nent, nst;
            int64_t g, ent0;
            item_of(t, b, sl, g);
            item_span(g, ent0, nent, nst);
            if ((int)(tl & 1) != grp) {  // the other group's item: pass its stages
                for (int js = 0; js < nst && ok; ++js) {
                    const int64_t it = tl * nst + js;
                    const int s = (int)(it % kSpStages);
                    if (*abort_flag || !tc::mbar_wait(&full[s], (uint32_t)(it / kSpStages) & 1, tc::kWaitBudget)) {
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&empty[s]);
                }
                if (!ok) break;
                continue;
            }
            const int j = sl * kSpCols + col;
            float mx = -INFINITY, l = 0.f, acc = 0.f;
            for (int js = 0; js < nst; ++js) {
                const int64_t it = tl * nst + js;  // the producer's stage count
                const int s = (int)(it % kSpStages);
                if (*abort_flag || !tc::mbar_wait(&full[s], (uint32_t)(it / kSpStages) & 1, tc::kWaitBudget)) {
                    *abort_flag = 1;
                    ok = false;
                    break;
                }
                const __nv_bfloat16* sz = reinterpret_cast<const __nv_bfloat16*>(smem + s * kSpStageBytes) + col;
                const __nv_bfloat16* sc = sz + kRows * kSpCols;
#pragma unroll
                for (int r0 = 0; r0 < kRows; r0 += 8) {
                    float zl[8], xv[8], cmax = -INFINITY;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int row = kRows * js + r0 + u;  // token within the entry
                        const float bz = a.Ba ? __ldg(&a.Ba[(int64_t)row * a.c + j]) : 0.f;
                        zl[u] = (__bfloat162float(sz[(r0 + u) * kSpCols]) + bz) * kL2e;
                        xv[u] = __bfloat162float(sc[(r0 + u) * kSpCols]);
                        cmax = fmaxf(cmax, zl[u]);
                    }
                    const float mn = fmaxf(mx, cmax);
                    const float f = tc::ex2_approx(mx - mn);  // 0 while the state is empty
                    l *= f;
                    acc *= f;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float p = tc::ex2_approx(zl[u] - mn);
                        l += p;
                        acc = fmaf(p, xv[u], acc);
                    }
                    mx = mn;
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&empty[s]);  // this warp is done with the stage
            }
            if (!ok) break;
            a.out[(int64_t)b * a.out_ld_batch + ent0 * a.c + j] = __float2bfloat16_rn(acc * tc::rcp_approx(l));
        }
        if (!ok) {
            // timeout: NaN into this group's unfinished entries
            for (; t < a.items; t += gridDim.x, ++tl) {
                if ((int)(tl & 1) != grp) continue;
                int b, sl;
                int64_t g;
                item_of(t, b, sl, g);
                a.out[(int64_t)b * a.out_ld_batch + (a.e0 + g) * a.c + sl * kSpCols + col] = __float2bfloat16_rn(NAN);
            }
        }
    } else {
        // ------------------------------------------------------------ CSA compute: thread = column
        const int col = threadIdx.x % kSpCols;
        const int q0 = (threadIdx.x / kSpCols) * kSpEntPerThread;  // this thread's first entry of a stage
        int it = 0;
        bool ok = true;
        int64_t t = blockIdx.x;
        for (; t < a.items && ok; t += gridDim.x) {
            int b, sl, nent, nst;
            int64_t g, ent0;
            item_of(t, b, sl, g);
            item_span(g, ent0, nent, nst);
            const int j = sl * kSpCols + col;
            __nv_bfloat16* orow = a.out + (int64_t)b * a.out_ld_batch + j;
            float ba[4], bb[4];  // biases in base-2 units
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                ba[r] = a.Ba ? __ldg(&a.Ba[r * a.c + j]) * kL2e : 0.f;
                bb[r] = a.Bb ? __ldg(&a.Bb[r * a.c + j]) * kL2e : 0.f;
            }
            for (int js = 0; js < nst; ++js, ++it) {
                const int s = it % kSpStages;
                if (*abort_flag || !tc::mbar_wait(&full[s], (it / kSpStages) & 1, tc::kWaitBudget)) {
                    *abort_flag = 1;
                    ok = false;
                    break;
                }
                const __nv_bfloat16* st = reinterpret_cast<const __nv_bfloat16*>(smem + s * kSpStageBytes) + col;
                const __nv_bfloat16* za = st;
                const __nv_bfloat16* ca = st + kRows * kSpCols;
                const __nv_bfloat16* zb = st + 2 * kRows * kSpCols;
                const __nv_bfloat16* cb = st + 3 * kRows * kSpCols;
                float res[kSpEntPerThread];
#pragma unroll
                for (int qq = 0; qq < kSpEntPerThread; ++qq) {
                    const int q = q0 + qq;
                    const int64_t i = ent0 + 4 * js + q;
                    const bool has_b = i > 0;  // entry 0 has no b-part
                    float zl[8], xv[8], mx = -INFINITY;
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        zl[r] = fmaf(__bfloat162float(za[(4 * q + r) * kSpCols]), kL2e, ba[r]);
                        xv[r] = __bfloat162float(ca[(4 * q + r) * kSpCols]);
                        zl[4 + r] = has_b ? fmaf(__bfloat162float(zb[(4 * q + r) * kSpCols]), kL2e, bb[r])
                                          : -INFINITY;
                        xv[4 + r] = has_b ? __bfloat162float(cb[(4 * q + r) * kSpCols]) : 0.f;
                    }
#pragma unroll
                    for (int r = 0; r < 8; ++r) mx = fmaxf(mx, zl[r]);
                    float l = 0.f, acc = 0.f;
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const float p = tc::ex2_approx(zl[r] - mx);
                        l += p;
                        acc = fmaf(p, xv[r], acc);
                    }
                    res[qq] = acc * tc::rcp_approx(l);  // l in [1, 8]
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&empty[s]);  // this warp is done with the stage
#pragma unroll
                for (int qq = 0; qq < kSpEntPerThread; ++qq) {
                    const int q = q0 + qq;
                    const int64_t i = ent0 + 4 * js + q;
                    if (4 * js + q < nent) orow[i * a.c] = __float2bfloat16_rn(res[qq]);
                }
            }
            if (!ok) break;
        }
        if (!ok) {
            // timeout: NaN into every entry of this item and of the CTA's later items
            for (; t < a.items; t += gridDim.x) {
                int b, sl, nent, nst;
                int64_t g, ent0;
                item_of(t, b, sl, g);
                item_span(g, ent0, nent, nst);
                __nv_bfloat16* orow = a.out + (int64_t)b * a.out_ld_batch + sl * kSpCols + col;
                for (int e = 0; e < nent; ++e) orow[(ent0 + e) * a.c] = __float2bfloat16_rn(NAN);
            }
        }
    }
}

// Vectorised (16-byte) path when every row offset of the call is 16-byte aligned,
// element path otherwise.
bool vector_ok(const PoolArgs& p, int dtype)
{
    const int V = 16 / elem_bytes(dtype);
    return p.c % V == 0 && p.ld_row % V == 0 && p.ld_batch % V == 0 && p.out_ld_batch % V == 0 &&
           aligned16(p.Xa) && aligned16(p.Za) && (!p.has_b || (aligned16(p.Xb) && aligned16(p.Zb))) &&
           aligned16(p.out) && (!p.Ba || aligned16(p.Ba)) && (!p.Bb || aligned16(p.Bb));
}

// The TMA-staged path for bf16 prefill-sized calls; false when the call does not fit it
// (odd widths or strides, m other than 4 for CSA or not a multiple of 32 for HCA, or too
// little work to fill the SMs), which then runs pool_kernel.
bool launch_stream_pool(const PoolArgs& p, cudaStream_t stream, int& status)
{
    if (p.has_b ? p.m != 4 : p.m % 32 != 0) return false;
    if (p.c % kSpCols != 0 || p.ld_row % 8 != 0 || (p.B > 1 && p.ld_batch % p.ld_row != 0)) return false;
    if (!aligned16(p.Xa) || !aligned16(p.Za) || !aligned16(p.Xb) || !aligned16(p.Zb)) return false;
    const int64_t nent = p.e1 - p.e0;
    SpArgs a;
    a.n_slices = p.c / kSpCols;
    a.groups = p.has_b ? (nent + kSpCsaEntries - 1) / kSpCsaEntries : nent;
    a.items = (int64_t)p.B * a.groups * a.n_slices;
    if (a.items < kNumSMs) return false;
    a.rows_per_batch = p.B > 1 ? p.ld_batch / p.ld_row : p.n_rows;
    const int64_t height = (int64_t)(p.B - 1) * a.rows_per_batch + p.n_rows;  // rows the buffers hold
    if (height + kSpCols >= (int64_t(1) << 31)) return false;
    a.tok0 = p.tok0;
    a.Ba = p.Ba;
    a.Bb = p.Bb;
    a.out = static_cast<__nv_bfloat16*>(p.out);
    a.out_ld_batch = p.out_ld_batch;
    a.c = p.c;
    a.m = p.m;
    a.e0 = p.e0;
    a.e1 = p.e1;
    CUtensorMap tm[4];
    const void* src[4] = {p.Za, p.Xa, p.has_b ? p.Zb : p.Za, p.has_b ? p.Xb : p.Xa};
    for (int i = 0; i < 4; ++i)
        if (!make_tmap_bf16_2d_plain(&tm[i], src[i], (uint64_t)height, (uint64_t)p.c, (uint64_t)p.ld_row, kSpCols,
                                     p.has_b ? 16 : 32)) {
            status = CSA_ERR_CUDA;
            return true;
        }
    const unsigned grid = (unsigned)(a.items < kNumSMs ? a.items : kNumSMs);
    if (p.has_b) {
        cudaFuncSetAttribute(stream_pool_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSpSmem);
        launch_pdl(stream_pool_kernel<true>, dim3(grid), dim3(kSpThreads), (size_t)kSpSmem, stream, tm[0], tm[1],
                   tm[2], tm[3], a);
    } else {
        cudaFuncSetAttribute(stream_pool_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSpSmem);
        launch_pdl(stream_pool_kernel<false>, dim3(grid), dim3(kSpThreads), (size_t)kSpSmem, stream, tm[0], tm[1],
                   tm[2], tm[3], a);
    }
    status = launch_status();
    return true;
}

int launch_pool(const PoolArgs& p, int dtype, cudaStream_t stream)
{
    int status = CSA_OK;
    if (dtype == CSA_BF16 && launch_stream_pool(p, stream, status)) return status;
    const bool vec = vector_ok(p, dtype);
    const int V = vec ? 16 / elem_bytes(dtype) : 1;
    const int64_t total = (int64_t)p.B * (p.e1 - p.e0) * (p.c / V);
    if (total == 0) return CSA_OK;
    if (const int chunk = small_pool_chunk(p)) {
        const dim3 grid((unsigned)(p.e1 - p.e0), (unsigned)p.B);
        const dim3 block((unsigned)((p.c + 31) / 32 * 32));
        const size_t smem = (size_t)chunk * p.c * 8;
        void (*kern)(PoolArgs, int) =
            dtype == CSA_BF16 ? (vec ? pool_small_kernel<__nv_bfloat16, 8> : pool_small_kernel<__nv_bfloat16, 1>)
                              : (vec ? pool_small_kernel<float, 4> : pool_small_kernel<float, 1>);
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_pdl(kern, grid, block, smem, stream, p, chunk);
        return launch_status();
    }
    int64_t blocks = (total + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)kNumSMs * 64;
    if (blocks > cap) blocks = cap;
    if (dtype == CSA_BF16) {
        launch_pdl(vec ? pool_kernel<__nv_bfloat16, 8> : pool_kernel<__nv_bfloat16, 1>, dim3((unsigned)blocks),
                   dim3(kThreads), 0, stream, p);
    } else {
        launch_pdl(vec ? pool_kernel<float, 4> : pool_kernel<float, 1>, dim3((unsigned)blocks), dim3(kThreads), 0,
                   stream, p);
    }
    return launch_status();
}

int check_common(int dtype, int B, int c, int m, int64_t e0, int64_t e1, int64_t n,
                 int64_t ld_row, int64_t ld_batch, int64_t out_ld_batch, int64_t first_row,
                 int64_t tok0)
{
    if (dtype != CSA_BF16 && dtype != CSA_F32) return CSA_ERR_DTYPE;
    if (B < 0 || c <= 0 || m <= 0 || m > 4096 || e0 < 0 || e1 < e0 || n < 0 || tok0 < 0)
        return CSA_ERR_ARG;
    if ((int64_t)m * e1 > n) return CSA_ERR_ARG;
    if (e1 > e0 && first_row < tok0) return CSA_ERR_ARG;
    if (ld_row < c || ld_batch < 0 || out_ld_batch < 0) return CSA_ERR_ARG;
    if (B > 1 && (ld_batch < (n - tok0) * ld_row || out_ld_batch < e1 * (int64_t)c))
        return CSA_ERR_ARG;
    return CSA_OK;
}

}  // namespace
}  // namespace csa

extern "C" int csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                            int64_t ld_row, int64_t ld_batch, int64_t tok0, int64_t n,
                            const float* Ba, const float* Bb, void* out, int64_t out_ld_batch,
                            int B, int c, int m, int64_t entry_begin, int64_t entry_end,
                            int dtype, csa_stream_t stream)
{
    using namespace csa;
    const int64_t first_row = entry_begin == 0 ? 0 : (int64_t)m * (entry_begin - 1);
    int st = check_common(dtype, B, c, m, entry_begin, entry_end, n, ld_row, ld_batch,
                          out_ld_batch, first_row, tok0);
    if (st != CSA_OK) return st;
    if (B == 0 || entry_end == entry_begin) return CSA_OK;
    if (!Ca || !Cb || !Za || !Zb || !out) return CSA_ERR_ARG;
    const uintptr_t eb = (uintptr_t)elem_bytes(dtype) - 1;
    if ((((uintptr_t)Ca | (uintptr_t)Cb | (uintptr_t)Za | (uintptr_t)Zb | (uintptr_t)out) & eb) ||
        (((uintptr_t)Ba | (uintptr_t)Bb) & 3))
        return CSA_ERR_ALIGN;
    PoolArgs p;
    p.Xa = Ca; p.Za = Za; p.Xb = Cb; p.Zb = Zb; p.Ba = Ba; p.Bb = Bb;
    p.ld_row = ld_row; p.ld_batch = ld_batch; p.tok0 = tok0;
    p.out = out; p.out_ld_batch = out_ld_batch;
    p.B = B; p.c = c; p.m = m; p.e0 = entry_begin; p.e1 = entry_end; p.has_b = 1;
    p.n_rows = n - tok0;
    return launch_pool(p, dtype, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int hca_compress(const void* C, const void* Z, int64_t ld_row, int64_t ld_batch,
                            int64_t tok0, int64_t n, const float* Bias, void* out,
                            int64_t out_ld_batch, int B, int c, int m_prime,
                            int64_t entry_begin, int64_t entry_end, int dtype,
                            csa_stream_t stream)
{
    using namespace csa;
    const int64_t first_row = (int64_t)m_prime * entry_begin;
    int st = check_common(dtype, B, c, m_prime, entry_begin, entry_end, n, ld_row, ld_batch,
                          out_ld_batch, first_row, tok0);
    if (st != CSA_OK) return st;
    if (B == 0 || entry_end == entry_begin) return CSA_OK;
    if (!C || !Z || !out) return CSA_ERR_ARG;
    const uintptr_t eb = (uintptr_t)elem_bytes(dtype) - 1;
    if ((((uintptr_t)C | (uintptr_t)Z | (uintptr_t)out) & eb) || ((uintptr_t)Bias & 3))
        return CSA_ERR_ALIGN;
    PoolArgs p;
    p.Xa = C; p.Za = Z; p.Xb = nullptr; p.Zb = nullptr; p.Ba = Bias; p.Bb = nullptr;
    p.ld_row = ld_row; p.ld_batch = ld_batch; p.tok0 = tok0;
    p.out = out; p.out_ld_batch = out_ld_batch;
    p.B = B; p.c = c; p.m = m_prime; p.e0 = entry_begin; p.e1 = entry_end; p.has_b = 0;
    p.n_rows = n - tok0;
    return launch_pool(p, dtype, reinterpret_cast<cudaStream_t>(stream));
}
