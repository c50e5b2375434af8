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

// Vectorised (16-byte) path when every row offset of the call is 16-byte aligned,
// element path otherwise.
bool vector_ok(const PoolArgs& p, int dtype)
{
    const int V = 16 / elem_bytes(dtype);
    return p.c % V == 0 && p.ld_row % V == 0 && p.ld_batch % V == 0 && p.out_ld_batch % V == 0 &&
           aligned16(p.Xa) && aligned16(p.Za) && (!p.has_b || (aligned16(p.Xb) && aligned16(p.Zb))) &&
           aligned16(p.out) && (!p.Ba || aligned16(p.Ba)) && (!p.Bb || aligned16(p.Bb));
}

int launch_pool(const PoolArgs& p, int dtype, cudaStream_t stream)
{
    const bool vec = vector_ok(p, dtype);
    const int V = vec ? 16 / elem_bytes(dtype) : 1;
    const int64_t total = (int64_t)p.B * (p.e1 - p.e0) * (p.c / V);
    if (total == 0) return CSA_OK;
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
    return launch_pool(p, dtype, reinterpret_cast<cudaStream_t>(stream));
}
