// Radix top-k select building blocks shared by the stand-alone select kernel
// (indexer.cu) and the scan kernel that selects in place (indexer_tc.cu)
// ("DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch", section 7: the k largest
// index scores of the visible entries; ties go to the smaller entry index).
//
// Every routine runs on a group of kSelThreads threads identified by `tid` (0..255)
// that synchronise through the barrier policy `Bar`: the whole CTA (__syncthreads) or
// a named barrier over the group.  Selection keys are 64-bit (order_key(score), index):
// larger is better, and among equal scores the smaller index wins.
#pragma once
#include "common.cuh"
#include "indexer.cuh"

namespace csa {
namespace sel {

constexpr int kSelThreads = 256;
constexpr int kListCap = 2048;  // candidates kept in shared memory by the resolving CTA
constexpr int kPer = 8;         // scores per thread per classification round
constexpr int kRound = kPer * kSelThreads;
static_assert(kRound <= kListCap, "a round's staging must fit the shared lists");
constexpr int kRankMax = 256;   // lists up to this size are finished by exact ranking

struct CtaBar {
    static CSA_DEV void sync() { __syncthreads(); }
};
template <int ID>
struct NamedBar {
    static CSA_DEV void sync() { asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(kSelThreads) : "memory"); }
};

// Shared scalars and scratch of one selecting group.
struct Shared {
    uint32_t scr[32];
    uint32_t bin, above, last, cnt, out, nt, nc, bt, bc, ok;
};

// Per-query outputs and workspace views.
struct Query {
    int k;
    int32_t* idx_out;   // [k]
    float* sc_out;      // [k] or null
    uint32_t* ctr;      // [kCtrs]
    uint32_t* hist0;    // [kBins]
    uint2* cand;        // [ld]
    uint2* cand2;       // [ld]
    int64_t ld;
};

CSA_DEV Query query_view(const TopkWs& ws, int g, int k, int32_t* idx_out, float* scores_out)
{
    Query q;
    q.k = k;
    q.idx_out = idx_out + (int64_t)g * k;
    q.sc_out = scores_out ? scores_out + (int64_t)g * k : nullptr;
    q.ctr = ws.ctr + (size_t)g * kCtrs;
    q.hist0 = ws.hist0 + (size_t)g * kBins;
    q.cand = ws.cand + (int64_t)g * ws.ld;
    q.cand2 = ws.cand2 + (int64_t)g * ws.ld;
    q.ld = ws.ld;
    return q;
}

CSA_DEV void emit(const Query& q, uint32_t pos, uint2 kv)
{
    if (pos < (uint32_t)q.k) {
        q.idx_out[pos] = (int32_t)kv.y;
        if (q.sc_out) q.sc_out[pos] = key_to_float(kv.x);
    }
}

// Bin holding the need-th largest element of hist[0..NBINS) (need >= 1, sum >= need):
// s->bin = that bin, s->above = count in the bins strictly above it.  hist in smem.
// Thread t owns PER consecutive bins, the top ones to thread 0, held in registers: one
// warp scan and one exchange of warp totals locate the owning thread, which then walks
// its own registers, so the dependent chain stays short.  A kBins histogram is in the
// hist_slot layout (PLAIN: in plain order), a 256-bin one in plain order.
template <int NBINS, class Bar, bool PLAIN = false>
CSA_DEV void find_threshold_bin(const uint32_t* hist, uint32_t need, Shared* s, int tid)
{
    constexpr int PER = NBINS / kSelThreads;
    static_assert(NBINS == 256 || NBINS == kBins, "256 bins (identity layout) or kBins (hist_slot layout)");
    const int lane = tid & 31, warp = tid >> 5;
    const int lo = NBINS - (tid + 1) * PER;  // this thread covers [lo, lo + PER)
    uint32_t v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = NBINS == kBins && !PLAIN ? hist[hist_slot((uint32_t)(lo + i))] : hist[lo + i];
    uint32_t local = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) local += v[i];
    uint32_t incl = local;  // inclusive scan in thread order (thread 0 = top bins)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    if (lane == 31) s->scr[warp] = incl;
    Bar::sync();
    uint32_t base = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) base += w < warp ? s->scr[w] : 0u;
    uint32_t cum = base + incl - local;  // count in the bins above this thread's range
    if (cum < need && need <= cum + local) {
        uint32_t bin = 0, above = 0;
        bool found = false;
#pragma unroll
        for (int i = PER - 1; i >= 0; --i) {  // from this thread's highest bin down
            const bool here = !found && cum + v[i] >= need;
            bin = here ? (uint32_t)(lo + i) : bin;
            above = here ? cum : above;
            found = found || here;
            cum += v[i];
        }
        s->bin = bin;
        s->above = above;
    }
    Bar::sync();
}

// find_threshold_bin over a kBins histogram in the hist_slot layout that also replaces
// each bin's count by the count of the bins above it (an exclusive suffix sum: the first
// output slot of the bin's entries when entries are placed from the top bin down) and
// sets s->cnt to the threshold bin's own count.
template <class Bar>
CSA_DEV void threshold_and_suffix(uint32_t* hist, uint32_t need, Shared* s, int tid)
{
    constexpr int PER = kBins / kSelThreads;
    const int lane = tid & 31, warp = tid >> 5;
    const int lo = kBins - (tid + 1) * PER;  // this thread covers [lo, lo + PER)
    uint32_t v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = hist[hist_slot((uint32_t)(lo + i))];
    uint32_t local = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) local += v[i];
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    if (lane == 31) s->scr[warp] = incl;
    Bar::sync();
    uint32_t base = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) base += w < warp ? s->scr[w] : 0u;
    uint32_t cum = base + incl - local;  // count in the bins above this thread's range
#pragma unroll
    for (int i = PER - 1; i >= 0; --i) {
        const uint32_t bin = (uint32_t)(lo + i);
        if (cum < need && need <= cum + v[i]) {
            s->bin = bin;
            s->above = cum;
            s->cnt = v[i];
        }
        hist[hist_slot(bin)] = cum;
        cum += v[i];
    }
    Bar::sync();
}

// Warp-aggregated append: this lane's slot in a list whose length counter is *ctr, for
// lanes with pred true.  All lanes of the warp call.
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

// Radix digits of the 64-bit key (kv.x << 32) | ~kv.y: level 0 = bits 63..52, level 1 =
// bits 51..40 (12-bit digits), levels 2..6 = 8-bit digits from bit 39 down to bit 0.
// Digits of the 64-bit key (score key << 32 | ~index), most significant first: level 0
// the top 12 bits (the scan's histogram), levels 1-6 eight bits each (bits 44-51 down
// to 4-11), level 7 the last four.  The narrow digits after level 0 keep the per-level
// histograms at 256 bins, which the threshold search covers with one bin per thread.
CSA_DEV uint32_t digit_shift(int level) { return level == 0 ? 52u : level < 7 ? (uint32_t)(52 - 8 * level) : 0u; }
CSA_DEV uint32_t digit_mask(int level) { return level == 0 ? 0xfffu : level < 7 ? 0xffu : 0xfu; }
CSA_DEV uint32_t digit_at(uint2 kv, uint32_t shift, uint32_t mask)
{
    const uint64_t key = ((uint64_t)kv.x << 32) | (uint32_t)~kv.y;
    return (uint32_t)(key >> shift) & mask;
}
CSA_DEV uint32_t digit_of(uint2 kv, int level) { return digit_at(kv, digit_shift(level), digit_mask(level)); }

// Global -> shared copy of a 4096-bin histogram with every load issued before the
// first store (one round trip instead of one per iteration).
CSA_DEV void load_hist(uint32_t* sh, const uint32_t* gh, int tid)
{
    constexpr int kQuads = kBins / 4 / kSelThreads;
    uint4 v[kQuads];
#pragma unroll
    for (int u = 0; u < kQuads; ++u) v[u] = __ldcg(reinterpret_cast<const uint4*>(gh) + tid + u * kSelThreads);
#pragma unroll
    for (int u = 0; u < kQuads; ++u) reinterpret_cast<uint4*>(sh)[tid + u * kSelThreads] = v[u];
}

// Zero n words of 16-byte-aligned memory (n a multiple of 4 * kSelThreads).
CSA_DEV void zero_words(uint32_t* p, int n, int tid)
{
    for (int i = tid; i < n / 4; i += kSelThreads) reinterpret_cast<uint4*>(p)[i] = make_uint4(0, 0, 0, 0);
}

// Exclusive prefix sum of v over the group in thread order; total = group sum (every
// thread receives it).
template <class Bar>
CSA_DEV uint32_t block_excl_scan(uint32_t v, Shared* s, int tid, uint32_t& total)
{
    const int lane = tid & 31, warp = tid >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    Bar::sync();  // scr may still be read by a previous use
    if (lane == 31) s->scr[warp] = incl;
    Bar::sync();
    uint32_t base = 0, sum = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
        const uint32_t x = s->scr[w];
        base += w < warp ? x : 0u;
        sum += x;
    }
    total = sum;
    return base + incl - v;
}

// Emit every entry of a list into the output slots counted by s->out.
CSA_DEV void emit_all(const Query& q, const uint2* list, bool in_smem, uint32_t count, Shared* s, int tid)
{
    for (uint32_t i = tid; i < ((count + 31) & ~31u); i += kSelThreads) {
        const bool in = i < count;
        const uint2 kv = in ? (in_smem ? list[i] : __ldcg(&list[i])) : make_uint2(0, 0);
        const uint32_t pos = warp_append(&s->out, in);
        if (in) emit(q, pos, kv);
    }
}

// Emit the `need` best entries of a shared-memory list of at most kSelThreads entries:
// an entry is selected when fewer than `need` entries beat it.
CSA_DEV void emit_by_rank(const Query& q, const uint2* list, uint32_t count, uint32_t need, Shared* s, int tid)
{
    const bool in = (uint32_t)tid < count;
    const uint2 me = in ? list[tid] : make_uint2(0, 0);
    uint32_t rank = 0;
    if (in)
        for (uint32_t j = 0; j < count; ++j) {
            const uint2 o = list[j];
            rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
        }
    const bool take = in && rank < need;
    const uint32_t pos = warp_append(&s->out, take);
    if (take) emit(q, pos, me);
}

// One classification round against the digit-0 threshold bin b0.  Each thread brings up
// to kPer (key, entry index) pairs (valid[u] false for none).  Entries above b0 are
// emitted; entries inside b0 are appended to the candidate list.  Slots come from one
// block-wide scan of the packed (emitted, candidate) counts and one global atomic per
// list and round, issued before the entries are staged so that the round trip overlaps.
template <class Bar>
CSA_DEV void classify_round(const Query& q, const uint32_t (&key)[kPer], const uint32_t (&eidx)[kPer],
                            const bool (&valid)[kPer], uint32_t b0, uint2* s_take, uint2* s_cand, Shared* s,
                            int tid)
{
    uint32_t cnt = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const uint32_t d0 = key[u] >> 20;
        if (valid[u]) cnt += d0 > b0 ? 1u : (d0 == b0 ? 0x10000u : 0u);
    }
    uint32_t tot;
    const uint32_t excl = block_excl_scan<Bar>(cnt, s, tid, tot);
    const uint32_t nt = tot & 0xffffu, nc = tot >> 16;
    uint32_t bt = 0, bc = 0;
    if (tid == 0) {
        if (nt) bt = atomicAdd(&q.ctr[0], nt);
        if (nc) bc = atomicAdd(&q.ctr[1], nc);
    }
    uint32_t tp = excl & 0xffffu, cp = excl >> 16;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        if (!valid[u]) continue;
        const uint32_t d0 = key[u] >> 20;
        if (d0 > b0)
            s_take[tp++] = make_uint2(key[u], eidx[u]);
        else if (d0 == b0)
            s_cand[cp++] = make_uint2(key[u], eidx[u]);
    }
    if (tid == 0) {
        s->bt = bt;
        s->bc = bc;
    }
    Bar::sync();
    bt = s->bt;
    bc = s->bc;
    for (uint32_t i = tid; i < nt; i += kSelThreads) emit(q, bt + i, s_take[i]);
    for (uint32_t i = tid; i < nc; i += kSelThreads)
        if (bc + i < (uint32_t)q.ld) q.cand[bc + i] = s_cand[i];
    Bar::sync();
}

// Resolution of a candidate list too long for shared memory (more than kListCap
// entries: heavy ties in the threshold bin).  Digit by digit over global lists, with
// warp-aggregated slots; lists that shrink below kListCap move into shared memory.
// Entry: sh zeroed, s->out = entries emitted so far, all threads synchronised.
template <class Bar>
CSA_DEV void resolve_long_list(const Query& q, uint32_t* sh, uint2* s_listA, uint2* s_listB, Shared* s,
                               int tid, uint32_t count)
{
    for (uint32_t i = tid; i < count; i += kSelThreads)
        atomicAdd(&sh[digit_of(__ldcg(&q.cand[i]), 1)], 1u);
    Bar::sync();
    uint32_t need = (uint32_t)q.k - s->out;
    uint2* list = q.cand;
    bool in_smem = false;
    for (int level = 1; need > 0; ++level) {
        if (need >= count) {  // every remaining candidate is selected
            emit_all(q, list, in_smem, count, s, tid);
            break;
        }
        if (in_smem && count <= kRankMax) {  // exact rank among a small list
            emit_by_rank(q, list, count, need, s, tid);
            break;
        }
        if (level > 7) break;  // unreachable: (score, index) keys are unique
        if (level >= 2) {
            for (int i = tid; i < 256; i += kSelThreads) sh[i] = 0;
            Bar::sync();
            for (uint32_t i = tid; i < count; i += kSelThreads)
                atomicAdd(&sh[digit_of(in_smem ? list[i] : __ldcg(&list[i]), level)], 1u);
            Bar::sync();
        }
        find_threshold_bin<256, Bar>(sh, need, s, tid);
        const uint32_t bt = s->bin, above = s->above, keep_n = sh[bt];
        const bool next_smem = keep_n <= (uint32_t)kListCap;
        uint2* next = next_smem ? (list == s_listA ? s_listB : s_listA) : (list == q.cand ? q.cand2 : q.cand);
        if (tid == 0) s->cnt = 0;
        Bar::sync();
        for (uint32_t i = tid; i < ((count + kSelThreads - 1) / kSelThreads) * kSelThreads; i += kSelThreads) {
            const bool in = i < count;
            const uint2 kv = in ? (in_smem ? list[i] : __ldcg(&list[i])) : make_uint2(0, 0);
            const uint32_t d = digit_of(kv, level);
            const bool take = in && d > bt;
            const bool keep = in && d == bt;
            const uint32_t pos = warp_append(&s->out, take);
            if (take) emit(q, pos, kv);
            const uint32_t npos = warp_append(&s->cnt, keep);
            if (keep && npos < (next_smem ? (uint32_t)kListCap : (uint32_t)q.ld)) next[npos] = kv;
        }
        __threadfence_block();
        Bar::sync();
        need -= above;
        count = s->cnt;
        list = next;
        in_smem = next_smem;
        Bar::sync();
    }
}

// Run by the last group to finish classifying: resolve the candidates of the digit-0
// threshold bin digit by digit on the 64-bit key.  The counters and the first kListCap
// candidate slots are fetched in one round trip (slots past the count are loaded but
// ignored).  A list of up to kListCap entries is resolved with the entries in registers
// (kListCap / kSelThreads per thread): per level one histogram of the next digit, one
// threshold search and one block scan that places the selected entries and compacts
// the tied ones into shared memory; lists of up to kRankMax entries are finished by
// exact ranking.
template <class Bar>
CSA_DEV void resolve_candidates(const Query& q, uint32_t* sh, uint2* s_listA, uint2* s_listB, Shared* s, int tid)
{
    constexpr int kPerT = kListCap / kSelThreads;
    const uint32_t nload = q.ld < kListCap ? (uint32_t)q.ld : (uint32_t)kListCap;
    uint32_t out = __ldcg(&q.ctr[0]);
    uint32_t count = __ldcg(&q.ctr[1]);
    uint2 v[kPerT];
#pragma unroll
    for (int u = 0; u < kPerT; ++u) {
        const uint32_t i = tid + u * kSelThreads;
        v[u] = i < nload ? __ldcg(&q.cand[i]) : make_uint2(0, 0);
    }
    zero_words(sh, kBins, tid);
    if (tid == 0) s->out = out;
    Bar::sync();
    if (count > (uint32_t)kListCap) {
        resolve_long_list<Bar>(q, sh, s_listA, s_listB, s, tid, count);
        return;
    }
    uint32_t need = (uint32_t)q.k - out;
    for (int level = 1; need > 0 && level <= 7; ++level) {
        // v[u] holds entry tid + u * kSelThreads of the current list (valid below count)
        if (need < count && count <= (uint32_t)kRankMax) {  // exact rank among a small list
            if (tid < (int)count) s_listA[tid] = v[0];
            Bar::sync();
            emit_by_rank(q, s_listA, count, need, s, tid);
            break;
        }
        const uint32_t dsh = digit_shift(level), dmask = digit_mask(level);
        uint32_t bt = 0xffffffffu;  // need >= count: every entry is taken
        if (need < count) {
            if (level > 1) {  // (level 1 starts from the zeroed histogram)
                for (int i = tid; i < 256; i += kSelThreads) sh[i] = 0;
                Bar::sync();
            }
#pragma unroll
            for (int u = 0; u < kPerT; ++u) {
                const uint32_t d = digit_at(v[u], dsh, dmask);
                if (tid + u * kSelThreads < (int)count) atomicAdd(&sh[d], 1u);
            }
            Bar::sync();
            find_threshold_bin<256, Bar>(sh, need, s, tid);
            bt = s->bin;
        }
        uint32_t cnt = 0;
#pragma unroll
        for (int u = 0; u < kPerT; ++u) {
            if (tid + u * kSelThreads >= (int)count) continue;
            const uint32_t d = bt == 0xffffffffu ? 0x1000u : digit_at(v[u], dsh, dmask);
            cnt += d > bt || bt == 0xffffffffu ? 1u : (d == bt ? 0x10000u : 0u);
        }
        uint32_t tot;
        const uint32_t excl = block_excl_scan<Bar>(cnt, s, tid, tot);
        uint32_t tp = out + (excl & 0xffffu), kp = excl >> 16;
#pragma unroll
        for (int u = 0; u < kPerT; ++u) {
            if (tid + u * kSelThreads >= (int)count) continue;
            const uint32_t d = bt == 0xffffffffu ? 0x1000u : digit_at(v[u], dsh, dmask);
            if (d > bt || bt == 0xffffffffu)
                emit(q, tp++, v[u]);
            else if (d == bt)
                s_listA[kp++] = v[u];
        }
        out += tot & 0xffffu;
        if (bt == 0xffffffffu) break;
        need -= tot & 0xffffu;
        count = tot >> 16;
        Bar::sync();
#pragma unroll
        for (int u = 0; u < kPerT; ++u) {
            const uint32_t i = tid + u * kSelThreads;
            v[u] = i < count ? s_listA[i] : make_uint2(0, 0);
        }
        if (tid == 0) s->out = out;
        Bar::sync();
    }
}

// Zero this query's histogram and counters for the next call.
CSA_DEV void reset_query(const Query& q, int tid, bool hist = true)
{
    if (hist) zero_words(q.hist0, kBins, tid);
    if (tid < kCtrs) q.ctr[tid] = 0;
}

}  // namespace sel
}  // namespace csa
