// topk_group.cuh -- selection primitives run cooperatively by a group of NT
// threads (whole warps, synchronised with one named barrier).
//
// Candidates are 64-bit keys: high word = order-preserving image of the fp32
// score, low word = bitwise NOT of the key index.  Comparing keys as unsigned
// integers therefore ranks by score (descending when taking the larger key)
// and, for equal scores, by lower index first -- the top-k rule of
// "StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming Top-k",
// abstract (top-k per query), with ties to the lower index.  Every real key is
// non-zero, so 0 marks an empty slot.
//
// Two families of selection live here:
//  * bucket selection (the fast path): scores are mapped monotonically onto
//    NB buckets spanning the candidates' [min, max] score range, one shared
//    histogram pass finds the bucket holding the k-th key, and a counting sort
//    over buckets plus a tiny per-bucket sort orders the result;
//  * radix selection over the 64-bit key (the exact fallback for degenerate
//    ranges, e.g. many equal scores) and a bitonic sort.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace csa {

// Score -> unsigned integer with the same order; -0.0 is folded onto +0.0.
__device__ __forceinline__ uint32_t ord_of_score(float f)
{
    const uint32_t b = __float_as_uint(f + 0.0f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float score_of_ord(uint32_t u)
{
    const uint32_t b = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
    return __uint_as_float(b);
}

__device__ __forceinline__ uint64_t make_key(uint32_t ord, uint32_t s)
{
    return (static_cast<uint64_t>(ord) << 32) | static_cast<uint32_t>(~s);
}

__device__ __forceinline__ int key_index(uint64_t k) { return static_cast<int>(~static_cast<uint32_t>(k)); }
__device__ __forceinline__ uint32_t key_ord(uint64_t k) { return static_cast<uint32_t>(k >> 32); }
__device__ __forceinline__ float key_score(uint64_t k) { return score_of_ord(key_ord(k)); }

// Small per-group scratch for broadcasts and scans.
struct GroupSmall {
    int bcast[8];
    uint32_t warp_sums[32];
};

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// All-thread AND over the group; doubles as the group barrier.
__device__ __forceinline__ bool group_all(int bar, int nthreads, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "r"(bar), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Exclusive prefix sum of v over the group (thread order); *total = group sum.
template <int NT>
__device__ __forceinline__ int group_excl_scan(int v, GroupSmall *gs, int bar, int tid, int *total)
{
    const int lane = tid & 31, wid = tid >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off)
            x += y;
    }
    if (lane == 31)
        gs->warp_sums[wid] = static_cast<uint32_t>(x);
    named_bar_sync(bar, NT);
    int base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const int s = static_cast<int>(gs->warp_sums[w]);
        base += w < wid ? s : 0;
        tot += s;
    }
    named_bar_sync(bar, NT);
    *total = tot;
    return base + x - v;
}

// Group-wide min of an unsigned value; every thread gets the result.
template <int NT>
__device__ __forceinline__ uint32_t group_min_u32(uint32_t v, GroupSmall *gs, int bar, int tid)
{
    const int lane = tid & 31, wid = tid >> 5;
    const uint32_t m = __reduce_min_sync(0xffffffffu, v);
    if (lane == 0)
        gs->warp_sums[wid] = m;
    named_bar_sync(bar, NT);
    uint32_t r = 0xFFFFFFFFu;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w)
        r = min(r, gs->warp_sums[w]);
    named_bar_sync(bar, NT);
    return r;
}

// Smallest and largest score order image among the group's non-zero keys.
template <int NT, int EPT>
__device__ __forceinline__ void group_ord_range(const uint64_t (&e)[EPT], GroupSmall *gs, int bar,
                                                int tid, uint32_t *mn, uint32_t *mx)
{
    const int lane = tid & 31, wid = tid >> 5;
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
        if (e[i] != 0) {
            lo = min(lo, key_ord(e[i]));
            hi = max(hi, key_ord(e[i]));
        }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
        gs->warp_sums[wid] = lo;
        gs->warp_sums[16 + wid] = hi;
    }
    named_bar_sync(bar, NT);
    uint32_t a = 0xFFFFFFFFu, b = 0u;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        a = min(a, gs->warp_sums[w]);
        b = max(b, gs->warp_sums[16 + w]);
    }
    named_bar_sync(bar, NT);
    *mn = a;
    *mx = b;
}

// Warp-aggregated counter increment: lanes with the same idx share one
// atomic.  Returns, for active lanes, the counter's old value plus the lane's
// rank among its peers (a unique slot).  All 32 lanes must call it.
__device__ __forceinline__ uint32_t agg_atomic_add(uint32_t *counters, int idx, bool active)
{
    const unsigned act = __ballot_sync(0xffffffffu, active);
    uint32_t res = 0;
    if (active) {
        const int lane = threadIdx.x & 31;
        const unsigned peers = __match_any_sync(act, idx);
        const int leader = __ffs(peers) - 1;
        uint32_t base = 0;
        if (lane == leader)
            base = atomicAdd(&counters[idx], static_cast<uint32_t>(__popc(peers)));
        base = __shfl_sync(peers, base, leader);
        res = base + static_cast<uint32_t>(__popc(peers & lanemask_lt()));
    }
    return res;
}

// ---------------------------------------------------------------------------- radix (exact)

// Radix select over the group's keys (EPT per thread, 0 = empty), most
// significant byte first.  Precondition: more than K non-zero keys, all
// distinct.  Returns a bound L such that the number of keys >= L lies in
// [K, K + slack] (exactly K when slack == 0); *kept = that number.  Every key
// below L has at least K keys above it, so dropping it never loses a top-K key.
template <int NT, int EPT>
__device__ uint64_t radix_bound(const uint64_t (&e)[EPT], int K, int slack, uint32_t *hist,
                                GroupSmall *gs, int bar, int tid, int *kept)
{
    const int lane = tid & 31;
    uint64_t prefix = 0, mask = 0;
    int need = K;
    int total_ge = 0;
    for (int pos = 56; pos >= 0; pos -= 8) {
        for (int i = tid; i < 256; i += NT)
            hist[i] = 0;
        named_bar_sync(bar, NT);
#pragma unroll
        for (int i = 0; i < EPT; ++i) {
            const uint64_t x = e[i];
            const bool match = x != 0 && (x & mask) == prefix;
            const uint32_t digit = static_cast<uint32_t>(x >> pos) & 255u;
            const unsigned act = __ballot_sync(0xffffffffu, match);
            if (match) {
                const unsigned peers = __match_any_sync(act, digit);
                if (lane == __ffs(peers) - 1)
                    atomicAdd(&hist[digit], static_cast<uint32_t>(__popc(peers)));
            }
        }
        named_bar_sync(bar, NT);
        if (tid < 32) {
            uint32_t c[8];
            uint32_t sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = hist[lane * 8 + j];
                sum += c[j];
            }
            uint32_t suf = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t t = __shfl_down_sync(0xffffffffu, suf, off);
                if (lane + off < 32)
                    suf += t;
            }
            const uint32_t above_lane = suf - sum;
            const uint32_t nd = static_cast<uint32_t>(need);
            if (above_lane < nd && nd <= suf) {
                uint32_t above = above_lane;
#pragma unroll
                for (int j = 7; j >= 0; --j) {
                    if (above + c[j] >= nd) {
                        gs->bcast[0] = lane * 8 + j;
                        gs->bcast[1] = static_cast<int>(above);
                        gs->bcast[2] = static_cast<int>(c[j]);
                        break;
                    }
                    above += c[j];
                }
            }
        }
        named_bar_sync(bar, NT);
        const int digit = gs->bcast[0];
        const int above = gs->bcast[1];
        const int inb = gs->bcast[2];
        named_bar_sync(bar, NT);
        need -= above;
        prefix |= static_cast<uint64_t>(digit) << pos;
        mask |= 0xFFull << pos;
        total_ge = K - need + inb;
        if (total_ge <= K + slack)
            break;
    }
    *kept = total_ge;
    return prefix;
}

// Bitonic sort of a[0..P) in shared memory, descending (P a power of two).
template <int NT>
__device__ void bitonic_sort_desc(uint64_t *a, int P, int bar, int tid)
{
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const int sh = __ffs(stride) - 1;
            for (int p = tid; p < (P >> 1); p += NT) {
                const int lo = ((p >> sh) << (sh + 1)) + (p & (stride - 1));
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const uint64_t x = a[lo], y = a[hi];
                if (desc ? (x < y) : (x > y)) {
                    a[lo] = y;
                    a[hi] = x;
                }
            }
            named_bar_sync(bar, NT);
        }
    }
}

// Keeps the keys >= L of e[] (all non-zero keys when L == 1) at out[0..total)
// in arbitrary order; returns total.  Also returns the smallest kept score
// order image in *min_ord (0xFFFFFFFF when nothing is kept).
template <int NT, int EPT>
__device__ int write_kept(const uint64_t (&e)[EPT], uint64_t L, uint64_t *out, GroupSmall *gs,
                          int bar, int tid, uint32_t *min_ord)
{
    int mine = 0;
    uint32_t mn = 0xFFFFFFFFu;
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
        const bool keep = e[i] != 0 && e[i] >= L;
        mine += keep ? 1 : 0;
        mn = keep ? min(mn, key_ord(e[i])) : mn;
    }
    int total;
    int off = group_excl_scan<NT>(mine, gs, bar, tid, &total);
#pragma unroll
    for (int i = 0; i < EPT; ++i)
        if (e[i] != 0 && e[i] >= L)
            out[off++] = e[i];
    *min_ord = group_min_u32<NT>(mn, gs, bar, tid);
    return total;
}

// ---------------------------------------------------------------------------- buckets

// Monotone map of scores in [lo, hi] onto buckets [0, NB): b(x) never
// decreases when x increases (fp32 subtraction, multiplication by a positive
// constant and truncation are all monotone), so bucket order is score order.
struct BucketMap {
    float lo, inv;
    bool ok;
};

__device__ __forceinline__ BucketMap bucket_map(uint32_t min_ord, uint32_t max_ord, int NB)
{
    BucketMap m;
    const float lo = score_of_ord(min_ord);
    const float hi = score_of_ord(max_ord);
    const float span = hi - lo;
    m.lo = lo;
    m.inv = static_cast<float>(NB) / span;
    m.ok = max_ord > min_ord && span > 0.0f && isfinite(span) && isfinite(m.inv) && isfinite(lo);
    return m;
}

__device__ __forceinline__ int bucket_of(float s, const BucketMap &m, int NB)
{
    const float x = (s - m.lo) * m.inv;
    int b = static_cast<int>(x);
    b = b < 0 ? 0 : b;
    return b > NB - 1 ? NB - 1 : b;
}

// After a histogram hist[0..NB) of the group's keys, find the bucket b* that
// holds the need-th largest key: above(b*) < need <= above(b*) + hist[b*],
// where above(b) counts keys in buckets > b.  gs->bcast = {b*, above(b*),
// hist[b*], largest bucket count among buckets >= b*}.  With write_above,
// hist[b] is replaced by above(b) (the first output slot of bucket b when
// buckets are laid out from the highest down).  Precondition: at least
// `need` keys in the histogram.
template <int NT, int NB>
__device__ void bucket_boundary(uint32_t *hist, int need, bool write_above, GroupSmall *gs, int bar,
                                int tid)
{
    constexpr int PER = NB / NT;
    const int lane = tid & 31, wid = tid >> 5;
    uint32_t c[PER];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        c[j] = hist[tid * PER + j];
        sum += c[j];
    }
    uint32_t suf = sum; // inclusive suffix over threads within the warp
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t t = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32)
            suf += t;
    }
    if (lane == 0)
        gs->warp_sums[wid] = suf; // the warp's total
    named_bar_sync(bar, NT);
    uint32_t higher = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w)
        higher += w > wid ? gs->warp_sums[w] : 0u;
    suf += higher;
    const uint32_t above_thread = suf - sum;
    const uint32_t nd = static_cast<uint32_t>(need);
    if (write_above) {
        uint32_t run = above_thread;
#pragma unroll
        for (int j = PER - 1; j >= 0; --j) {
            hist[tid * PER + j] = run;
            run += c[j];
        }
    }
    if (above_thread < nd && nd <= suf) {
        uint32_t above = above_thread;
#pragma unroll
        for (int j = PER - 1; j >= 0; --j) {
            if (above + c[j] >= nd) {
                gs->bcast[0] = tid * PER + j;
                gs->bcast[1] = static_cast<int>(above);
                gs->bcast[2] = static_cast<int>(c[j]);
                break;
            }
            above += c[j];
        }
    }
    named_bar_sync(bar, NT);
    // largest bucket at or above b*
    const int bstar = gs->bcast[0];
    uint32_t mx = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j)
        mx = (tid * PER + j >= bstar) ? max(mx, c[j]) : mx;
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0)
        gs->warp_sums[wid] = mx;
    named_bar_sync(bar, NT);
    if (tid == 0) {
        uint32_t m = 0;
        for (int w = 0; w < NT / 32; ++w)
            m = max(m, gs->warp_sums[w]);
        gs->bcast[3] = static_cast<int>(m);
    }
    named_bar_sync(bar, NT);
}

// Square-root bucket map: b(x) = floor(NB * sqrt((x - lo) / (hi - lo))).
// Still monotone (each step is), but it spreads the dense low end of a
// candidate list -- scores just above the admission bound -- over many more
// buckets than a linear map, so fewer keys share a bucket (and an atomic).
__device__ __forceinline__ int bucket_of_sqrt(float s, const BucketMap &m, int NB)
{
    const float u = (s - m.lo) * m.inv; // m.inv = 1 / span for this map
    const float r = sqrtf(u > 0.0f ? u : 0.0f) * static_cast<float>(NB);
    int b = static_cast<int>(r);
    return b > NB - 1 ? NB - 1 : b;
}

__device__ __forceinline__ BucketMap bucket_map_unit(uint32_t min_ord, uint32_t max_ord)
{
    BucketMap m;
    const float lo = score_of_ord(min_ord);
    const float hi = score_of_ord(max_ord);
    const float span = hi - lo;
    m.lo = lo;
    m.inv = 1.0f / span;
    m.ok = max_ord > min_ord && span > 0.0f && isfinite(span) && isfinite(m.inv) && isfinite(lo);
    return m;
}

// ---------------------------------------------------------------------------- bitonic in registers
// 64-bit compare-exchange keeping the larger key in a when `big_first`.
__device__ __forceinline__ void cex(uint64_t &a, uint64_t &b, bool big_first)
{
    const bool sw = big_first ? (a < b) : (a > b);
    const uint64_t x = sw ? b : a;
    const uint64_t y = sw ? a : b;
    a = x;
    b = y;
}

// Sorts P = 128 * EPT keys held by a 128-thread group (element j = tid * EPT
// + r lives in a[r] of thread tid) into descending order.  Pairs closer than
// EPT are exchanged inside a thread, pairs within a warp through shuffles,
// and the few cross-warp steps through `buf` (P keys of shared memory).
template <int EPT>
__device__ void bitonic_sort_regs(uint64_t (&a)[EPT], uint64_t *buf, int bar, int tid)
{
    constexpr int P = 128 * EPT;
    const int lane = tid & 31;
    const int base = tid * EPT;
    for (int k = 2; k <= P; k <<= 1) {
        for (int s = k >> 1; s >= EPT; s >>= 1) {
            // partner lives in another thread: lane ^ (s / EPT), or another warp
            const bool lower = (base & s) == 0;
            const bool desc = (base & k) == 0;
            const bool keep_big = lower == desc;
            if (s < 32 * EPT) {
                const int m = s / EPT;
#pragma unroll
                for (int r = 0; r < EPT; ++r) {
                    const uint64_t o = __shfl_xor_sync(0xffffffffu, a[r], m);
                    a[r] = keep_big ? (a[r] > o ? a[r] : o) : (a[r] < o ? a[r] : o);
                }
            } else {
#pragma unroll
                for (int r = 0; r < EPT; ++r)
                    buf[base + r] = a[r];
                named_bar_sync(bar, 128);
#pragma unroll
                for (int r = 0; r < EPT; ++r) {
                    const uint64_t o = buf[(base + r) ^ s];
                    a[r] = keep_big ? (a[r] > o ? a[r] : o) : (a[r] < o ? a[r] : o);
                }
                named_bar_sync(bar, 128);
            }
            (void)lane;
        }
        // partner in the same thread
#pragma unroll
        for (int sc = EPT / 2; sc >= 1; sc >>= 1) {
            if (sc < k) {
#pragma unroll
                for (int r = 0; r < EPT; ++r) {
                    if ((r & sc) == 0) {
                        const bool desc = ((base + r) & k) == 0;
                        cex(a[r], a[r | sc], desc);
                    }
                }
            }
        }
    }
}

__host__ __device__ constexpr int pow2_at_least(int x)
{
    int p = 2;
    while (p < x)
        p <<= 1;
    return p;
}

} // namespace csa
