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
// Here: the key encoding, group-wide scans and votes, the monotone bucket map
// of the select kernel's counting sort (scores mapped onto NB buckets that
// span the candidates' [min, max] score range), and the bitonic sort it falls
// back to for degenerate ranges (e.g. many equal scores).
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace csa {

// Score -> unsigned integer with the same order; -0.0 is folded onto +0.0.
// Negative scores are complemented, the rest get the sign bit set: the XOR
// mask is the sign spread by an arithmetic shift, with bit 31 forced on.
__device__ __forceinline__ uint32_t ord_of_score(float f)
{
    const uint32_t b = __float_as_uint(f + 0.0f);
    return b ^ (static_cast<uint32_t>(static_cast<int32_t>(b) >> 31) | 0x80000000u);
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

// Monotone map of score images in [lo, hi] onto NB buckets (NB a power of
// two), ascending with the score: integer ranges of the image when both ends
// share a sign (the image is then roughly logarithmic in the score, which
// spreads the dense scores just above a cut), linear in the score otherwise.
// ok is false when every score is equal or the range is not finite.
struct RangeMap {
    uint32_t mn;
    int shift;
    bool by_ord;
    bool ok;
    BucketMap bm;
};

__device__ __forceinline__ RangeMap range_map(uint32_t lo, uint32_t hi, int NB)
{
    RangeMap m;
    m.mn = lo;
    m.by_ord = (lo >> 31) == (hi >> 31);
    const uint32_t span = hi - lo;
    const int nb_bits = 31 - __clz(NB);
    m.shift = span < static_cast<uint32_t>(NB) ? 0 : 32 - __clz(span) - nb_bits;
    m.bm = bucket_map(lo, hi, NB);
    m.ok = hi > lo && (m.by_ord || m.bm.ok);
    return m;
}

__device__ __forceinline__ int range_bucket(uint32_t o, const RangeMap &m, int NB)
{
    if (m.by_ord) {
        const uint32_t b = (o > m.mn ? o - m.mn : 0u) >> m.shift;
        return b > static_cast<uint32_t>(NB - 1) ? NB - 1 : static_cast<int>(b);
    }
    return bucket_of(score_of_ord(o), m.bm, NB);
}

// The smallest score image in [lo, hi] whose bucket is at least b (b at most
// the bucket of hi): every image at or above it maps to b or higher, every
// image below it to a lower bucket.  Integer ranges: the bucket's first
// image.  Linear ranges: the image of the bucket's lower edge, moved to the
// exact boundary by a few one-ulp steps (bisection if rounding put it far).
__device__ __forceinline__ uint32_t range_bucket_floor(uint32_t lo, uint32_t hi, int b,
                                                       const RangeMap &m, int NB)
{
    if (m.by_ord) {
        const unsigned long long f = static_cast<unsigned long long>(m.mn) +
                                     (static_cast<unsigned long long>(b) << m.shift);
        return f < lo ? lo : (f > hi ? hi : static_cast<uint32_t>(f));
    }
    uint32_t o = ord_of_score(m.bm.lo + static_cast<float>(b) / m.bm.inv);
    o = o < lo ? lo : (o > hi ? hi : o);
    for (int step = 0; step < 16; ++step) {
        if (o > lo && range_bucket(o - 1, m, NB) >= b)
            --o;
        else if (o < hi && range_bucket(o, m, NB) < b)
            ++o;
        else
            return o;
    }
    while (lo < hi) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (range_bucket(mid, m, NB) >= b)
            hi = mid;
        else
            lo = mid + 1;
    }
    return lo;
}

__host__ __device__ constexpr int pow2_at_least(int x)
{
    int p = 2;
    while (p < x)
        p <<= 1;
    return p;
}

} // namespace csa
