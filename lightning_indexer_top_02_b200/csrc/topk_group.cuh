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
__device__ __forceinline__ float key_score(uint64_t k) { return score_of_ord(static_cast<uint32_t>(k >> 32)); }

struct GroupScratch {
    uint32_t hist[256];
    int bcast[4];
    int warp_sums[32];
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
__device__ __forceinline__ int group_excl_scan(int v, GroupScratch *sc, int bar, int tid, int *total)
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
        sc->warp_sums[wid] = x;
    named_bar_sync(bar, NT);
    int base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const int s = sc->warp_sums[w];
        base += w < wid ? s : 0;
        tot += s;
    }
    named_bar_sync(bar, NT);
    *total = tot;
    return base + x - v;
}

// Radix select over the group's keys (EPT per thread, 0 = empty), most
// significant byte first.  Precondition: more than K non-zero keys, all
// distinct.  Returns a bound L such that the number of keys >= L lies in
// [K, K + slack] (exactly K when slack == 0); *kept = that number.  Every key
// below L has at least K keys above it, so dropping it never loses a top-K key.
template <int NT, int EPT>
__device__ uint64_t radix_bound(const uint64_t (&e)[EPT], int K, int slack, GroupScratch *sc,
                                int bar, int tid, int *kept)
{
    const int lane = tid & 31;
    uint64_t prefix = 0, mask = 0;
    int need = K;
    int total_ge = 0;
    for (int pos = 56; pos >= 0; pos -= 8) {
        for (int i = tid; i < 256; i += NT)
            sc->hist[i] = 0;
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
                    atomicAdd(&sc->hist[digit], static_cast<uint32_t>(__popc(peers)));
            }
        }
        named_bar_sync(bar, NT);
        if (tid < 32) {
            uint32_t c[8];
            uint32_t sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = sc->hist[lane * 8 + j];
                sum += c[j];
            }
            uint32_t suf = sum; // keys whose digit lies in this lane's bins or above
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
                        sc->bcast[0] = lane * 8 + j;
                        sc->bcast[1] = static_cast<int>(above);
                        sc->bcast[2] = static_cast<int>(c[j]);
                        break;
                    }
                    above += c[j];
                }
            }
        }
        named_bar_sync(bar, NT);
        const int digit = sc->bcast[0];
        const int above = sc->bcast[1];
        const int inb = sc->bcast[2];
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
            for (int p = tid; p < (P >> 1); p += NT) {
                const int lo = 2 * stride * (p / stride) + (p % stride);
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

// Shrinks the candidate list buf[0..n) (global memory, keys unique) to at
// most K + slack keys that still contain the top K, in place.  Returns the
// new length; *bound_ord receives the high word of the cut, so a later key
// can only matter if its score's order image is >= *bound_ord.
template <int NT, int EPT>
__device__ int compact_candidates(uint64_t *buf, int n, int K, int slack, GroupScratch *sc, int bar,
                                  int tid, uint32_t *bound_ord)
{
    uint64_t e[EPT];
#pragma unroll
    for (int i = 0; i < EPT; ++i) {
        const int j = i * NT + tid;
        e[i] = j < n ? buf[j] : 0ull;
    }
    int kept;
    const uint64_t L = radix_bound<NT, EPT>(e, K, slack, sc, bar, tid, &kept);
    int mine = 0;
#pragma unroll
    for (int i = 0; i < EPT; ++i)
        mine += (e[i] != 0 && e[i] >= L) ? 1 : 0;
    int total;
    int off = group_excl_scan<NT>(mine, sc, bar, tid, &total);
#pragma unroll
    for (int i = 0; i < EPT; ++i)
        if (e[i] != 0 && e[i] >= L)
            buf[off++] = e[i];
    *bound_ord = static_cast<uint32_t>(L >> 32);
    named_bar_sync(bar, NT); // writes visible to the whole group before reuse
    return total;
}

// Exact selection of the min(K, #non-zero) largest keys among e[] into
// out[0..kept) (shared memory, unordered), zero-filled up to `pad_to`.
template <int NT, int EPT>
__device__ int select_topk(const uint64_t (&e)[EPT], int n, int K, uint64_t *out, int pad_to,
                           GroupScratch *sc, int bar, int tid)
{
    uint64_t L = 1;
    int kept = n;
    if (n > K) {
        L = radix_bound<NT, EPT>(e, K, 0, sc, bar, tid, &kept);
    }
    int mine = 0;
#pragma unroll
    for (int i = 0; i < EPT; ++i)
        mine += (e[i] != 0 && e[i] >= L) ? 1 : 0;
    int total;
    int off = group_excl_scan<NT>(mine, sc, bar, tid, &total);
#pragma unroll
    for (int i = 0; i < EPT; ++i)
        if (e[i] != 0 && e[i] >= L)
            out[off++] = e[i];
    for (int i = total + tid; i < pad_to; i += NT)
        out[i] = 0ull;
    named_bar_sync(bar, NT);
    return total;
}

__host__ __device__ constexpr int pow2_at_least(int x)
{
    int p = 2;
    while (p < x)
        p <<= 1;
    return p;
}

} // namespace csa
