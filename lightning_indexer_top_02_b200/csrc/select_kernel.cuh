// select_kernel.cuh -- the exact top k of each query, sorted, from the
// candidate lists the fused kernel leaves behind (one list per key-range
// split).
//
// "StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", abstract: a partition-merge top-k that never materialises the full
// score tensor.  Here the partitions are the key ranges of one query; every
// list already holds a superset of its range's top k, so the union of a
// query's lists holds its global top k.  Ranking: larger score first, equal
// scores by lower key index (one comparison of the 64-bit keys).
//
// One CTA of 256 threads per query row at a time, several CTAs per SM:
//   1. The row's keys go to registers (16 per thread).  Lists longer than
//      that in total (key-range splits) first go through one histogram pass
//      over the lists in global memory, and the keys at or above the bucket of
//      the k-th largest are gathered; if that bucket is too full, a radix
//      select over the 64-bit keys (one byte per pass) finds the k-th largest
//      key L exactly and the k keys >= L are gathered.
//   2. A histogram over NB buckets spanning the keys' own [min, max] (integer
//      ranges of the score image when all scores share a sign, else linear in
//      the score) finds the bucket holding the k-th largest key; the keys of
//      that bucket and above are scattered into bucket order (a counting
//      sort); each key is then ranked among the keys of its own bucket and
//      written straight to its output slot (the buckets average a few keys).
//      A bucket too full for that -- many equal or near-equal scores -- sends
//      the row to a bitonic sort instead.
//   3. The slots past min(k, n) are padded with (-1, -inf).
// While a row is processed, the next row's list is prefetched into L2.
#pragma once
#include <cstdint>

#include "ptx.cuh"
#include "topk_group.cuh"

namespace csa {

constexpr int kSelThreads = 256;
constexpr int kSelEpt = 16;                       // keys per thread in registers
constexpr int kSelKeys = kSelThreads * kSelEpt;   // 4096
constexpr int kSelNb = 2048;                      // histogram buckets
constexpr int kSelSmallBucket = 64;               // largest bucket ordered by ranking
constexpr int kSelMaxSplits = 64;

struct SelParams {
    const uint64_t *lists;  // [rows][nsplit][cap]
    const int *counts;      // [rows][nsplit]
    int rows;               // list rows in this launch
    int nsplit, cap, topk;
    // list row r -> output row: b = r / (nqb * qps), q = qb_lo * qps + r % (nqb * qps)
    int B, S, qps, nqb, qb_lo;
    int32_t *out_idx;
    float *out_score;
};

struct SelSmem {
    GroupSmall gs;
    int split_off[kSelMaxSplits + 1];
    int misc[4];
    uint32_t hist[kSelNb];
    uint64_t out[kSelKeys];
    uint16_t out_b[kSelKeys]; // bucket of out[i] (fast path)
};

__device__ __forceinline__ void sel_prefetch_l2(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)),
                 "r"(bytes)
                 : "memory");
}

// Calls f(key) for every key of a row's lists in global memory, with
// kSelBatch loads per thread in flight before any of them is used: these
// passes are bound by L2 latency, one round trip per batch instead of per key.
constexpr int kSelBatch = 8;
template <typename F>
__device__ __forceinline__ void sel_for_each_key(const SelParams &sp, const uint64_t *row_lists,
                                                 const SelSmem *sm, int tid, F &&f)
{
    for (int s = 0; s < sp.nsplit; ++s) {
        const uint64_t *src = row_lists + static_cast<size_t>(s) * sp.cap;
        const int n = sm->split_off[s + 1] - sm->split_off[s];
        for (int j0 = 0; j0 < n; j0 += kSelBatch * kSelThreads) {
            uint64_t x[kSelBatch];
#pragma unroll
            for (int u = 0; u < kSelBatch; ++u) {
                const int j = j0 + u * kSelThreads + tid;
                x[u] = j < n ? __ldg(src + j) : 0ull;
            }
#pragma unroll
            for (int u = 0; u < kSelBatch; ++u)
                if (j0 + u * kSelThreads + tid < n)
                    f(x[u]);
        }
    }
}

// For rows whose lists hold more keys than fit in registers: one histogram
// pass over the lists in global memory (buckets = top 11 bits of the score
// image) finds the bucket of the k-th largest key; returns the key L such that
// every key >= L is at or above that bucket, with *count keys >= L.  With
// b1 >= 0 the pass histograms only the keys of top-level bucket b1, by the
// next 11 bits, for the `need`-th largest of them; *count then counts keys of
// bucket b1 at or above the cut and *above those in higher sub-buckets.
__device__ uint64_t sel_prefilter_global(const SelParams &sp, const uint64_t *row_lists,
                                         SelSmem *sm, int tid, int *count, int *above_out,
                                         int b1 = -1, int need = -1)
{
    const int lane = tid & 31, wid = tid >> 5;
    for (int i = tid; i < kSelNb; i += kSelThreads)
        sm->hist[i] = 0;
    __syncthreads();
    sel_for_each_key(sp, row_lists, sm, tid, [&](uint64_t x) {
        const uint32_t o = key_ord(x);
        if (b1 < 0)
            atomicAdd(&sm->hist[o >> 21], 1u);
        else if ((o >> 21) == static_cast<uint32_t>(b1))
            atomicAdd(&sm->hist[(o >> 10) & (kSelNb - 1)], 1u);
    });
    __syncthreads();
    // bucket of the k-th largest, top bucket first
    constexpr int PER = kSelNb / kSelThreads;
    uint32_t c[PER];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        c[j] = sm->hist[tid * PER + j];
        sum += c[j];
    }
    uint32_t suf = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t t = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32)
            suf += t;
    }
    if (lane == 0)
        sm->gs.warp_sums[wid] = suf;
    __syncthreads();
    uint32_t higher = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w)
        higher += w > wid ? sm->gs.warp_sums[w] : 0u;
    const uint32_t above_thread = suf - sum + higher;
    const uint32_t nd = static_cast<uint32_t>(b1 < 0 ? sp.topk : need);
    if (above_thread < nd && nd <= above_thread + sum) {
        uint32_t above = above_thread;
#pragma unroll
        for (int j = PER - 1; j >= 0; --j) {
            if (above + c[j] >= nd) {
                sm->misc[0] = tid * PER + j;
                sm->misc[1] = static_cast<int>(above + c[j]);
                sm->misc[3] = static_cast<int>(above);
                break;
            }
            above += c[j];
        }
    }
    __syncthreads();
    *count = sm->misc[1];
    *above_out = sm->misc[3];
    const uint32_t cut = b1 < 0 ? static_cast<uint32_t>(sm->misc[0]) << 21
                                : (static_cast<uint32_t>(b1) << 21) |
                                      (static_cast<uint32_t>(sm->misc[0]) << 10);
    const uint64_t L = static_cast<uint64_t>(cut) << 32;
    __syncthreads();
    return L;
}

// Radix select over the row's lists in global memory: the largest L such that
// exactly `need` keys are >= L (keys are distinct and non-zero; n > need).
__device__ uint64_t sel_radix_global(const SelParams &sp, const uint64_t *row_lists, SelSmem *sm,
                                     int need, int tid)
{
    const int lane = tid & 31;
    uint64_t prefix = 0, mask = 0;
    for (int pos = 56; pos >= 0; pos -= 8) {
        for (int i = tid; i < 256; i += kSelThreads)
            sm->hist[i] = 0;
        __syncthreads();
        sel_for_each_key(sp, row_lists, sm, tid, [&](uint64_t x) {
            if ((x & mask) == prefix)
                atomicAdd(&sm->hist[static_cast<uint32_t>(x >> pos) & 255u], 1u);
        });
        __syncthreads();
        if (tid < 32) {
            uint32_t c[8];
            uint32_t sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = sm->hist[lane * 8 + j];
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
                        sm->gs.bcast[0] = lane * 8 + j;
                        sm->gs.bcast[1] = static_cast<int>(above);
                        sm->gs.bcast[2] = static_cast<int>(c[j]);
                        break;
                    }
                    above += c[j];
                }
            }
        }
        __syncthreads();
        const int digit = sm->gs.bcast[0];
        const int above = sm->gs.bcast[1];
        const int inb = sm->gs.bcast[2];
        __syncthreads();
        need -= above;
        prefix |= static_cast<uint64_t>(digit) << pos;
        mask |= 0xFFull << pos;
        if (inb == need)
            break; // every key with this prefix is in
    }
    return prefix;
}

// Bucket of a score image over the row's own [min, max], numbered from the
// top score down (range_map: integer ranges of the image when every key has
// the same sign, linear in the score otherwise).
__device__ __forceinline__ int sel_bucket(uint32_t o, const RangeMap &m)
{
    return kSelNb - 1 - range_bucket(o, m, kSelNb);
}

__device__ __forceinline__ void sel_store(int32_t *oi, float *os, int slot, uint64_t key)
{
    oi[slot] = key_index(key);
    os[slot] = key_score(key);
}

// Writes the top `kept` (kept <= n) of the n keys of e[] (0 = empty slot,
// n <= kSelKeys) in descending order to oi/os[0..kept).
__device__ void sel_sort_regs(SelSmem *sm, const uint64_t (&e)[kSelEpt], int n, int kept, int tid,
                              int32_t *oi, float *os)
{
    const int lane = tid & 31, wid = tid >> 5;
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
    for (int i = 0; i < kSelEpt; ++i) {
        if (e[i] != 0) {
            lo = min(lo, key_ord(e[i]));
            hi = max(hi, key_ord(e[i]));
        }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
        sm->gs.warp_sums[wid] = lo;
        sm->gs.warp_sums[16 + wid] = hi;
    }
    for (int i = tid; i < kSelNb; i += kSelThreads)
        sm->hist[i] = 0;
    __syncthreads();
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
        mn = min(mn, sm->gs.warp_sums[w]);
        mx = max(mx, sm->gs.warp_sums[16 + w]);
    }
    const RangeMap map = range_map(mn, mx, kSelNb);
    int total = n;
    bool fallback = !map.ok;
    if (!fallback) {
        // histogram, buckets numbered from the top score down
        int db[kSelEpt];
#pragma unroll
        for (int i = 0; i < kSelEpt; ++i) {
            db[i] = e[i] != 0 ? sel_bucket(key_ord(e[i]), map) : kSelNb;
            if (db[i] < kSelNb)
                atomicAdd(&sm->hist[db[i]], 1u);
        }
        __syncthreads();
        // exclusive prefix over buckets: hist[b] becomes the first slot of
        // bucket b; find the bucket db* that holds slot kept-1
        constexpr int PER = kSelNb / kSelThreads;
        uint32_t c[PER];
        uint32_t sum = 0;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            c[j] = sm->hist[tid * PER + j];
            sum += c[j];
        }
        uint32_t inc = sum; // inclusive prefix over the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off)
                inc += t;
        }
        if (lane == 31)
            sm->gs.warp_sums[wid] = inc; // the min/max reads finished before the last barrier
        __syncthreads();
        uint32_t run = inc - sum;
#pragma unroll
        for (int w = 0; w < kSelThreads / 32; ++w)
            run += w < wid ? sm->gs.warp_sums[w] : 0u;
        int biggest = 0;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const uint32_t start = run;
            sm->hist[tid * PER + j] = start;
            run += c[j];
            if (start < static_cast<uint32_t>(kept) && run >= static_cast<uint32_t>(kept)) {
                sm->misc[0] = tid * PER + j;          // db*
                sm->misc[1] = static_cast<int>(run);  // keys in buckets <= db*
            }
            if (start < static_cast<uint32_t>(kept))
                biggest = max(biggest, static_cast<int>(c[j]));
        }
        biggest = __reduce_max_sync(0xffffffffu, biggest);
        __syncthreads(); // warp_sums reads done
        if (lane == 0)
            sm->gs.warp_sums[wid] = static_cast<uint32_t>(biggest);
        __syncthreads();
        const int dstar = sm->misc[0];
        total = sm->misc[1];
        int big = 0;
#pragma unroll
        for (int w = 0; w < kSelThreads / 32; ++w)
            big = max(big, static_cast<int>(sm->gs.warp_sums[w]));
        // scatter the keys of buckets <= db* into bucket order
#pragma unroll
        for (int i = 0; i < kSelEpt; ++i) {
            if (db[i] <= dstar) {
                const uint32_t slot = atomicAdd(&sm->hist[db[i]], 1u);
                if (CSA_CHECK_INDEX(kChkSelOut, slot, kSelKeys)) {
                    sm->out[slot] = e[i];
                    sm->out_b[slot] = static_cast<uint16_t>(db[i]);
                }
            }
        }
        __syncthreads();
        if (big <= kSelSmallBucket) {
            // Rank each placed key inside its bucket (keys are distinct) and
            // write it to bucket start + rank when that slot is among the
            // first `kept`.  Keys go to threads in slot order, so the lanes of
            // a warp see buckets of similar size.
            for (int a = tid; a < total; a += kSelThreads) {
                const uint64_t x = sm->out[a];
                const int b = sm->out_b[a];
                const int lo_s = b == 0 ? 0 : static_cast<int>(sm->hist[b - 1]);
                const int hi_s = static_cast<int>(sm->hist[b]);
                int to = lo_s;
                for (int j = lo_s; j < hi_s; ++j)
                    to += sm->out[j] > x ? 1 : 0;
                if (to < kept)
                    sel_store(oi, os, to, x);
            }
            return;
        }
    } else {
        // degenerate range (one score for every key): all keys to out[]
        int mine = 0;
#pragma unroll
        for (int i = 0; i < kSelEpt; ++i)
            mine += e[i] != 0;
        int tot;
        int off = group_excl_scan<kSelThreads>(mine, &sm->gs, 0, tid, &tot);
#pragma unroll
        for (int i = 0; i < kSelEpt; ++i)
            if (e[i] != 0)
                sm->out[off++] = e[i];
        total = tot;
    }
    // bitonic sort of out[0..total) padded with empty keys to a power of two
    const int P = pow2_at_least(total);
    for (int i = total + tid; i < P; i += kSelThreads)
        sm->out[i] = 0ull;
    __syncthreads();
    bitonic_sort_desc<kSelThreads>(sm->out, P, 0, tid);
    for (int i = tid; i < kept; i += kSelThreads)
        if (CSA_CHECK_INDEX(kChkSelOut, i, P))
            sel_store(oi, os, i, sm->out[i]);
}

constexpr int kSelCtasPerSm = 3;

__global__ void __launch_bounds__(kSelThreads, kSelCtasPerSm)
    select_topk_kernel(const SelParams sp)
{
    extern __shared__ uint8_t sel_smem_raw[];
    SelSmem *sm = reinterpret_cast<SelSmem *>(
        (reinterpret_cast<uintptr_t>(sel_smem_raw) + 15) & ~static_cast<uintptr_t>(15));
    const int tid = threadIdx.x;
    const int per_b = sp.nqb * sp.qps;
    for (int r = blockIdx.x; r < sp.rows; r += gridDim.x) {
        const int b = r / per_b;
        const int q = sp.qb_lo * sp.qps + r % per_b;
        if (q >= sp.S)
            continue;
        const size_t orow = static_cast<size_t>(b) * sp.S + q;
        const uint64_t *row_lists = sp.lists + static_cast<size_t>(r) * sp.nsplit * sp.cap;
        if (tid < 32) {
            // list lengths -> offsets (nsplit <= 64: two per lane)
            const int lane = tid;
            const int c0 = lane < sp.nsplit ? sp.counts[static_cast<size_t>(r) * sp.nsplit + lane] : 0;
            const int c1 = lane + 32 < sp.nsplit
                               ? sp.counts[static_cast<size_t>(r) * sp.nsplit + lane + 32]
                               : 0;
            int x0 = c0, x1 = c1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int t0 = __shfl_up_sync(0xffffffffu, x0, off);
                const int t1 = __shfl_up_sync(0xffffffffu, x1, off);
                if (lane >= off) {
                    x0 += t0;
                    x1 += t1;
                }
            }
            const int tot0 = __shfl_sync(0xffffffffu, x0, 31);
            if (lane == 0)
                sm->split_off[0] = 0;
            if (lane < sp.nsplit)
                sm->split_off[lane + 1] = x0;
            if (lane + 32 < sp.nsplit)
                sm->split_off[lane + 33] = tot0 + x1;
        } else if (tid == 32) {
            // Warm L2 with the next row's first list.  Rows past the last
            // query of a partial query block have no list (their count slots
            // were never written), and a count is never trusted beyond cap.
            const int rn = r + gridDim.x;
            if (rn < sp.rows && sp.qb_lo * sp.qps + rn % per_b < sp.S) {
                int cn = sp.counts[static_cast<size_t>(rn) * sp.nsplit];
                cn = cn < 0 ? 0 : (cn > sp.cap ? sp.cap : cn);
                const uint32_t bytes = static_cast<uint32_t>((cn * 8 + 15) & ~15);
                if (bytes > 0)
                    sel_prefetch_l2(sp.lists + static_cast<size_t>(rn) * sp.nsplit * sp.cap, bytes);
            }
        }
        __syncthreads();
        const int n_all = sm->split_off[sp.nsplit];
        int n = n_all;
        uint64_t e[kSelEpt];
        if (n_all > kSelKeys) {
            // keys at or above the histogram bucket of the k-th largest; an
            // exact radix cut when that bucket is too full
            int kept_pre, above_pre;
            uint64_t L = sel_prefilter_global(sp, row_lists, sm, tid, &kept_pre, &above_pre);
            if (kept_pre > kSelKeys) {
                // the boundary bucket is too full: split it by the next 11 bits
                const int b1 = static_cast<int>(static_cast<uint32_t>(L >> 32) >> 21);
                int kept2, above2;
                const uint64_t L2 = sel_prefilter_global(sp, row_lists, sm, tid, &kept2, &above2,
                                                         b1, sp.topk - above_pre);
                if (above_pre + kept2 <= kSelKeys) {
                    L = L2;
                    n = above_pre + kept2;
                } else {
                    L = sel_radix_global(sp, row_lists, sm, sp.topk, tid);  // near-ties
                }
            } else {
                n = kept_pre;
            }
            if (tid == 0)
                sm->misc[2] = 0;
            __syncthreads();
            sel_for_each_key(sp, row_lists, sm, tid, [&](uint64_t x) {
                if (x >= L) {
                    const int slot = atomicAdd(&sm->misc[2], 1);
                    if (CSA_CHECK_INDEX(kChkSelOut, slot, kSelKeys))
                        sm->out[slot] = x;
                }
            });
            __syncthreads();
            if (n == n_all)
                n = sp.topk; // the radix cut keeps exactly k
#pragma unroll
            for (int i = 0; i < kSelEpt; ++i) {
                const int j = i * kSelThreads + tid;
                e[i] = j < n ? sm->out[j] : 0ull;
            }
            __syncthreads(); // out[] is rewritten below
        } else if (sp.nsplit == 1) {
#pragma unroll
            for (int i = 0; i < kSelEpt; ++i) {
                const int j = i * kSelThreads + tid;
                e[i] = j < n ? row_lists[j] : 0ull;
            }
        } else {
            for (int s = 0; s < sp.nsplit; ++s) {
                const uint64_t *src = row_lists + static_cast<size_t>(s) * sp.cap;
                const int o = sm->split_off[s];
                const int ns = sm->split_off[s + 1] - o;
                // kSelBatch loads in flight per thread, as in sel_for_each_key
                for (int j0 = 0; j0 < ns; j0 += kSelBatch * kSelThreads) {
                    uint64_t x[kSelBatch];
#pragma unroll
                    for (int u = 0; u < kSelBatch; ++u) {
                        const int j = j0 + u * kSelThreads + tid;
                        x[u] = j < ns ? __ldg(src + j) : 0ull;
                    }
#pragma unroll
                    for (int u = 0; u < kSelBatch; ++u) {
                        const int j = j0 + u * kSelThreads + tid;
                        if (j < ns)
                            sm->out[o + j] = x[u];
                    }
                }
            }
            __syncthreads();
#pragma unroll
            for (int i = 0; i < kSelEpt; ++i) {
                const int j = i * kSelThreads + tid;
                e[i] = j < n ? sm->out[j] : 0ull;
            }
            __syncthreads(); // out[] is rewritten below
        }
        const int kept = min(n, sp.topk);
        int32_t *oi = sp.out_idx + orow * sp.topk;
        float *os = sp.out_score + orow * sp.topk;
        if (kept > 0)
            sel_sort_regs(sm, e, n, kept, tid, oi, os);
        for (int i = kept + tid; i < sp.topk; i += kSelThreads) {
            oi[i] = -1;
            os[i] = -__int_as_float(0x7f800000);
        }
        __syncthreads();
    }
}

} // namespace csa
