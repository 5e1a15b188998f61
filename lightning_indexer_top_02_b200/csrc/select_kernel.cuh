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
// One CTA per query row at a time:
//   1. If the lists hold more keys than fit in shared memory, a radix select
//      over the 64-bit keys, reading them from global memory one byte per
//      pass, finds the k-th largest key L; the k keys >= L are gathered.
//      Otherwise every key is copied to shared memory.
//   2. A histogram over NB buckets linear in the score, spanning the keys'
//      own [min, max], finds the bucket holding the k-th largest key; the keys
//      of that bucket and above are scattered into bucket order (a counting
//      sort), and each bucket is then sorted on its own (insertion sort; the
//      buckets average a few keys).  A bucket too full for that -- many equal
//      or near-equal scores -- sends the row to a bitonic sort instead.
//   3. The first min(k, n) keys become (index, score) pairs; the rest of the
//      row is padded with (-1, -inf).
#pragma once
#include <cstdint>

#include "ptx.cuh"
#include "topk_group.cuh"

namespace csa {

constexpr int kSelThreads = 512;
constexpr int kSelNb = 2048;          // histogram buckets
constexpr int kSelKeys = 4096;        // keys held in shared memory
constexpr int kSelSmallBucket = 24;   // largest bucket sorted by one thread
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
    uint64_t in[kSelKeys];
    uint64_t out[kSelKeys];
};

// Block-wide min and max of the score order images of a[0..n).
__device__ __forceinline__ void sel_ord_range(const uint64_t *a, int n, GroupSmall *gs, int tid,
                                              uint32_t *mn, uint32_t *mx)
{
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (int i = tid; i < n; i += kSelThreads) {
        const uint32_t o = key_ord(a[i]);
        lo = min(lo, o);
        hi = max(hi, o);
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    const int lane = tid & 31, wid = tid >> 5;
    if (lane == 0) {
        gs->warp_sums[wid] = lo;
        gs->warp_sums[16 + wid] = hi;
    }
    __syncthreads();
    uint32_t a0 = 0xFFFFFFFFu, b0 = 0u;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) {
        a0 = min(a0, gs->warp_sums[w]);
        b0 = max(b0, gs->warp_sums[16 + w]);
    }
    __syncthreads();
    *mn = a0;
    *mx = b0;
}

// Radix select over the row's lists in global memory: the largest L such that
// exactly `need` keys are >= L (keys are distinct and non-zero; n > need).
__device__ uint64_t sel_radix_global(const SelParams &sp, const uint64_t *row_lists,
                                     const SelSmem *ro, SelSmem *sm, int need, int tid)
{
    const int lane = tid & 31;
    uint64_t prefix = 0, mask = 0;
    for (int pos = 56; pos >= 0; pos -= 8) {
        for (int i = tid; i < 256; i += kSelThreads)
            sm->hist[i] = 0;
        __syncthreads();
        for (int s = 0; s < sp.nsplit; ++s) {
            const uint64_t *src = row_lists + static_cast<size_t>(s) * sp.cap;
            const int n = ro->split_off[s + 1] - ro->split_off[s];
            for (int j = tid; j < n; j += kSelThreads) {
                const uint64_t x = src[j];
                if ((x & mask) == prefix)
                    atomicAdd(&sm->hist[static_cast<uint32_t>(x >> pos) & 255u], 1u);
            }
        }
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

// Sorts the keys of in[0..n) that belong to the top `kept` (kept <= n) into
// descending order.  Returns the buffer holding them at [0, kept).
__device__ uint64_t *sel_sort_top(SelSmem *sm, int n, int kept, int tid)
{
    uint32_t mn, mx;
    sel_ord_range(sm->in, n, &sm->gs, tid, &mn, &mx);
    const BucketMap bm = bucket_map(mn, mx, kSelNb);
    bool fallback = !bm.ok;
    int total = n;
    uint64_t *res = sm->in;
    if (!fallback) {
        // histogram with buckets numbered from the top score down
        for (int i = tid; i < kSelNb; i += kSelThreads)
            sm->hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += kSelThreads)
            atomicAdd(&sm->hist[kSelNb - 1 - bucket_of(key_score(sm->in[i]), bm, kSelNb)], 1u);
        __syncthreads();
        // exclusive prefix over buckets (top first): hist[b] becomes the first
        // slot of bucket b; find the bucket db* holding slot kept-1
        constexpr int PER = kSelNb / kSelThreads;
        uint32_t c[PER];
        uint32_t sum = 0;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            c[j] = sm->hist[tid * PER + j];
            sum += c[j];
        }
        int tot;
        const int base = group_excl_scan<kSelThreads>(static_cast<int>(sum), &sm->gs, 0, tid, &tot);
        uint32_t run = static_cast<uint32_t>(base);
        int biggest = 0;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const uint32_t start = run;
            sm->hist[tid * PER + j] = start;
            run += c[j];
            if (start < static_cast<uint32_t>(kept) && run >= static_cast<uint32_t>(kept)) {
                sm->misc[0] = tid * PER + j;   // db*
                sm->misc[1] = static_cast<int>(run); // keys in buckets <= db*
            }
            if (start < static_cast<uint32_t>(kept))
                biggest = max(biggest, static_cast<int>(c[j]));
        }
        biggest = __reduce_max_sync(0xffffffffu, biggest);
        if ((tid & 31) == 0)
            sm->gs.warp_sums[tid >> 5] = static_cast<uint32_t>(biggest);
        __syncthreads();
        const int dstar = sm->misc[0];
        total = sm->misc[1];
        int big = 0;
#pragma unroll
        for (int w = 0; w < kSelThreads / 32; ++w)
            big = max(big, static_cast<int>(sm->gs.warp_sums[w]));
        __syncthreads();
        // scatter the keys of buckets <= db* into bucket order
        for (int i = tid; i < n; i += kSelThreads) {
            const uint64_t x = sm->in[i];
            const int db = kSelNb - 1 - bucket_of(key_score(x), bm, kSelNb);
            if (db <= dstar)
                sm->out[atomicAdd(&sm->hist[db], 1u)] = x;
        }
        __syncthreads();
        res = sm->out;
        if (big > kSelSmallBucket) {
            fallback = true;
        } else {
            // bucket db now spans [end(db-1), end(db)) where end = hist after the scatter
            for (int db = tid; db <= dstar; db += kSelThreads) {
                const int lo = db == 0 ? 0 : static_cast<int>(sm->hist[db - 1]);
                const int hi = static_cast<int>(sm->hist[db]);
                for (int a = lo + 1; a < hi; ++a) {
                    const uint64_t x = sm->out[a];
                    int b = a - 1;
                    while (b >= lo && sm->out[b] < x) {
                        sm->out[b + 1] = sm->out[b];
                        --b;
                    }
                    sm->out[b + 1] = x;
                }
            }
            __syncthreads();
        }
    }
    if (fallback) {
        // bitonic sort of res[0..total) padded with empty keys to a power of two
        const int P = pow2_at_least(total);
        for (int i = total + tid; i < P; i += kSelThreads)
            res[i] = 0ull;
        __syncthreads();
        bitonic_sort_desc<kSelThreads>(res, P, 0, tid);
    }
    return res;
}

__global__ void __launch_bounds__(kSelThreads)
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
        if (tid == 0) {
            int off = 0;
            sm->split_off[0] = 0;
            for (int s = 0; s < sp.nsplit; ++s) {
                off += sp.counts[static_cast<size_t>(r) * sp.nsplit + s];
                sm->split_off[s + 1] = off;
            }
        }
        __syncthreads();
        const int n_all = sm->split_off[sp.nsplit];
        int n = n_all;
        if (n_all > kSelKeys) {
            const uint64_t L = sel_radix_global(sp, row_lists, sm, sm, sp.topk, tid);
            if (tid == 0)
                sm->misc[2] = 0;
            __syncthreads();
            for (int s = 0; s < sp.nsplit; ++s) {
                const uint64_t *src = row_lists + static_cast<size_t>(s) * sp.cap;
                const int ns = sm->split_off[s + 1] - sm->split_off[s];
                for (int j = tid; j < ns; j += kSelThreads) {
                    const uint64_t x = src[j];
                    if (x >= L)
                        sm->in[atomicAdd(&sm->misc[2], 1)] = x;
                }
            }
            n = sp.topk;
        } else {
            for (int s = 0; s < sp.nsplit; ++s) {
                const uint64_t *src = row_lists + static_cast<size_t>(s) * sp.cap;
                const int o = sm->split_off[s];
                const int ns = sm->split_off[s + 1] - o;
                for (int j = tid; j < ns; j += kSelThreads)
                    sm->in[o + j] = src[j];
            }
        }
        __syncthreads();
        const int kept = min(n, sp.topk);
        const uint64_t *res = kept > 0 ? sel_sort_top(sm, n, kept, tid) : sm->in;
        int32_t *oi = sp.out_idx + orow * sp.topk;
        float *os = sp.out_score + orow * sp.topk;
        for (int i = tid; i < sp.topk; i += kSelThreads) {
            if (i < kept) {
                const uint64_t key = res[i];
                oi[i] = key_index(key);
                os[i] = key_score(key);
            } else {
                oi[i] = -1;
                os[i] = -__int_as_float(0x7f800000);
            }
        }
        __syncthreads();
    }
}

} // namespace csa
