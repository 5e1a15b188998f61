// union_kernel.cuh -- OR-union of several layers' selections per query.
//
// "FlashMemory-DeepSeek-V4: Lightning Index Ultra-Long Context via Lookahead
// Sparse Attention", "What carries the argument": gated indexers sit on a few
// intermediate layers and their binarised decisions are combined by
// OR-union.  For every query row the union of the key indices the given
// selection lists hold (entries outside [0, T) are padding) is written in
// ascending key order, at most `cap` of them, the rest padded with -1, with
// the number written in `count`.
//
// One CTA per row at a time (grid-stride): a bitmap of the row's T keys in
// shared memory collects the lists (atomicOr), then a block-wide prefix sum
// over the words' population counts places every set bit at its output
// position, so the output comes out sorted without a sort.
#pragma once
#include <cstdint>

namespace csa {
namespace uni {

constexpr int kThreads = 256;
constexpr int kMaxLists = 8;

struct UnionParams {
    const int32_t *lists[kMaxLists];   // [rows, topk] each
    int n_lists, rows, topk, T, cap, words;
    int32_t *out;                      // [rows, cap]
    int32_t *count;                    // [rows]
};

__global__ void __launch_bounds__(kThreads) union_kernel(const UnionParams p)
{
    extern __shared__ uint32_t bm[];              // [words] bitmap, then [kThreads/32] scan
    uint32_t *warp_tot = bm + p.words;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // each thread owns words [w0, w1) for the placement pass
    const int per = (p.words + kThreads - 1) / kThreads;
    const int w0 = min(p.words, tid * per), w1 = min(p.words, w0 + per);
    for (int r = blockIdx.x; r < p.rows; r += gridDim.x) {
        for (int w = tid; w < p.words; w += kThreads)
            bm[w] = 0u;
        __syncthreads();
        for (int l = 0; l < p.n_lists; ++l) {
            const int32_t *src = p.lists[l] + static_cast<size_t>(r) * p.topk;
            for (int j = tid; j < p.topk; j += kThreads) {
                const int32_t s = src[j];
                if (s >= 0 && s < p.T)
                    atomicOr(&bm[s >> 5], 1u << (s & 31));
            }
        }
        __syncthreads();
        // exclusive prefix of the set bits over the thread's words
        int mine = 0;
        for (int w = w0; w < w1; ++w)
            mine += __popc(bm[w]);
        int incl = mine;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off)
                incl += t;
        }
        if (lane == 31)
            warp_tot[wid] = static_cast<uint32_t>(incl);
        __syncthreads();
        int base = 0, total = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            base += w < wid ? static_cast<int>(warp_tot[w]) : 0;
            total += static_cast<int>(warp_tot[w]);
        }
        int pos = base + incl - mine;
        int32_t *out = p.out + static_cast<size_t>(r) * p.cap;
        for (int w = w0; w < w1 && pos < p.cap; ++w) {
            uint32_t bits = bm[w];
            while (bits && pos < p.cap) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1;
                out[pos++] = 32 * w + b;
            }
        }
        const int n = total < p.cap ? total : p.cap;
        for (int j = n + tid; j < p.cap; j += kThreads)
            out[j] = -1;
        if (tid == 0)
            p.count[r] = n;
        __syncthreads();                          // bm and warp_tot are reused by the next row
    }
}

} // namespace uni
} // namespace csa
