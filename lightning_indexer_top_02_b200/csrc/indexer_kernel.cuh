// indexer_kernel.cuh -- the fused lightning-indexer + streaming top-k kernel.
//
// One persistent CTA per SM walks work items (batch b, block of qps queries,
// range of key tiles).  For each 128-key tile the tensor cores compute the
// logits L[s, (t,h)] = k[s,:] . q[t,h,:] for every head of the item's queries
// ("StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", abstract: the lightning indexer scores compressed keys per query),
// with keys as the MMA's M dimension so that each TMEM lane -- one epilogue
// thread -- holds one key's logits for every (query, head).  The epilogue
// applies ReLU and the head weights without leaving the thread, masks keys the
// query may not see, and streams the surviving (score, index) pairs into a
// per-query candidate list that is cut back to the top k plus slack whenever
// it could overflow.  When an item's key range is done, a separate warpgroup
// reduces each list to the exact top k and sorts it while the next item's
// tiles already flow through the tensor cores, so the [B,S,H_I,T] score tensor
// never exists and the selection stays off the MMA's critical path.
//
// Warp roles (448 threads):
//   warp 0       TMA producer: the query block once per item (with an L2
//                prefetch of the next item's), key tiles into a ring
//   warp 1       TMEM owner and MMA issuer (one thread): per key tile, d/16
//                tcgen05.mma (M = 128 keys, N = qps*H_I) into one of two
//                256-column TMEM accumulators
//   warps 2..5   epilogue warpgroup 0: the first half of the item's queries
//   warps 6..9   epilogue warpgroup 1: the second half (idle when qps == 1)
//   warps 10..13 finalizer: exact top-k + sort of each finished query, from
//                double-buffered candidate lists
#pragma once
#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"
#include "topk_group.cuh"

namespace csa {

constexpr int kTileKeys = 128;   // MMA M: keys per tile
constexpr int kSlotCols = 256;   // TMEM columns per accumulator slot
constexpr int kThreads = 448;
constexpr int kGroupThreads = 128;
constexpr int kBarWg0 = 1, kBarWg1 = 2, kBarFin = 3;  // named barriers
constexpr int kEpt = 32;         // candidate keys per thread in a group (cap <= 4096)
constexpr int kMaxStages = 8;
constexpr int kMaxTopk = 2048;
constexpr int kNbCompact = 1024; // buckets of the compaction histogram
constexpr int kNbFinal = 1024;   // buckets of the final selection histogram
constexpr int kGatherMax = 128;  // keys of the boundary bucket resolved in place
constexpr int kBucketSortMax = 32; // larger buckets take the exact fallback

enum Role : int { kRoleProducer = 1, kRoleMma = 2, kRoleEpilogue = 3, kRoleFinal = 4 };

struct Params {
    int B, S, T, H, d, m, topk, causal, mode, key_fp8;
    long long q_offset;
    int qps;      // queries per item
    int N;        // MMA N = qps * H (<= 256)
    int n_wg;     // epilogue warpgroups in use (1 or 2)
    int qpw;      // queries per epilogue warpgroup = qps / n_wg
    int nqb;      // query blocks per batch
    int nsplit;   // key-range splits per query block
    int n_items;
    int stages;
    int cap;      // candidate list capacity per query
    int slack;    // compaction keeps at most topk + slack when it must cut exactly
    int row_bytes;   // bytes of one swizzled operand row: min(128, 2*d)
    int n_chunks;    // d*2 / row_bytes
    // shared memory carve-up (byte offsets from the 1024-aligned base)
    int off_q, off_k, off_w, off_state, off_wg, off_fin, off_bar, smem_bytes;
    int wg_bytes;    // per-warpgroup scratch
    const uint16_t *q; // only for L2 prefetch; loads go through the tensor map
    const float *w;
    const float *k_scale;
    int32_t *out_idx;
    float *out_score;
    uint64_t *cand;  // [gridDim.x][2][qps][cap]
    uint64_t *part;  // [B*S][nsplit][topk] (nsplit > 1)
    long long wait_limit;
};

struct Item {
    int b, q0, nq, tile_begin, tile_end, split;
};

__device__ __forceinline__ int visible_count(const Params &p, long long t)
{
    if (!p.causal)
        return p.T;
    // key s is visible iff (s+1)*m - 1 <= t  <=>  s < floor((t+1)/m)
    if (t + 1 <= 0)
        return 0;
    const long long v = (t + 1) / p.m;
    return static_cast<int>(v > p.T ? p.T : v);
}

// Items run heaviest first: the last query blocks of a causal batch see the
// most keys.
__device__ __forceinline__ Item decode_item(const Params &p, int id)
{
    Item it;
    it.split = id % p.nsplit;
    const int r = id / p.nsplit;
    it.b = r % p.B;
    const int qb = p.nqb - 1 - r / p.B;
    it.q0 = qb * p.qps;
    it.nq = min(p.qps, p.S - it.q0);
    const int nvis = visible_count(p, static_cast<long long>(it.q0 + it.nq - 1) + p.q_offset);
    const int nkt = (nvis + kTileKeys - 1) / kTileKeys;
    it.tile_begin = static_cast<int>(static_cast<long long>(it.split) * nkt / p.nsplit);
    it.tile_end = static_cast<int>(static_cast<long long>(it.split + 1) * nkt / p.nsplit);
    return it;
}

struct Barriers {
    uint64_t q_full, q_empty, drain, pad0;
    uint64_t k_full[kMaxStages], k_empty[kMaxStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t fin_full[2], fin_empty[2];
    uint32_t tmem_addr;
    int abort;
};

// Per-query streaming state (double-buffered by item parity).
struct QueryState {
    int cnt;          // candidates in the list
    uint32_t bound;   // admit a key only if ord(score) >= bound
    uint32_t min_ord; // smallest / largest score order image in the list
    uint32_t max_ord;
    int vis_end;      // keys s < vis_end are visible to this query
    int pad[3];
};

// Bounded wait used when unwinding: ignores the abort flag and the (possibly
// shrunk) per-wait budget, so that copies and MMAs already in flight land
// before the CTA frees its shared memory and TMEM.  Work in flight finishes in
// microseconds; the fixed budget (about a second) only bounds a broken GPU.
constexpr long long kDrainLimit = 1ll << 31;

__device__ __forceinline__ void wait_drain(uint64_t *bar, uint32_t parity, long long limit = kDrainLimit)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit)
            return;
    }
}

// Hint: bring [src, src+bytes) into L2 (16-byte aligned, multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)),
                 "r"(bytes)
                 : "memory");
}

// ------------------------------------------------------------------ producer
__device__ void run_producer(const Params &p, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                             uint8_t *smem, Barriers *bars, const WaitCtl &ctl)
{
    int kload = 0, qload = 0;
    const uint32_t q_bytes = static_cast<uint32_t>(p.N * p.d * 2);
    const uint32_t k_bytes = static_cast<uint32_t>(kTileKeys * p.d * 2);
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        if (!wait_bounded(&bars->q_empty, (qload & 1) ^ 1, ctl, kRoleProducer, id))
            goto unwind;
        const size_t wrow = static_cast<size_t>(it.b) * p.S + it.q0;
        if (it.tile_end > it.tile_begin) {
            mbar_arrive_expect_tx(&bars->q_full, q_bytes);
            const int row0 = static_cast<int>(wrow) * p.H;
            for (int c = 0; c < p.n_chunks; ++c)
                tma_load_2d(smem + p.off_q + c * p.N * p.row_bytes, tmQ, &bars->q_full,
                            c * (p.row_bytes / 2), row0);
        } else {
            mbar_arrive(&bars->q_full);
        }
        ++qload;
        // Warm L2 with the next item's query block while this one streams keys.
        {
            const int nid = id + gridDim.x;
            if (nid < p.n_items) {
                const Item nx = decode_item(p, nid);
                const size_t nrow = static_cast<size_t>(nx.b) * p.S + nx.q0;
                if (nx.tile_end > nx.tile_begin)
                    prefetch_l2(p.q + nrow * p.H * p.d,
                                static_cast<uint32_t>(nx.nq * p.H * p.d * 2));
            }
        }
        for (int t = it.tile_begin; t < it.tile_end; ++t) {
            const int stage = kload % p.stages;
            if (!wait_bounded(&bars->k_empty[stage], ((kload / p.stages) & 1) ^ 1, ctl,
                              kRoleProducer, id))
                goto unwind;
            mbar_arrive_expect_tx(&bars->k_full[stage], k_bytes);
            uint8_t *dst = smem + p.off_k + stage * kTileKeys * p.d * 2;
            const int row = it.b * p.T + t * kTileKeys;
            for (int c = 0; c < p.n_chunks; ++c)
                tma_load_2d(dst + c * kTileKeys * p.row_bytes, tmK, &bars->k_full[stage],
                            c * (p.row_bytes / 2), row);
            ++kload;
        }
    }
unwind:
    // Let every copy already issued land before the CTA can exit.
    for (int s = 0; s < p.stages; ++s) {
        if (kload > s) {
            const int fills = (kload - s + p.stages - 1) / p.stages;
            wait_drain(&bars->k_full[s], (fills - 1) & 1);
        }
    }
    if (qload > 0)
        wait_drain(&bars->q_full, (qload - 1) & 1);
}

// ------------------------------------------------------------------ MMA issuer
__device__ void run_mma(const Params &p, uint8_t *smem, Barriers *bars, uint32_t tmem_base,
                        const WaitCtl &ctl)
{
    int kuse = 0, quse = 0, acc_use = 0;
    const uint32_t idesc = instr_desc_f16(p.N, p.key_fp8 ? 0 : 1);
    const int ksteps_per_chunk = p.row_bytes / 32;  // 16 elements (32 B) per MMA K step
    const uint32_t q_base = smem_u32(smem + p.off_q);
    const uint32_t k_base = smem_u32(smem + p.off_k);
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        if (!wait_bounded(&bars->q_full, quse & 1, ctl, kRoleMma, id))
            goto unwind;
        tc_fence_after();
        for (int t = it.tile_begin; t < it.tile_end; ++t) {
            const int stage = kuse % p.stages;
            if (!wait_bounded(&bars->k_full[stage], (kuse / p.stages) & 1, ctl, kRoleMma, id))
                goto unwind;
            const int slot = acc_use & 1;
            if (!wait_bounded(&bars->acc_empty[slot], ((acc_use >> 1) & 1) ^ 1, ctl, kRoleMma, id))
                goto unwind;
            tc_fence_after();
            const uint32_t a_tile = k_base + stage * kTileKeys * p.d * 2;
            const uint32_t d_tmem = tmem_base + slot * kSlotCols;
            for (int c = 0; c < p.n_chunks; ++c) {
                for (int ks = 0; ks < ksteps_per_chunk; ++ks) {
                    const uint64_t adesc = smem_desc_kmajor(
                        a_tile + c * kTileKeys * p.row_bytes + ks * 32, p.row_bytes);
                    const uint64_t bdesc =
                        smem_desc_kmajor(q_base + c * p.N * p.row_bytes + ks * 32, p.row_bytes);
                    mma_f16_ss(d_tmem, adesc, bdesc, idesc, (c | ks) != 0);
                }
            }
            mma_commit(&bars->acc_full[slot]);
            mma_commit(&bars->k_empty[stage]);
            ++acc_use;
            ++kuse;
        }
        if (it.tile_end > it.tile_begin)
            mma_commit(&bars->q_empty);
        else
            mbar_arrive(&bars->q_empty);
        ++quse;
    }
unwind:
    mma_commit(&bars->drain);
    wait_drain(&bars->drain, 0);
}

// ------------------------------------------------------------------ group scratch
struct WgScratch {          // one per epilogue warpgroup
    GroupSmall gs;
    uint32_t hist[kNbCompact];
};

struct FinScratch {         // the finalizer's
    GroupSmall gs;
    int gather_n;
    int pad[3];
    uint32_t hist[kNbFinal];
    uint64_t gather[kGatherMax];
    uint64_t stage[kMaxTopk];
};

// ------------------------------------------------------------------ compaction
// Cuts a query's list back when it could overflow: keeps every key whose
// bucket is at or above the bucket of the k-th largest key (a superset of the
// top k), or -- when the score range is degenerate or that bucket is too full
// -- the radix-exact top k plus slack.  Updates cnt, bound and min_ord.
__device__ void compact_list(const Params &p, uint64_t *list, QueryState &st, WgScratch *sc,
                             int bar, int tid)
{
    const int n = st.cnt;
    uint64_t e[kEpt];
#pragma unroll
    for (int i = 0; i < kEpt; ++i) {
        const int j = i * kGroupThreads + tid;
        e[i] = j < n ? list[j] : 0ull;
    }
    const BucketMap bm = bucket_map(st.min_ord, st.max_ord, kNbCompact);
    bool done = false;
    uint32_t newmin = 0xFFFFFFFFu;
    int kept = 0;
    if (bm.ok) {
        for (int i = tid; i < kNbCompact; i += kGroupThreads)
            sc->hist[i] = 0;
        named_bar_sync(bar, kGroupThreads);
#pragma unroll
        for (int i = 0; i < kEpt; ++i)
            if (e[i] != 0)
                atomicAdd(&sc->hist[bucket_of(key_score(e[i]), bm, kNbCompact)], 1u);
        named_bar_sync(bar, kGroupThreads);
        bucket_boundary<kGroupThreads, kNbCompact>(sc->hist, p.topk, false, &sc->gs, bar, tid);
        const int bstar = sc->gs.bcast[0];
        const int cand_kept = sc->gs.bcast[1] + sc->gs.bcast[2];
        named_bar_sync(bar, kGroupThreads);
        if (cand_kept <= p.cap - 2 * kTileKeys) {
            int mine = 0;
            uint32_t mn = 0xFFFFFFFFu;
            bool keep[kEpt];
#pragma unroll
            for (int i = 0; i < kEpt; ++i) {
                keep[i] = e[i] != 0 && bucket_of(key_score(e[i]), bm, kNbCompact) >= bstar;
                mine += keep[i] ? 1 : 0;
                mn = keep[i] ? min(mn, key_ord(e[i])) : mn;
            }
            int total;
            int off = group_excl_scan<kGroupThreads>(mine, &sc->gs, bar, tid, &total);
#pragma unroll
            for (int i = 0; i < kEpt; ++i)
                if (keep[i])
                    list[off++] = e[i];
            newmin = group_min_u32<kGroupThreads>(mn, &sc->gs, bar, tid);
            kept = total;
            done = true;
        }
    }
    if (!done) {
        int k2;
        const uint64_t L = radix_bound<kGroupThreads, kEpt>(e, p.topk, p.slack, sc->hist, &sc->gs,
                                                            bar, tid, &k2);
        kept = write_kept<kGroupThreads, kEpt>(e, L, list, &sc->gs, bar, tid, &newmin);
    }
    named_bar_sync(bar, kGroupThreads); // list writes and scratch reads done
    if (tid == 0) {
        st.cnt = kept;
        st.bound = max(st.bound, newmin);
        st.min_ord = newmin;
    }
    named_bar_sync(bar, kGroupThreads);
}

// ------------------------------------------------------------------ epilogue
template <bool kHeadsGe32>
__device__ void run_epilogue(const Params &p, uint8_t *smem, Barriers *bars, uint32_t tmem_base,
                             const WaitCtl &ctl, int wg)
{
    const int tid = (threadIdx.x - 64) & (kGroupThreads - 1); // 0..127 within the warpgroup
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int bar = wg == 0 ? kBarWg0 : kBarWg1;
    const int quarter = warp & 3;             // TMEM lanes this warp may read
    const int key_local = quarter * 32 + lane;
    float *w_s = reinterpret_cast<float *>(smem + p.off_w);
    QueryState *qs_all = reinterpret_cast<QueryState *>(smem + p.off_state);
    WgScratch *sc = reinterpret_cast<WgScratch *>(smem + p.off_wg + wg * p.wg_bytes);
    uint64_t *cand_cta = p.cand + static_cast<size_t>(blockIdx.x) * 2 * p.qps * p.cap;
    const uint32_t bound0 = p.mode == 1 ? 0x80000001u : 0u; // gate: score > 0
    const int j0 = wg * p.qpw;                 // first query slot this group owns
    const int col0 = j0 * p.H;                 // first TMEM column it reads
    const int ncols = p.qpw * p.H;             // TMEM columns it reads
    const int nchunk = ncols / 32;             // in 32-column chunks
    int acc_use = 0, it_count = 0;
    constexpr int kWRegs = kSlotCols / kGroupThreads;
    float wnext[kWRegs];
    {
        const Item it0 = decode_item(p, blockIdx.x);
        const size_t row = static_cast<size_t>(it0.b) * p.S + it0.q0;
        for (int r = 0; r < kWRegs; ++r) {
            const int c = tid + r * kGroupThreads;
            wnext[r] = (blockIdx.x < p.n_items && c < ncols && j0 + c / p.H < it0.nq)
                           ? p.w[(row + j0) * p.H + c]
                           : 0.0f;
        }
    }

    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        const int buf = it_count & 1;
        QueryState *qs = qs_all + buf * p.qps;
        uint64_t *lists = cand_cta + static_cast<size_t>(buf) * p.qps * p.cap;
        // The finalizer must be done with this list buffer (item it_count - 2).
        bool ok = wait_bounded(&bars->fin_empty[buf], ((it_count >> 1) & 1) ^ 1, ctl,
                               kRoleEpilogue, id);
        ok = group_all(bar, kGroupThreads, ok);
        if (!ok) {
            *ctl.abort = 1;
            break;
        }
        for (int j = j0 + tid; j < j0 + p.qpw; j += kGroupThreads) {
            const int i = it.q0 + j;
            QueryState st;
            st.cnt = 0;
            st.bound = bound0;
            st.min_ord = 0xFFFFFFFFu;
            st.max_ord = 0u;
            st.vis_end = i < p.S ? visible_count(p, static_cast<long long>(i) + p.q_offset) : 0;
            st.pad[0] = st.pad[1] = st.pad[2] = 0;
            qs[j] = st;
        }
        // This group's head weights for the item: registers loaded one item
        // ahead, stored to the group's own columns of w_s (nothing else reads
        // them), then the next item's loads are issued.
        for (int r = 0; r < kWRegs; ++r) {
            const int c = tid + r * kGroupThreads;
            if (c < ncols)
                w_s[col0 + c] = wnext[r];
        }
        {
            const int nid = id + gridDim.x;
            if (nid < p.n_items) {
                const Item nx = decode_item(p, nid);
                const size_t nrow = static_cast<size_t>(nx.b) * p.S + nx.q0;
                for (int r = 0; r < kWRegs; ++r) {
                    const int c = tid + r * kGroupThreads;
                    wnext[r] = (c < ncols && j0 + c / p.H < nx.nq) ? p.w[(nrow + j0) * p.H + c] : 0.0f;
                }
            }
        }
        named_bar_sync(bar, kGroupThreads);

        for (int t = it.tile_begin; t < it.tile_end; ++t) {
            const int s = t * kTileKeys + key_local;
            float kscale = 1.0f;
            if (p.key_fp8 && s < p.T)
                kscale = p.k_scale[static_cast<size_t>(it.b) * p.T + s];
            const int slot = acc_use & 1;
            ok = wait_bounded(&bars->acc_full[slot], (acc_use >> 1) & 1, ctl, kRoleEpilogue, id);
            ok = group_all(bar, kGroupThreads, ok);
            if (!ok)
                break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   slot * kSlotCols + col0;
            const float *wsub = w_s + col0;

            auto emit = [&](int jq, float score) {
                QueryState &st = qs[jq];
                const uint32_t ord = ord_of_score(score * kscale);
                const bool pass = s < st.vis_end && ord >= st.bound;
                const unsigned bal = __ballot_sync(0xffffffffu, pass);
                if (bal) {
                    const uint32_t mx = __reduce_max_sync(0xffffffffu, pass ? ord : 0u);
                    const uint32_t mn = __reduce_min_sync(0xffffffffu, pass ? ord : 0xFFFFFFFFu);
                    int base = 0;
                    if (lane == 0) {
                        base = atomicAdd(&st.cnt, __popc(bal));
                        atomicMax(&st.max_ord, mx);
                        atomicMin(&st.min_ord, mn);
                    }
                    base = __shfl_sync(0xffffffffu, base, 0);
                    if (pass)
                        lists[static_cast<size_t>(jq) * p.cap + base + __popc(bal & lanemask_lt())] =
                            make_key(ord, static_cast<uint32_t>(s));
                }
            };

            float acc = 0.0f;
            uint32_t v[32];
            __syncwarp();
            tmem_ld_32x32b_x32(taddr, v);
            for (int c = 0; c < nchunk; ++c) {
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    reg_fence(v[i]);
                float x[32];
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    x[i] = fmaxf(__uint_as_float(v[i]), 0.0f);
                if (c + 1 < nchunk) {
                    __syncwarp();
                    tmem_ld_32x32b_x32(taddr + (c + 1) * 32, v);
                }
                const float *wc = wsub + c * 32;
                if (kHeadsGe32) {
                    // packed fp32 FMA over pairs of heads
                    unsigned long long a0 = 0ull, a1 = 0ull;
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        const float4 w4 = *reinterpret_cast<const float4 *>(wc + i);
                        unsigned long long xa, xb, wa, wb;
                        asm("mov.b64 %0, {%1, %2};" : "=l"(xa) : "f"(x[i]), "f"(x[i + 1]));
                        asm("mov.b64 %0, {%1, %2};" : "=l"(xb) : "f"(x[i + 2]), "f"(x[i + 3]));
                        asm("mov.b64 %0, {%1, %2};" : "=l"(wa) : "f"(w4.x), "f"(w4.y));
                        asm("mov.b64 %0, {%1, %2};" : "=l"(wb) : "f"(w4.z), "f"(w4.w));
                        asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a0) : "l"(xa), "l"(wa));
                        asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a1) : "l"(xb), "l"(wb));
                    }
                    float p0, p1, p2, p3;
                    asm("mov.b64 {%0, %1}, %2;" : "=f"(p0), "=f"(p1) : "l"(a0));
                    asm("mov.b64 {%0, %1}, %2;" : "=f"(p2), "=f"(p3) : "l"(a1));
                    acc += (p0 + p1) + (p2 + p3);
                    if (((c + 1) * 32) % p.H == 0) {
                        emit(j0 + (c * 32) / p.H, acc);
                        acc = 0.0f;
                    }
                } else {
                    // H < 32 (a power of two): each 32-column chunk holds 32/H queries
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        acc = fmaf(x[i], wc[i], acc);
                        if (((i + 1) & (p.H - 1)) == 0) {
                            emit(j0 + (c * 32 + i) / p.H, acc);
                            acc = 0.0f;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->acc_empty[slot]);
            ++acc_use;
            named_bar_sync(bar, kGroupThreads);
            // Cut back any list that the next tile could overflow.
            for (int jq = j0; jq < j0 + p.qpw; ++jq) {
                if (qs[jq].cnt > p.cap - kTileKeys)
                    compact_list(p, lists + static_cast<size_t>(jq) * p.cap, qs[jq], sc, bar, tid);
            }
        }
        if (!ok) {
            *ctl.abort = 1;
            break;
        }
        // Hand the finished lists to the finalizer.
        mbar_arrive(&bars->fin_full[buf]);
        ++it_count;
    }
}

// ------------------------------------------------------------------ finalizer
// Exact top-k of one finished list, sorted by (score desc, index asc):
// histogram over [min, max] score buckets, resolve the boundary bucket in
// place, counting-sort the selected keys by bucket and sort each (small)
// bucket.  Degenerate cases take the radix-exact path and a bitonic sort.
// Returns the number of keys, in order, in sc->stage.
__device__ int final_select(const Params &p, const uint64_t *list, const QueryState &st,
                            FinScratch *sc, int bar, int tid)
{
    const int n = st.cnt;
    const int K = p.topk;
    const int kept = min(n, K);
    if (kept == 0)
        return 0;
    uint64_t e[kEpt];
#pragma unroll
    for (int i = 0; i < kEpt; ++i) {
        const int j = i * kGroupThreads + tid;
        e[i] = j < n ? list[j] : 0ull;
    }
    const BucketMap bm = bucket_map(st.min_ord, st.max_ord, kNbFinal);
    if (bm.ok) {
        for (int i = tid; i < kNbFinal; i += kGroupThreads)
            sc->hist[i] = 0;
        if (tid == 0)
            sc->gather_n = 0;
        named_bar_sync(bar, kGroupThreads);
#pragma unroll
        for (int i = 0; i < kEpt; ++i)
            if (e[i] != 0)
                atomicAdd(&sc->hist[bucket_of(key_score(e[i]), bm, kNbFinal)], 1u);
        named_bar_sync(bar, kGroupThreads);
        bucket_boundary<kGroupThreads, kNbFinal>(sc->hist, kept, true, &sc->gs, bar, tid);
        const int bstar = sc->gs.bcast[0];
        const int above = sc->gs.bcast[1];
        const int inb = sc->gs.bcast[2];
        const int biggest = sc->gs.bcast[3];
        named_bar_sync(bar, kGroupThreads);
        if (biggest <= kBucketSortMax && inb <= kGatherMax) {
            const int r = kept - above; // keys taken from the boundary bucket
            // gather the boundary bucket when only part of it is taken
            if (r < inb) {
#pragma unroll
                for (int i = 0; i < kEpt; ++i)
                    if (e[i] != 0 && bucket_of(key_score(e[i]), bm, kNbFinal) == bstar)
                        sc->gather[atomicAdd(&sc->gather_n, 1)] = e[i];
                named_bar_sync(bar, kGroupThreads);
            }
            // counting-sort scatter: hist[b] holds the next free slot of bucket b
#pragma unroll
            for (int i = 0; i < kEpt; ++i) {
                if (e[i] == 0)
                    continue;
                const int b = bucket_of(key_score(e[i]), bm, kNbFinal);
                bool sel = b > bstar;
                if (b == bstar) {
                    if (r < inb) {
                        int rank = 0;
                        for (int g = 0; g < inb; ++g)
                            rank += sc->gather[g] > e[i] ? 1 : 0;
                        sel = rank < r;
                    } else {
                        sel = true;
                    }
                }
                if (sel)
                    sc->stage[atomicAdd(&sc->hist[b], 1u)] = e[i];
            }
            named_bar_sync(bar, kGroupThreads);
            // per-bucket insertion sort, descending: bucket b spans
            // [end of bucket b+1, end of bucket b) after the scatter
            for (int b = tid; b < kNbFinal; b += kGroupThreads) {
                if (b < bstar)
                    continue;
                const int end = static_cast<int>(sc->hist[b]);
                const int beg = b + 1 < kNbFinal ? static_cast<int>(sc->hist[b + 1]) : 0;
                for (int x = beg + 1; x < end; ++x) {
                    const uint64_t key = sc->stage[x];
                    int y = x - 1;
                    while (y >= beg && sc->stage[y] < key) {
                        sc->stage[y + 1] = sc->stage[y];
                        --y;
                    }
                    sc->stage[y + 1] = key;
                }
            }
            named_bar_sync(bar, kGroupThreads);
            return kept;
        }
    }
    // exact fallback: radix select + bitonic sort
    const int P = pow2_at_least(kept);
    uint64_t L = 1;
    if (n > K) {
        int k2;
        L = radix_bound<kGroupThreads, kEpt>(e, K, 0, sc->hist, &sc->gs, bar, tid, &k2);
    }
    uint32_t mn;
    const int total = write_kept<kGroupThreads, kEpt>(e, L, sc->stage, &sc->gs, bar, tid, &mn);
    for (int i = total + tid; i < P; i += kGroupThreads)
        sc->stage[i] = 0ull;
    named_bar_sync(bar, kGroupThreads);
    bitonic_sort_desc<kGroupThreads>(sc->stage, P, bar, tid);
    return kept;
}

__device__ void run_finalizer(const Params &p, uint8_t *smem, Barriers *bars, const WaitCtl &ctl)
{
    const int tid = threadIdx.x - 320; // warps 10..13
    QueryState *qs_all = reinterpret_cast<QueryState *>(smem + p.off_state);
    FinScratch *sc = reinterpret_cast<FinScratch *>(smem + p.off_fin);
    const uint64_t *cand_cta = p.cand + static_cast<size_t>(blockIdx.x) * 2 * p.qps * p.cap;
    int it_count = 0;
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        const int buf = it_count & 1;
        bool ok = wait_bounded(&bars->fin_full[buf], (it_count >> 1) & 1, ctl, kRoleFinal, id);
        ok = group_all(kBarFin, kGroupThreads, ok);
        if (!ok) {
            *ctl.abort = 1;
            break;
        }
        const QueryState *qs = qs_all + buf * p.qps;
        const uint64_t *lists = cand_cta + static_cast<size_t>(buf) * p.qps * p.cap;
        for (int j = 0; j < it.nq; ++j) {
            const QueryState st = qs[j];
            const int kept = final_select(p, lists + static_cast<size_t>(j) * p.cap, st, sc,
                                          kBarFin, tid);
            const size_t row = static_cast<size_t>(it.b) * p.S + it.q0 + j;
            if (p.nsplit == 1) {
                for (int slot = tid; slot < p.topk; slot += kGroupThreads) {
                    const size_t o = row * p.topk + slot;
                    if (slot < kept) {
                        const uint64_t key = sc->stage[slot];
                        p.out_idx[o] = key_index(key);
                        p.out_score[o] = key_score(key);
                    } else {
                        p.out_idx[o] = -1;
                        p.out_score[o] = -__int_as_float(0x7f800000);
                    }
                }
            } else {
                uint64_t *dst = p.part + (row * p.nsplit + it.split) * p.topk;
                for (int slot = tid; slot < p.topk; slot += kGroupThreads)
                    dst[slot] = slot < kept ? sc->stage[slot] : 0ull;
            }
            named_bar_sync(kBarFin, kGroupThreads);
        }
        mbar_arrive(&bars->fin_empty[buf]);
        ++it_count;
    }
}

// ------------------------------------------------------------------ kernel
template <bool kHeadsGe32>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_topk_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Barriers *bars = reinterpret_cast<Barriers *>(smem + p.off_bar);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int epi_warps = 4 * p.n_wg;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        mbar_init(&bars->drain, 1);
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->acc_full[s], 1);
            mbar_init(&bars->acc_empty[s], epi_warps);
            mbar_init(&bars->fin_full[s], 32 * epi_warps);
            mbar_init(&bars->fin_empty[s], kGroupThreads);
        }
        bars->abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_addr, 2 * kSlotCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_addr;
    WaitCtl ctl{&bars->abort, p.wait_limit};

    if (warp == 0) {
        if (lane == 0)
            run_producer(p, &tmQ, &tmK, smem, bars, ctl);
    } else if (warp == 1) {
        if (lane == 0)
            run_mma(p, smem, bars, tmem_base, ctl);
    } else if (warp < 6) {
        run_epilogue<kHeadsGe32>(p, smem, bars, tmem_base, ctl, 0);
    } else if (warp < 10) {
        if (p.n_wg == 2)
            run_epilogue<kHeadsGe32>(p, smem, bars, tmem_base, ctl, 1);
    } else {
        run_finalizer(p, smem, bars, ctl);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, 2 * kSlotCols);
    }
}

// ------------------------------------------------------------------ split merge
// Merges the nsplit partial lists of one query row into its final top-k:
// "StreamIndex ...", abstract (a partition-merge top-k that never materialises
// the full score tensor); here the partitions are key ranges of one query.
constexpr int kMergeThreads = 256;
constexpr int kMergeEpt = 32; // nsplit * topk <= 8192

__global__ void __launch_bounds__(kMergeThreads)
    merge_splits_kernel(const uint64_t *__restrict__ part, int rows, int nsplit, int topk,
                        int32_t *__restrict__ out_idx, float *__restrict__ out_score)
{
    __shared__ GroupSmall gs;
    __shared__ uint32_t hist[256];
    __shared__ uint64_t sortbuf[kMaxTopk];
    const int tid = threadIdx.x;
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
        const uint64_t *src = part + static_cast<size_t>(row) * nsplit * topk;
        const int n_all = nsplit * topk;
        uint64_t e[kMergeEpt];
        int mine = 0;
#pragma unroll
        for (int i = 0; i < kMergeEpt; ++i) {
            const int x = i * kMergeThreads + tid;
            e[i] = x < n_all ? src[x] : 0ull;
            mine += e[i] != 0;
        }
        int n;
        group_excl_scan<kMergeThreads>(mine, &gs, 0, tid, &n);
        const int kept = min(n, topk);
        const int P = pow2_at_least(kept);
        uint64_t L = 1;
        if (n > topk) {
            int k2;
            L = radix_bound<kMergeThreads, kMergeEpt>(e, topk, 0, hist, &gs, 0, tid, &k2);
        }
        uint32_t mn;
        const int total = write_kept<kMergeThreads, kMergeEpt>(e, L, sortbuf, &gs, 0, tid, &mn);
        for (int i = total + tid; i < P; i += kMergeThreads)
            sortbuf[i] = 0ull;
        __syncthreads();
        bitonic_sort_desc<kMergeThreads>(sortbuf, P, 0, tid);
        for (int slot = tid; slot < topk; slot += kMergeThreads) {
            const size_t o = static_cast<size_t>(row) * topk + slot;
            if (slot < kept) {
                const uint64_t key = sortbuf[slot];
                out_idx[o] = key_index(key);
                out_score[o] = key_score(key);
            } else {
                out_idx[o] = -1;
                out_score[o] = -__int_as_float(0x7f800000);
            }
        }
        __syncthreads();
    }
}

} // namespace csa
