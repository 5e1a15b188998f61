// indexer_kernel.cuh -- the fused lightning-indexer + streaming top-k kernel.
//
// One persistent CTA per SM walks work items (batch b, block of queries,
// range of key tiles).  For each 128-key tile the tensor cores compute the
// logits L[s, (t,h)] = k[s,:] . q[t,h,:] for all heads of the block's queries
// ("StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", abstract: the lightning indexer scores compressed keys per query),
// with keys as the MMA's M dimension so that each TMEM lane -- one epilogue
// thread -- holds one key's logits for every (query, head).  The epilogue
// applies ReLU and the head weights without leaving the thread, masks keys the
// query may not see, and streams the surviving (score, index) pairs into a
// per-query candidate list that is periodically cut back to the top k plus
// some slack.  At the end of its key range each query's list is reduced to the
// exact top k and sorted, so the [B,S,H_I,T] score tensor never exists.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: the query block once per item, key tiles into a
//               ring of shared-memory stages
//   warp 1      TMEM owner and MMA issuer (one thread): per key tile and
//               query sub-block, d/16 tcgen05.mma into one of two TMEM slots
//   warps 2..5  epilogue: TMEM -> registers, ReLU + head-weighted sum, causal
//               mask, candidate filter/append, compaction, final top-k
#pragma once
#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"
#include "topk_group.cuh"

namespace csa {

constexpr int kTileKeys = 128;   // MMA M: keys per tile
constexpr int kSlotCols = 256;   // TMEM columns per accumulator slot
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kEpiBar = 1;       // named barrier of the epilogue warps
constexpr int kEpt = 32;         // candidate keys per epilogue thread (cap <= 4096)
constexpr int kMaxStages = 8;
constexpr int kMaxTopk = 2048;

enum Role : int { kRoleProducer = 1, kRoleMma = 2, kRoleEpilogue = 3, kRoleMerge = 4 };

struct Params {
    int B, S, T, H, d, m, topk, causal, mode, key_fp8;
    long long q_offset;
    int qps;      // queries per sub-block
    int N;        // MMA N = qps * H (columns of one sub-block)
    int nsub;     // sub-blocks per item (1 or 2)
    int qpb;      // queries per item = nsub * qps
    int nqb;      // query blocks per batch
    int nsplit;   // key-range splits per query block
    int n_items;
    int stages;
    int cap;      // candidate list capacity per query
    int slack;    // compaction keeps at most topk + slack
    int row_bytes;   // bytes of one swizzled operand row: min(128, 2*d)
    int n_chunks;    // d*2 / row_bytes
    // shared memory carve-up (byte offsets from the 1024-aligned base)
    int off_q, off_k, off_sort, off_w, off_state, off_scratch, off_bar, smem_bytes;
    const float *w;
    const float *k_scale;
    int32_t *out_idx;
    float *out_score;
    uint64_t *cand;  // [gridDim.x][qpb][cap]
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
    long long v = (t + 1) / p.m;
    if (t + 1 < 0)
        v = 0;
    return static_cast<int>(v < 0 ? 0 : (v > p.T ? p.T : v));
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
    it.q0 = qb * p.qpb;
    it.nq = min(p.qpb, p.S - it.q0);
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
    uint32_t tmem_addr;
    int abort;
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

// ------------------------------------------------------------------ producer
__device__ void run_producer(const Params &p, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                             uint8_t *smem, Barriers *bars, const WaitCtl &ctl)
{
    int kload = 0, qload = 0;
    const uint32_t q_bytes = static_cast<uint32_t>(p.nsub * p.N * p.d * 2);
    const uint32_t k_bytes = static_cast<uint32_t>(kTileKeys * p.d * 2);
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        if (it.tile_end <= it.tile_begin)
            continue;
        if (!wait_bounded(&bars->q_empty, (qload & 1) ^ 1, ctl, kRoleProducer, id))
            goto unwind;
        mbar_arrive_expect_tx(&bars->q_full, q_bytes);
        for (int sub = 0; sub < p.nsub; ++sub) {
            const int row0 = (it.b * p.S + it.q0) * p.H + sub * p.N;
            uint8_t *dst = smem + p.off_q + sub * p.N * p.d * 2;
            for (int c = 0; c < p.n_chunks; ++c)
                tma_load_2d(dst + c * p.N * p.row_bytes, tmQ, &bars->q_full,
                            c * (p.row_bytes / 2), row0);
        }
        ++qload;
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
        if (it.tile_end <= it.tile_begin)
            continue;
        if (!wait_bounded(&bars->q_full, quse & 1, ctl, kRoleMma, id))
            goto unwind;
        tc_fence_after();
        for (int t = it.tile_begin; t < it.tile_end; ++t) {
            const int stage = kuse % p.stages;
            if (!wait_bounded(&bars->k_full[stage], (kuse / p.stages) & 1, ctl, kRoleMma, id))
                goto unwind;
            tc_fence_after();
            const uint32_t a_tile = k_base + stage * kTileKeys * p.d * 2;
            for (int sub = 0; sub < p.nsub; ++sub) {
                const int slot = acc_use & 1;
                if (!wait_bounded(&bars->acc_empty[slot], ((acc_use >> 1) & 1) ^ 1, ctl, kRoleMma,
                                  id))
                    goto unwind;
                tc_fence_after();
                const uint32_t b_tile = q_base + sub * p.N * p.d * 2;
                const uint32_t d_tmem = tmem_base + slot * kSlotCols;
                for (int c = 0; c < p.n_chunks; ++c) {
                    for (int ks = 0; ks < ksteps_per_chunk; ++ks) {
                        const uint64_t adesc = smem_desc_kmajor(
                            a_tile + c * kTileKeys * p.row_bytes + ks * 32, p.row_bytes);
                        const uint64_t bdesc =
                            smem_desc_kmajor(b_tile + c * p.N * p.row_bytes + ks * 32, p.row_bytes);
                        mma_f16_ss(d_tmem, adesc, bdesc, idesc, (c | ks) != 0);
                    }
                }
                mma_commit(&bars->acc_full[slot]);
                ++acc_use;
            }
            mma_commit(&bars->k_empty[stage]);
            ++kuse;
        }
        mma_commit(&bars->q_empty);
        ++quse;
    }
unwind:
    mma_commit(&bars->drain);
    wait_drain(&bars->drain, 0);
}

// ------------------------------------------------------------------ epilogue
struct QueryState {
    int cnt;        // candidates in the list
    uint32_t bound; // admit a key only if ord(score) >= bound
    int vis_end;    // keys s < vis_end are visible to this query
    int pad;
};

template <bool kHeadsGe32>
__device__ void run_epilogue(const Params &p, uint8_t *smem, Barriers *bars, uint32_t tmem_base,
                             const WaitCtl &ctl)
{
    const int etid = threadIdx.x - 64;        // 0..127
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int quarter = warp & 3;             // TMEM lanes this warp may read
    const int key_local = quarter * 32 + lane;
    float *w_s = reinterpret_cast<float *>(smem + p.off_w);
    QueryState *qs = reinterpret_cast<QueryState *>(smem + p.off_state);
    GroupScratch *sc = reinterpret_cast<GroupScratch *>(smem + p.off_scratch);
    uint64_t *sortbuf = reinterpret_cast<uint64_t *>(smem + p.off_sort);
    uint64_t *cand_cta = p.cand + static_cast<size_t>(blockIdx.x) * p.qpb * p.cap;
    const uint32_t bound0 = p.mode == 1 ? 0x80000001u : 0u; // gate: score > 0
    int acc_use = 0;

    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        // ---- per-item state
        for (int j = etid; j < p.qpb; j += kEpiThreads) {
            const int i = it.q0 + j;
            QueryState st;
            st.cnt = 0;
            st.bound = bound0;
            st.vis_end = i < p.S ? visible_count(p, static_cast<long long>(i) + p.q_offset) : 0;
            st.pad = 0;
            qs[j] = st;
        }
        for (int c = etid; c < p.qpb * p.H; c += kEpiThreads) {
            const int j = c / p.H;
            w_s[c] = it.q0 + j < p.S
                         ? p.w[(static_cast<size_t>(it.b) * p.S + it.q0) * p.H + c]
                         : 0.0f;
        }
        named_bar_sync(kEpiBar, kEpiThreads);

        bool ok = true;
        for (int t = it.tile_begin; t < it.tile_end && ok; ++t) {
            const int s = t * kTileKeys + key_local;
            float kscale = 1.0f;
            if (p.key_fp8 && s < p.T)
                kscale = p.k_scale[static_cast<size_t>(it.b) * p.T + s];
            for (int sub = 0; sub < p.nsub; ++sub) {
                const int slot = acc_use & 1;
                ok = wait_bounded(&bars->acc_full[slot], (acc_use >> 1) & 1, ctl, kRoleEpilogue, id);
                ok = group_all(kEpiBar, kEpiThreads, ok);
                if (!ok) {
                    *ctl.abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr =
                    tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + slot * kSlotCols;
                const float *wsub = w_s + sub * p.N;
                const int jq0 = sub * p.qps;

                auto emit = [&](int jq, float score) {
                    const QueryState st = qs[jq];
                    const uint32_t ord = ord_of_score(score * kscale);
                    const bool pass = s < st.vis_end && ord >= st.bound;
                    const unsigned bal = __ballot_sync(0xffffffffu, pass);
                    if (bal) {
                        int base = 0;
                        if (lane == 0)
                            base = atomicAdd(&qs[jq].cnt, __popc(bal));
                        base = __shfl_sync(0xffffffffu, base, 0);
                        if (pass)
                            cand_cta[static_cast<size_t>(jq) * p.cap + base +
                                     __popc(bal & lanemask_lt())] = make_key(ord, static_cast<uint32_t>(s));
                    }
                };

                float acc = 0.0f;
                for (int c = 0; c < p.N / 32; ++c) {
                    uint32_t v[32];
                    __syncwarp(); // tcgen05.ld is warp-aligned: reconverge after emit()
                    tmem_ld_32x32b_x32(taddr + c * 32, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        reg_fence(v[i]);
                    const float *wc = wsub + c * 32;
                    if (kHeadsGe32) {
                        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            const float4 w4 = *reinterpret_cast<const float4 *>(wc + i);
                            a0 = fmaf(fmaxf(__uint_as_float(v[i + 0]), 0.f), w4.x, a0);
                            a1 = fmaf(fmaxf(__uint_as_float(v[i + 1]), 0.f), w4.y, a1);
                            a2 = fmaf(fmaxf(__uint_as_float(v[i + 2]), 0.f), w4.z, a2);
                            a3 = fmaf(fmaxf(__uint_as_float(v[i + 3]), 0.f), w4.w, a3);
                        }
                        acc += (a0 + a1) + (a2 + a3);
                        if (((c + 1) * 32) % p.H == 0) {
                            emit(jq0 + (c * 32) / p.H, acc);
                            acc = 0.0f;
                        }
                    } else {
                        // H < 32 (a power of two): each 32-column chunk holds 32/H queries
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            acc = fmaf(fmaxf(__uint_as_float(v[i]), 0.f), wc[i], acc);
                            if (((i + 1) & (p.H - 1)) == 0) {
                                emit(jq0 + (c * 32 + i) / p.H, acc);
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
                named_bar_sync(kEpiBar, kEpiThreads);
                // Cut back any list that the next tile could overflow.
                for (int jq = jq0; jq < jq0 + p.qps; ++jq) {
                    const int n = qs[jq].cnt;
                    if (n > p.cap - kTileKeys) {
                        uint32_t bound;
                        const int kept = compact_candidates<kEpiThreads, kEpt>(
                            cand_cta + static_cast<size_t>(jq) * p.cap, n, p.topk, p.slack, sc,
                            kEpiBar, etid, &bound);
                        if (etid == 0) {
                            qs[jq].cnt = kept;
                            qs[jq].bound = max(qs[jq].bound, bound);
                        }
                        named_bar_sync(kEpiBar, kEpiThreads);
                    }
                }
            }
        }
        if (!ok)
            break;

        // ---- final exact top-k per query of the item
        for (int j = 0; j < it.nq; ++j) {
            const int n = qs[j].cnt;
            const uint64_t *buf = cand_cta + static_cast<size_t>(j) * p.cap;
            uint64_t e[kEpt];
#pragma unroll
            for (int i = 0; i < kEpt; ++i) {
                const int x = i * kEpiThreads + etid;
                e[i] = x < n ? buf[x] : 0ull;
            }
            const int kept_max = min(n, p.topk);
            const int P = pow2_at_least(kept_max);
            const int kept =
                select_topk<kEpiThreads, kEpt>(e, n, p.topk, sortbuf, P, sc, kEpiBar, etid);
            const size_t row = static_cast<size_t>(it.b) * p.S + it.q0 + j;
            if (p.nsplit == 1) {
                bitonic_sort_desc<kEpiThreads>(sortbuf, P, kEpiBar, etid);
                for (int slot = etid; slot < p.topk; slot += kEpiThreads) {
                    const size_t o = row * p.topk + slot;
                    if (slot < kept) {
                        const uint64_t key = sortbuf[slot];
                        p.out_idx[o] = key_index(key);
                        p.out_score[o] = key_score(key);
                    } else {
                        p.out_idx[o] = -1;
                        p.out_score[o] = -__int_as_float(0x7f800000);
                    }
                }
            } else {
                uint64_t *dst = p.part + (row * p.nsplit + it.split) * p.topk;
                for (int slot = etid; slot < p.topk; slot += kEpiThreads)
                    dst[slot] = slot < kept ? sortbuf[slot] : 0ull;
            }
            named_bar_sync(kEpiBar, kEpiThreads);
        }
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
            mbar_init(&bars->acc_empty[s], kEpiThreads / 32);
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
    } else {
        run_epilogue<kHeadsGe32>(p, smem, bars, tmem_base, ctl);
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
    __shared__ GroupScratch sc;
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
        group_excl_scan<kMergeThreads>(mine, &sc, 0, tid, &n);
        const int kept_max = min(n, topk);
        const int P = pow2_at_least(kept_max);
        const int kept = select_topk<kMergeThreads, kMergeEpt>(e, n, topk, sortbuf, P, &sc, 0, tid);
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
