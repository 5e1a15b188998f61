// indexer_kernel.cuh -- the fused lightning-indexer scoring + streaming
// candidate filter.
//
// One persistent CTA per SM walks work items (batch b, block of qps queries,
// range of key tiles).  For each 128-key tile the tensor cores compute the
// logits L[s, (t,h)] = k[s,:] . q[t,h,:] for every head of the item's queries
// ("StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", abstract: the lightning indexer scores compressed keys per query),
// with keys as the MMA's M dimension so that each TMEM lane holds one key's
// logits for every (query, head).  The epilogue applies ReLU and the head
// weights, masks keys the query may not see, and streams the surviving
// (score, index) pairs into the query's candidate list in global memory; a
// list that could overflow is cut back in place to the top k plus slack and
// the admission bound rises to the smallest score kept.  When an item's key
// range is done the list holds a superset of the query's top k over that
// range; select_kernel.cuh turns the lists into the exact, sorted top k.  The
// [B,S,H_I,T] score tensor never exists and the extra memory is O(S * k).
//
// Warp roles (384 threads, three warpgroups):
//   warps 0..3  epilogue warpgroup 0: the first half of the item's queries
//   warps 4..7  epilogue warpgroup 1: the second half (idle when qps == 1)
//   warp 8      TMA producer: the query block once per item (with an L2
//               prefetch of the next item's), key tiles into a ring
//   warp 9      TMEM owner and MMA issuer (one thread): per key tile, d/16
//               tcgen05.mma (M = 128 keys, N = qps*H_I) into one of two
//               256-column TMEM accumulators
//   warps 10,11 E4M3 keys only: converters.  The producer lands each FP8 key
//               tile in a staging ring; the converters rewrite it as f16
//               into the MMA's swizzled key ring (exact: every E4M3 value is
//               an f16 normal) and convert the item's query block from bf16
//               to f16 in place (exact for |q| < 65504), so the MMA runs
//               kind::f16 with both operands f16.  The key's fp32 scale
//               multiplies its score after the head reduction (scale > 0).
// The block launches with 168 registers per thread; the producer/MMA
// warpgroup gives most of its share to the two epilogue warpgroups
// (3 x 128 x 168 = 2 x 128 x kEpiRegs + 128 x kCtlRegs).
//
// Epilogue fast path (H_I >= 32, at most 128 TMEM columns per warpgroup): a
// warp reads its 32 TMEM lanes with two 16-lane x 256-bit loads, so every
// thread sees a fixed quarter of the columns of four keys; the head weights of
// that quarter stay in registers for the whole item, the accumulator slot is
// handed back to the MMA as soon as the loads land, and two butterfly shuffles
// leave each thread with one key's complete scores.  Other shapes read one key
// per thread with 32-lane loads and weights from shared memory.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "ptx.cuh"
#include "topk_group.cuh"

namespace csa {

constexpr int kTileKeys = 128;   // MMA M: keys per tile
constexpr int kSlotCols = 256;   // TMEM columns per accumulator slot
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;  // registers per thread the kernel must be built with
constexpr int kEpiRegs = 216;     // after the split: epilogue warpgroups
constexpr int kCtlRegs = 72;      //                  producer / MMA warpgroup
static_assert(2 * 128 * kEpiRegs + 128 * kCtlRegs == kThreads * kLaunchRegs,
              "register split must match the launch budget");
constexpr int kGroupThreads = 128;
constexpr int kBarWg0 = 1, kBarWg1 = 2;  // named barriers of the epilogue warpgroups
constexpr int kEpt = 32;         // candidate keys per thread in a group (cap <= 4096)
constexpr int kMaxStages = 8;
constexpr int kMaxTopk = 2048;
constexpr int kNbCompact = 1024; // buckets of the compaction histogram

enum Role : int { kRoleProducer = 1, kRoleMma = 2, kRoleEpilogue = 3, kRoleSelect = 4, kRoleConvert = 5 };

// Optional per-role cycle counters (built only with -DCSA_PROFILE): where each
// role spends its time, recorded by one thread per role and CTA.
enum ProfSlot : int {
    kPfProdQEmpty, kPfProdKEmpty, kPfMmaQFull, kPfMmaKFull, kPfMmaAccEmpty, kPfMmaTotal,
    kPfEpiAccFull, kPfEpiCompact, kPfEpiTotal, kPfEpiCompactCount, kPfEpiTiles, kPfEpiMath,
    kPfEpiTileBar, kPfSlots
};
#ifdef CSA_PROFILE
constexpr int kProfCtas = 160;
__device__ unsigned long long g_csa_prof[kProfCtas][32];

struct ProfAcc {
    unsigned long long v[kPfSlots];
    __device__ __forceinline__ ProfAcc()
    {
#pragma unroll
        for (int i = 0; i < kPfSlots; ++i)
            v[i] = 0;
    }
    __device__ __forceinline__ void flush(bool rec)
    {
        if (rec && blockIdx.x < kProfCtas) {
#pragma unroll
            for (int i = 0; i < kPfSlots; ++i)
                if (v[i])
                    atomicAdd(&g_csa_prof[blockIdx.x][i], v[i]);
        }
    }
};

struct Prof {
    long long t0;
    __device__ __forceinline__ void start() { t0 = clock64(); }
    __device__ __forceinline__ void add(ProfAcc &a, int slot, bool rec)
    {
        if (rec)
            a.v[slot] += static_cast<unsigned long long>(clock64() - t0);
    }
    __device__ __forceinline__ void count(ProfAcc &a, int slot, bool rec)
    {
        if (rec)
            a.v[slot] += 1;
    }
};
#else
struct ProfAcc {
    __device__ __forceinline__ void flush(bool) {}
};
struct Prof {
    __device__ __forceinline__ void start() {}
    __device__ __forceinline__ void add(ProfAcc &, int, bool) {}
    __device__ __forceinline__ void count(ProfAcc &, int, bool) {}
};
#endif

struct Params {
    int B, S, T, H, d, m, topk, causal, mode, key_fp8;
    long long q_offset;
    int qps;      // queries per item
    int N;        // MMA N = qps * H (<= 256)
    int n_wg;     // epilogue warpgroups in use (1 or 2)
    int qpw;      // queries per epilogue warpgroup = qps / n_wg
    int qb_lo;    // first query block (per batch) of this launch
    int nqb;      // query blocks per batch in this launch
    int nsplit;   // key-range splits per query block
    int n_items;
    int stages;
    int cap;      // candidate list capacity per query and split
    int slack;    // compaction keeps at most topk + slack when it must cut exactly
    int row_bytes;   // bytes of one swizzled operand row: min(128, 2*d)
    int n_chunks;    // d*2 / row_bytes
    // shared memory carve-up (byte offsets from the 1024-aligned base)
    int off_q, off_k, off_w, off_state, off_wg, off_bar, smem_bytes;
    int off_k8;      // E4M3 keys: staging ring of raw key tiles
    int wg_bytes;    // per-warpgroup scratch
    const uint16_t *q; // only for L2 prefetch; loads go through the tensor map
    const float *w;
    const float *k_scale;
    uint64_t *lists; // [list row][nsplit][cap] candidate keys
    int *counts;     // [list row][nsplit] keys in each list
    long long wait_limit;
};

// List row of query j of query block qb (relative to qb_lo) in batch b:
// (b * nqb + qb) * qps + j.
struct Item {
    int b, q0, nq, tile_begin, tile_end, split, lrow;
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
    const int qbr = p.nqb - 1 - r / p.B;
    it.q0 = (p.qb_lo + qbr) * p.qps;
    it.nq = min(p.qps, p.S - it.q0);
    it.lrow = (it.b * p.nqb + qbr) * p.qps;
    const int nvis = visible_count(p, static_cast<long long>(it.q0 + it.nq - 1) + p.q_offset);
    const int nkt = (nvis + kTileKeys - 1) / kTileKeys;
    it.tile_begin = static_cast<int>(static_cast<long long>(it.split) * nkt / p.nsplit);
    it.tile_end = static_cast<int>(static_cast<long long>(it.split + 1) * nkt / p.nsplit);
    return it;
}

struct Barriers {
    uint64_t q_full, q_empty, drain, q_ready;
    uint64_t k_full[kMaxStages], k_empty[kMaxStages];
    uint64_t k8_full[kMaxStages], k8_empty[kMaxStages];  // E4M3 staging ring
    uint64_t acc_full[2], acc_empty[2];
    uint32_t tmem_addr;
    int abort;
};

// Per-query streaming state of the current item.
struct QueryState {
    int cnt;          // candidates in the list
    uint32_t bound;   // admit a key only if ord(score) >= bound
    int vis_end;      // keys s < vis_end are visible to this query
    int pad;
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
    ProfAcc pa;
    Prof pf;
    const uint32_t q_bytes = static_cast<uint32_t>(p.N * p.d * 2);
    const uint32_t k_bytes = static_cast<uint32_t>(kTileKeys * p.d * 2);
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        pf.start();
        if (!wait_bounded(&bars->q_empty, (qload & 1) ^ 1, ctl, kRoleProducer, id))
            goto unwind;
        pf.add(pa, kPfProdQEmpty, true);
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
            const int row = it.b * p.T + t * kTileKeys;
            pf.start();
            if (p.key_fp8) {
                // raw E4M3 tile (128 rows x d bytes) into the staging ring
                if (!wait_bounded(&bars->k8_empty[stage], ((kload / p.stages) & 1) ^ 1, ctl,
                                  kRoleProducer, id))
                    goto unwind;
                pf.add(pa, kPfProdKEmpty, true);
                mbar_arrive_expect_tx(&bars->k8_full[stage], static_cast<uint32_t>(kTileKeys * p.d));
                tma_load_2d(smem + p.off_k8 + stage * kTileKeys * p.d, tmK, &bars->k8_full[stage],
                            0, row);
            } else {
                if (!wait_bounded(&bars->k_empty[stage], ((kload / p.stages) & 1) ^ 1, ctl,
                                  kRoleProducer, id))
                    goto unwind;
                pf.add(pa, kPfProdKEmpty, true);
                mbar_arrive_expect_tx(&bars->k_full[stage], k_bytes);
                uint8_t *dst = smem + p.off_k + stage * kTileKeys * p.d * 2;
                for (int c = 0; c < p.n_chunks; ++c)
                    tma_load_2d(dst + c * kTileKeys * p.row_bytes, tmK, &bars->k_full[stage],
                                c * (p.row_bytes / 2), row);
            }
            ++kload;
        }
    }
unwind:
    // Let every copy already issued land before the CTA can exit.
    for (int s = 0; s < p.stages; ++s) {
        if (kload > s) {
            const int fills = (kload - s + p.stages - 1) / p.stages;
            wait_drain(p.key_fp8 ? &bars->k8_full[s] : &bars->k_full[s], (fills - 1) & 1);
        }
    }
    if (qload > 0)
        wait_drain(&bars->q_full, (qload - 1) & 1);
    pa.flush(true);
}

// ------------------------------------------------------------------ MMA issuer
__device__ void run_mma(const Params &p, uint8_t *smem, Barriers *bars, uint32_t tmem_base,
                        const WaitCtl &ctl)
{
    int kuse = 0, quse = 0, acc_use = 0;
    ProfAcc pa;
    Prof pf, pt;
    pt.start();
    const uint32_t idesc = instr_desc_f16(p.N, p.key_fp8 ? 0 : 1); // f16 x f16 for E4M3 keys
    const int ksteps_per_chunk = p.row_bytes / 32;  // 16 elements (32 B) per MMA K step
    const uint32_t q_base = smem_u32(smem + p.off_q);
    const uint32_t k_base = smem_u32(smem + p.off_k);
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        pf.start();
        if (!wait_bounded(p.key_fp8 ? &bars->q_ready : &bars->q_full, quse & 1, ctl, kRoleMma, id))
            goto unwind;
        pf.add(pa, kPfMmaQFull, true);
        tc_fence_after();
        for (int t = it.tile_begin; t < it.tile_end; ++t) {
            const int stage = kuse % p.stages;
            pf.start();
            if (!wait_bounded(&bars->k_full[stage], (kuse / p.stages) & 1, ctl, kRoleMma, id))
                goto unwind;
            pf.add(pa, kPfMmaKFull, true);
            const int slot = acc_use & 1;
            pf.start();
            if (!wait_bounded(&bars->acc_empty[slot], ((acc_use >> 1) & 1) ^ 1, ctl, kRoleMma, id))
                goto unwind;
            pf.add(pa, kPfMmaAccEmpty, true);
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
    pt.add(pa, kPfMmaTotal, true);
    mma_commit(&bars->drain);
    wait_drain(&bars->drain, 0);
    pa.flush(true);
}

// ------------------------------------------------------------------ E4M3 converters
// Byte offset of 16-byte unit `unit` of row r inside one swizzled operand
// chunk (rows of row_bytes = 128 -> 128-byte swizzle, 64 -> 64-byte swizzle):
// the unit index is XORed with row bits, as the TMA swizzle modes lay it out.
__device__ __forceinline__ uint32_t swizzled_unit(int r, int unit, int row_bytes)
{
    const uint32_t o = static_cast<uint32_t>(r * row_bytes + unit * 16);
    const uint32_t mask = row_bytes == 128 ? (7u << 7) : (3u << 7);
    return o ^ ((o & mask) >> 3);
}

// Four E4M3 values (one 32-bit word) -> four f16 (two words), exact.
__device__ __forceinline__ uint2 e4m3x4_to_f16x4(uint32_t b)
{
    uint2 r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}\n"
        : "=r"(r.x), "=r"(r.y)
        : "r"(b));
    return r;
}

// Two bf16 (one word) -> two f16 (one word), round to nearest.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;"
        : "=r"(r)
        : "f"(__uint_as_float(w & 0xFFFF0000u)), "f"(__uint_as_float(w << 16)));
    return r;
}

constexpr int kConvThreads = 64;
constexpr int kConvUnits = kTileKeys * 128 / 16 / kConvThreads; // 16-value units per thread (d <= 128)

// Two warps (64 threads, `ct` = 0..63).  Per item: the query block, once the
// TMA has landed it, from bf16 to f16 in place.  Per key tile: the staged
// E4M3 tile to f16 in the swizzled key ring; a thread's units (and so its
// source and destination offsets) are the same for every tile.  Each hand-off
// fences the generic-proxy writes for the tensor cores, then one arrive per
// warp.
__device__ void run_converter(const Params &p, uint8_t *smem, Barriers *bars, const WaitCtl &ctl,
                              int ct)
{
    const int lane = ct & 31;
    int kuse = 0, quse = 0;
    const int units_q = p.N * p.d / 8;                 // 16-byte units of the query block
    const int units_per_row = p.d / 16;                // 16 E4M3 values per unit
    const int n_units = kTileKeys * units_per_row / kConvThreads;
    const int elems_per_chunk_row = p.row_bytes / 2;
    // Unit i of this thread is u = 64 i + ct: row 64 i / units_per_row + ct /
    // units_per_row (a multiple of 8 rows apart for d <= 128, so the swizzle
    // term is the same for every i) and the same columns for every i.
    uint32_t dst_base[2];
    {
        const int r0 = ct / units_per_row;
        const int j0 = (ct % units_per_row) * 16;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int j = j0 + 8 * half;
            const int c = j / elems_per_chunk_row;
            const int unit = (j % elems_per_chunk_row) / 8;
            dst_base[half] =
                static_cast<uint32_t>(c * kTileKeys * p.row_bytes) + swizzled_unit(r0, unit, p.row_bytes);
        }
    }
    const uint32_t dst_step = static_cast<uint32_t>(kConvThreads / units_per_row * p.row_bytes);
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        bool ok = wait_bounded(&bars->q_full, quse & 1, ctl, kRoleConvert, id);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok)
            return;
        if (it.tile_end > it.tile_begin) {
            uint4 *qv = reinterpret_cast<uint4 *>(smem + p.off_q);
            for (int u = ct; u < units_q; u += kConvThreads) {
                uint4 x = qv[u];
                x.x = bf16x2_to_f16x2(x.x);
                x.y = bf16x2_to_f16x2(x.y);
                x.z = bf16x2_to_f16x2(x.z);
                x.w = bf16x2_to_f16x2(x.w);
                qv[u] = x;
            }
            fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&bars->q_ready);
        ++quse;
        for (int t = it.tile_begin; t < it.tile_end; ++t) {
            const int stage = kuse % p.stages;
            const uint32_t par = (kuse / p.stages) & 1;
            ok = wait_bounded(&bars->k8_full[stage], par, ctl, kRoleConvert, id);
            ok = ok && wait_bounded(&bars->k_empty[stage], par ^ 1, ctl, kRoleConvert, id);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                return;
            const uint4 *src =
                reinterpret_cast<const uint4 *>(smem + p.off_k8 + stage * kTileKeys * p.d);
            uint8_t *dst = smem + p.off_k + stage * kTileKeys * p.d * 2;
#pragma unroll
            for (int i = 0; i < kConvUnits; ++i) {
                if (i < n_units) {
                    const uint4 x = src[i * kConvThreads + ct];
                    const uint2 a = e4m3x4_to_f16x4(x.x);
                    const uint2 b = e4m3x4_to_f16x4(x.y);
                    const uint2 c = e4m3x4_to_f16x4(x.z);
                    const uint2 d = e4m3x4_to_f16x4(x.w);
                    *reinterpret_cast<uint4 *>(dst + dst_base[0] + i * dst_step) = make_uint4(a.x, a.y, b.x, b.y);
                    *reinterpret_cast<uint4 *>(dst + dst_base[1] + i * dst_step) = make_uint4(c.x, c.y, d.x, d.y);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->k_full[stage]);
                mbar_arrive(&bars->k8_empty[stage]);
            }
            ++kuse;
        }
    }
}

// ------------------------------------------------------------------ group scratch
struct WgScratch {          // one per epilogue warpgroup
    GroupSmall gs;
    uint32_t hist[kNbCompact];
};

// ------------------------------------------------------------------ compaction
// Bucket of the k-th largest key over a 1024-bucket histogram of the group:
// {b*, keys in buckets above b*, keys in b*} with above < need <= above + in.
// Thread tid owns buckets [8 tid, 8 tid + 8); two group barriers.
__device__ __forceinline__ void compact_boundary(const uint32_t *hist, int need, GroupSmall *gs,
                                                 int bar, int tid, int (&out)[3])
{
    constexpr int PER = kNbCompact / kGroupThreads;
    const int lane = tid & 31, wid = tid >> 5;
    uint32_t c[PER];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        c[j] = hist[tid * PER + j];
        sum += c[j];
    }
    uint32_t suf = sum; // inclusive suffix sum over the warp's threads
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t t = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32)
            suf += t;
    }
    if (lane == 0)
        gs->warp_sums[wid] = suf;
    named_bar_sync(bar, kGroupThreads);
    uint32_t higher = 0;
#pragma unroll
    for (int w = 0; w < kGroupThreads / 32; ++w)
        higher += w > wid ? gs->warp_sums[w] : 0u;
    const uint32_t above_thread = suf - sum + higher;
    const uint32_t nd = static_cast<uint32_t>(need);
    if (above_thread < nd && nd <= above_thread + sum) {
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
    named_bar_sync(bar, kGroupThreads);
    out[0] = gs->bcast[0];
    out[1] = gs->bcast[1];
    out[2] = gs->bcast[2];
}

// Cuts a query's list back when it could overflow: keeps every key whose
// bucket is at or above the bucket of the k-th largest key -- a superset of
// the top k -- or, when that bucket is too full, the radix-exact top k plus
// slack.  Buckets split the list's own [min, max] range of score order images
// into 1024 equal integer ranges.  Warp w owns list slots [1024 w, 1024 w +
// 1024) (lane l: slots 1024 w + 64 i + 2 l and the one after) and writes the
// keys it keeps back with coalesced stores.  Updates cnt and raises bound to
// the smallest kept score.  The group's histogram is all zero on entry and on
// return.
__device__ void compact_list(const Params &p, uint64_t *list, QueryState &st, WgScratch *sc,
                             int bar, int tid)
{
    const int n = st.cnt;
    const int lane = tid & 31, wid = tid >> 5;
    uint64_t e[kEpt];
#pragma unroll
    for (int i = 0; i < kEpt / 2; ++i) {
        const int j = wid * (kEpt * 32) + i * 64 + 2 * lane;
        if (j + 1 < n) {
            const ulonglong2 v = *reinterpret_cast<const ulonglong2 *>(list + j);
            e[2 * i] = v.x;
            e[2 * i + 1] = v.y;
        } else {
            e[2 * i] = j < n ? list[j] : 0ull;
            e[2 * i + 1] = 0ull;
        }
    }
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
    for (int i = 0; i < kEpt; ++i) {
        if (e[i] != 0) {
            lo = min(lo, key_ord(e[i]));
            hi = max(hi, key_ord(e[i]));
        }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
        sc->gs.warp_sums[wid] = lo;
        sc->gs.warp_sums[16 + wid] = hi;
    }
    named_bar_sync(bar, kGroupThreads);
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
    for (int w = 0; w < kGroupThreads / 32; ++w) {
        mn = min(mn, sc->gs.warp_sums[w]);
        mx = max(mx, sc->gs.warp_sums[16 + w]);
    }
    const uint32_t span = mx - mn;
    const int shift = span < static_cast<uint32_t>(kNbCompact) ? 0 : 32 - __clz(span) - 10;
    int bk[kEpt]; // each key's bucket, -1 for an empty slot
#pragma unroll
    for (int i = 0; i < kEpt; ++i) {
        bk[i] = e[i] != 0 ? static_cast<int>((key_ord(e[i]) - mn) >> shift) : -1;
        if (bk[i] >= 0)
            atomicAdd(&sc->hist[bk[i]], 1u);
    }
    named_bar_sync(bar, kGroupThreads);
    int bd[3];
    compact_boundary(sc->hist, p.topk, &sc->gs, bar, tid, bd);
    // every thread read its own buckets in compact_boundary: clear them
#pragma unroll
    for (int j = 0; j < kNbCompact / kGroupThreads; ++j)
        sc->hist[tid * (kNbCompact / kGroupThreads) + j] = 0;
    const int bstar = bd[0];
    const int cand_kept = bd[1] + bd[2];
    uint32_t newmin = 0xFFFFFFFFu;
    int kept = 0;
    if (cand_kept <= p.cap - 2 * kTileKeys) {
        uint32_t keep = 0;
        int mine = 0;
        uint32_t kmin = 0xFFFFFFFFu;
#pragma unroll
        for (int i = 0; i < kEpt; ++i) {
            const bool k = bk[i] >= bstar;
            keep |= k ? (1u << i) : 0u;
            mine += k ? 1 : 0;
            kmin = k ? min(kmin, key_ord(e[i])) : kmin;
        }
        const int wcount = __reduce_add_sync(0xffffffffu, mine);
        kmin = __reduce_min_sync(0xffffffffu, kmin);
        if (lane == 0) {
            sc->gs.warp_sums[wid] = static_cast<uint32_t>(wcount);
            sc->gs.warp_sums[16 + wid] = kmin;
        }
        named_bar_sync(bar, kGroupThreads);
        int pos = 0;
#pragma unroll
        for (int w = 0; w < kGroupThreads / 32; ++w) {
            const int c = static_cast<int>(sc->gs.warp_sums[w]);
            pos += w < wid ? c : 0;
            kept += c;
            newmin = min(newmin, sc->gs.warp_sums[16 + w]);
        }
        const unsigned lt = lanemask_lt();
#pragma unroll
        for (int i = 0; i < kEpt; ++i) {
            const bool k = (keep >> i) & 1u;
            const unsigned m = __ballot_sync(0xffffffffu, k);
            if (k)
                list[pos + __popc(m & lt)] = e[i];
            pos += __popc(m);
        }
    } else {
        int k2;
        const uint64_t L = radix_bound<kGroupThreads, kEpt>(e, p.topk, p.slack, sc->hist, &sc->gs,
                                                            bar, tid, &k2);
        kept = write_kept<kGroupThreads, kEpt>(e, L, list, &sc->gs, bar, tid, &newmin);
        for (int i = tid; i < kNbCompact; i += kGroupThreads)
            sc->hist[i] = 0;
    }
    named_bar_sync(bar, kGroupThreads); // list writes and scratch reads done
    if (tid == 0) {
        st.cnt = kept;
        st.bound = max(st.bound, newmin);
    }
    named_bar_sync(bar, kGroupThreads);
}

// ------------------------------------------------------------------ emission
// Appends this warp's surviving (score, key) pairs of Q queries to their
// candidate lists: one ballot per query, the lane-0 atomics back to back.
// Query j's list starts at lbase + j * lstride.
template <int Q>
__device__ __forceinline__ void emit_batch(const float *sc, int j0, int s, float kscale,
                                           QueryState *qs, uint64_t *lbase, size_t lstride,
                                           int lane)
{
    uint32_t ord[Q];
    unsigned bal[Q];
    int base[Q];
#pragma unroll
    for (int q = 0; q < Q; ++q) {
        const QueryState st = qs[j0 + q];
        ord[q] = ord_of_score(sc[q] * kscale);
        bal[q] = __ballot_sync(0xffffffffu, s < st.vis_end && ord[q] >= st.bound);
    }
    if (lane == 0) {
#pragma unroll
        for (int q = 0; q < Q; ++q)
            base[q] = bal[q] ? atomicAdd(&qs[j0 + q].cnt, __popc(bal[q])) : 0;
    }
#pragma unroll
    for (int q = 0; q < Q; ++q) {
        base[q] = __shfl_sync(0xffffffffu, base[q], 0);
        if (bal[q] & (1u << lane))
            lbase[static_cast<size_t>(j0 + q) * lstride + base[q] +
                  __popc(bal[q] & lanemask_lt())] = make_key(ord[q], static_cast<uint32_t>(s));
    }
}

// ------------------------------------------------------------------ fast tile math
template <int FC> struct Ld16x256;
template <> struct Ld16x256<64> {
    static __device__ __forceinline__ void ld(uint32_t a, uint32_t (&v)[32]) { tmem_ld_16x256b_x8(a, v); }
};
template <> struct Ld16x256<128> {
    static __device__ __forceinline__ void ld(uint32_t a, uint32_t (&v)[64]) { tmem_ld_16x256b_x16(a, v); }
};

// This thread's head weights for a warpgroup that reads FC columns holding FQ
// queries: weight 2i+e belongs to column 8i + 2(lane%4) + e.
template <int FC, int FQ>
__device__ __forceinline__ void fast_load_w(const Params &p, const Item &it, int j0, int lane,
                                            float2 (&wr)[FC / 8])
{
    constexpr int RPQ = FC / 8 / FQ;  // 8-column repetitions per query
#pragma unroll
    for (int i = 0; i < FC / 8; ++i) {
        const int j = j0 + i / RPQ;
        const int h = 8 * (i % RPQ) + 2 * (lane & 3);
        float a = 0.0f, b = 0.0f;
        if (j < it.nq) {
            const float *src = p.w + (static_cast<size_t>(it.b) * p.S + it.q0 + j) * p.H + h;
            a = src[0];
            b = src[1];
        }
        wr[i] = make_float2(a, b);
    }
}

__device__ __forceinline__ float2 relu2(uint32_t a, uint32_t b)
{
    return make_float2(fmaxf(__uint_as_float(a), 0.0f), fmaxf(__uint_as_float(b), 0.0f));
}

// Scores of FQ queries for one key per thread.  The warp's two 16-lane loads
// cover its 32 keys; thread t holds columns 8i + 2(t%4) + {0,1} of keys
// t/4 + {0, 8, 16, 24}.  After the loads land the accumulator slot is released
// (one arrive per warp).  Each thread then forms per-key partial sums over its
// columns (column pairs with one packed FMA); the quad (threads sharing t/4)
// exchanges halves twice so that thread t ends with the complete scores of
// key row 16*((t>>1)&1) + 8*(t&1) + t/4 of the warp's 32.
template <int FC, int FQ>
__device__ __forceinline__ void fast_tile_scores(uint32_t taddr, const float2 (&wr)[FC / 8],
                                                 uint64_t *acc_empty, int lane, float (&F)[FQ])
{
    constexpr int NV = FC / 2;
    constexpr int REPS = FC / 8;
    constexpr int RPQ = REPS / FQ;
    uint32_t va[NV], vb[NV];
    __syncwarp();
    Ld16x256<FC>::ld(taddr, va);
    Ld16x256<FC>::ld(taddr + (16u << 16), vb);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        reg_fence(va[i]);
        reg_fence(vb[i]);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
        mbar_arrive(acc_empty);
    float2 P[4][FQ];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int j = 0; j < FQ; ++j)
            P[k][j] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < REPS; ++i) {
        const int j = i / RPQ;
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
            P[sub][j] = __ffma2_rn(relu2(va[4 * i + 2 * sub], va[4 * i + 2 * sub + 1]), wr[i],
                                   P[sub][j]);
            P[2 + sub][j] = __ffma2_rn(relu2(vb[4 * i + 2 * sub], vb[4 * i + 2 * sub + 1]), wr[i],
                                       P[2 + sub][j]);
        }
    }
    const bool b1 = (lane >> 1) & 1;
    const bool b0 = lane & 1;
#pragma unroll
    for (int j = 0; j < FQ; ++j) {
        float R[2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const float lo = P[m][j].x + P[m][j].y;          // key m (first 16 lanes)
            const float hi = P[2 + m][j].x + P[2 + m][j].y;  // key 2+m (last 16 lanes)
            const float send = b1 ? lo : hi;
            const float keep = b1 ? hi : lo;
            R[m] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
        }
        const float send = b0 ? R[0] : R[1];
        const float keep = b0 ? R[1] : R[0];
        F[j] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
}

// Appends this warp's surviving keys of FQ queries (one key per thread, the
// queries' admission bounds and visibility ends cached in registers).
template <int FQ>
__device__ __forceinline__ void fast_emit(const float (&F)[FQ], const uint32_t (&bnd)[FQ],
                                          const int (&vend)[FQ], int j0, int s, float kscale,
                                          QueryState *qs, uint64_t *lbase, size_t lstride,
                                          int lane)
{
    uint32_t ord[FQ];
    unsigned bal[FQ];
    int base[FQ];
#pragma unroll
    for (int q = 0; q < FQ; ++q) {
        ord[q] = ord_of_score(F[q] * kscale);
        bal[q] = __ballot_sync(0xffffffffu, s < vend[q] && ord[q] >= bnd[q]);
    }
    if (lane == 0) {
#pragma unroll
        for (int q = 0; q < FQ; ++q)
            base[q] = bal[q] ? atomicAdd(&qs[j0 + q].cnt, __popc(bal[q])) : 0;
    }
#pragma unroll
    for (int q = 0; q < FQ; ++q) {
        if (bal[q]) {
            base[q] = __shfl_sync(0xffffffffu, base[q], 0);
            if (bal[q] & (1u << lane))
                lbase[static_cast<size_t>(j0 + q) * lstride + base[q] +
                      __popc(bal[q] & lanemask_lt())] = make_key(ord[q], static_cast<uint32_t>(s));
        }
    }
}

// ------------------------------------------------------------------ generic tile math
// One 32-column TMEM chunk: sum over the chunk's heads of w * ReLU(logit),
// four independent accumulators.
__device__ __forceinline__ float chunk_dot(const uint32_t (&v)[32], const float *wc)
{
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        const float4 w4 = *reinterpret_cast<const float4 *>(wc + i);
        a0 = fmaf(fmaxf(__uint_as_float(v[i + 0]), 0.0f), w4.x, a0);
        a1 = fmaf(fmaxf(__uint_as_float(v[i + 1]), 0.0f), w4.y, a1);
        a2 = fmaf(fmaxf(__uint_as_float(v[i + 2]), 0.0f), w4.z, a2);
        a3 = fmaf(fmaxf(__uint_as_float(v[i + 3]), 0.0f), w4.w, a3);
    }
    return (a0 + a1) + (a2 + a3);
}

__device__ __forceinline__ void fence_regs(uint32_t (&v)[32])
{
#pragma unroll
    for (int i = 0; i < 32; ++i)
        reg_fence(v[i]);
}

// ------------------------------------------------------------------ epilogue
// FC > 0: fast path for FC columns and FQ queries per warpgroup.  FC == 0:
// generic path (kHeadsGe32 tells whether a query spans whole 32-column chunks).
template <int FC, int FQ, bool kHeadsGe32>
__device__ void run_epilogue(const Params &p, uint8_t *smem, Barriers *bars, uint32_t tmem_base,
                             const WaitCtl &ctl, int wg)
{
    const int tid = threadIdx.x & (kGroupThreads - 1); // 0..127 within the warpgroup
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int bar = wg == 0 ? kBarWg0 : kBarWg1;
    const int quarter = warp & 3;             // TMEM lanes this warp may read
    float *w_s = reinterpret_cast<float *>(smem + p.off_w);
    QueryState *qs = reinterpret_cast<QueryState *>(smem + p.off_state);
    WgScratch *sc = reinterpret_cast<WgScratch *>(smem + p.off_wg + wg * p.wg_bytes);
    const uint32_t bound0 = p.mode == 1 ? 0x80000001u : 0u; // gate: score > 0
    const int j0 = wg * p.qpw;                 // first query slot this group owns
    const int col0 = j0 * p.H;                 // first TMEM column it reads
    const int ncols = p.qpw * p.H;             // TMEM columns it reads
    const int nchunk = ncols / 32;             // in 32-column chunks (generic path)
    const int cpq_shift = p.H >= 32 ? __ffs(p.H / 32) - 1 : 0;
    const int h_shift = __ffs(p.H) - 1;
    const size_t lstride = static_cast<size_t>(p.nsplit) * p.cap;
    // the key row (of the warp's 32) whose scores this thread ends up with
    const int key_local =
        FC > 0 ? quarter * 32 + 16 * ((lane >> 1) & 1) + 8 * (lane & 1) + (lane >> 2)
               : quarter * 32 + lane;
    int acc_use = 0;
    ProfAcc pa;
    Prof pf, pt;
    const bool rec = wg == 0 && tid == 0;
    pt.start();

    // Generic path: the group's weights go through shared memory, loaded into
    // registers one item ahead.
    constexpr int kWRegs = FC > 0 ? 1 : kSlotCols / kGroupThreads;
    float wnext[kWRegs];
    if (FC == 0) {
        const Item it0 = decode_item(p, blockIdx.x);
        const size_t row = static_cast<size_t>(it0.b) * p.S + it0.q0;
        for (int r = 0; r < kWRegs; ++r) {
            const int c = tid + r * kGroupThreads;
            wnext[r] = (blockIdx.x < p.n_items && c < ncols && j0 + c / p.H < it0.nq)
                           ? p.w[(row + j0) * p.H + c]
                           : 0.0f;
        }
    }
    float2 wr[FC > 0 ? FC / 8 : 1];
    constexpr int CQ = FC > 0 ? FQ : 1;
    uint32_t bnd[CQ];   // fast path: this group's admission bounds and
    int vend[CQ];       // visibility ends, cached from qs

    for (int i = tid; i < kNbCompact; i += kGroupThreads)
        sc->hist[i] = 0;
    named_bar_sync(bar, kGroupThreads);

    bool ok = true;
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        uint64_t *lbase = p.lists + (static_cast<size_t>(it.lrow) * p.nsplit + it.split) * p.cap;
        for (int j = j0 + tid; j < j0 + p.qpw; j += kGroupThreads) {
            const int i = it.q0 + j;
            QueryState st;
            st.cnt = 0;
            st.bound = bound0;
            st.vis_end = i < p.S ? visible_count(p, static_cast<long long>(i) + p.q_offset) : 0;
            st.pad = 0;
            qs[j] = st;
        }
        if constexpr (FC > 0) {
            fast_load_w<FC, FQ>(p, it, j0, lane, wr);
        } else {
            for (int r = 0; r < kWRegs; ++r) {
                const int c = tid + r * kGroupThreads;
                if (c < ncols)
                    w_s[col0 + c] = wnext[r];
            }
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
        if constexpr (FC > 0) {
#pragma unroll
            for (int q = 0; q < CQ; ++q) {
                bnd[q] = qs[j0 + q].bound;
                vend[q] = qs[j0 + q].vis_end;
            }
        }

        for (int t = it.tile_begin; t < it.tile_end; ++t) {
            const int s = t * kTileKeys + key_local;
            float kscale = 1.0f;
            if (p.key_fp8 && s < p.T)
                kscale = p.k_scale[static_cast<size_t>(it.b) * p.T + s];
            const int slot = acc_use & 1;
            pf.start();
            ok = wait_bounded(&bars->acc_full[slot], (acc_use >> 1) & 1, ctl, kRoleEpilogue, id);
            // the TMEM loads below are warp-collective: agree on the outcome first
            ok = __all_sync(0xffffffffu, ok);
            pf.add(pa, kPfEpiAccFull, rec);
            pf.count(pa, kPfEpiTiles, rec);
            if (ok) {
                tc_fence_after();
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                       slot * kSlotCols + col0;
                pf.start();
                if constexpr (FC > 0) {
                    float F[FQ];
                    fast_tile_scores<FC, FQ>(taddr, wr, &bars->acc_empty[slot], lane, F);
                    fast_emit<FQ>(F, bnd, vend, j0, s, kscale, qs, lbase, lstride, lane);
                } else {
                    // One chunk at a time, each query emitted as it completes.
                    auto emit = [&](int jq, float score) {
                        QueryState &st = qs[jq];
                        const uint32_t ord = ord_of_score(score * kscale);
                        const bool pass = s < st.vis_end && ord >= st.bound;
                        const unsigned bal = __ballot_sync(0xffffffffu, pass);
                        if (bal) {
                            int base = 0;
                            if (lane == 0)
                                base = atomicAdd(&st.cnt, __popc(bal));
                            base = __shfl_sync(0xffffffffu, base, 0);
                            if (pass)
                                lbase[static_cast<size_t>(jq) * lstride + base +
                                      __popc(bal & lanemask_lt())] =
                                    make_key(ord, static_cast<uint32_t>(s));
                        }
                    };
                    const float *wsub = w_s + col0;
                    float acc = 0.0f;
                    uint32_t v[32];
                    for (int c = 0; c < nchunk; ++c) {
                        __syncwarp();
                        tmem_ld_32x32b_x32(taddr + c * 32, v);
                        tmem_ld_wait();
                        fence_regs(v);
                        const float *wc = wsub + c * 32;
                        if (kHeadsGe32) {
                            acc += chunk_dot(v, wc);
                            if (((c + 1) & ((1 << cpq_shift) - 1)) == 0) {
                                emit(j0 + (c >> cpq_shift), acc);
                                acc = 0.0f;
                            }
                        } else {
                            // H < 32 (a power of two): each 32-column chunk holds 32/H queries
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                acc = fmaf(fmaxf(__uint_as_float(v[i]), 0.0f), wc[i], acc);
                                if (((i + 1) & (p.H - 1)) == 0) {
                                    emit(j0 + ((c * 32 + i) >> h_shift), acc);
                                    acc = 0.0f;
                                }
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bars->acc_empty[slot]);
                }
                pf.add(pa, kPfEpiMath, rec);
            }
            ++acc_use;
            pf.start();
            ok = group_all(bar, kGroupThreads, ok);
            pf.add(pa, kPfEpiTileBar, rec);
            if (!ok)
                break;
            // Cut back any list that the next tile could overflow.
            for (int jq = j0; jq < j0 + p.qpw; ++jq) {
                if (qs[jq].cnt > p.cap - kTileKeys) {
                    pf.start();
                    compact_list(p, lbase + static_cast<size_t>(jq) * lstride, qs[jq], sc, bar, tid);
                    pf.add(pa, kPfEpiCompact, rec);
                    pf.count(pa, kPfEpiCompactCount, rec);
                    if constexpr (FC > 0) {
#pragma unroll
                        for (int q = 0; q < CQ; ++q)
                            bnd[q] = qs[j0 + q].bound;
                    }
                }
            }
        }
        if (!ok) {
            *ctl.abort = 1;
            break;
        }
        // Publish the list lengths (rows past the end of the batch get 0).
        for (int j = j0 + tid; j < j0 + p.qpw; j += kGroupThreads)
            p.counts[static_cast<size_t>(it.lrow + j) * p.nsplit + it.split] =
                j < it.nq ? qs[j].cnt : 0;
        named_bar_sync(bar, kGroupThreads);
    }
    pt.add(pa, kPfEpiTotal, rec);
    pa.flush(rec);
}

// ------------------------------------------------------------------ kernel
template <int FC, int FQ, bool kHeadsGe32>
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
        mbar_init(&bars->q_ready, 2);
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&bars->k_full[s], p.key_fp8 ? 2 : 1); // converters, or the TMA's tx
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->k8_full[s], 1);
            mbar_init(&bars->k8_empty[s], 2);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->acc_full[s], 1);
            mbar_init(&bars->acc_empty[s], epi_warps);
        }
        bars->abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
    }
    if (warp == 9) {
        tmem_alloc(&bars->tmem_addr, 2 * kSlotCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bars->tmem_addr;
    WaitCtl ctl{&bars->abort, p.wait_limit};

    if (warp < 8) {
        regs_inc<kEpiRegs>();
        const int wg = warp >> 2;
        if (wg < p.n_wg)
            run_epilogue<FC, FQ, kHeadsGe32>(p, smem, bars, tmem_base, ctl, wg);
    } else {
        regs_dec<kCtlRegs>();
        if (warp == 8 && lane == 0)
            run_producer(p, &tmQ, &tmK, smem, bars, ctl);
        else if (warp == 9 && lane == 0)
            run_mma(p, smem, bars, tmem_base, ctl);
        else if (warp >= 10 && p.key_fp8)
            run_converter(p, smem, bars, ctl, threadIdx.x - 320);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) {
        __syncwarp();
        tmem_dealloc(tmem_base, 2 * kSlotCols);
    }
}

} // namespace csa
