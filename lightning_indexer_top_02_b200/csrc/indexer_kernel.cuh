// indexer_kernel.cuh -- the fused lightning-indexer scoring + candidate
// selection kernel.
//
// One persistent CTA per SM walks work items (batch b, block of qps queries,
// range of key tiles).  For each 128-key tile the tensor cores compute the
// logits L[s, (t,h)] = k[s,:] . q[t,h,:] for every head of the item's queries
// ("StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", abstract: the lightning indexer scores compressed keys per query),
// with keys as the MMA's M dimension so that each TMEM lane holds one key's
// logits for every (query, head).  The epilogue applies ReLU and the head
// weights and writes one fp32 score per (query, key) into the CTA's score
// buffer for the item (two halves, alternating between items).  A selector
// warpgroup then cuts each query's scores of a finished item down to a
// candidate list of at most `cap` keys that holds the query's top k over the
// item's key range (exactly the top k when a cut is needed), while the
// epilogue already fills the other half.  select_kernel.cuh turns the lists
// into the exact, sorted top k.  No score tensor over all queries exists: the
// buffers are per CTA (grid x 2 x qps x keys per item) and the lists O(S*k).
//
// Warp roles (512 threads, four warpgroups):
//   warps 0..3   epilogue warpgroup 0: the first half of the item's queries
//   warps 4..7   epilogue warpgroup 1: the second half (with one query per
//                item both warpgroups read every column of alternate tile groups)
//   warp 8       TMA producer: the query block once per item (with an L2
//                prefetch of the next item's), key tiles into a ring
//   warp 9       TMEM owner and MMA issuer (one thread): per key tile, d/16
//                tcgen05.mma kind::f16 (M = 128 keys, N = qps*H_I) into one
//                of two 256-column TMEM accumulators (up to four tiles side by
//                side when N <= 128); with E4M3 keys, 2*d/32
//                kind::f8f6f4 MMAs (the key tile as stored, times the two
//                E4M3 pieces of the query block, summed in one accumulator)
//   warps 10,11  E4M3 keys only: query splitter.  Each item's bf16 query rows
//                become sigma * (hi8 + lo8) (run_qsplit); sigma folds into the
//                head weights and the key's fp32 scale multiplies its score
//                after the head reduction (both scales > 0).
//   warps 12..15 selector
// The block launches with 128 registers per thread; the two control
// warpgroups give most of their share to the epilogue warpgroups
// (4 x 128 x 128 = 2 x 128 x kEpiRegs + 128 x kCtlRegs + 128 x kSelRegs).
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
constexpr int kThreads = 512;
constexpr int kLaunchRegs = 128;  // registers per thread the kernel must be built with
constexpr int kEpiRegs = 160;     // after the split: epilogue warpgroups
constexpr int kCtlRegs = 96;      //                  producer / MMA / splitter
constexpr int kSelRegs = 96;      //                  selector
static_assert(2 * 128 * kEpiRegs + 128 * kCtlRegs + 128 * kSelRegs == kThreads * kLaunchRegs,
              "register split must match the launch budget");
constexpr int kGroupThreads = 128;
constexpr int kBarWg0 = 1, kBarWg1 = 2, kBarSelect = 3;  // named barriers
constexpr int kMaxStages = 12;
constexpr int kMaxTpg = 4;        // key tiles sharing one accumulator slot (small N)
constexpr int kMaxTopk = 2048;
constexpr int kNbSelect = 2048;  // buckets of the selector's histogram
constexpr int kMaxItemKeys = 65536; // keys of one work item (longer ranges are split)

enum Role : int { kRoleProducer = 1, kRoleMma = 2, kRoleEpilogue = 3, kRoleSelect = 4, kRoleSplit = 5 };

// Optional per-role cycle counters (built only with -DCSA_PROFILE): where each
// role spends its time, recorded by one thread per role and CTA.
enum ProfSlot : int {
    kPfProdQEmpty, kPfProdKEmpty, kPfMmaQFull, kPfMmaKFull, kPfMmaAccEmpty, kPfMmaTotal,
    kPfEpiAccFull, kPfEpiBufEmpty, kPfEpiTotal, kPfEpiTiles, kPfEpiMath, kPfSelBufFull,
    kPfSelBusy, kPfSelTotal, kPfSelCut, kPfSplitWait, kPfSplitWork, kPfSplitTotal, kPfMmaIssue,
    kPfMmaCommit, kPfSlots
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
    int q_pieces;   // E4M3 keys: query pieces per (query, head) row (2: exact split, 1: one E4M3 rounding)
    long long q_offset;
    int qps;      // queries per item
    int N;        // MMA N = qps * H (<= 256)
    int n_wg;     // epilogue warpgroups in use (1 or 2)
    int qpw;      // queries per epilogue warpgroup = qps / n_wg (or qps when tile_split)
    int tile_split; // one query per item: both warpgroups take every column, alternate tiles
    int tpg;        // key tiles per accumulator slot (slot columns / N, at most kMaxTpg)
    int qb_lo;    // first query block (per batch) of this launch
    int nqb;      // query blocks per batch in this launch
    int nsplit;   // key-range splits per query block
    int n_items;
    int stages;   // key tiles in the MMA's ring (bf16, or E4M3 as stored)
    int cap;      // candidate list capacity per query and split
    int nmax;     // score-buffer keys per query (the longest item's key range)
    int row_bytes;   // bytes of one swizzled bf16 operand row: min(128, 2*d)
    int n_chunks;    // d*2 / row_bytes
    // shared memory carve-up (byte offsets from the 1024-aligned base)
    int off_q, off_k, off_w, off_sel, off_bar, smem_bytes;
    int off_e;       // E4M3 keys: the query block split into two E4M3 pieces
    int off_sig;     // E4M3 keys: per-row query scales, two item halves
    const uint16_t *q; // only for L2 prefetch; loads go through the tensor map
    const float *w;
    const float *k_scale;
    uint64_t *lists; // [list row][nsplit][cap] candidate keys
    int *counts;     // [list row][nsplit] keys in each list
    float *scores;   // [gridDim.x][2][qps][nmax] the item's scores
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

// Items run heaviest first within a (batch, split): the last query blocks of
// a causal batch see the most keys.  Query blocks vary fastest, so the CTAs
// running at one time share a few sequences' key ranges and their key tiles
// are read from HBM about once and then from L2.
__device__ __forceinline__ Item decode_item(const Params &p, int id)
{
    Item it;
    const int qbr = p.nqb - 1 - id % p.nqb;
    const int r = id / p.nqb;
    it.split = r % p.nsplit;
    it.b = r / p.nsplit;
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
    uint64_t e_empty;                                     // E4M3: MMAs done with the pieces
    uint64_t sig_full[2], sig_empty[2];                   // E4M3: row scales per item half
    uint64_t k_full[kMaxStages], k_empty[kMaxStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t buf_full[2], buf_empty[2];                   // score-buffer halves
    uint32_t tmem_addr;
    int abort;
};


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
    int stage = 0, kphase = 0;   // ring position of the next key tile
    ProfAcc pa;
    Prof pf;
    const uint32_t q_bytes = static_cast<uint32_t>(p.N * p.d * 2);
    const int k_elem = p.key_fp8 ? 1 : 2;
    const uint32_t k_bytes = static_cast<uint32_t>(kTileKeys * p.d * k_elem);
    // One key tile into the ring (waits for its slot).
    auto load_tile = [&](const Item &it, int t, int id) -> bool {
        const int row = it.b * p.T + t * kTileKeys;
        pf.start();
        if (!wait_bounded(&bars->k_empty[stage], kphase ^ 1, ctl, kRoleProducer, id))
            return false;
        pf.add(pa, kPfProdKEmpty, true);
        if (!CSA_CHECK_INDEX(kChkKeyStage, stage, p.stages)) {
            mbar_arrive(&bars->k_full[stage]);     // debug build: skip the copy, never hang
            return true;
        }
        mbar_arrive_expect_tx(&bars->k_full[stage], k_bytes);
        uint8_t *dst = smem + p.off_k + stage * k_bytes;
        if (p.key_fp8) {
            // E4M3 tile as stored: 128 rows of d bytes, swizzled at width d
            tma_load_2d(dst, tmK, &bars->k_full[stage], 0, row);
        } else {
            for (int c = 0; c < p.n_chunks; ++c)
                tma_load_2d(dst + c * kTileKeys * p.row_bytes, tmK, &bars->k_full[stage],
                            c * (p.row_bytes / 2), row);
        }
        ++kload;
        if (++stage == p.stages) {
            stage = 0;
            kphase ^= 1;
        }
        return true;
    };
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        // The item's first key tiles go into the ring as slots free up, before
        // the query block, which waits for the previous item's MMAs: at the
        // item boundary only the query block's latency is left exposed.
        const int pre = min(it.tile_end - it.tile_begin, p.stages);
        for (int t = it.tile_begin; t < it.tile_begin + pre; ++t)
            if (!load_tile(it, t, id))
                goto unwind;
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
        for (int t = it.tile_begin + pre; t < it.tile_end; ++t)
            if (!load_tile(it, t, id))
                goto unwind;
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
    pa.flush(true);
}

// ------------------------------------------------------------------ MMA issuer
// MS selects the issue loop: 1 = bf16 keys with d = 128, 2 = E4M3 keys with
// d = 128 (both fully unrolled with constant operand offsets, since this one
// thread's instruction latency between tiles idles the tensor pipe), 0 = any
// other head dimension.
template <int MS>
__device__ void run_mma(const Params &p, uint8_t *smem, Barriers *bars, uint32_t tmem_base,
                        const WaitCtl &ctl)
{
    int quse = 0, acc_use = 0;
    // Ring position of the next key tile, kept incrementally: this thread's
    // instruction latency between two tiles' MMAs idles the tensor pipe.
    int stage = 0, kphase = 0;
    ProfAcc pa;
    Prof pf, pt;
    pt.start();
    // bf16 x bf16 (kind::f16), or E4M3 keys x E4M3 query pieces (kind::f8f6f4)
    const uint32_t idesc = instr_desc_f16(p.N, p.key_fp8 ? 0 : 1);
    const int ksteps_per_chunk = p.row_bytes / 32;  // 16 elements (32 B) per MMA K step
    const uint32_t q_base = smem_u32(smem + p.off_q);
    const uint32_t e_base = smem_u32(smem + p.off_e);
    const uint32_t k_base = smem_u32(smem + p.off_k);
    const int k_tile_bytes = kTileKeys * p.d * (p.key_fp8 ? 1 : 2);
    // Descriptors count 16-byte units: byte offsets inside an operand add >> 4.
    const uint64_t a_desc0 = smem_desc_kmajor(k_base, 128);
    const uint32_t a_stage = static_cast<uint32_t>(k_tile_bytes >> 4);
    const uint64_t b_desc0 = smem_desc_kmajor(MS >= 2 ? e_base : q_base, 128);
    const uint32_t b_chunk = static_cast<uint32_t>((p.N * 128) >> 4);  // bf16: next 64 elements; E4M3: lo8 block
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        pf.start();
        if (!wait_bounded(p.key_fp8 ? &bars->q_ready : &bars->q_full, quse & 1, ctl, kRoleMma, id))
            goto unwind;
        pf.add(pa, kPfMmaQFull, true);
        tc_fence_after();
        // Groups of up to tpg key tiles fill one accumulator slot side by side
        // (N columns each), so that small N still hands the epilogue a full slot.
        for (int t = it.tile_begin; t < it.tile_end; ++t) {
            const int g = (t - it.tile_begin) & (p.tpg - 1);     // place in the group
            const bool last = g == p.tpg - 1 || t + 1 == it.tile_end;
            const int slot = acc_use & 1;
            if (g == 0) {
                pf.start();
                if (!wait_bounded(&bars->acc_empty[slot], ((acc_use >> 1) & 1) ^ 1, ctl, kRoleMma,
                                  id))
                    goto unwind;
                pf.add(pa, kPfMmaAccEmpty, true);
            }
            pf.start();
            if (!wait_bounded(&bars->k_full[stage], kphase, ctl, kRoleMma, id))
                goto unwind;
            pf.add(pa, kPfMmaKFull, true);
            tc_fence_after();
            const uint32_t a_tile = k_base + stage * k_tile_bytes;
            const uint32_t d_tmem = tmem_base + slot * kSlotCols + g * p.N;
            pf.start();
            if (!CSA_CHECK_INDEX(kChkTmemMma, slot * kSlotCols + (g + 1) * p.N - 1, 2 * kSlotCols)) {
                // debug build: a tile that would write past the allocation is skipped
            } else if constexpr (MS == 1) {
                const uint64_t a = a_desc0 + stage * a_stage;
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_f16_ss(d_tmem, a + (c * ((kTileKeys * 128) >> 4) + 2 * ks),
                                   b_desc0 + (c * b_chunk + 2 * ks), idesc, (c | ks) != 0);
            } else if constexpr (MS == 2) {
                const uint64_t a = a_desc0 + stage * a_stage;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    mma_f8_ss(d_tmem, a + 2 * ks, b_desc0 + 2 * ks, idesc, ks != 0);
                    mma_f8_ss(d_tmem, a + 2 * ks, b_desc0 + (b_chunk + 2 * ks), idesc, 1);
                }
            } else if constexpr (MS == 3) {
                // one query piece: the key tile meets hi8 only
                const uint64_t a = a_desc0 + stage * a_stage;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_f8_ss(d_tmem, a + 2 * ks, b_desc0 + 2 * ks, idesc, ks != 0);
            } else if (p.key_fp8) {
                // 32 E4M3 per K step; the keys meet every query piece, which
                // sum in the one accumulator
                for (int ks = 0; ks < p.d / 32; ++ks) {
                    const uint64_t adesc = smem_desc_kmajor(a_tile + ks * 32, p.d);
                    mma_f8_ss(d_tmem, adesc, smem_desc_kmajor(e_base + ks * 32, p.d), idesc,
                              ks != 0);
                    if (p.q_pieces == 2)
                        mma_f8_ss(d_tmem, adesc,
                                  smem_desc_kmajor(e_base + p.N * p.d + ks * 32, p.d), idesc, 1);
                }
            } else {
                for (int c = 0; c < p.n_chunks; ++c) {
                    for (int ks = 0; ks < ksteps_per_chunk; ++ks) {
                        const uint64_t adesc = smem_desc_kmajor(
                            a_tile + c * kTileKeys * p.row_bytes + ks * 32, p.row_bytes);
                        const uint64_t bdesc = smem_desc_kmajor(
                            q_base + c * p.N * p.row_bytes + ks * 32, p.row_bytes);
                        mma_f16_ss(d_tmem, adesc, bdesc, idesc, (c | ks) != 0);
                    }
                }
            }
            pf.add(pa, kPfMmaIssue, true);
            pf.start();
            if (last) {
                mma_commit(&bars->acc_full[slot]);
                ++acc_use;
            }
            mma_commit(&bars->k_empty[stage]);
            pf.add(pa, kPfMmaCommit, true);
            if (++stage == p.stages) {
                stage = 0;
                kphase ^= 1;
            }
        }
        // the query operand's buffer is free once this item's MMAs are done
        uint64_t *done = p.key_fp8 ? &bars->e_empty : &bars->q_empty;
        if (it.tile_end > it.tile_begin)
            mma_commit(done);
        else
            mbar_arrive(done);
        ++quse;
    }
unwind:
    pt.add(pa, kPfMmaTotal, true);
    mma_commit(&bars->drain);
    wait_drain(&bars->drain, 0);
    pa.flush(true);
}

// ------------------------------------------------------------------ query splitter (E4M3 keys)
// Byte offset of 16-byte unit `unit` of row r in a swizzled operand block
// whose rows are row_bytes (128, 64 or 32) long: the unit index is XORed with
// row bits, as the TMA swizzle mode of that width lays it out.
__device__ __forceinline__ uint32_t swizzled_unit(int r, int unit, int row_bytes)
{
    const uint32_t o = static_cast<uint32_t>(r * row_bytes + unit * 16);
    const uint32_t mask = row_bytes == 128 ? (7u << 7) : (row_bytes == 64 ? (3u << 7) : (1u << 7));
    return o ^ ((o & mask) >> 3);
}

// Two fp32 -> two E4M3, round to nearest even (|x| < 448 here); lo in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi)
{
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two E4M3 (low byte first) -> two fp32, exact.
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t b)
{
    float2 r;
    asm("{\n\t.reg .b16 lo, hi;\n\t.reg .b32 h;\n\t"
        "cvt.rn.f16x2.e4m3x2 h, %2;\n\t"
        "mov.b32 {lo, hi}, h;\n\t"
        "cvt.f32.f16 %0, lo;\n\t"
        "cvt.f32.f16 %1, hi;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "h"(static_cast<unsigned short>(b)));
    return r;
}

// Four bf16 (two words, element 0 in the low half of w0) times inv -> the two
// E4M3 pieces: hi8 = E4M3(x), lo8 = E4M3(x - hi8), four bytes each.
__device__ __forceinline__ void split4(uint32_t w0, uint32_t w1, float inv, uint32_t &hi8,
                                       uint32_t &lo8)
{
    const float x0 = __uint_as_float(w0 << 16) * inv;
    const float x1 = __uint_as_float(w0 & 0xFFFF0000u) * inv;
    const float x2 = __uint_as_float(w1 << 16) * inv;
    const float x3 = __uint_as_float(w1 & 0xFFFF0000u) * inv;
    const uint32_t h01 = f32x2_to_e4m3x2(x0, x1);
    const uint32_t h23 = f32x2_to_e4m3x2(x2, x3);
    const float2 b01 = e4m3x2_to_f32x2(h01);
    const float2 b23 = e4m3x2_to_f32x2(h23);
    hi8 = h01 | (h23 << 16);
    lo8 = f32x2_to_e4m3x2(x0 - b01.x, x1 - b01.y) | (f32x2_to_e4m3x2(x2 - b23.x, x3 - b23.y) << 16);
}

// Four bf16 (two words) times inv, each rounded once to E4M3 (the one-piece
// query): four bytes, element 0 in the low byte.
__device__ __forceinline__ uint32_t round4(uint32_t w0, uint32_t w1, float inv)
{
    const float x0 = __uint_as_float(w0 << 16) * inv;
    const float x1 = __uint_as_float(w0 & 0xFFFF0000u) * inv;
    const float x2 = __uint_as_float(w1 << 16) * inv;
    const float x3 = __uint_as_float(w1 & 0xFFFF0000u) * inv;
    return f32x2_to_e4m3x2(x0, x1) | (f32x2_to_e4m3x2(x2, x3) << 16);
}

// E4M3 keys: the tensor core multiplies E4M3 by E4M3, so warps 10-11 carry
// each bf16 query row (one (query, head) pair) as sigma * (hi8 + lo8): sigma a
// power of two that puts the row's largest |q| in [128, 256), hi8 the E4M3
// rounding of q / sigma and lo8 the E4M3 rounding of what is left.  The
// remainder has at most four significant bits, so the pair is exact whenever
// it lies on E4M3's grid: for every element of at least 2^-9 of the row's
// largest, and within 2^-17 of that largest otherwise (rows whose largest is
// below 2^-100 take the scale of 2^-100).  hi8 and lo8 go to two
// K-major operand blocks (rows of d bytes, swizzled at width d); sigma goes to
// the epilogue, which folds it into the head weight (ReLU(sigma x) = sigma
// ReLU(x) for sigma > 0).  With one piece (q_pieces == 1) only hi8 is formed
// and multiplied: half the tensor work, each query element rounded once to
// E4M3 (relative error up to 2^-4).
constexpr int kSplitThreads = 64;

__device__ void run_qsplit(const Params &p, uint8_t *smem, Barriers *bars, const WaitCtl &ctl,
                           int ct)
{
    const int lane = ct & 31;
    const int units = p.row_bytes / 16;     // 8 bf16 per 16-byte unit, per chunk
    const int eunits = p.d / 16;            // 16 E4M3 per 16-byte unit
    const uint8_t *qs = smem + p.off_q;
    uint8_t *e_hi = smem + p.off_e;
    uint8_t *e_lo = e_hi + p.N * p.d;
    int quse = 0;
    ProfAcc pa;
    Prof pf, pt;
    const bool rec = ct == 0;
    pt.start();
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        const int par = quse & 1;
        pf.start();
        bool ok = wait_bounded(&bars->q_full, quse & 1, ctl, kRoleSplit, id);
        // the MMAs of the previous item are done with the pieces, and the
        // epilogue with this half's scales
        ok = ok && wait_bounded(&bars->e_empty, (quse & 1) ^ 1, ctl, kRoleSplit, id);
        ok = ok && wait_bounded(&bars->sig_empty[par], ((quse >> 1) & 1) ^ 1, ctl, kRoleSplit, id);
        pf.add(pa, kPfSplitWait, rec);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok)
            return;
        pf.start();
        float *sig = reinterpret_cast<float *>(smem + p.off_sig) + par * p.N;
        if (it.tile_end > it.tile_begin) {
            for (int r = ct; r < p.N; r += kSplitThreads) {
                uint32_t m2 = 0;
                for (int g = 0; g < p.d / 8; ++g) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(
                        qs + (g / units) * p.N * p.row_bytes + swizzled_unit(r, g % units, p.row_bytes));
                    m2 = __vmaxu2(m2, x.x & 0x7FFF7FFFu);
                    m2 = __vmaxu2(m2, x.y & 0x7FFF7FFFu);
                    m2 = __vmaxu2(m2, x.z & 0x7FFF7FFFu);
                    m2 = __vmaxu2(m2, x.w & 0x7FFF7FFFu);
                }
                const uint32_t mb = max(m2 & 0xFFFFu, m2 >> 16);   // bf16 bits of max |q|
                int e = static_cast<int>((mb >> 7) & 0xFF) - 127;  // floor(log2 max |q|)
                e = e < -100 ? -100 : (e > 127 ? 127 : e);
                const float inv = __uint_as_float(static_cast<uint32_t>(7 - e + 127) << 23);
                sig[r] = __uint_as_float(static_cast<uint32_t>(e - 7 + 127) << 23);
                for (int v = 0; v < eunits; ++v) {
                    uint32_t w[8];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int g = 2 * v + h;
                        const uint4 x = *reinterpret_cast<const uint4 *>(
                            qs + (g / units) * p.N * p.row_bytes + swizzled_unit(r, g % units, p.row_bytes));
                        w[4 * h + 0] = x.x;
                        w[4 * h + 1] = x.y;
                        w[4 * h + 2] = x.z;
                        w[4 * h + 3] = x.w;
                    }
                    uint32_t hi[4], lo[4];
                    const uint32_t o = swizzled_unit(r, v, p.d);
                    if (p.q_pieces == 2) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            split4(w[2 * j], w[2 * j + 1], inv, hi[j], lo[j]);
                        *reinterpret_cast<uint4 *>(e_lo + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            hi[j] = round4(w[2 * j], w[2 * j + 1], inv);
                    }
                    *reinterpret_cast<uint4 *>(e_hi + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                }
            }
            fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&bars->q_empty);       // the bf16 block may be overwritten
            mbar_arrive(&bars->q_ready);       // the pieces are in place
            mbar_arrive(&bars->sig_full[par]); // and the scales
        }
        pf.add(pa, kPfSplitWork, rec);
        ++quse;
    }
    pt.add(pa, kPfSplitTotal, rec);
    pa.flush(rec);
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
// queries: weight 2i+e belongs to column 8i + 2(lane%4) + e.  They are held
// halved, because the tile math multiplies them by twice the ReLU (relu2x2).
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
        wr[i] = make_float2(0.5f * a, 0.5f * b);
    }
}

// E4M3 keys: multiply the weights of fast_load_w by their rows' query scales.
template <int FC, int FQ>
__device__ __forceinline__ void fast_scale_w(const float *sig, int H, int j0, int lane,
                                             float2 (&wr)[FC / 8])
{
    constexpr int RPQ = FC / 8 / FQ;
#pragma unroll
    for (int i = 0; i < FC / 8; ++i) {
        const int j = j0 + i / RPQ;
        const int h = 8 * (i % RPQ) + 2 * (lane & 3);
        const float2 sg = *reinterpret_cast<const float2 *>(sig + j * H + h);
        wr[i].x *= sg.x;
        wr[i].y *= sg.y;
    }
}

// Twice the ReLU of a logit pair, x + |x| in one packed FP32 add: exactly 0
// for x <= 0 and exactly 2x otherwise.  With the weights held halved, the
// packed FMA after it forms the same exact product w * ReLU(x) as
// max(x, 0) * w (for normal weights and |x| below half the largest float),
// and the pair costs one instruction instead of two max operations.
__device__ __forceinline__ float2 relu2x2(uint32_t a, uint32_t b)
{
    const float x = __uint_as_float(a), y = __uint_as_float(b);
    return __fadd2_rn(make_float2(x, y), make_float2(fabsf(x), fabsf(y)));
}

// Scores of FQ queries for one key per thread.  The warp's two 16-lane loads
// cover its 32 keys; thread t holds columns 8i + 2(t%4) + {0,1} of keys
// t/4 + {0, 8, 16, 24}.  The second load (the warp's upper 16 lanes) is in
// flight while the first one's columns are reduced, and the accumulator slot
// is released (one arrive per warp) as soon as it has landed.  Each thread
// forms per-key partial sums over its columns (column pairs with one packed
// FMA); the quad (threads sharing t/4) exchanges halves twice so that thread
// t ends with the complete scores of key row 16*((t>>1)&1) + 8*(t&1) + t/4 of
// the warp's 32.
template <int FC, int FQ>
__device__ __forceinline__ void fast_tile_scores(uint32_t taddr, const float2 (&wr)[FC / 8],
                                                 uint64_t *acc_empty, int lane, float (&F)[FQ])
{
    constexpr int NV = FC / 2;
    constexpr int REPS = FC / 8;
    constexpr int RPQ = REPS / FQ;
    uint32_t va[NV], vb[NV];
    float2 P[4][FQ];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int j = 0; j < FQ; ++j)
            P[k][j] = make_float2(0.0f, 0.0f);
    __syncwarp();
    Ld16x256<FC>::ld(taddr, va);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < NV; ++i)
        reg_fence(va[i]);
    Ld16x256<FC>::ld(taddr + (16u << 16), vb);      // lands while va is reduced
#pragma unroll
    for (int i = 0; i < REPS; ++i) {
        const int j = i / RPQ;
#pragma unroll
        for (int sub = 0; sub < 2; ++sub)
            P[sub][j] = __ffma2_rn(relu2x2(va[4 * i + 2 * sub], va[4 * i + 2 * sub + 1]), wr[i],
                                   P[sub][j]);
    }
#pragma unroll
    for (int j = 0; j < FQ; ++j) {                  // va's sums are formed before the wait
        fence_f32(P[0][j].x);
        fence_f32(P[0][j].y);
        fence_f32(P[1][j].x);
        fence_f32(P[1][j].y);
    }
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < NV; ++i)
        reg_fence(vb[i]);
    tc_fence_before();
    __syncwarp();
    if (lane == 0 && acc_empty)
        mbar_arrive(acc_empty);
#pragma unroll
    for (int i = 0; i < REPS; ++i) {
        const int j = i / RPQ;
#pragma unroll
        for (int sub = 0; sub < 2; ++sub)
            P[2 + sub][j] = __ffma2_rn(relu2x2(vb[4 * i + 2 * sub], vb[4 * i + 2 * sub + 1]), wr[i],
                                       P[2 + sub][j]);
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

// The fast tile math in chunks, for the software pipeline across tiles.  A
// chunk is one 16-lane x 64-column TMEM load (16x256b.x8, 32 registers):
// half h (0: the warp's lanes 0-15, 1: lanes 16-31) and column group cg (64
// columns = repetitions 8cg .. 8cg+7 of the tile's FC/8).  ft_chunk adds a
// chunk's ReLU(logit) x weight pairs to the per-key partial sums; ft_finish
// leaves each thread its key's FQ scores.
template <int FC, int FQ>
__device__ __forceinline__ void ft_chunk(const uint32_t (&x)[32], const float2 (&wr)[FC / 8],
                                         float2 (&P)[4][FQ], int h, int cg)
{
    constexpr int RPQ = (FC / 8) / FQ;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int i = 8 * cg + r;
        const int j = i / RPQ;
#pragma unroll
        for (int sub = 0; sub < 2; ++sub)
            P[2 * h + sub][j] =
                __ffma2_rn(relu2x2(x[4 * r + 2 * sub], x[4 * r + 2 * sub + 1]), wr[i], P[2 * h + sub][j]);
    }
}

template <int FQ>
__device__ __forceinline__ void ft_finish(const float2 (&P)[4][FQ], int lane, float (&F)[FQ])
{
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

// TMEM address of chunk c (of NC = 2 * FC/64) of a tile: halves outermost.
template <int FC>
__device__ __forceinline__ uint32_t ft_chunk_addr(uint32_t tile_addr, int c)
{
    constexpr int CGS = FC / 64;
    return tile_addr + ((c / CGS) ? (16u << 16) : 0u) + 64u * static_cast<uint32_t>(c % CGS);
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
// Writes the score of every (query, key) of the item into the score buffer;
// the selector decides what to keep.
template <int FC, int FQ, bool kHeadsGe32>
__device__ void run_epilogue(const Params &p, uint8_t *smem, Barriers *bars, uint32_t tmem_base,
                             const WaitCtl &ctl, int wg)
{
    const int tid = threadIdx.x & (kGroupThreads - 1); // 0..127 within the warpgroup
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int bar = wg == 0 ? kBarWg0 : kBarWg1;
    const int quarter = warp & 3;             // TMEM lanes this warp may read
    const int j0 = p.tile_split ? 0 : wg * p.qpw; // first query slot this group owns
    const int col0 = j0 * p.H;                 // first TMEM column it reads
    const int ncols = p.qpw * p.H;             // TMEM columns it reads
    const int nchunk = ncols / 32;             // in 32-column chunks (generic path)
    const int cpq_shift = p.H >= 32 ? __ffs(p.H / 32) - 1 : 0;
    const int h_shift = __ffs(p.H) - 1;
    // the key row (of the warp's 32) whose scores this thread ends up with
    const int key_local =
        FC > 0 ? quarter * 32 + 16 * ((lane >> 1) & 1) + 8 * (lane & 1) + (lane >> 2)
               : quarter * 32 + lane;
    int acc_use = 0, it_count = 0;
    int gtile = 0; // tile groups of this CTA so far (tile_split: even ones are group 0's)
    ProfAcc pa;
    Prof pf, pt;
    const bool rec = wg == 0 && tid == 0;
    pt.start();

    // Generic path: the group's weights go through shared memory (one half
    // per item parity; per group when tile_split), loaded into registers one
    // item ahead.
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

    bool ok = true;
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        const int par = it_count & 1;
        // tile_split: both groups use every column, so each has its own halves
        // (a group can run up to two items ahead of the other)
        float *w_s = reinterpret_cast<float *>(smem + p.off_w) +
                     ((p.tile_split ? wg : 0) * 2 + par) * p.qps * p.H;
        // E4M3 keys: the splitter's per-row query scales of this item
        const float *sig = reinterpret_cast<const float *>(smem + p.off_sig) + par * p.N;
        bool oks = true;
        if (p.key_fp8) {
            pf.start();
            oks = wait_bounded(&bars->sig_full[par], (it_count >> 1) & 1, ctl, kRoleEpilogue, id);
            pf.add(pa, kPfEpiBufEmpty, rec);
        }
        if constexpr (FC > 0) {
            fast_load_w<FC, FQ>(p, it, j0, lane, wr);
            if (p.key_fp8 && oks)
                fast_scale_w<FC, FQ>(sig, p.H, j0, lane, wr);
        } else {
            for (int r = 0; r < kWRegs; ++r) {
                const int c = tid + r * kGroupThreads;
                if (c < ncols)
                    w_s[col0 + c] = (p.key_fp8 && oks) ? wnext[r] * sig[col0 + c] : wnext[r];
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
        if (p.key_fp8) {
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->sig_empty[par]);    // scales read
        }
        // The selector must be done with this half (item it_count - 2).
        pf.start();
        const bool okw =
            wait_bounded(&bars->buf_empty[par], ((it_count >> 1) & 1) ^ 1, ctl, kRoleEpilogue, id);
        pf.add(pa, kPfEpiBufEmpty, rec);
        ok = group_all(bar, kGroupThreads, ok && okw && oks); // also publishes w_s
        if (!ok)
            break;
        float *buf = p.scores + (static_cast<size_t>(blockIdx.x) * 2 + par) * p.qps * p.nmax +
                     static_cast<size_t>(j0) * p.nmax;

        if constexpr (FC > 0) {
            if (p.tpg == 1 && !p.tile_split) {
                // One tile per accumulator slot: a software pipeline across the
                // item's tiles in chunks of 16 lanes x 64 columns, two buffers of
                // 32 registers: the next chunk (of this tile, or the first of the
                // next tile) loads while the current one is reduced.  The slot
                // goes back to the MMA once the tile's last chunk has landed.
                constexpr int NC = 2 * (FC / 64);
                uint32_t xa[32], xb[32];
                const uint32_t lane_base =
                    tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + col0;
                int slot = 0;
                if (it.tile_begin < it.tile_end) {
                    slot = acc_use & 1;
                    pf.start();
                    ok = wait_bounded(&bars->acc_full[slot], (acc_use >> 1) & 1, ctl,
                                      kRoleEpilogue, id);
                    ok = __all_sync(0xffffffffu, ok);
                    pf.add(pa, kPfEpiAccFull, rec);
                    ++acc_use;
                    if (ok) {
                        tc_fence_after();
                        __syncwarp();
                        tmem_ld_16x256b_x8(ft_chunk_addr<FC>(lane_base + slot * kSlotCols, 0), xa);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            reg_fence(xa[i]);
                    }
                }
                for (int t = it.tile_begin; t < it.tile_end && ok; ++t) {
                    pf.count(pa, kPfEpiTiles, rec);
                    const int s = t * kTileKeys + key_local;
                    const size_t off = static_cast<size_t>(t - it.tile_begin) * kTileKeys + key_local;
                    float kscale = 1.0f;
                    if (p.key_fp8 && s < p.T)
                        kscale = p.k_scale[static_cast<size_t>(it.b) * p.T + s];
                    const bool in_buf = CSA_CHECK_INDEX(kChkScoreBuf, off, p.nmax);
                    (void)in_buf;
                    pf.start();
                    const uint32_t tile_addr = lane_base + slot * kSlotCols;
                    const bool next = t + 1 < it.tile_end;
                    float2 P[4][FQ];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
#pragma unroll
                        for (int j = 0; j < FQ; ++j)
                            P[k][j] = make_float2(0.0f, 0.0f);
#pragma unroll
                    for (int c = 0; c < NC; ++c) {
                        uint32_t(&cur)[32] = (c & 1) ? xb : xa;
                        uint32_t(&nxt)[32] = (c & 1) ? xa : xb;
                        bool more = true;
                        if (c + 1 < NC) {
                            tmem_ld_16x256b_x8(ft_chunk_addr<FC>(tile_addr, c + 1), nxt);
                        } else {
                            // every chunk of tile t has landed: the slot is free
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0)
                                mbar_arrive(&bars->acc_empty[slot]);
                            more = next;
                            if (next) {
                                slot = acc_use & 1;
                                ok = wait_bounded(&bars->acc_full[slot], (acc_use >> 1) & 1, ctl,
                                                  kRoleEpilogue, id);
                                ok = __all_sync(0xffffffffu, ok);
                                ++acc_use;
                                more = ok;
                                if (ok) {
                                    tc_fence_after();
                                    __syncwarp();
                                    tmem_ld_16x256b_x8(
                                        ft_chunk_addr<FC>(lane_base + slot * kSlotCols, 0), nxt);
                                }
                            }
                        }
                        ft_chunk<FC, FQ>(cur, wr, P, c / (FC / 64), c % (FC / 64));
#pragma unroll
                        for (int j = 0; j < FQ; ++j) {   // the sums are formed before the wait
                            fence_f32(P[0][j].x);
                            fence_f32(P[1][j].x);
                            fence_f32(P[2][j].x);
                            fence_f32(P[3][j].x);
                        }
                        if (more) {
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                reg_fence(nxt[i]);
                        }
                    }
                    float F[FQ];
                    ft_finish<FQ>(P, lane, F);
#pragma unroll
                    for (int q = 0; q < FQ; ++q)
                        if (in_buf)
                            buf[static_cast<size_t>(q) * p.nmax + off] = F[q] * kscale;
                    pf.add(pa, kPfEpiMath, rec);
                }
                // Hand this half to the selector (one arrive per warp).
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&bars->buf_full[par]);
                if (!ok)
                    *ctl.abort = 1;
                ++it_count;
                continue;
            }
        }

        int slot = 0;      // accumulator slot of the current tile group
        bool mine = true;  // tile_split: the current group is this warpgroup's
        for (int t = it.tile_begin; t < it.tile_end && ok; ++t) {
            // tiles come in groups of tpg sharing one slot (as the MMA fills them)
            const int g = (t - it.tile_begin) & (p.tpg - 1);
            const bool last = g == p.tpg - 1 || t + 1 == it.tile_end;
            if (g == 0) {
                mine = !p.tile_split || (gtile++ & 1) == wg;
                if (mine) {
                    // tile_split: group w always drains slot w, every use flips its phase
                    slot = p.tile_split ? wg : acc_use & 1;
                    const uint32_t par = p.tile_split ? (acc_use & 1) : ((acc_use >> 1) & 1);
                    pf.start();
                    ok = wait_bounded(&bars->acc_full[slot], par, ctl, kRoleEpilogue, id);
                    // the TMEM loads below are warp-collective: agree on the outcome first
                    ok = __all_sync(0xffffffffu, ok);
                    pf.add(pa, kPfEpiAccFull, rec);
                    pf.count(pa, kPfEpiTiles, rec);
                    ++acc_use;
                    if (!ok)
                        break;
                    tc_fence_after();
                }
            }
            if (!mine)
                continue;                            // the other warpgroup's group
            const int s = t * kTileKeys + key_local;
            const size_t off = static_cast<size_t>(t - it.tile_begin) * kTileKeys + key_local;
            float kscale = 1.0f;
            if (p.key_fp8 && s < p.T)
                kscale = p.k_scale[static_cast<size_t>(it.b) * p.T + s];
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   slot * kSlotCols + g * p.N + col0;
            const bool in_tmem =
                CSA_CHECK_INDEX(kChkTmemEpi, slot * kSlotCols + g * p.N + col0 + ncols - 1, 2 * kSlotCols);
            const bool in_buf = CSA_CHECK_INDEX(kChkScoreBuf, off, p.nmax);
            (void)in_tmem;
            (void)in_buf;
            pf.start();
            if constexpr (FC > 0) {
                float F[FQ];
                // the slot goes back to the MMA once its group's last tile is loaded
                fast_tile_scores<FC, FQ>(taddr, wr, last ? &bars->acc_empty[slot] : nullptr, lane,
                                         F);
#pragma unroll
                for (int q = 0; q < FQ; ++q)
                    if (in_buf)
                        buf[static_cast<size_t>(q) * p.nmax + off] = F[q] * kscale;
            } else {
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
                            buf[static_cast<size_t>(c >> cpq_shift) * p.nmax + off] = acc * kscale;
                            acc = 0.0f;
                        }
                    } else {
                        // H < 32 (a power of two): each 32-column chunk holds 32/H queries
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            acc = fmaf(fmaxf(__uint_as_float(v[i]), 0.0f), wc[i], acc);
                            if (((i + 1) & (p.H - 1)) == 0) {
                                buf[static_cast<size_t>((c * 32 + i) >> h_shift) * p.nmax + off] =
                                    acc * kscale;
                                acc = 0.0f;
                            }
                        }
                    }
                }
                if (last) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bars->acc_empty[slot]);
                }
            }
            pf.add(pa, kPfEpiMath, rec);
        }
        // Hand this half to the selector (one arrive per warp, after every
        // lane's stores).
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&bars->buf_full[par]);
        if (!ok)
            *ctl.abort = 1;
        ++it_count;
    }
    pt.add(pa, kPfEpiTotal, rec);
    pa.flush(rec);
}

// ------------------------------------------------------------------ selector
// The selector reads a query's scores in chunks of kSelChunk (16 per thread,
// four 16-byte loads issued together), so a pass costs one memory round trip
// per chunk.  Histogram buckets are the top 11 bits of the score's order
// image (sign, exponent, two mantissa bits): fixed, so no range pass.
constexpr int kSelPer = 16;
constexpr int kSelChunk = kGroupThreads * kSelPer;   // 2048 scores
constexpr int kSelShift = 21;                         // 2048 buckets
constexpr int kSelShift2 = kSelShift - 11;            // second level inside one bucket

struct SelectorScratch {
    GroupSmall gs;
    int out_cnt;
    int pad[3];
    uint32_t hist[kNbSelect];
};

// Scores base .. base+kSelChunk of sj into v (index base + 512 r + 4 tid + e
// in v[4 r + e]); slots at or past n get the order image 0 (never kept).
__device__ __forceinline__ void sel_load(const float *sj, int base, int n, int tid,
                                         uint32_t (&o)[kSelPer])
{
    float4 x[kSelPer / 4];
#pragma unroll
    for (int r = 0; r < kSelPer / 4; ++r) {
        const int i = base + r * (kGroupThreads * 4) + 4 * tid;
        x[r] = i < n ? *reinterpret_cast<const float4 *>(sj + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int r = 0; r < kSelPer / 4; ++r) {
        const int i = base + r * (kGroupThreads * 4) + 4 * tid;
        o[4 * r + 0] = i + 0 < n ? ord_of_score(x[r].x) : 0u;
        o[4 * r + 1] = i + 1 < n ? ord_of_score(x[r].y) : 0u;
        o[4 * r + 2] = i + 2 < n ? ord_of_score(x[r].z) : 0u;
        o[4 * r + 3] = i + 3 < n ? ord_of_score(x[r].w) : 0u;
    }
}

// sel_load for a chunk that lies wholly below n: no bounds tests
__device__ __forceinline__ void sel_load_full(const float *sj, int base, int tid, uint32_t (&o)[kSelPer])
{
    float4 x[kSelPer / 4];
#pragma unroll
    for (int r = 0; r < kSelPer / 4; ++r)
        x[r] = *reinterpret_cast<const float4 *>(sj + base + r * (kGroupThreads * 4) + 4 * tid);
#pragma unroll
    for (int r = 0; r < kSelPer / 4; ++r) {
        o[4 * r + 0] = ord_of_score(x[r].x);
        o[4 * r + 1] = ord_of_score(x[r].y);
        o[4 * r + 2] = ord_of_score(x[r].z);
        o[4 * r + 3] = ord_of_score(x[r].w);
    }
}

__device__ __forceinline__ int sel_index(int base, int e, int tid)
{
    return base + (e >> 2) * (kGroupThreads * 4) + 4 * tid + (e & 3);
}

// Appends every key of sj[0..n) (key index key0 + i) that is >= lo to `list`
// in arbitrary order; returns how many.  One shared atomic per warp and chunk.
__device__ int sel_emit(const float *sj, int n, int key0, uint64_t lo, uint64_t *list, int cap,
                        SelectorScratch *sc, int tid)
{
    const int lane = tid & 31;
    if (tid == 0)
        sc->out_cnt = 0;
    named_bar_sync(kBarSelect, kGroupThreads);
    for (int base = 0; base < n; base += kSelChunk) {
        uint32_t o[kSelPer];
        const bool full = base + kSelChunk <= n;
        if (full)
            sel_load_full(sj, base, tid, o);
        else
            sel_load(sj, base, n, tid, o);
        uint32_t keep = 0;
        int mine = 0;
#pragma unroll
        for (int e = 0; e < kSelPer; ++e) {
            const int i = sel_index(base, e, tid);
            const bool k = (full || i < n) && make_key(o[e], static_cast<uint32_t>(key0 + i)) >= lo;
            keep |= k ? (1u << e) : 0u;
            mine += k;
        }
        int incl = mine; // inclusive scan over the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off)
                incl += t;
        }
        const int wtot = __shfl_sync(0xffffffffu, incl, 31);
        int wbase = 0;
        if (lane == 0 && wtot)
            wbase = atomicAdd(&sc->out_cnt, wtot);
        int pos = __shfl_sync(0xffffffffu, wbase, 0) + incl - mine;
#pragma unroll
        for (int e = 0; e < kSelPer; ++e)
            if (keep & (1u << e)) {
                if (CSA_CHECK_INDEX(kChkListPos, pos, cap))
                    list[pos] = make_key(o[e], static_cast<uint32_t>(key0 + sel_index(base, e, tid)));
                ++pos;
            }
    }
    named_bar_sync(kBarSelect, kGroupThreads);
    const int c = sc->out_cnt;
    named_bar_sync(kBarSelect, kGroupThreads); // out_cnt is reset by the next call
    return c;
}

// Bucket of the need-th largest count in hist[0..kNbSelect) (thread tid owns
// buckets [16 tid, 16 tid + 16)): {b*, keys above b*, keys in b*, all keys}.
__device__ void sel_boundary(const uint32_t *hist, int need, GroupSmall *gs, int tid, int (&out)[4])
{
    constexpr int PER = kNbSelect / kGroupThreads;
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
    if (tid == 0)
        gs->bcast[0] = -1;
    named_bar_sync(kBarSelect, kGroupThreads);
    uint32_t higher = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kGroupThreads / 32; ++w) {
        higher += w > wid ? gs->warp_sums[w] : 0u;
        total += gs->warp_sums[w];
    }
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
    named_bar_sync(kBarSelect, kGroupThreads);
    out[0] = gs->bcast[0];
    out[1] = gs->bcast[1];
    out[2] = gs->bcast[2];
    out[3] = static_cast<int>(total);
    named_bar_sync(kBarSelect, kGroupThreads);
}

// Exact cut: the largest 64-bit key L such that exactly `need` keys with score
// image >= lo_ord are >= L (more than `need` such keys exist; keys distinct).
// Only for near-ties: even the second histogram level's boundary bucket holds
// too many keys to keep.
__device__ uint64_t sel_radix(const float *sj, int n, int key0, uint32_t lo_ord, int need,
                              SelectorScratch *sc, int tid)
{
    const int lane = tid & 31;
    uint64_t prefix = 0, mask = 0;
    for (int pos = 56; pos >= 0; pos -= 8) {
        for (int i = tid; i < 256; i += kGroupThreads)
            sc->hist[i] = 0;
        named_bar_sync(kBarSelect, kGroupThreads);
        for (int base = 0; base < n; base += kSelChunk) {
            uint32_t o[kSelPer];
            sel_load(sj, base, n, tid, o);
#pragma unroll
            for (int e = 0; e < kSelPer; ++e) {
                const int i = sel_index(base, e, tid);
                const uint64_t key = make_key(o[e], static_cast<uint32_t>(key0 + i));
                if (i < n && o[e] >= lo_ord && (key & mask) == prefix)
                    atomicAdd(&sc->hist[static_cast<uint32_t>(key >> pos) & 255u], 1u);
            }
        }
        named_bar_sync(kBarSelect, kGroupThreads);
        if (tid < 32) {
            uint32_t c[8];
            uint32_t sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = sc->hist[lane * 8 + j];
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
                        sc->gs.bcast[0] = lane * 8 + j;
                        sc->gs.bcast[1] = static_cast<int>(above);
                        sc->gs.bcast[2] = static_cast<int>(c[j]);
                        break;
                    }
                    above += c[j];
                }
            }
        }
        named_bar_sync(kBarSelect, kGroupThreads);
        const int digit = sc->gs.bcast[0];
        const int above = sc->gs.bcast[1];
        const int inb = sc->gs.bcast[2];
        named_bar_sync(kBarSelect, kGroupThreads);
        need -= above;
        prefix |= static_cast<uint64_t>(digit) << pos;
        mask |= 0xFFull << pos;
        if (inb == need)
            break;
    }
    return prefix;
}

// One query of a finished item: its n visible scores (keys key0..key0+n-1)
// become a list of at most cap keys holding its top k -- all of them when
// they fit (gated mode: all positive ones), else the keys at or above the
// histogram bucket of the k-th largest, else at or above its sub-bucket one
// level down, else exactly the top k.
__device__ int sel_query(const Params &p, const float *sj, int n, int key0, uint64_t *list,
                         SelectorScratch *sc, int tid, ProfAcc &pa, bool rec)
{
    const uint32_t lo_ord = p.mode == 1 ? 0x80000001u : 0u; // gate: score > 0
    const uint64_t lo_key = static_cast<uint64_t>(lo_ord) << 32;
    if (n <= 0)
        return 0;
    if (n <= p.cap)
        return sel_emit(sj, n, key0, lo_key, list, p.cap, sc, tid);
    Prof pf;
    pf.start();
    for (int i = tid; i < kNbSelect; i += kGroupThreads)
        sc->hist[i] = 0;
    named_bar_sync(kBarSelect, kGroupThreads);
    for (int base = 0; base < n; base += kSelChunk) {
        uint32_t o[kSelPer];
        if (base + kSelChunk <= n) {
            // whole chunks skip the per-score bounds test, and in top-k mode
            // (lo_ord == 0) every score passes the floor test
            sel_load_full(sj, base, tid, o);
            if (lo_ord == 0) {
#pragma unroll
                for (int e = 0; e < kSelPer; ++e)
                    atomicAdd(&sc->hist[o[e] >> kSelShift], 1u);
            } else {
#pragma unroll
                for (int e = 0; e < kSelPer; ++e)
                    if (o[e] >= lo_ord)
                        atomicAdd(&sc->hist[o[e] >> kSelShift], 1u);
            }
        } else {
            sel_load(sj, base, n, tid, o);
#pragma unroll
            for (int e = 0; e < kSelPer; ++e)
                if (sel_index(base, e, tid) < n && o[e] >= lo_ord)
                    atomicAdd(&sc->hist[o[e] >> kSelShift], 1u);
        }
    }
    named_bar_sync(kBarSelect, kGroupThreads);
    int bd[4];
    sel_boundary(sc->hist, p.topk, &sc->gs, tid, bd);
    uint64_t lo;
    if (bd[3] <= p.cap) {
        lo = lo_key;                                   // every candidate fits
    } else if (bd[1] + bd[2] <= p.cap) {
        lo = static_cast<uint64_t>(static_cast<uint32_t>(bd[0]) << kSelShift) << 32;
    } else {
        // The boundary bucket (a quarter binade) holds too many keys: one
        // more pass histograms its keys by the next 11 bits of the order image.
        const uint32_t b1 = static_cast<uint32_t>(bd[0]);
        const int above1 = bd[1];
        for (int i = tid; i < kNbSelect; i += kGroupThreads)
            sc->hist[i] = 0;
        named_bar_sync(kBarSelect, kGroupThreads);
        for (int base = 0; base < n; base += kSelChunk) {
            uint32_t o[kSelPer];
            const bool full = base + kSelChunk <= n;
            if (full)
                sel_load_full(sj, base, tid, o);
            else
                sel_load(sj, base, n, tid, o);
#pragma unroll
            for (int e = 0; e < kSelPer; ++e)
                if ((full || sel_index(base, e, tid) < n) && o[e] >= lo_ord && (o[e] >> kSelShift) == b1)
                    atomicAdd(&sc->hist[(o[e] >> kSelShift2) & (kNbSelect - 1)], 1u);
        }
        named_bar_sync(kBarSelect, kGroupThreads);
        int bd2[4];
        sel_boundary(sc->hist, p.topk - above1, &sc->gs, tid, bd2);
        if (above1 + bd2[1] + bd2[2] <= p.cap)
            lo = static_cast<uint64_t>((b1 << kSelShift) |
                                       (static_cast<uint32_t>(bd2[0]) << kSelShift2))
                 << 32;
        else
            lo = sel_radix(sj, n, key0, lo_ord, p.topk, sc, tid);  // near-ties
    }
    pf.add(pa, kPfSelCut, rec);
    return sel_emit(sj, n, key0, lo > lo_key ? lo : lo_key, list, p.cap, sc, tid);
}

__device__ void run_selector(const Params &p, uint8_t *smem, Barriers *bars, const WaitCtl &ctl)
{
    const int tid = threadIdx.x & (kGroupThreads - 1);
    const int lane = tid & 31;
    SelectorScratch *sc = reinterpret_cast<SelectorScratch *>(smem + p.off_sel);
    int it_count = 0;
    ProfAcc pa;
    Prof pf, pt;
    const bool rec = tid == 0;
    pt.start();
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
        const Item it = decode_item(p, id);
        const int par = it_count & 1;
        pf.start();
        bool ok = wait_bounded(&bars->buf_full[par], (it_count >> 1) & 1, ctl, kRoleSelect, id);
        ok = group_all(kBarSelect, kGroupThreads, ok);
        pf.add(pa, kPfSelBufFull, rec);
        if (!ok)
            break;
        pf.start();
        const float *buf = p.scores + (static_cast<size_t>(blockIdx.x) * 2 + par) * p.qps * p.nmax;
        const int key0 = it.tile_begin * kTileKeys;
        const int key_end = it.tile_end * kTileKeys;
        for (int j = 0; j < it.nq; ++j) {
            const int vis = visible_count(p, static_cast<long long>(it.q0 + j) + p.q_offset);
            const int n = max(0, min(vis, key_end) - key0);
            uint64_t *list = p.lists + (static_cast<size_t>(it.lrow + j) * p.nsplit + it.split) * p.cap;
            const int c = sel_query(p, buf + static_cast<size_t>(j) * p.nmax, n, key0, list, sc, tid,
                                    pa, rec);
            if (tid == 0)
                p.counts[static_cast<size_t>(it.lrow + j) * p.nsplit + it.split] = c;
        }
        // every read of this half is done
        named_bar_sync(kBarSelect, kGroupThreads);
        pf.add(pa, kPfSelBusy, rec);
        if (lane == 0)
            mbar_arrive(&bars->buf_empty[par]);
        ++it_count;
    }
    pt.add(pa, kPfSelTotal, rec);
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
        mbar_init(&bars->q_empty, p.key_fp8 ? 2 : 1); // the splitter warps, or the MMA's commit
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->q_ready, 2);
        mbar_init(&bars->e_empty, 1);
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->sig_full[s], 2);
            mbar_init(&bars->sig_empty[s], epi_warps);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->acc_full[s], 1);
            mbar_init(&bars->acc_empty[s], p.tile_split ? 4 : epi_warps);
            mbar_init(&bars->buf_full[s], epi_warps);
            mbar_init(&bars->buf_empty[s], kGroupThreads / 32);
        }
        bars->abort = 0;
#ifdef CSA_DEBUG
        // debug build: the plan's shared-memory carve-up fits the allocation
        const int q_end = p.off_q + p.N * p.d * 2;
        const int k_end = p.off_k + p.stages * kTileKeys * p.d * (p.key_fp8 ? 1 : 2);
        if (!CSA_CHECK_INDEX(kChkQueryBlock, q_end - 1, p.key_fp8 ? p.off_e : p.off_k) ||
            !CSA_CHECK_INDEX(kChkKeyStage, k_end - 1, p.off_w))
            bars->abort = 1;
#endif
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
    } else if (warp < 12) {
        regs_dec<kCtlRegs>();
        if (warp == 8 && lane == 0)
            run_producer(p, &tmQ, &tmK, smem, bars, ctl);
        else if (warp == 9 && lane == 0) {
            if (p.d == 128) {
                if (!p.key_fp8)
                    run_mma<1>(p, smem, bars, tmem_base, ctl);
                else if (p.q_pieces == 2)
                    run_mma<2>(p, smem, bars, tmem_base, ctl);
                else
                    run_mma<3>(p, smem, bars, tmem_base, ctl);
            } else
                run_mma<0>(p, smem, bars, tmem_base, ctl);
        }
        else if (warp >= 10 && p.key_fp8)
            run_qsplit(p, smem, bars, ctl, threadIdx.x - 320);
    } else {
        regs_dec<kSelRegs>();
        run_selector(p, smem, bars, ctl);
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
