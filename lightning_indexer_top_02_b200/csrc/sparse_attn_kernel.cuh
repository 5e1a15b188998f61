// sparse_attn_kernel.cuh -- sparse attention over the keys the indexer
// selected ("StreamIndex: Memory-Bounded Compressed Sparse Attention via
// Streaming Top-k", abstract: the indexer selects the top-k compressed keys
// per query, and a sparse attention kernel reads only those).
//
// For every query row (b, i) and head g < HA:
//   J     = the selected keys idx[b,i,0..topk) (the indexer lists them first
//           and pads with -1; entries outside [0, T) are ignored)
//   o[g]  = softmax_j( scale * qa[g] . kc[J_j] ) . vc[J_j]     (0 if J is empty)
// with one compressed cache row per key shared by every head; the value row
// of key s is read from vc + (b*T + s) * ld_v, so values may be a prefix of
// each key row (a latent cache) or a separate array.
//
// One persistent CTA per SM walks query rows.  Per row the selected keys go
// through in tiles of 128:
//   warp 4 (producer): the row's query block [128 head rows x Dk] by TMA, and
//     per tile the 128 selected key rows and value rows by TMA gather (four
//     rows per instruction) into a two-stage ring;
//   warp 5 (MMA issuer, one thread; owns the TMEM allocation):
//     S(t) = Q . K(t)^T into one of two 128-column TMEM slots (M = 128 head
//     rows, N = 128 keys), then, once the softmax has written P(t-1),
//     O += P(t-1) . V(t-1) into TMEM columns 256.. (N = Dv, V as an MN-major
//     operand exactly as gathered);
//   warps 0-3 (softmax, thread = head row = TMEM lane): online softmax over
//     the row's tiles in the exp2 domain with the running maximum raised only
//     when a tile exceeds it by more than 2^8 (then O is rescaled in TMEM),
//     P in bf16 written to shared memory as the next MMA's K-major A
//     operand, and at the end O / l to global memory (fp32).
// Head rows past HA are computed and discarded (the MMA's M is 128).
#pragma once
#include <cuda.h>
#include <cstdint>

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace csa {
namespace attn {

constexpr int kKeys = 128;      // selected keys per tile (S's N, P.V's K)
constexpr int kRows = 128;      // MMA M: head rows
constexpr int kThreads = 192;   // warps 0-3 softmax, 4 producer, 5 MMA
constexpr int kMaxStages = 2;
constexpr int kOCol = 256;      // first TMEM column of O (S slots take 0..255)
constexpr float kRescaleLog2 = 8.0f; // raise the running max only past 2^8

enum Role : int { kRoleProducer = 21, kRoleMma = 22, kRoleSoftmax = 23 };

struct AttnParams {
    int B, S, T, HA, Dk, Dv, topk;
    int stages;
    float sl2;              // scale * log2(e)
    const int32_t *idx;     // [B*S, topk]
    float *out;             // [B*S, HA, Dv]
    int off_q, off_k, off_v, off_p, off_bar;   // shared-memory carve-up
    int k_stage_bytes, v_stage_bytes;
    long long wait_limit;
};

struct AttnBarriers {
    uint64_t q_full, q_empty;
    uint64_t kv_full[kMaxStages], kv_empty[kMaxStages];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full, pv_done, o_empty;
    uint64_t drain;
    uint32_t tmem_addr;
    int abort;
};

__device__ __forceinline__ bool key_ok(int32_t s, int T) { return s >= 0 && s < T; }

// Selected keys of a query row: the indexer lists them first and pads with
// -1, so the count is the first slot that holds no key (a full row is
// recognised by its last slot; otherwise a bisection on that prefix).
__device__ __forceinline__ int selected_count(const int32_t *row, int topk, int T)
{
    if (key_ok(__ldg(row + topk - 1), T))
        return topk;
    int lo = 0, hi = topk - 1;        // row[hi] holds no key
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (key_ok(__ldg(row + mid), T))
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

// ------------------------------------------------------------------ producer
__device__ void attn_producer(const AttnParams &p, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                              const CUtensorMap *tmV, uint8_t *smem, AttnBarriers *bars,
                              const WaitCtl &ctl)
{
    const int lane = threadIdx.x & 31;
    int gt = 0, rows_used = 0;
    const uint32_t kv_bytes = static_cast<uint32_t>(p.k_stage_bytes + p.v_stage_bytes);
    const uint32_t q_bytes = static_cast<uint32_t>(kRows * p.Dk * 2);
    bool ok = true;
    for (int r = blockIdx.x; r < p.B * p.S && ok; r += gridDim.x) {
        const int32_t *row = p.idx + static_cast<size_t>(r) * p.topk;
        const int n = selected_count(row, p.topk, p.T);
        const int ntiles = (n + kKeys - 1) / kKeys;
        if (ntiles == 0)
            continue;
        const int b = r / p.S;
        // the query block: rows r*HA .. r*HA+127 of [B*S*HA, Dk] (padding head
        // rows read the next rows or the zero fill past the end)
        if (lane == 0) {
            ok = wait_bounded(&bars->q_empty, (rows_used & 1) ^ 1, ctl, kRoleProducer, r);
            if (ok) {
                mbar_arrive_expect_tx(&bars->q_full, q_bytes);
                for (int c = 0; c < p.Dk / 64; ++c)
                    tma_load_2d(smem + p.off_q + c * kRows * 128, tmQ, &bars->q_full, 64 * c,
                                r * p.HA);
            }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok)
            break;
        ++rows_used;
        for (int t = 0; t < ntiles && ok; ++t, ++gt) {
            const int stage = gt % p.stages;
            if (lane == 0) {
                ok = wait_bounded(&bars->kv_empty[stage], ((gt / p.stages) & 1) ^ 1, ctl,
                                  kRoleProducer, r);
                if (ok)
                    mbar_arrive_expect_tx(&bars->kv_full[stage], kv_bytes);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok)
                break;
            // lane l gathers keys 4l .. 4l+3 of the tile; slots holding no key
            // read row 0 of the batch (their scores are masked)
            int rr[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int slot = t * kKeys + 4 * lane + e;
                const int32_t s = slot < p.topk ? __ldg(row + slot) : -1;
                rr[e] = b * p.T + (key_ok(s, p.T) ? s : 0);
            }
            uint8_t *kdst = smem + p.off_k + stage * p.k_stage_bytes + 4 * lane * 128;
            uint8_t *vdst = smem + p.off_v + stage * p.v_stage_bytes + 4 * lane * 128;
            for (int c = 0; c < p.Dk / 64; ++c)
                tma_gather4(kdst + c * kKeys * 128, tmK, &bars->kv_full[stage], 64 * c, rr[0],
                            rr[1], rr[2], rr[3]);
            for (int c = 0; c < p.Dv / 64; ++c)
                tma_gather4(vdst + c * kKeys * 128, tmV, &bars->kv_full[stage], 64 * c, rr[0],
                            rr[1], rr[2], rr[3]);
        }
    }
    // every copy issued lands before the CTA can exit
    if (lane == 0) {
        for (int s = 0; s < p.stages; ++s)
            if (gt > s) {
                const int fills = (gt - s + p.stages - 1) / p.stages;
                wait_drain(&bars->kv_full[s], (fills - 1) & 1);
            }
        if (rows_used > 0)
            wait_drain(&bars->q_full, (rows_used - 1) & 1);
    }
}

// ------------------------------------------------------------------ MMA issuer
__device__ void attn_mma(const AttnParams &p, uint8_t *smem, AttnBarriers *bars, uint32_t tmem,
                         const WaitCtl &ctl)
{
    int gt = 0, rows_used = 0;
    const uint32_t idesc_s = instr_desc_f16(kKeys, 1);
    const uint32_t idesc_pv = instr_desc_f16(p.Dv, 1) | (1u << 16);  // B (V) MN-major
    const uint32_t q_base = smem_u32(smem + p.off_q);
    const uint32_t k_base = smem_u32(smem + p.off_k);
    const uint32_t v_base = smem_u32(smem + p.off_v);
    const uint32_t p_base = smem_u32(smem + p.off_p);
    auto issue_pv = [&](int gu, bool first) -> bool {
        if (!wait_bounded(&bars->p_full, gu & 1, ctl, kRoleMma, gu))
            return false;
        // the row's first P.V overwrites O: the previous row's O must have been read out
        if (first && rows_used > 0 &&
            !wait_bounded(&bars->o_empty, (rows_used - 1) & 1, ctl, kRoleMma, gu))
            return false;
        tc_fence_after();
        const int stage = gu % p.stages;
        const uint32_t vst = v_base + stage * p.v_stage_bytes;
#pragma unroll
        for (int ks = 0; ks < kKeys / 16; ++ks) {
            const uint64_t adesc = smem_desc_kmajor(p_base + (ks >> 2) * kRows * 128 + (ks & 3) * 32, 128);
            const uint64_t bdesc = smem_desc_mn_sw128(vst + ks * 16 * 128, kKeys * 128, 1024);
            mma_f16_ss(tmem + kOCol, adesc, bdesc, idesc_pv, (!first || ks > 0) ? 1u : 0u);
        }
        mma_commit(&bars->kv_empty[stage]);
        mma_commit(&bars->pv_done);
        return true;
    };
    bool ok = true;
    for (int r = blockIdx.x; r < p.B * p.S && ok; r += gridDim.x) {
        const int32_t *row = p.idx + static_cast<size_t>(r) * p.topk;
        const int n = selected_count(row, p.topk, p.T);
        const int ntiles = (n + kKeys - 1) / kKeys;
        if (ntiles == 0)
            continue;
        if (!wait_bounded(&bars->q_full, rows_used & 1, ctl, kRoleMma, r))
            break;
        tc_fence_after();
        const int g0 = gt;
        for (int t = 0; t < ntiles; ++t, ++gt) {
            const int stage = gt % p.stages;
            const int slot = gt & 1;
            // one stage: tile t's keys replace tile t-1's values, so P.V of
            // tile t-1 goes first; with two, S(t) overlaps the softmax of t-1
            if (p.stages == 1 && t > 0 && !(ok = issue_pv(gt - 1, gt - 1 == g0)))
                break;
            ok = wait_bounded(&bars->kv_full[stage], (gt / p.stages) & 1, ctl, kRoleMma, r) &&
                 wait_bounded(&bars->s_empty[slot], ((gt >> 1) & 1) ^ 1, ctl, kRoleMma, r);
            if (!ok)
                break;
            tc_fence_after();
            const uint32_t kst = k_base + stage * p.k_stage_bytes;
            for (int ks = 0; ks < p.Dk / 16; ++ks) {
                const uint32_t co = (ks >> 2) * kRows * 128 + (ks & 3) * 32;
                mma_f16_ss(tmem + slot * kKeys, smem_desc_kmajor(q_base + co, 128),
                           smem_desc_kmajor(kst + co, 128), idesc_s, ks > 0 ? 1u : 0u);
            }
            mma_commit(&bars->s_full[slot]);
            if (p.stages > 1 && t > 0 && !(ok = issue_pv(gt - 1, gt - 1 == g0)))
                break;
        }
        if (!ok)
            break;
        mma_commit(&bars->q_empty);                  // the query block is free
        ok = issue_pv(gt - 1, gt - 1 == g0);
        ++rows_used;
    }
    mma_commit(&bars->drain);
    wait_drain(&bars->drain, 0);
}

// ------------------------------------------------------------------ softmax
// Validity of the tile's 128 key slots as four 32-bit masks (bit j of mask w
// = slot 32w + j), formed by each warp from the index row.
__device__ __forceinline__ void tile_masks(const int32_t *row, int topk, int n, int T, int t,
                                           int lane, uint32_t (&mask)[4])
{
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const int slot = t * kKeys + 32 * w + lane;
        const bool ok = slot < n && key_ok(__ldg(row + slot), T);
        mask[w] = __ballot_sync(0xffffffffu, ok);
    }
}

__device__ void attn_softmax(const AttnParams &p, uint8_t *smem, AttnBarriers *bars, uint32_t tmem,
                             const WaitCtl &ctl)
{
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int hrow = threadIdx.x;                 // head row = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    uint8_t *pbuf = smem + p.off_p;
    int gt = 0, rows_used = 0;
    bool ok = true;
    for (int r = blockIdx.x; r < p.B * p.S && ok; r += gridDim.x) {
        const int32_t *row = p.idx + static_cast<size_t>(r) * p.topk;
        const int n = selected_count(row, p.topk, p.T);
        const int ntiles = (n + kKeys - 1) / kKeys;
        float *orow = p.out + (static_cast<size_t>(r) * p.HA + hrow) * p.Dv;
        if (ntiles == 0) {
            if (hrow < p.HA)
                for (int e = 0; e < p.Dv; e += 4)
                    *reinterpret_cast<float4 *>(orow + e) = make_float4(0.f, 0.f, 0.f, 0.f);
            continue;
        }
        float m = -INFINITY, l = 0.0f;
        for (int t = 0; t < ntiles; ++t, ++gt) {
            const int slot = gt & 1;
            uint32_t mask[4];
            tile_masks(row, p.topk, n, p.T, t, lane, mask);
            ok = wait_bounded(&bars->s_full[slot], (gt >> 1) & 1, ctl, kRoleSoftmax, r);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                break;
            tc_fence_after();
            float x[kKeys];
            {
                uint32_t v[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    tmem_ld_32x32b_x32(lane_base + slot * kKeys + 32 * c, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        x[32 * c + j] = ((mask[c] >> j) & 1u) ? __uint_as_float(v[j]) * p.sl2
                                                              : -INFINITY;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->s_empty[slot]);     // the S slot may be overwritten
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < kKeys; ++j)
                mt = fmaxf(mt, x[j]);
            float m_use = m, alpha = 1.0f;
            bool rescale = false;
            if (m == -INFINITY) {
                m_use = mt;                            // first keys of the row
            } else if (mt > m + kRescaleLog2) {
                m_use = mt;
                alpha = exp2f(m - mt);
                rescale = true;
            }
            float sum = 0.0f;
            uint32_t pk[kKeys / 2];
#pragma unroll
            for (int j = 0; j < kKeys; j += 2) {
                const float p0 = m_use == -INFINITY ? 0.0f : exp2f(x[j] - m_use);
                const float p1 = m_use == -INFINITY ? 0.0f : exp2f(x[j + 1] - m_use);
                sum += p0 + p1;
                const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                pk[j / 2] = *reinterpret_cast<const uint32_t *>(&h);
            }
            l = l * alpha + sum;
            m = m_use;
            // the previous tile's P.V is done: P may be overwritten and O is stable
            if (t > 0) {
                ok = wait_bounded(&bars->pv_done, (gt - 1) & 1, ctl, kRoleSoftmax, r);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok)
                    break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
                    // O (TMEM, this thread's row) *= alpha, 32 columns at a time
                    for (int c = 0; c < p.Dv / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(lane_base + kOCol + 32 * c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
                        tmem_st_32x32b_x32(lane_base + kOCol + 32 * c, v);
                    }
                    tmem_st_wait();
                }
            }
            // P row: 128 bf16 keys as two 64-key chunks of the K-major operand
            // (128-byte rows, 16-byte units swizzled by the row's low 3 bits)
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int c = u >> 3, uu = u & 7;
                uint8_t *dst = pbuf + c * kRows * 128 + hrow * 128 + ((uu ^ (hrow & 7)) << 4);
                *reinterpret_cast<uint4 *>(dst) =
                    make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->p_full);
        }
        if (!ok)
            break;
        // the row's last P.V, then O / l to global memory
        ok = wait_bounded(&bars->pv_done, (gt - 1) & 1, ctl, kRoleSoftmax, r);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok)
            break;
        tc_fence_after();
        const float inv = l > 0.0f ? 1.0f / l : 0.0f;
        for (int c = 0; c < p.Dv / 32; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(lane_base + kOCol + 32 * c, v);
            tmem_ld_wait();
            if (hrow < p.HA) {
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(orow + 32 * c + j) =
                        make_float4(__uint_as_float(v[j]) * inv, __uint_as_float(v[j + 1]) * inv,
                                    __uint_as_float(v[j + 2]) * inv, __uint_as_float(v[j + 3]) * inv);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&bars->o_empty);
        ++rows_used;
    }
    if (!ok)
        *ctl.abort = 1;
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    AttnBarriers *bars = reinterpret_cast<AttnBarriers *>(smem + p.off_bar);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 1);
        for (int s = 0; s < kMaxStages; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->s_empty[s], 4);
        }
        mbar_init(&bars->p_full, 4);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->o_empty, 4);
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (warp == 5) {
        tmem_alloc(&bars->tmem_addr, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_addr;
    WaitCtl ctl{&bars->abort, p.wait_limit};
    if (warp < 4)
        attn_softmax(p, smem, bars, tmem, ctl);
    else if (warp == 4)
        attn_producer(p, &tmQ, &tmK, &tmV, smem, bars, ctl);
    else if (lane == 0)
        attn_mma(p, smem, bars, tmem, ctl);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) {
        __syncwarp();
        tmem_dealloc(tmem, 512);
    }
}

} // namespace attn
} // namespace csa
