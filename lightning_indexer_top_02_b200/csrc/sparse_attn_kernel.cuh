// sparse_attn_kernel.cuh -- sparse attention over the keys the indexer
// selected ("StreamIndex: Memory-Bounded Compressed Sparse Attention via
// Streaming Top-k", abstract: the indexer selects the top-k compressed keys
// per query, and a sparse attention kernel reads only those).
//
// For every query row (b, i) and head g < HA:
//   J     = the entries of idx[b,i,0..topk) in [0, T), in slot order (the
//           indexer lists its selection first and pads with -1; any entry
//           outside [0, T) is padding, wherever it stands)
//   o[g]  = softmax_j( scale * qa[g] . kc[J_j] ) . vc[J_j]     (0 if J is empty)
// with one compressed cache row per key shared by every head; the value row
// of key s is read from vc + (b*T + s) * ld_v, so values may be a prefix of
// each key row (a latent cache) or a separate array.
//
// One persistent CTA per SM walks query rows.  Per row the slots up to the
// last one that holds a key go through in tiles of 128:
//   warp 13 (control): scans each row's index slots ahead of the others and
//     publishes its tile count through a two-entry ring; loads the row's
//     query block [128 head rows x Dk] by TMA (for HA <= 64 a 64-row block,
//     loaded twice, into rows 0-63 and 64-127);
//   warps 4-11 (gather, 16 tile rows each, two per SM sub-partition): per
//     tile the selected key rows and value rows by cp.async, 16 bytes per
//     thread, written straight into the 128-byte-swizzled K-major layout,
//     into separate key and value rings (a key stage frees as soon as its S
//     is computed); every thread's arrival on the stage's barrier fires when
//     its copies have landed;
//   warp 12 (MMA issuer, one thread; owns the TMEM allocation):
//     S(t) = Q . K(t)^T into one of two 128-column TMEM slots (M = 128 head
//     rows, N = 128 keys), then, once the softmax has written P(t-1) over
//     that tile's slot, O += P(t-1) . V(t-1) with P read from TMEM (N = Dv, V
//     as an MN-major operand exactly as gathered) into TMEM columns 256..;
//     that P.V's completion frees the slot;
//   warps 0-3 (softmax, thread = head row = TMEM lane): online softmax over
//     the row's tiles in the exp2 domain with the running maximum raised only
//     when a tile exceeds it by more than 2^8 (then O is rescaled in TMEM),
//     P in bf16 written back to TMEM over the first 64 columns of its S slot,
//     and at the end O / l to global memory (fp32).  The tile's slot
//     validity comes from index loads issued one tile ahead.
// Head rows past HA are computed by the MMA and discarded; a softmax warp
// whose 32 rows are all past HA only keeps the barrier protocol.  Warps 14-15
// only complete the last warpgroup; registers move to the softmax
// warpgroup (setmaxnreg).
#pragma once
#include <cuda.h>
#include <cstdint>

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace csa {
namespace attn {

constexpr int kKeys = 128;      // selected keys per tile (S's N, P.V's K)
constexpr int kRows = 128;      // MMA M: head rows
constexpr int kThreads = 512;   // warps 0-3 softmax, 4-11 gather, 12 MMA, 13 control
constexpr int kGatherWarps = 8;  // two warpgroups
constexpr int kGatherRows = kKeys / kGatherWarps;   // tile rows per gather warp
constexpr int kMmaWarp = 4 + kGatherWarps, kControlWarp = kMmaWarp + 1;
// register split (setmaxnreg): launched with kLaunchRegs per thread, the
// softmax warpgroup raises its count to kSoftmaxRegs, each gather warpgroup
// lowers its count to kGatherRegs, the MMA / control warpgroup keeps the
// launch count.  An increase must not go below, a decrease not above, the
// count a warpgroup holds, and the increase can only take what the decreases
// released.
constexpr int kLaunchRegs = 128;
constexpr int kSoftmaxRegs = 248, kGatherRegs = 64;
static_assert(kSoftmaxRegs >= kLaunchRegs && kGatherRegs <= kLaunchRegs &&
                  kSoftmaxRegs % 8 == 0 && kGatherRegs % 8 == 0 && kSoftmaxRegs <= 256 &&
                  kGatherRegs >= 24,
              "setmaxnreg counts: increases from, decreases to at most, the launch count");
static_assert(kSoftmaxRegs - kLaunchRegs <= 2 * (kLaunchRegs - kGatherRegs),
              "the softmax increase must fit in what the gather warpgroups release");
static_assert(128 * (kSoftmaxRegs + 2 * kGatherRegs + kLaunchRegs) <= kThreads * kLaunchRegs,
              "the register split must fit in the launch's registers");
static_assert(kGatherRows <= 32 && kGatherWarps % 4 == 0, "one index slot per gather lane");
constexpr int kMaxStages = 2;   // per ring (keys, values)
constexpr int kOCol = 256;      // first TMEM column of O (S slots take 0..255)
constexpr int kScanChunk = 256; // index slots the producer scans per step (8 per lane)
constexpr float kRescaleLog2 = 8.0f; // raise the running max only past 2^8

enum Role : int { kRoleProducer = 21, kRoleMma = 22, kRoleSoftmax = 23, kRoleGather = 24 };

struct AttnParams {
    int B, S, T, HA, Dk, Dv, topk;
    int k_stages, v_stages;
    int split;              // HA <= 64: each query block loaded twice, keys split over warp pairs
    float sl2;              // scale * log2(e)
    const int32_t *idx;     // [B*S, topk]
    const uint8_t *k;       // key rows, Dk bf16 each
    const uint8_t *v;       // value rows, ld_v bf16 apart
    long long v_row_bytes;  // ld_v * 2
    float *out;             // [B*S, HA, Dv]
    int off_q, off_k, off_v, off_p, off_bar;   // shared-memory carve-up
    int k_stage_bytes, v_stage_bytes;
    long long wait_limit;
};

struct AttnBarriers {
    uint64_t q_full, q_empty;
    uint64_t k_full[kMaxStages], k_empty[kMaxStages];
    uint64_t v_full[kMaxStages], v_empty[kMaxStages];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2], pv_done, o_empty;       // p_full: tile g's P in TMEM, entry g & 1
    uint64_t row_full[2], row_empty[2];
    uint64_t drain;
    int row_tiles[2];       // tile count of the row published in each ring entry
    int gather_rows[kGatherWarps][kGatherRows];   // global key rows of the tile, per gather warp
    uint64_t xbar[2][2];    // split mode: per head-row pair, two exchange phases
    float xchg[2][4][32];   // split mode: exchanged partial maxima / sums
    uint32_t tmem_addr;
    int abort;
};

__device__ __forceinline__ bool key_ok(int32_t s, int T) { return s >= 0 && s < T; }

// Index slots base + 32u + lane (u < 8) of a row, -1 past topk.
__device__ __forceinline__ void scan_load(const int32_t *row, int base, int topk, int lane,
                                          int32_t (&v)[8])
{
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int slot = base + 32 * u + lane;
        v[u] = slot < topk ? __ldg(row + slot) : -1;
    }
}

// The last slot of the chunk that holds a key, or -1 (warp-uniform).
__device__ __forceinline__ int scan_last(const int32_t (&v)[8], int base, int T)
{
    int last = -1;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const uint32_t b = __ballot_sync(0xffffffffu, key_ok(v[u], T));
        if (b)
            last = base + 32 * u + 31 - __clz(b);
    }
    return last;
}

// ------------------------------------------------------------------ control
__device__ void attn_control(const AttnParams &p, const CUtensorMap *tmQ, uint8_t *smem,
                             AttnBarriers *bars, const WaitCtl &ctl)
{
    const int lane = threadIdx.x & 31;
    const int rows = p.B * p.S;
    int rows_used = 0;
    const uint32_t q_bytes = static_cast<uint32_t>(kRows * p.Dk * 2);
    // tile count of row r: the slots up to the last one that holds a key
    auto row_tiles = [&](int r) -> int {
        const int32_t *row = p.idx + static_cast<size_t>(r) * p.topk;
        int last = -1;
        for (int base = 0; base < p.topk; base += 2 * kScanChunk) {
            int32_t v0[8], v1[8];
            scan_load(row, base, p.topk, lane, v0);
            scan_load(row, base + kScanChunk, p.topk, lane, v1);
            last = max(last, scan_last(v0, base, p.T));
            last = max(last, scan_last(v1, base + kScanChunk, p.T));
        }
        return (last + kKeys) / kKeys;
    };
    // publishes the tile count of the CTA's i-th row
    auto publish = [&](int i, int nt) -> bool {
        bool good = true;
        if (lane == 0) {
            good = wait_bounded(&bars->row_empty[i & 1], ((i >> 1) & 1) ^ 1, ctl, kRoleProducer, i);
            if (good) {
                bars->row_tiles[i & 1] = nt;
                mbar_arrive(&bars->row_full[i & 1]);    // release: the count is visible
            }
        }
        return __shfl_sync(0xffffffffu, good, 0);
    };
    int r = blockIdx.x;
    int nt = row_tiles(r);
    bool ok = publish(0, nt);
    for (int i = 0; r < rows && ok; r += gridDim.x, ++i) {
        if (nt > 0) {
            // the query block: rows r*HA .. r*HA+127 of [B*S*HA, Dk] (padding
            // head rows read the next rows or the zero fill past the end)
            if (lane == 0) {
                ok = wait_bounded(&bars->q_empty, (rows_used & 1) ^ 1, ctl, kRoleProducer, r);
                if (ok) {
                    mbar_arrive_expect_tx(&bars->q_full, q_bytes);
                    // split mode: a 64-row box, loaded into rows 0-63 and 64-127
                    for (int c = 0; c < p.Dk / 64; ++c)
                        for (int d = 0; d < (p.split ? 2 : 1); ++d)
                            tma_load_2d(smem + p.off_q + c * kRows * 128 + d * 64 * 128, tmQ,
                                        &bars->q_full, 64 * c, r * p.HA);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok)
                break;
            ++rows_used;
        }
        const int rn = r + gridDim.x;
        if (rn >= rows)
            break;
        nt = row_tiles(rn);
        ok = publish(i + 1, nt);
    }
    // the query copies issued land before the CTA can exit
    if (lane == 0 && rows_used > 0)
        wait_drain(&bars->q_full, (rows_used - 1) & 1);
}

// ------------------------------------------------------------------ gather
// Tile rows row0 .. row0+nrows-1 of one ring stage from global rows
// grows[k] (row_bytes apart; 16-byte units, `units` per row), in the
// 128-byte-swizzled K-major layout: 64-element chunk c of tile row k at
// stage + c*128*128 + k*128, 16-byte unit u of the chunk at (u ^ (k & 7))*16.
// Lane l copies unit q = l % units of rows k = l / units, + rpi, ...
__device__ __forceinline__ void gather_stage(uint32_t stage, const uint8_t *base, long long row_bytes,
                                             const int *grows, int row0, int nrows, int q, int k0,
                                             int rpi)
{
    const int c = q >> 3, u = q & 7;
    const uint32_t dst0 = stage + c * kRows * 128;
    for (int k = k0; k < nrows; k += rpi) {
        const int row = row0 + k;
        cp_async_16(dst0 + row * 128 + ((u ^ (row & 7)) << 4),
                    base + grows[k] * row_bytes + q * 16);
    }
}

__device__ void attn_gather(const AttnParams &p, uint8_t *smem, AttnBarriers *bars, const WaitCtl &ctl)
{
    const int lane = threadIdx.x & 31;
    const int gw = (threadIdx.x >> 5) - 4;        // gather warp 0 .. kGatherWarps-1
    const int row0 = gw * kGatherRows;            // its rows of every tile
    const int rows = p.B * p.S;
    int *grows = bars->gather_rows[gw];
    const uint32_t k_base = smem_u32(smem + p.off_k);
    const uint32_t v_base = smem_u32(smem + p.off_v);
    // lane -> (unit, first row, rows per instruction) for each operand width
    const int ku = p.Dk / 8, vu = p.Dv / 8;
    const int k_rpi = ku >= 32 ? 1 : 32 / ku, v_rpi = vu >= 32 ? 1 : 32 / vu;
    const int k_q = lane % ku, v_q = lane % vu;
    const int k_k0 = lane < k_rpi * ku ? lane / ku : kGatherRows;   // idle lanes copy nothing
    const int v_k0 = lane < v_rpi * vu ? lane / vu : kGatherRows;
    int gt = 0;
    bool ok = true;
    int32_t pf = -1;                              // the next tile's slot row0 + lane
    auto prefetch = [&](int r, int t) {
        const int slot = t * kKeys + row0 + lane;
        pf = lane < kGatherRows && slot < p.topk
                 ? __ldg(p.idx + static_cast<size_t>(r) * p.topk + slot) : -1;
    };
    prefetch(blockIdx.x, 0);
    for (int r = blockIdx.x, i = 0; r < rows && ok; r += gridDim.x, ++i) {
        int nt = 0;
        if (lane == 0) {
            ok = wait_bounded(&bars->row_full[i & 1], (i >> 1) & 1, ctl, kRoleGather, r);
            if (ok)
                nt = *reinterpret_cast<volatile int *>(&bars->row_tiles[i & 1]);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        nt = __shfl_sync(0xffffffffu, nt, 0);
        if (!ok)
            break;
        if (lane == 0)
            mbar_arrive(&bars->row_empty[i & 1]);
        const int rn = r + gridDim.x;
        const int bT = (r / p.S) * p.T;
        if (nt == 0 && rn < rows)
            prefetch(rn, 0);
        for (int t = 0; t < nt; ++t, ++gt) {
            // this tile's global key rows (slots holding no key read row 0 of
            // the batch: their scores are masked)
            __syncwarp();                         // the previous tile's copies have read grows
            if (lane < kGatherRows)
                grows[lane] = bT + (key_ok(pf, p.T) ? pf : 0);
            if (t + 1 < nt)
                prefetch(r, t + 1);
            else if (rn < rows)
                prefetch(rn, 0);
            __syncwarp();
            const int ks = gt % p.k_stages, vs = gt % p.v_stages;
            if (lane == 0)
                ok = wait_bounded(&bars->k_empty[ks], ((gt / p.k_stages) & 1) ^ 1, ctl, kRoleGather, r);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok)
                break;
            gather_stage(k_base + ks * p.k_stage_bytes, p.k, static_cast<long long>(p.Dk) * 2, grows,
                         row0, kGatherRows, k_q, k_k0, k_rpi);
            cp_async_arrive_noinc(&bars->k_full[ks]);
            if (lane == 0)
                ok = wait_bounded(&bars->v_empty[vs], ((gt / p.v_stages) & 1) ^ 1, ctl, kRoleGather, r);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok)
                break;
            gather_stage(v_base + vs * p.v_stage_bytes, p.v, p.v_row_bytes, grows, row0, kGatherRows,
                         v_q, v_k0, v_rpi);
            cp_async_arrive_noinc(&bars->v_full[vs]);
        }
    }
    if (!ok)
        *ctl.abort = 1;
    cp_async_wait_all();                          // every copy lands before the CTA can exit
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
    // O (+)= P(g) . V(g) for the CTA's g-th tile; P(g) is read from TMEM, where
    // the softmax wrote it over its own S slot (packed bf16 pairs, 64 columns)
    auto issue_pv = [&](int g, bool first) -> bool {
        const int vs = g % p.v_stages;
        if (!wait_bounded(&bars->p_full[g & 1], (g >> 1) & 1, ctl, kRoleMma, g) ||
            !wait_bounded(&bars->v_full[vs], (g / p.v_stages) & 1, ctl, kRoleMma, g))
            return false;
        // the row's first P.V overwrites O: the previous row's O must have been read out
        if (first && rows_used > 0 &&
            !wait_bounded(&bars->o_empty, (rows_used - 1) & 1, ctl, kRoleMma, g))
            return false;
        fence_proxy_async_smem();                    // cp.async (generic) writes -> tensor core reads
        tc_fence_after();
        const uint32_t vst = v_base + vs * p.v_stage_bytes;
        const uint32_t p_tmem = tmem + (g & 1) * kKeys;
#pragma unroll
        for (int ks = 0; ks < kKeys / 16; ++ks) {
            const uint64_t bdesc = smem_desc_mn_sw128(vst + ks * 16 * 128, kKeys * 128, 1024);
            mma_f16_ts(tmem + kOCol, p_tmem + 8 * ks, bdesc, idesc_pv, (!first || ks > 0) ? 1u : 0u);
        }
        mma_commit(&bars->v_empty[vs]);
        mma_commit(&bars->s_empty[g & 1]);           // the slot (S, then P) is free
        mma_commit(&bars->pv_done);
        return true;
    };
    bool ok = true;
    for (int r = blockIdx.x, i = 0; r < p.B * p.S && ok; r += gridDim.x, ++i) {
        if (!wait_bounded(&bars->row_full[i & 1], (i >> 1) & 1, ctl, kRoleMma, r))
            break;
        const int nt = *reinterpret_cast<volatile int *>(&bars->row_tiles[i & 1]);
        mbar_arrive(&bars->row_empty[i & 1]);
        if (nt == 0)
            continue;
        if (!wait_bounded(&bars->q_full, rows_used & 1, ctl, kRoleMma, r))
            break;
        tc_fence_after();
        const int g0 = gt;
        for (int t = 0; t < nt; ++t, ++gt) {
            const int ks = gt % p.k_stages;
            const int slot = gt & 1;
            // P(t-1) already written while K(t) is still arriving: its P.V goes first
            bool pv_pending = t > 0;
            if (pv_pending && mbar_try_wait(&bars->p_full[(gt - 1) & 1], ((gt - 1) >> 1) & 1, false) &&
                mbar_try_wait(&bars->v_full[(gt - 1) % p.v_stages], ((gt - 1) / p.v_stages) & 1, false) &&
                !mbar_try_wait(&bars->k_full[ks], (gt / p.k_stages) & 1, false)) {
                if (!(ok = issue_pv(gt - 1, gt - 1 == g0)))
                    break;
                pv_pending = false;
            }
            ok = wait_bounded(&bars->k_full[ks], (gt / p.k_stages) & 1, ctl, kRoleMma, r) &&
                 wait_bounded(&bars->s_empty[slot], ((gt >> 1) & 1) ^ 1, ctl, kRoleMma, r);
            if (!ok)
                break;
            fence_proxy_async_smem();                // cp.async (generic) writes -> tensor core reads
            tc_fence_after();
            const uint32_t kst = k_base + ks * p.k_stage_bytes;
            for (int kk = 0; kk < p.Dk / 16; ++kk) {
                const uint32_t co = (kk >> 2) * kRows * 128 + (kk & 3) * 32;
                mma_f16_ss(tmem + slot * kKeys, smem_desc_kmajor(q_base + co, 128),
                           smem_desc_kmajor(kst + co, 128), idesc_s, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bars->s_full[slot]);
            mma_commit(&bars->k_empty[ks]);
            // S(t) is queued: P(t-1) . V(t-1) overlaps the softmax of tile t
            if (pv_pending && !(ok = issue_pv(gt - 1, gt - 1 == g0)))
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
// Raw extreme of a thread's NC scores of the tile (v = TMEM image, mk = their
// slot validity, bit j of word j/32): the maximum for a non-negative scale,
// the minimum otherwise (the one that becomes the largest scale * s).
// Masked slots are skipped; NaN when none is valid.
template <bool kMasked, int NC>
__device__ __forceinline__ float tile_extreme(const uint32_t (&v)[NC], const uint32_t (&mk)[NC / 32],
                                              bool up)
{
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        a[k] = kMasked ? NAN : __uint_as_float(v[k]);
    auto pick = [&](int j) -> float {
        const float x = __uint_as_float(v[j]);
        return kMasked && !((mk[j >> 5] >> (j & 31)) & 1u) ? NAN : x;
    };
    if (up) {
#pragma unroll
        for (int j = kMasked ? 0 : 8; j < NC; ++j)
            a[j & 7] = fmaxf(a[j & 7], pick(j));
#pragma unroll
        for (int k = 1; k < 8; ++k)
            a[0] = fmaxf(a[0], a[k]);
    } else {
#pragma unroll
        for (int j = kMasked ? 0 : 8; j < NC; ++j)
            a[j & 7] = fminf(a[j & 7], pick(j));
#pragma unroll
        for (int k = 1; k < 8; ++k)
            a[0] = fminf(a[0], a[k]);
    }
    return a[0];
}

// The running maximum (log2 domain) after a tile whose raw extreme is e: the
// maximum is raised only when the tile exceeds it by more than 2^8; alpha is
// the factor O and l must then be scaled by (1 when it was kept).
__device__ __forceinline__ float next_max(float e, float sl2, float m, float &alpha)
{
    const float mt = e == e ? e * sl2 : -INFINITY;
    alpha = 1.0f;
    if (m == -INFINITY)
        return mt;                                   // first keys of the row
    if (mt > m + kRescaleLog2) {
        alpha = ex2_approx(m - mt);
        return mt;
    }
    return m;
}

// P for a thread's NC keys: p_j = 2^(sl2 * v_j - m) (0 for masked slots),
// rounded to bf16 and packed in pairs (the lower half holds the even key), as
// the P.V MMA reads its A operand from TMEM.  Returns the sum of the thread's
// p (fp32).
template <bool kMasked, int NC>
__device__ __forceinline__ float tile_probs(const uint32_t (&v)[NC], const uint32_t (&mk)[NC / 32],
                                            float sl2, float m, uint32_t (&pk)[NC / 2])
{
    float s[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const float nm = -m;
#pragma unroll
    for (int j = 0; j < NC; j += 2) {
        float p0 = ex2_approx(fmaf(__uint_as_float(v[j]), sl2, nm));
        float p1 = ex2_approx(fmaf(__uint_as_float(v[j + 1]), sl2, nm));
        if (kMasked) {
            p0 = ((mk[j >> 5] >> (j & 31)) & 1u) ? p0 : 0.0f;
            p1 = ((mk[(j + 1) >> 5] >> ((j + 1) & 31)) & 1u) ? p1 : 0.0f;
        }
        s[(j >> 1) & 3] += p0 + p1;
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
        pk[j / 2] = *reinterpret_cast<const uint32_t *>(&b2);
    }
    return (s[0] + s[1]) + (s[2] + s[3]);
}

// Index slots 32w + lane (w < 4) of tile t of row r, -1 past topk.
__device__ __forceinline__ void mask_slots(const AttnParams &p, int r, int t, int lane,
                                           int32_t (&v)[4])
{
    const int32_t *row = p.idx + static_cast<size_t>(r) * p.topk;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const int slot = t * kKeys + 32 * w + lane;
        v[w] = slot < p.topk ? __ldg(row + slot) : -1;
    }
}

// Softmax warps.  Full mode (HA > 64): warp w owns head rows 32w.. (its TMEM
// lane quarter) and all 128 keys of a tile.  Split mode (HA <= 64, the query
// block loaded twice so that TMEM lanes 64-127 repeat rows 0-63): warps w and
// w ^ 2 own the same 32 head rows, w the keys 64 * (w >> 1) .. +63 of every
// tile; the pair exchanges its partial row maxima per tile and its partial sums
// per row through shared memory (bounded waits on a pair barrier).  P goes to
// TMEM over the S slot it came from (64 columns of packed bf16 pairs); in split
// mode each copy of a row holds its own keys and zeros for the partner's, so
// O's lanes 0-63 and 64-127 collect the two key halves, summed at the row's end.
template <bool kSplit>
__device__ void attn_softmax(const AttnParams &p, uint8_t *smem, AttnBarriers *bars, uint32_t tmem,
                             const WaitCtl &ctl)
{
    constexpr int NC = kSplit ? kKeys / 2 : kKeys;   // keys per thread per tile
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int q = kSplit ? (warp & 1) : warp;        // head-row quarter
    const int half = kSplit ? (warp >> 1) : 0;       // key / output-column half
    const int hrow = 32 * q + lane;                  // head row
    const bool active = 32 * q < p.HA;               // the warp's rows include heads
    const int rows = p.B * p.S;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const bool up = p.sl2 >= 0.0f;
    // split mode: partial O of the partner's output columns, [q][half][col][lane]
    float *xo = reinterpret_cast<float *>(smem + p.off_p);
    const int xo_cols = p.Dv / 2 < 64 ? p.Dv / 2 : 64;   // columns per exchange round
    int gt = 0, xc = 0;
    bool ok = true;
    // P.V of the CTA's tile g is done.  The barrier completes one phase per
    // P.V, and a parity wait is exact only when the barrier stands at that
    // phase or the next: every tile waits for the previous tile's P.V before
    // it hands over its own P, which keeps the softmax within that window
    // (P.V(g-1) cannot start the phase after next without P(g)).
    auto wait_pv = [&](int g) -> bool {
        const bool good = wait_bounded(&bars->pv_done, g & 1, ctl, kRoleSoftmax, g);
        return __all_sync(0xffffffffu, good);
    };
    // pair barrier (split mode): both warps of the pair have arrived
    auto pair_sync = [&]() -> bool {
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&bars->xbar[q][xc & 1]);
        const bool good = wait_bounded(&bars->xbar[q][xc & 1], (xc >> 1) & 1, ctl, kRoleSoftmax, xc);
        ++xc;
        return __all_sync(0xffffffffu, good);
    };
    // pair exchange (split mode): write own value, sync, read the partner's
    auto exchange = [&](float mine) -> float {
        float *buf = bars->xchg[xc & 1][warp];
        buf[lane] = mine;
        const int x = xc & 1;
        ok = pair_sync();
        return bars->xchg[x][warp ^ 2][lane];
    };
    int32_t pf[4] = {-1, -1, -1, -1};             // the next tile's index slots, in flight
    if (active)
        mask_slots(p, blockIdx.x, 0, lane, pf);
    for (int r = blockIdx.x, i = 0; r < rows && ok; r += gridDim.x, ++i) {
        int nt = 0;
        if (lane == 0) {
            ok = wait_bounded(&bars->row_full[i & 1], (i >> 1) & 1, ctl, kRoleSoftmax, r);
            if (ok)
                nt = *reinterpret_cast<volatile int *>(&bars->row_tiles[i & 1]);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        nt = __shfl_sync(0xffffffffu, nt, 0);
        if (!ok)
            break;
        if (lane == 0)
            mbar_arrive(&bars->row_empty[i & 1]);
        const int rn = r + gridDim.x;
        float *orow = p.out + (static_cast<size_t>(r) * p.HA + hrow) * p.Dv;
        if (nt == 0) {
            const int c0 = kSplit ? half * (p.Dv / 2) : 0, nc = kSplit ? p.Dv / 2 : p.Dv;
            if (hrow < p.HA)
                for (int e = c0; e < c0 + nc; e += 4)
                    *reinterpret_cast<float4 *>(orow + e) = make_float4(0.f, 0.f, 0.f, 0.f);
            if (active && rn < rows)
                mask_slots(p, rn, 0, lane, pf);
            continue;
        }
        float m = -INFINITY, l = 0.0f;
        for (int t = 0; t < nt; ++t, ++gt) {
            const int slot = gt & 1;
            uint32_t mask[4] = {0u, 0u, 0u, 0u};
            if (active) {
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    mask[w] = __ballot_sync(0xffffffffu, key_ok(pf[w], p.T));
                if (t + 1 < nt)
                    mask_slots(p, r, t + 1, lane, pf);
                else if (rn < rows)
                    mask_slots(p, rn, 0, lane, pf);
            }
            ok = wait_bounded(&bars->s_full[slot], (gt >> 1) & 1, ctl, kRoleSoftmax, r);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                break;
            tc_fence_after();
            if (active) {
                uint32_t v[NC];
#pragma unroll
                for (int c = 0; c < NC / 32; ++c)
                    tmem_ld_32x32b_x32(lane_base + slot * kKeys + half * NC + 32 * c,
                                       *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c));
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < NC; ++j)
                    reg_fence(v[j]);
                uint32_t mk[NC / 32];
#pragma unroll
                for (int w = 0; w < NC / 32; ++w)
                    mk[w] = kSplit ? (half ? mask[2 + w] : mask[w]) : mask[w];
                bool full = true;
#pragma unroll
                for (int w = 0; w < NC / 32; ++w)
                    full = full && mk[w] == 0xFFFFFFFFu;
                float e = full ? tile_extreme<false, NC>(v, mk, up) : tile_extreme<true, NC>(v, mk, up);
                if (kSplit) {
                    const float o = exchange(e);
                    if (!ok)
                        break;
                    e = up ? fmaxf(e, o) : fminf(e, o);
                }
                float alpha;
                const float m_new = next_max(e, p.sl2, m, alpha);
                // a raised maximum rescales O (this warp's lanes, every column)
                // once the previous tile's P.V is done
                if (t > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                    if (!(ok = wait_pv(gt - 1)))
                        break;
                    tc_fence_after();
                    for (int c = 0; c < p.Dv; c += 32) {
                        uint32_t o[32];
                        tmem_ld_32x32b_x32(lane_base + kOCol + c, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                        tmem_st_32x32b_x32(lane_base + kOCol + c, o);
                    }
                }
                uint32_t pk[NC / 2];
                float sum = 0.0f;
                if (m_new != -INFINITY) {
                    sum = full ? tile_probs<false, NC>(v, mk, p.sl2, m_new, pk)
                               : tile_probs<true, NC>(v, mk, p.sl2, m_new, pk);
                } else {
#pragma unroll
                    for (int j = 0; j < NC / 2; ++j)    // no key yet: P = 0
                        pk[j] = 0u;
                }
                l = l * alpha + sum;
                m = m_new;
                // P over the slot's first 64 columns (the S values are in registers)
                const uint32_t pcol = lane_base + slot * kKeys;
                if (kSplit) {
                    uint32_t z[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        z[j] = 0u;
                    tmem_st_32x32b_x32(pcol + 32 * half, *reinterpret_cast<uint32_t(*)[32]>(pk));
                    tmem_st_32x32b_x32(pcol + 32 * (1 - half), z);
                } else {
                    tmem_st_32x32b_x32(pcol, *reinterpret_cast<uint32_t(*)[32]>(pk));
                    tmem_st_32x32b_x32(pcol + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
                }
                tmem_st_wait();
            }
            // (see wait_pv; on the first tile of a row this is the previous row's last)
            if (gt > 0 && !(ok = wait_pv(gt - 1)))
                break;
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bars->p_full[gt & 1]);
        }
        if (!ok)
            break;
        // the row's sum over all its keys (split: both halves)
        if (kSplit && active) {
            l += exchange(l);
            if (!ok)
                break;
        }
        // the row's last P.V, then O / l to global memory
        if (!(ok = wait_pv(gt - 1)))
            break;
        tc_fence_after();
        const float inv = l > 0.0f ? 1.0f / l : 0.0f;
        if (kSplit && active) {
            // this warp writes columns half * Dv/2 ..: its own partial plus the
            // partner's, exchanged through shared memory xo_cols at a time
            float *mine = xo + static_cast<size_t>(q * 2 + half) * xo_cols * 32;
            const float *theirs = xo + static_cast<size_t>(q * 2 + (1 - half)) * xo_cols * 32;
            for (int c0 = 0; c0 < p.Dv / 2 && ok; c0 += xo_cols) {
                // this round's columns: xo_cols, or what is left of the half
                // (Dv is a multiple of 64, so a multiple of 32)
                const int cw = p.Dv / 2 - c0 < xo_cols ? p.Dv / 2 - c0 : xo_cols;
                const int pc = (1 - half) * (p.Dv / 2) + c0;   // the partner's columns
                for (int cc = 0; cc < cw; cc += 32) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(lane_base + kOCol + pc + cc, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        mine[(cc + j) * 32 + lane] = __uint_as_float(o[j]);
                }
                if (!(ok = pair_sync()))
                    break;
                const int mc = half * (p.Dv / 2) + c0;         // this warp's columns
                for (int cc = 0; cc < cw; cc += 32) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(lane_base + kOCol + mc + cc, o);
                    tmem_ld_wait();
                    if (hrow < p.HA) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4 *>(orow + mc + cc + j) = make_float4(
                                (__uint_as_float(o[j]) + theirs[(cc + j) * 32 + lane]) * inv,
                                (__uint_as_float(o[j + 1]) + theirs[(cc + j + 1) * 32 + lane]) * inv,
                                (__uint_as_float(o[j + 2]) + theirs[(cc + j + 2) * 32 + lane]) * inv,
                                (__uint_as_float(o[j + 3]) + theirs[(cc + j + 3) * 32 + lane]) * inv);
                    }
                }
                ok = pair_sync();                          // the buffer may be rewritten
            }
            if (!ok)
                break;
        } else if (active) {
            for (int c = 0; c < p.Dv; c += 32) {
                uint32_t o[32];
                tmem_ld_32x32b_x32(lane_base + kOCol + c, o);
                tmem_ld_wait();
                if (hrow < p.HA) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(orow + c + j) =
                            make_float4(__uint_as_float(o[j]) * inv, __uint_as_float(o[j + 1]) * inv,
                                        __uint_as_float(o[j + 2]) * inv, __uint_as_float(o[j + 3]) * inv);
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&bars->o_empty);
    }
    if (!ok)
        *ctl.abort = 1;
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const AttnParams p)
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
            mbar_init(&bars->k_full[s], kGatherWarps * 32);   // one arrival per gather thread
            mbar_init(&bars->k_empty[s], 1);
            mbar_init(&bars->v_full[s], kGatherWarps * 32);
            mbar_init(&bars->v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->s_full[s], 1);
            mbar_init(&bars->s_empty[s], 1);        // P.V of the slot's tile is done
            mbar_init(&bars->row_full[s], 1);
            mbar_init(&bars->row_empty[s], 5 + kGatherWarps);   // MMA, softmax and gather warps
        }
        for (int q = 0; q < 2; ++q)
            for (int k = 0; k < 2; ++k)
                mbar_init(&bars->xbar[q][k], 2);    // the pair's two warps
        for (int b = 0; b < 2; ++b)
            mbar_init(&bars->p_full[b], 4);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->o_empty, 4);
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tmQ);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&bars->tmem_addr, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_addr;
    WaitCtl ctl{&bars->abort, p.wait_limit};
    if (warp < 4) {
        regs_inc<kSoftmaxRegs>();
        if (p.split)
            attn_softmax<true>(p, smem, bars, tmem, ctl);
        else
            attn_softmax<false>(p, smem, bars, tmem, ctl);
    } else if (warp < 4 + kGatherWarps) {      // whole warpgroups
        regs_dec<kGatherRegs>();
        attn_gather(p, smem, bars, ctl);
    } else {
        if (warp == kMmaWarp) {
            if (lane == 0)
                attn_mma(p, smem, bars, tmem, ctl);
        } else if (warp == kControlWarp) {
            attn_control(p, &tmQ, smem, bars, ctl);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) {
        __syncwarp();
        tmem_dealloc(tmem, 512);
    }
}

} // namespace attn
} // namespace csa
